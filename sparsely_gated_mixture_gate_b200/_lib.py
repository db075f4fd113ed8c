"""ctypes declarations of the C ABI in include/moe.h (libmoe_b200.so)."""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_EINVAL, MOE_EWORKSPACE, MOE_ECUDA, MOE_EDEVICE = 0, -1, -2, -3, -4
ROUTER_NOISY_TOPK, ROUTER_SWITCH = 0, 1
F32, BF16 = 0, 1
GATE_FP32, GATE_TF32X3 = 0, 1
STATUS_NONFINITE, STATUS_BAD_INDEX, STATUS_TIMEOUT, STATUS_OVERFLOW = 1, 2, 4, 8

# every symbol include/moe.h declares
EXPORTS = ("moe_strerror", "moe_validate", "moe_capacity", "moe_workspace_size", "moe_gate",
           "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_balance_losses", "moe_forward",
           "moe_trace_enable", "moe_trace_reset", "moe_trace_count", "moe_trace_get",
           "moe_launch_count", "moe_dispatch_noalloc", "moe_sel_bias_update", "moe_backward",
           "moe_noise_step", "moe_fma_probe", "moe_test_expert_wait", "moe_gather_rows",
           "moe_balance_from_totals")


class moe_config(C.Structure):
    _fields_ = [
        ("T", C.c_int32), ("d", C.c_int32), ("n", C.c_int32), ("k", C.c_int32), ("f", C.c_int32),
        ("hier_a", C.c_int32), ("hier_b", C.c_int32), ("hier_k1", C.c_int32), ("hier_k2", C.c_int32),
        ("router", C.c_int32), ("noise", C.c_int32), ("expert_dtype", C.c_int32),
        ("seed", C.c_uint64), ("capacity_factor", C.c_double), ("overflow_passthrough", C.c_int32),
        ("w_importance", C.c_float), ("w_load", C.c_float), ("alpha_aux", C.c_float),
        ("gate_precision", C.c_int32), ("shared_expert", C.c_int32), ("router_stats", C.c_int32),
        ("backward", C.c_int32), ("w_z", C.c_float), ("w_entropy", C.c_float),
        ("token_base", C.c_int64),
    ]


class moe_gate_params(C.Structure):
    _fields_ = [("W_g", C.c_void_p), ("b_g", C.c_void_p), ("W_noise", C.c_void_p),
                ("W_g2", C.c_void_p), ("b_g2", C.c_void_p), ("W_noise2", C.c_void_p),
                ("sel_bias", C.c_void_p), ("seed_dev", C.c_void_p)]


class moe_expert_params(C.Structure):
    _fields_ = [("W1", C.c_void_p), ("b1", C.c_void_p), ("W2", C.c_void_p), ("b2", C.c_void_p),
                ("W1s", C.c_void_p), ("b1s", C.c_void_p), ("W2s", C.c_void_p), ("b2s", C.c_void_p)]


class moe_grads(C.Structure):
    _fields_ = [(name, C.c_void_p) for name in (
        "dW_g", "db_g", "dW_noise", "dW1", "db1", "dW2", "db2", "dW1s", "db1s", "dW2s", "db2s",
        "dgate", "dlogits", "dW_g2", "db_g2", "dW_noise2")]


_lib = None


def load():
    """Load the library; raise loudly if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: run `python -m sparsely_gated_mixture_gate_b200.build` "
                          "(the CUDA library is the only compute path; there is no fallback)")
    L = C.CDLL(LIB_PATH)
    vp, i32, sz = C.c_void_p, C.c_int, C.c_size_t
    cfgp = C.POINTER(moe_config)
    L.moe_strerror.argtypes = [i32]
    L.moe_strerror.restype = C.c_char_p
    L.moe_validate.argtypes = [cfgp]
    L.moe_capacity.argtypes = [cfgp, C.POINTER(C.c_int64)]
    L.moe_workspace_size.argtypes = [cfgp, C.POINTER(C.c_size_t)]
    L.moe_gate.argtypes = [cfgp, vp, C.POINTER(moe_gate_params), vp, vp, vp, vp, vp, sz, vp, vp]
    L.moe_dispatch.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    L.moe_dispatch_noalloc.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.moe_sel_bias_update.argtypes = [cfgp, vp, C.c_float, vp, vp]
    L.moe_noise_step.argtypes = [vp, vp]
    L.moe_fma_probe.argtypes = [vp, i32, i32, i32, vp]
    L.moe_test_expert_wait.argtypes = [C.c_ulonglong, i32]
    i64 = C.c_int64
    L.moe_gather_rows.argtypes = [vp, vp, vp, i64, i64, i64, vp, vp]
    L.moe_balance_from_totals.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.moe_expert_ffn.argtypes = [cfgp, vp, vp, C.POINTER(moe_expert_params), vp, vp, sz, vp, vp]
    L.moe_combine.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp]
    L.moe_balance_losses.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    L.moe_forward.argtypes = [cfgp, vp, C.POINTER(moe_gate_params), C.POINTER(moe_expert_params),
                              vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    L.moe_backward.argtypes = [cfgp, vp, C.POINTER(moe_gate_params), C.POINTER(moe_expert_params),
                               vp, vp, vp, vp, vp, vp, vp, C.POINTER(moe_grads), vp, sz, vp, vp]
    L.moe_trace_enable.argtypes = [i32]
    L.moe_trace_get.argtypes = [i32, C.POINTER(C.c_char_p), C.POINTER(C.c_int), C.POINTER(C.c_double)]
    L.moe_launch_count.restype = C.c_longlong
    for name in EXPORTS:
        if name not in ("moe_strerror", "moe_launch_count"):
            getattr(L, name).restype = i32
    _lib = L
    return L
