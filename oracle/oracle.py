"""ctypes front end of the plain C oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The product package never imports
it.  Every function takes and returns numpy arrays; the arithmetic lives in the
C file, in fp64.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libmoe_oracle.so")
_SRC = [os.path.join(_HERE, "moe_oracle.c")]
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc -O2 (single-threaded, no vectorisation flags
    beyond -O2's defaults)."""
    newest = max(os.path.getmtime(p) for p in _SRC + [os.path.join(_HERE, "moe_oracle.h")])
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < newest:
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, *_SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


class OrcCfg(C.Structure):
    _fields_ = [
        ("T", C.c_int), ("d", C.c_int), ("n", C.c_int), ("k", C.c_int), ("f", C.c_int),
        ("hier_a", C.c_int), ("hier_b", C.c_int), ("hier_k1", C.c_int), ("hier_k2", C.c_int),
        ("router", C.c_int), ("noise", C.c_int), ("seed", C.c_uint64),
        ("capacity_factor", C.c_double), ("passthrough", C.c_int), ("expert_bf16", C.c_int),
        ("w_importance", C.c_double), ("w_load", C.c_double), ("alpha", C.c_double),
        ("shared_expert", C.c_int), ("router_stats", C.c_int),
        ("w_z", C.c_double), ("w_entropy", C.c_double),
    ]


class OrcInputs(C.Structure):
    _fields_ = [
        ("x", C.c_void_p), ("Wg", C.c_void_p), ("bg", C.c_void_p), ("Wn", C.c_void_p),
        ("Wg2", C.c_void_p), ("bg2", C.c_void_p), ("Wn2", C.c_void_p),
        ("W1", C.c_void_p), ("b1", C.c_void_p), ("W2", C.c_void_p), ("b2", C.c_void_p),
        ("sel_bias", C.c_void_p),
        ("W1s", C.c_void_p), ("b1s", C.c_void_p), ("W2s", C.c_void_p), ("b2s", C.c_void_p),
    ]


class OrcOutputs(C.Structure):
    _fields_ = [
        ("y", C.c_void_p), ("topk_idx", C.c_void_p), ("topk_gate", C.c_void_p),
        ("importance", C.c_void_p), ("load", C.c_void_p), ("prob_sum", C.c_void_p),
        ("counts", C.c_void_p), ("row_of", C.c_void_p), ("losses", C.c_void_p),
        ("near_tie", C.c_void_p),
    ]


class OrcGrads(C.Structure):
    _fields_ = [(name, C.c_void_p) for name in (
        "dx", "dWg", "dbg", "dWn", "dW1", "db1", "dW2", "db2", "dW1s", "db1s", "dW2s", "db2s",
        "dgate", "dlogits", "dnoise", "dWg2", "dbg2", "dWn2")]


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_SO)
        vp, u32, i32, f64 = C.c_void_p, C.c_uint32, C.c_int, C.c_double
        L.orc_philox4x32_10.argtypes = [vp, vp, vp]
        L.orc_box_muller.argtypes = [u32, u32, i32]
        L.orc_box_muller.restype = f64
        L.orc_noise.argtypes = [C.c_uint64, u32, u32, u32]
        L.orc_noise.restype = f64
        L.orc_softplus.argtypes = [f64]
        L.orc_softplus.restype = f64
        L.orc_phi.argtypes = [f64]
        L.orc_phi.restype = f64
        L.orc_cv2.argtypes = [vp, i32]
        L.orc_cv2.restype = f64
        L.orc_bf16_round.argtypes = [C.c_float]
        L.orc_bf16_round.restype = C.c_float
        L.orc_capacity.argtypes = [i32, i32, i32, f64]
        L.orc_capacity.restype = C.c_int64
        L.orc_gate_row.argtypes = [i32, i32, i32, i32, i32, C.c_uint64, u32, u32,
                                   vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.orc_sel_bias_update.argtypes = [i32, i32, i32, vp, C.c_float, vp]
        L.orc_router_stats.argtypes = [C.POINTER(OrcCfg), C.POINTER(OrcInputs), vp, vp]
        L.orc_router_stats.restype = i32
        L.orc_load_row.argtypes = [i32, i32, i32, vp, vp, vp, vp]
        L.orc_dispatch.argtypes = [i32, i32, i32, C.c_int64, vp, vp, vp, vp, vp, vp, vp]
        L.orc_expert_row.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp]
        L.orc_gate_batch.argtypes = [C.POINTER(OrcCfg), C.POINTER(OrcInputs), vp, vp, vp, vp, vp]
        L.orc_gate_batch.restype = i32
        L.orc_gate_tokens.argtypes = [C.POINTER(OrcCfg), C.POINTER(OrcInputs), vp, i32, vp, vp, vp, vp,
                                      vp]
        L.orc_gate_tokens.restype = i32
        L.orc_combine.argtypes = [i32, i32, i32, vp, vp, vp, vp, i32, vp]
        L.orc_balance.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, C.c_int64, i32, f64, f64, f64,
                                  vp, vp]
        L.orc_forward.argtypes = [C.POINTER(OrcCfg), C.POINTER(OrcInputs), C.POINTER(OrcOutputs)]
        L.orc_forward.restype = i32
        L.orc_cv2_grad.argtypes = [vp, i32, vp]
        L.orc_backward.argtypes = [C.POINTER(OrcCfg), C.POINTER(OrcInputs), vp, C.POINTER(OrcGrads)]
        L.orc_backward.restype = i32
        L.orc_expert_backward.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                          vp, vp, vp, vp]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- noise
def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32)
    k = np.asarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def box_muller(w0: int, w1: int, branch: int = 0) -> float:
    """branch 0: r cos(2 pi u2); branch 1: r sin(2 pi u2)."""
    return lib().orc_box_muller(w0, w1, branch)


def noise(seed: int, token: int, expert: int, gate_id: int = 0) -> float:
    return lib().orc_noise(seed, token, expert, gate_id)


def softplus(z: float) -> float:
    return lib().orc_softplus(z)


def phi(z: float) -> float:
    return lib().orc_phi(z)


def cv2(v) -> float:
    a = _c(v, np.float64)
    return lib().orc_cv2(_p(a), a.size)


def bf16_round(v: float) -> float:
    return lib().orc_bf16_round(v)


def capacity(T: int, k: int, n: int, cf: float) -> int:
    return lib().orc_capacity(T, k, n, cf)


# ---------------------------------------------------------------- gate
def gate_row(x, Wg, k, *, bg=None, Wn=None, router=0, noise=True, seed=0, token=0, gate_id=0,
             sel_bias=None):
    x = _c(x, np.float32)
    Wg = _c(Wg, np.float32)
    d, n = Wg.shape
    bg = _c(bg, np.float32)
    Wn = _c(Wn, np.float32) if noise else None
    sb = _c(sel_bias, np.float32)
    c = np.zeros(n); s = np.zeros(n); H = np.zeros(n, np.float32)
    order = np.zeros(n, np.int32); gates = np.zeros(k); p = np.zeros(n)
    lib().orc_gate_row(d, n, k, router, int(bool(noise)), seed, token, gate_id, _p(x), _p(Wg),
                       _p(bg), _p(Wn), _p(c), _p(s), _p(H), _p(order), _p(gates), _p(p), _p(sb))
    return dict(c=c, s=s, H=H, order=order, gates=gates, idx=order[:k].copy(), p=p)


def sel_bias_update(counts, T: int, k: int, gamma: float, bias) -> np.ndarray:
    """Router 2's selection-bias update; returns the new bias (fp32)."""
    counts = _c(counts, np.int32)
    b = np.array(bias, dtype=np.float32, copy=True)
    lib().orc_sel_bias_update(counts.size, T, k, _p(counts), gamma, _p(b))
    return b


def load_row(c, s, H, k, noise=True) -> np.ndarray:
    c = _c(c, np.float64); s = _c(s, np.float64); H = _c(H, np.float32)
    P = np.zeros(c.size)
    lib().orc_load_row(c.size, k, int(bool(noise)), _p(c), _p(s), _p(H), _p(P))
    return P


# ---------------------------------------------------------------- dispatch
def dispatch(idx, n: int, C: int):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.zeros(n, np.int32); offsets = np.zeros(n + 1, np.int32)
    S = max(T * k, 1)
    perm_token = np.full(S, -1, np.int32); perm_slot = np.full(S, -1, np.int32)
    row_of = np.zeros((T, k), np.int32)
    ninv = np.zeros(1, np.int64)
    lib().orc_dispatch(T, k, n, C, _p(idx), _p(counts), _p(offsets), _p(perm_token),
                       _p(perm_slot), _p(row_of), _p(ninv))
    R = int(offsets[-1])
    return dict(counts=counts, offsets=offsets, perm_token=perm_token[:R], perm_slot=perm_slot[:R],
                row_of=row_of, n_invalid=int(ninv[0]))


# ---------------------------------------------------------------- expert
def expert_row(x, W1, b1, W2, b2, bf16: bool) -> np.ndarray:
    """W1: [f][d], W2: [d][f]; bf16 weights are passed as uint16 bit patterns."""
    x = _c(x, np.float32)
    wdt = np.uint16 if bf16 else np.float32
    W1 = _c(W1, wdt); W2 = _c(W2, wdt)
    f, d = W1.shape
    b1 = _c(b1, np.float32); b2 = _c(b2, np.float32)
    y = np.zeros(d)
    lib().orc_expert_row(d, f, int(bool(bf16)), _p(x), _p(W1), _p(b1), _p(W2), _p(b2), _p(y))
    return y


# ---------------------------------------------------------------- forward
_CFG_KEYS = ("T", "d", "n", "k", "f", "hier_a", "hier_b", "hier_k1", "hier_k2", "router", "noise",
             "seed", "capacity_factor", "passthrough", "expert_bf16", "w_importance", "w_load", "alpha",
             "shared_expert", "router_stats", "w_z", "w_entropy")


def make_cfg(**kw) -> OrcCfg:
    base = dict(hier_a=0, hier_b=0, hier_k1=0, hier_k2=0, router=0, noise=1, seed=0,
                capacity_factor=0.0, passthrough=0, expert_bf16=0, w_importance=0.1,
                w_load=0.1, alpha=0.01, shared_expert=0, router_stats=0, w_z=0.0, w_entropy=0.0)
    base.update({k: v for k, v in kw.items() if k in _CFG_KEYS})
    return OrcCfg(**{k: base[k] for k in _CFG_KEYS})


def _inputs(oc, inp):
    wdt = np.uint16 if oc.expert_bf16 else np.float32
    keep = {}
    for name, dt in (("x", np.float32), ("Wg", np.float32), ("bg", np.float32), ("Wn", np.float32),
                     ("Wg2", np.float32), ("bg2", np.float32), ("Wn2", np.float32),
                     ("W1", wdt), ("b1", np.float32), ("W2", wdt), ("b2", np.float32),
                     ("sel_bias", np.float32), ("W1s", wdt), ("b1s", np.float32), ("W2s", wdt),
                     ("b2s", np.float32)):
        keep[name] = _c(inp.get(name), dt)
    return keep, OrcInputs(**{name: _p(a) for name, a in keep.items()})


def gate_batch(cfg: dict, inp: dict) -> dict:
    """Gate of the whole batch (flat, Switch or hierarchical); expert weights
    are not needed."""
    oc = make_cfg(**cfg)
    keep, ins = _inputs(oc, inp)
    T, n, k = oc.T, oc.n, oc.k
    out = dict(topk_idx=np.zeros((T, k), np.int32), topk_gate=np.zeros((T, k)), load=np.zeros(n),
               prob_sum=np.zeros(n), near_tie=np.zeros(T, np.float32))
    rc = lib().orc_gate_batch(C.byref(oc), C.byref(ins), _p(out["topk_idx"]), _p(out["topk_gate"]),
                              _p(out["load"]), _p(out["prob_sum"]), _p(out["near_tie"]))
    if rc != 0:
        raise ValueError(f"oracle rejected the configuration {cfg}")
    return out


def gate_tokens(cfg: dict, inp: dict, tokens) -> dict:
    """The gate for the listed tokens only (x rows and noise counters of those
    tokens); load / prob_sum are sums over the listed tokens."""
    oc = make_cfg(**cfg)
    keep, ins = _inputs(oc, inp)
    toks = _c(tokens, np.int32)
    m, n, k = toks.size, oc.n, oc.k
    out = dict(topk_idx=np.zeros((m, k), np.int32), topk_gate=np.zeros((m, k)), load=np.zeros(n),
               prob_sum=np.zeros(n), near_tie=np.zeros(m, np.float32))
    rc = lib().orc_gate_tokens(C.byref(oc), C.byref(ins), _p(toks), m, _p(out["topk_idx"]),
                               _p(out["topk_gate"]), _p(out["load"]), _p(out["prob_sum"]),
                               _p(out["near_tie"]))
    if rc != 0:
        raise ValueError(f"oracle rejected the configuration {cfg}")
    return out


def router_stats(cfg: dict, inp: dict):
    """(sum of squared logit norms, sum of softmax entropies) over the tokens
    of the flat / primary gate."""
    oc = make_cfg(**cfg)
    keep, ins = _inputs(oc, inp)
    z = C.c_double(); h = C.c_double()
    if lib().orc_router_stats(C.byref(oc), C.byref(ins), C.byref(z), C.byref(h)) != 0:
        raise ValueError(f"oracle rejected the configuration {cfg}")
    return z.value, h.value


def combine(Y, gate, row_of, x=None, passthrough=False) -> np.ndarray:
    Y = _c(Y, np.float64); gate = _c(gate, np.float64); row_of = _c(row_of, np.int32)
    T, k = row_of.shape
    d = Y.shape[1]
    x = _c(x, np.float32)
    y = np.zeros((T, d))
    lib().orc_combine(T, k, d, _p(Y), _p(gate), _p(row_of), _p(x), int(bool(passthrough)), _p(y))
    return y


def balance(n, topk_idx, topk_gate, counts, load, prob_sum=None, C=2**63 - 1, router=0,
            w_importance=0.1, w_load=0.1, alpha=0.01):
    idx = _c(topk_idx, np.int32); g = _c(topk_gate, np.float64)
    T, k = idx.shape
    counts = _c(counts, np.int32); load = _c(load, np.float64); ps = _c(prob_sum, np.float64)
    imp = np.zeros(n); losses = np.zeros(8)
    lib().orc_balance(n, T, k, _p(idx), _p(g), _p(counts), _p(load), _p(ps), C, router,
                      w_importance, w_load, alpha, _p(imp), _p(losses))
    return imp, losses


def forward(cfg: dict, inp: dict) -> dict:
    """Run the whole layer.  ``cfg`` holds the fields of ``OrcCfg``; ``inp``
    holds numpy arrays x, Wg, bg, Wn, Wg2, bg2, Wn2, W1, b1, W2, b2, and for
    router 2 / a shared expert sel_bias, W1s, b1s, W2s, b2s (bf16 expert
    weights as uint16 bit patterns)."""
    oc = make_cfg(**cfg)
    T, d, n, k = oc.T, oc.d, oc.n, oc.k
    keep, ins = _inputs(oc, inp)
    out = dict(y=np.zeros((T, d)), topk_idx=np.zeros((T, k), np.int32), topk_gate=np.zeros((T, k)),
               importance=np.zeros(n), load=np.zeros(n), prob_sum=np.zeros(n),
               counts=np.zeros(n, np.int32), row_of=np.zeros((T, k), np.int32),
               losses=np.zeros(10), near_tie=np.zeros(T, np.float32))
    outs = OrcOutputs(**{name: _p(a) for name, a in out.items()})
    rc = lib().orc_forward(C.byref(oc), C.byref(ins), C.byref(outs))
    if rc != 0:
        raise ValueError(f"oracle rejected the configuration {cfg}")
    return out


# ---------------------------------------------------------------- backward
def cv2_grad(v) -> np.ndarray:
    a = _c(v, np.float64)
    g = np.zeros(a.size)
    lib().orc_cv2_grad(_p(a), a.size, _p(g))
    return g


def backward(cfg: dict, inp: dict, dy) -> dict:
    """Gradients of L = sum(dy * y) + losses[0] + losses[1] + losses[3]
    + w_z losses[8] - w_entropy losses[9] of
    ``forward(cfg, inp)`` with respect to x and every parameter; also dL/d
    topk_gate ("dgate") and, for flat layers, dL/d clean logits ("dlogits")
    and dL/d (x W_noise) ("dnoise").  Hierarchical layers: dWg, dbg, dWn are
    the primary gate's, dWg2, dbg2, dWn2 the secondary gates'."""
    oc = make_cfg(**cfg)
    T, d, n, k, f = oc.T, oc.d, oc.n, oc.k, oc.f
    keep, ins = _inputs(oc, inp)
    dy = _c(dy, np.float32)
    gn = oc.hier_a if oc.hier_a else n   # width of the flat or primary gate
    out = dict(dx=np.zeros((T, d)), dWg=np.zeros((d, gn)), dbg=np.zeros(gn), dWn=np.zeros((d, gn)),
               dW1=np.zeros((n, f, d)), db1=np.zeros((n, f)), dW2=np.zeros((n, d, f)),
               db2=np.zeros((n, d)), dgate=np.zeros((T, k)), dlogits=np.zeros((T, n)),
               dnoise=np.zeros((T, n)))
    if oc.hier_a:
        a_, b_ = oc.hier_a, oc.hier_b
        out.update(dWg2=np.zeros((a_, d, b_)), dbg2=np.zeros((a_, b_)), dWn2=np.zeros((a_, d, b_)))
    if oc.shared_expert:
        out.update(dW1s=np.zeros((f, d)), db1s=np.zeros(f), dW2s=np.zeros((d, f)), db2s=np.zeros(d))
    g = OrcGrads(**{name: _p(a) for name, a in out.items()})
    if lib().orc_backward(C.byref(oc), C.byref(ins), _p(dy), C.byref(g)) != 0:
        raise ValueError(f"oracle backward rejected the configuration {cfg}")
    return out


def expert_backward(x_rows, g, dy_rows, W1, b1, W2, b2, bf16: bool) -> dict:
    """One expert's part of the backward over the given rows (see
    orc_expert_backward): its weight and bias gradients, dL/dgate per row and
    its part of dx per row.  bf16 weights as uint16 bit patterns."""
    x_rows = _c(x_rows, np.float32); dy_rows = _c(dy_rows, np.float32)
    g = _c(g, np.float64)
    wdt = np.uint16 if bf16 else np.float32
    W1 = _c(W1, wdt); W2 = _c(W2, wdt)
    f, d = W1.shape
    b1 = _c(b1, np.float32); b2 = _c(b2, np.float32)
    R = x_rows.shape[0]
    out = dict(dW1=np.zeros((f, d)), db1=np.zeros(f), dW2=np.zeros((d, f)), db2=np.zeros(d),
               dgate=np.zeros(R), dx=np.zeros((R, d)))
    lib().orc_expert_backward(d, f, int(bool(bf16)), R, _p(x_rows), _p(g), _p(dy_rows), _p(W1),
                              _p(b1), _p(W2), _p(b2), _p(out["dW1"]), _p(out["db1"]),
                              _p(out["dW2"]), _p(out["db2"]), _p(out["dgate"]), _p(out["dx"]))
    return out
