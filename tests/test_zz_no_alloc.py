"""moe_dispatch_noalloc against moe_dispatch, through the C ABI.

The allocation-free dispatch is for callers that only get their input and
output buffers and cannot allocate scratch device memory (for example a
plugin of an inference engine that plans all memory up front, or a serving
loop that must not call cudaMalloc after start-up).  Its results must equal
those of the workspace-based moe_dispatch; two calls in a row check that the
shared scratch array left by the first call does not leak into the second.
This file is collected last on purpose.
"""
import ctypes as C

import pytest
import torch

from sparsely_gated_mixture_gate_b200 import _lib, build, synth
from sparsely_gated_mixture_gate_b200 import moe as M

DEV = "cuda"


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _outputs(cfg, with_x):
    S = max(cfg.T * cfg.k, 1)
    return dict(counts=torch.full((cfg.n,), -7, dtype=torch.int32, device=DEV),
                offsets=torch.full((cfg.n + 1,), -7, dtype=torch.int32, device=DEV),
                perm_token=torch.full((S,), -7, dtype=torch.int32, device=DEV),
                row_of=torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device=DEV),
                x_perm=torch.zeros(S, cfg.d, dtype=cfg.expert_dtype, device=DEV) if with_x else None,
                status=torch.zeros(1, dtype=torch.int32, device=DEV))


def _run_both(L, cfg, x, idx):
    c = cfg.c()
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    a = _outputs(cfg, x is not None)
    ws = M.workspace(cfg, DEV)
    rc = L.moe_dispatch(C.byref(c), _p(x), _p(idx), _p(a["counts"]), _p(a["offsets"]), _p(a["perm_token"]),
                        _p(a["row_of"]), _p(a["x_perm"]), _p(ws), ws.numel(), _p(a["status"]), stream)
    assert rc == _lib.MOE_OK
    b = _outputs(cfg, x is not None)
    rc = L.moe_dispatch_noalloc(C.byref(c), _p(x), _p(idx), _p(b["counts"]), _p(b["offsets"]),
                                _p(b["perm_token"]), _p(b["row_of"]), _p(b["x_perm"]), _p(b["status"]),
                                stream)
    assert rc == _lib.MOE_OK
    torch.cuda.synchronize()
    return a, b


def _same(a, b, R):
    for key in ("counts", "offsets", "row_of", "status"):
        assert torch.equal(a[key], b[key]), key
    assert torch.equal(a["perm_token"][:R], b["perm_token"][:R])
    if a["x_perm"] is not None:
        xa, xb = a["x_perm"][:R], b["x_perm"][:R]
        if xa.dtype == torch.bfloat16:
            xa, xb = xa.view(torch.int16), xb.view(torch.int16)
        assert torch.equal(xa, xb)


@pytest.mark.gpu
def test_noalloc_dispatch_matches_workspace_dispatch_twice():
    build.build()
    L = _lib.load()
    # first call: LM-shaped routing with a capacity limit
    cfg1 = M.Config(T=8192, d=512, n=256, k=4, f=1024, capacity_factor=1.0)
    idx1 = synth.random_routing(cfg1.T, cfg1.k, cfg1.n, device=DEV, skew=0.8, seed=1)
    x1 = torch.randn(cfg1.T, cfg1.d, device=DEV)
    a, b = _run_both(L, cfg1, x1, idx1)
    _same(a, b, int(a["offsets"][-1]))
    assert int(a["offsets"][-1]) < cfg1.T * cfg1.k  # the cap dropped slots
    # second call right after, other sizes and ids: nothing of the first call
    # may survive in the shared scratch
    cfg2 = M.Config(T=3000, d=64, n=37, k=3, f=64, expert_bf16=0)
    idx2 = synth.random_routing(cfg2.T, cfg2.k, cfg2.n, device=DEV, skew=1.2, seed=2)
    x2 = torch.randn(cfg2.T, cfg2.d, device=DEV)
    a, b = _run_both(L, cfg2, x2, idx2)
    _same(a, b, int(a["offsets"][-1]))
    assert int(b["counts"].sum()) == cfg2.T * cfg2.k


@pytest.mark.gpu
@pytest.mark.parametrize("n,T_max", [(256, 524032), (4096, 4064)])
def test_noalloc_dispatch_size_limit_is_exact(n, T_max):
    """The documented limits: T_max tokens fit the fixed array (and give
    moe_dispatch's results), T_max + 1 is refused before any device work."""
    build.build()
    L = _lib.load()
    cfg = M.Config(T=T_max, d=8, n=n, k=4, f=8)
    idx = synth.random_routing(T_max, 4, n, device=DEV, skew=0.5, seed=n)
    x = torch.randn(T_max, 8, device=DEV)
    a, b = _run_both(L, cfg, x, idx)
    _same(a, b, int(a["offsets"][-1]))
    c = M.Config(T=T_max + 1, d=8, n=n, k=4, f=8).c()
    dummy = torch.zeros(16, dtype=torch.int32, device=DEV)
    p = _p(dummy)
    rc = L.moe_dispatch_noalloc(C.byref(c), None, p, p, p, p, p, None, p,
                                C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.MOE_EWORKSPACE
    torch.cuda.synchronize()
    assert int(dummy.abs().sum()) == 0


@pytest.mark.gpu
def test_noalloc_dispatch_rejects_sizes_beyond_its_array():
    build.build()
    L = _lib.load()
    cfg = M.Config(T=65536, d=512, n=4096, k=4, f=1024)
    c = cfg.c()
    dummy = torch.zeros(16, dtype=torch.int32, device=DEV)
    p = _p(dummy)
    rc = L.moe_dispatch_noalloc(C.byref(c), None, p, p, p, p, p, None, p,
                                C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.MOE_EWORKSPACE
    torch.cuda.synchronize()
    assert int(dummy.abs().sum()) == 0  # nothing was launched
