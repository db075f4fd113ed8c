"""Failure detection and bounds checks on the GPU, without faulting it.

Timeout: the fused expert kernel's GEMM2 tiles wait, bounded, for the GEMM1
tiles of their M-block to publish the hidden rows.  The test hook
moe_test_expert_wait shortens that limit and withholds one M-block's publish,
so the wait can only end by running out: the call must return, report
MOE_STATUS_TIMEOUT in the status word, and leave the context usable (the
next normal call is correct).

Guard zones: compute-sanitizer is closed here, so every output and the
workspace of every C-ABI call is placed between two 4 KiB zones of a
sentinel byte; after the calls (stage calls, moe_forward, moe_backward) on
odd, ragged shapes the zones must be untouched, and the results must equal
those of the same calls on ordinary buffers.
"""
import ctypes as C
import dataclasses

import numpy as np
import pytest
import torch

from parity_util import rel_fro
from sparsely_gated_mixture_gate_b200 import _lib, build, synth
from sparsely_gated_mixture_gate_b200 import moe as M

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 4096     # bytes on each side
SENTINEL = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


# ------------------------------------------------------------------ timeout
def _expert_case(d, f, counts, seed):
    n, S = len(counts), sum(counts)
    g = torch.Generator().manual_seed(seed)
    xp = torch.randn(S, d, generator=g).bfloat16()
    W1 = (torch.randn(n, f, d, generator=g) / d ** 0.5).bfloat16()
    W2 = (torch.randn(n, d, f, generator=g) / f ** 0.5).bfloat16()
    b1 = torch.randn(n, f, generator=g) * 0.1
    b2 = torch.randn(n, d, generator=g) * 0.1
    offsets = torch.tensor([0] + list(np.cumsum(counts)), dtype=torch.int32)
    return xp, W1, b1, W2, b2, offsets


def test_expert_wait_runs_out_and_the_context_stays_usable(orc):
    L = _lib.load()
    d, f, counts = 256, 1024, [300, 200, 5, 130]
    xp, W1, b1, W2, b2, offsets = _expert_case(d, f, counts, seed=3)
    S = sum(counts)
    cfg = M.Config(T=S, d=d, n=len(counts), k=1, f=f)
    params = dict(W1=W1.to(DEV), b1=b1.to(DEV), W2=W2.to(DEV), b2=b2.to(DEV))
    xd, od = xp.to(DEV), offsets.to(DEV)
    try:
        # 1 ms for the cross-CTA wait; M-block 0 (expert 0's first 128 rows)
        # never published: its GEMM2 tiles can only give up
        assert L.moe_test_expert_wait(1_000_000, 0) == _lib.MOE_OK
        bad = M.expert_ffn(cfg, xd, od, params)
        torch.cuda.synchronize()  # the kernel ended
        assert M.status_bits(bad["status"]) & M._lib.STATUS_TIMEOUT
    finally:
        L.moe_test_expert_wait(0, -1)
    good = M.expert_ffn(cfg, xd, od, params)
    torch.cuda.synchronize()
    assert M.status_bits(good["status"]) == 0
    got = good["y_perm"].float().cpu().numpy()
    off = offsets.numpy()
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    for r in sorted({0, 127, 128, 299, 300, 499, 500, 504, S - 1}):
        e = int(np.searchsorted(off, r, side="right") - 1)
        want = orc.expert_row(xp[r].float().numpy(), bits(W1[e]), b1[e].numpy(), bits(W2[e]),
                              b2[e].numpy(), bf16=True)
        assert rel_fro(got[r], want) < 3e-2, (r, e)


def test_layer_reports_timeout_through_moe_forward():
    """The same hook through the fused layer: moe_forward returns with
    MOE_STATUS_TIMEOUT set, and the next forward pass is bitwise the one
    before the hook."""
    L = _lib.load()
    w = synth.WORKLOADS["lm-flat"].with_(T=512)
    inp = {k: (v.to(DEV) if v is not None else None) for k, v in synth.make_inputs(w).items()}
    layer = M.MoELayer(M.Config.from_workload(w), inp, torch.device(DEV), resample_noise=False)
    layer.forward_(inp["x"])
    torch.cuda.synchronize()
    want = layer.y.clone()
    try:
        assert L.moe_test_expert_wait(1_000_000, 1) == _lib.MOE_OK
        layer.forward_(inp["x"])
        torch.cuda.synchronize()
        assert M.status_bits(layer.status) & M._lib.STATUS_TIMEOUT
    finally:
        L.moe_test_expert_wait(0, -1)
    layer.status.zero_()
    layer.forward_(inp["x"])
    torch.cuda.synchronize()
    assert M.status_bits(layer.status) == 0
    assert torch.equal(layer.y, want)


# ------------------------------------------------------------------ guard zones
class Guarded:
    """A device tensor between two GUARD-byte zones of SENTINEL bytes."""

    def __init__(self, shape, dtype):
        shape = tuple(shape)
        n = int(np.prod(shape)) if shape else 1
        esz = torch.empty(0, dtype=dtype).element_size()
        g = GUARD // esz
        self.buf = torch.empty(n + 2 * g, dtype=dtype, device=DEV)
        self.buf.view(torch.uint8).fill_(SENTINEL)
        self.t = self.buf[g:g + n].view(shape)

    def intact(self):
        b = self.buf.view(torch.uint8)
        return bool((b[:GUARD] == SENTINEL).all()) and bool((b[-GUARD:] == SENTINEL).all())


def _check(bufs):
    torch.cuda.synchronize()
    bad = [name for name, g in bufs.items() if not g.intact()]
    assert not bad, f"guard zones overwritten next to {bad}"


GUARD_CASES = {
    "noisy-T1": synth.WORKLOADS["lm-flat"].with_(T=1, d=40, f=24, n=8, k=2),
    "noisy-T33": synth.WORKLOADS["lm-flat"].with_(T=33, d=40, f=24, n=8, k=2),
    "noisy-T777": synth.WORKLOADS["lm-flat"].with_(T=777, d=40, f=24, n=13, k=3),
    "switch-capacity-T777": synth.VARIANTS["switch-skew"].with_(T=777, d=40, f=24, n=8),
    "fp32-T33": synth.WORKLOADS["tiny-flat"].with_(T=33, d=40, f=24),
    "hier-T777": synth.WORKLOADS["hierarchical"].with_(T=777, d=40, f=24, n=4 * 8, hier_a=4,
                                                       hier_b=8),
    "sigmoid-shared-T33": synth.VARIANTS["deepseek-tiny"].with_(T=33, d=40, f=24),
    # 2048 experts: a wide gate (16 column tiles per projection)
    "wide-gate-T33": synth.WORKLOADS["many-expert"].with_(T=33, d=40, f=24, n=2048, k=2),
}


@pytest.mark.parametrize("name", list(GUARD_CASES))
def test_stage_calls_stay_inside_their_buffers(name):
    w = GUARD_CASES[name]
    L = _lib.load()
    cfg = M.Config.from_workload(w)
    c = cfg.c()
    inp = {k: (v.to(DEV) if v is not None else None) for k, v in synth.make_inputs(w).items()}
    T, k, n, d, S = w.T, w.k, w.n, w.d, w.T * w.k
    ws_bytes = M.workspace_size(cfg)
    G = dict(ws=Guarded((ws_bytes,), torch.uint8), status=Guarded((1,), torch.int32),
             idx=Guarded((T, k), torch.int32), gate=Guarded((T, k), torch.float32),
             load=Guarded((n,), torch.float32), psum=Guarded((n,), torch.float32),
             counts=Guarded((n,), torch.int32), offsets=Guarded((n + 1,), torch.int32),
             perm_token=Guarded((S,), torch.int32), row_of=Guarded((T, k), torch.int32),
             x_perm=Guarded((S, d), cfg.expert_dtype), y_perm=Guarded((S, d), cfg.expert_dtype),
             y=Guarded((T, d), torch.float32), importance=Guarded((n,), torch.float32),
             losses=Guarded((10,), torch.float32))
    t = {key: g.t for key, g in G.items()}
    t["status"].zero_()
    gp, ep = M.gate_params(inp), M.expert_params(inp)
    ws = (_p(t["ws"]), ws_bytes)
    assert L.moe_gate(C.byref(c), _p(inp["x"]), C.byref(gp), _p(t["idx"]), _p(t["gate"]), _p(t["load"]),
                      _p(t["psum"]), *ws, _p(t["status"]), _stream()) == 0
    _check(G)
    assert L.moe_dispatch(C.byref(c), _p(inp["x"]), _p(t["idx"]), _p(t["counts"]), _p(t["offsets"]),
                          _p(t["perm_token"]), _p(t["row_of"]), _p(t["x_perm"]), *ws, _p(t["status"]),
                          _stream()) == 0
    _check(G)
    assert L.moe_expert_ffn(C.byref(c), _p(t["x_perm"]), _p(t["offsets"]), C.byref(ep), _p(t["y_perm"]),
                            *ws, _p(t["status"]), _stream()) == 0
    _check(G)
    assert L.moe_combine(C.byref(c), _p(t["y_perm"]), _p(t["gate"]), _p(t["row_of"]), _p(inp["x"]),
                         _p(t["y"]), _p(t["status"]), _stream()) == 0
    _check(G)
    assert L.moe_balance_losses(C.byref(c), _p(t["idx"]), _p(t["gate"]), _p(t["counts"]), _p(t["load"]),
                                _p(t["psum"]), _p(t["importance"]), _p(t["losses"]), *ws,
                                _p(t["status"]), _stream()) == 0
    _check(G)
    assert M.status_bits(t["status"]) == 0
    # the same answers as the wrappers' ordinary buffers
    ref = M.gate(cfg, inp["x"], inp)
    assert torch.equal(ref["topk_idx"], t["idx"]) and torch.equal(ref["topk_gate"], t["gate"])
    assert torch.equal(ref["load"], t["load"])


def _guard_layer(layer, cfg):
    """Swap a MoELayer's workspace and outputs for guarded buffers of the
    same shapes; returns the guards."""
    G = {"ws": Guarded((layer.ws.numel(),), torch.uint8)}
    for key in ("y", "topk_idx", "topk_gate", "importance", "load", "counts", "losses", "status"):
        old = getattr(layer, key)
        G[key] = Guarded(old.shape, old.dtype)
        setattr(layer, key, G[key].t)
    layer.ws = G["ws"].t
    layer.status.zero_()
    return G


@pytest.mark.parametrize("name", list(GUARD_CASES))
def test_forward_and_backward_stay_inside_their_buffers(name):
    w = GUARD_CASES[name]
    inp = {k: (v.to(DEV) if v is not None else None) for k, v in synth.make_inputs(w).items()}
    backward = True
    cfg = dataclasses.replace(M.Config.from_workload(w), backward=int(backward))
    plain = M.MoELayer(cfg, inp, torch.device(DEV))
    plain.forward_(inp["x"])
    layer = M.MoELayer(cfg, inp, torch.device(DEV))
    G = _guard_layer(layer, cfg)
    layer.forward_(inp["x"])
    _check(G)
    assert M.status_bits(layer.status) == 0
    assert torch.equal(layer.y, plain.y) and torch.equal(layer.losses, plain.losses)
    if not backward:
        return
    dy = synth.make_dy(w).to(DEV)
    gref = {k: v.clone() for k, v in plain.backward_(inp["x"], dy).items()}
    grads = {k: Guarded(v.shape, v.dtype) for k, v in plain.grads().items()}
    layer._grads = {k: g.t for k, g in grads.items()}
    gg = layer._grads
    layer._mg = _lib.moe_grads(
        dW_g=_p(gg["dWg"]), db_g=_p(gg["dbg"]), dW_noise=_p(gg.get("dWn")), dW1=_p(gg["dW1"]),
        db1=_p(gg["db1"]), dW2=_p(gg["dW2"]), db2=_p(gg["db2"]), dW1s=_p(gg.get("dW1s")),
        db1s=_p(gg.get("db1s")), dW2s=_p(gg.get("dW2s")), db2s=_p(gg.get("db2s")),
        dW_g2=_p(gg.get("dWg2")), db_g2=_p(gg.get("dbg2")), dW_noise2=_p(gg.get("dWn2")))
    layer.backward_(inp["x"], dy)
    _check(G)
    _check(grads)
    assert M.status_bits(layer.status) == 0
    for k, v in gref.items():
        assert torch.equal(gg[k], v), k
