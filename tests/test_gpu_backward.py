"""GPU parity of the backward pass (moe_backward through the C ABI) against
the oracle's backward in its bf16 mode, on the same seeded inputs.

The oracle takes the kernels' rounding points (bf16 expert-row gradients,
hidden-layer gradient and input-row gradients; fp32 gates), so what remains
is fp32-versus-fp64 accumulation order and the odd bf16 rounding that lands
on the other side of a tie: every gradient within 1e-2 relative Frobenius
of the oracle's (bf16 carries 8 bits), the gate gradient dL/dgate within
5e-3.  With fp32 experts nothing is rounded: 1e-4 for all.  Cases whose routing has near ties (k-th and (k+1)-th logits closer
than 1e-5) are skipped: a flipped choice changes the whole token."""
import dataclasses

import numpy as np
import pytest
import torch

from sparsely_gated_mixture_gate_b200 import build, synth
from sparsely_gated_mixture_gate_b200 import moe as M

pytestmark = pytest.mark.gpu
DEV = "cuda"
TIE = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def to_dev(inp):
    return {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}


def np_inputs(inp):
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif v.dtype == torch.bfloat16:
            out[k] = synth.bf16_bits(v)
        else:
            out[k] = v.detach().cpu().numpy()
    return out


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


W = synth.WORKLOADS
V = synth.VARIANTS
LOSSES = dict(w_importance=0.3, w_load=0.4)
CASES = {
    # noisy top-k, ragged d and f (not multiples of 64), capacity drops and pass-through
    "noisy-ragged-capacity": W["lm-flat"].with_(T=300, n=24, k=2, d=200, f=136, capacity_factor=1.0,
                                                passthrough=1, bias_var=0.1, logit_bias_var=0.1,
                                                **LOSSES),
    # the lm-flat layer's shape on 512 tokens: about 8 rows per expert, so nearly every
    # weight-gradient K loop ends in a partial 16-row step
    "lm-flat-512": W["lm-flat"].with_(T=512, **LOSSES),
    "noise-free": W["lm-flat"].with_(T=256, n=16, k=2, d=64, f=64, noise=0, **LOSSES),
    "k1-noisy": W["lm-flat"].with_(T=333, n=8, k=1, d=64, f=192, **LOSSES),
    "kn-equal": W["tiny-flat"].with_(T=65, n=3, k=3, d=16, f=24, expert_bf16=1, **LOSSES),
    "empty-experts": W["lm-flat"].with_(T=40, n=64, k=1, d=64, f=64, **LOSSES),
    "many-rows": W["lm-flat"].with_(T=2048, n=4, k=2, d=128, f=256, **LOSSES),
    "switch-capacity": V["switch-skew"].with_(T=1024, d=128, n=16, f=128, alpha=0.5,
                                              w_importance=0.3),
    "sigmoid-shared": V["deepseek-tiny"].with_(w_importance=0.3),
    "sigmoid-shared-256": V["deepseek-flat"].with_(T=256, d=128, n=32, k=4, f=128,
                                                   w_importance=0.3),
    "shared-noisy-passthrough": W["lm-flat"].with_(T=200, n=32, k=2, d=64, f=64, shared_expert=1,
                                                   capacity_factor=0.5, passthrough=1, **LOSSES),
    # the largest slot count, and a gate wider than the register path (n > 1024)
    "k8-n64": W["lm-flat"].with_(T=200, n=64, k=8, d=64, f=64, **LOSSES),
    "wide-n2000": W["lm-flat"].with_(T=128, n=2000, k=2, d=64, f=32, **LOSSES),
    # the router z-loss and gate entropy as weighted loss terms, on each router
    "zloss-entropy-noisy": W["lm-flat"].with_(T=300, n=24, k=2, d=64, f=64, router_stats=1,
                                              w_z=0.5, w_entropy=0.8, **LOSSES),
    "zloss-entropy-switch": V["switch-skew"].with_(T=512, d=64, n=16, f=64, alpha=0.5,
                                                   w_importance=0.3, w_z=0.5, w_entropy=0.8),
    "zloss-entropy-sigmoid": V["deepseek-tiny"].with_(w_importance=0.3, w_z=0.5, w_entropy=0.8),
    # fp32 experts (everything fp32: 1e-4)
    "f32-tiny": W["tiny-flat"].with_(**LOSSES),
    "f32-capacity": W["tiny-flat"].with_(T=200, n=6, k=2, d=40, f=24, capacity_factor=0.7,
                                         passthrough=1, bias_var=0.1, **LOSSES),
    "f32-sigmoid-shared": V["deepseek-tiny-f32"].with_(w_importance=0.3),
    # the hierarchical layer: both gate levels, the product-form load
    "hier-noisy": W["hierarchical"].with_(T=256, d=64, n=8 * 16, hier_a=8, hier_b=16, f=64,
                                          **LOSSES),
    "hier-capacity-ragged": W["hierarchical"].with_(T=300, d=40, n=4 * 8, hier_a=4, hier_b=8, f=24,
                                                    capacity_factor=1.0, passthrough=1,
                                                    logit_bias_var=0.2, **LOSSES),
    "hier-nonoise-zloss": W["hierarchical"].with_(T=200, d=64, n=8 * 16, hier_a=8, hier_b=16, f=64,
                                                  noise=0, router_stats=1, w_z=0.5, w_entropy=0.8,
                                                  **LOSSES),
    "hier-f32": W["hierarchical"].with_(T=64, d=32, n=4 * 4, hier_a=4, hier_b=4, f=32,
                                        expert_bf16=0, **LOSSES),
    # 64 experts in routing tiles of 20 rows: the routing kernel's two-rows-per-warp
    # instance, whose thresholds and kept gates the gate's backward reads
    "narrow-routing": W["lm-flat"].with_(T=20000, n=64, k=2, d=32, f=32, **LOSSES),
}

GRAD_KEYS = [("dx", "dx"), ("dWg", "dWg"), ("dbg", "dbg"), ("dWn", "dWn"), ("dW1", "dW1"),
             ("db1", "db1"), ("dW2", "dW2"), ("db2", "db2"), ("dW1s", "dW1s"), ("db1s", "db1s"),
             ("dW2s", "dW2s"), ("db2s", "db2s"), ("dlogits", "dlogits"), ("dWg2", "dWg2"),
             ("dbg2", "dbg2"), ("dWn2", "dWn2")]


def run_backward(w, inp, dy):
    cfg = dataclasses.replace(M.Config.from_workload(w), backward=1)
    dinp = to_dev(inp)
    layer = M.MoELayer(cfg, dinp, torch.device(DEV))
    x = dinp["x"]
    layer.forward_(x)
    layer.grads(intermediates=True)
    g = layer.backward_(x, dy.to(DEV))
    torch.cuda.synchronize()
    out = {k: v.cpu().numpy() for k, v in g.items()}
    fwd = {k: v.cpu() for k, v in layer.outputs().items()}
    return out, fwd


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(orc, name):
    w = CASES[name]
    inp = synth.make_inputs(w)
    dy = synth.make_dy(w)
    got, fwd = run_backward(w, inp, dy)
    assert M.status_bits(fwd["status"]) == 0
    ref_f = orc.forward(w.cfg(), np_inputs(inp))
    # the gradients are whole-batch functions of the routing, so every case
    # uses inputs (seed 0) on which no token has a near tie: checked here
    nt = int((ref_f["near_tie"] < TIE).sum())
    assert nt == 0, f"{name}: {nt} near-tie tokens; the case needs a tie-free seed"
    assert np.array_equal(fwd["topk_idx"].numpy(), ref_f["topk_idx"])
    assert np.array_equal(fwd["counts"].numpy(), ref_f["counts"])
    ref = orc.backward(w.cfg(), np_inputs(inp), dy.numpy())
    tol, tol_g = (1e-2, 5e-3) if w.expert_bf16 else (1e-4, 1e-4)
    assert rel_fro(got["dgate"], ref["dgate"]) < tol_g
    for gk, rk in GRAD_KEYS:
        if gk not in got or rk not in ref:
            continue
        if not np.any(ref[rk]) and not np.any(got[gk]):
            continue
        err = rel_fro(got[gk], ref[rk])
        assert err < tol, (gk, err)
    # experts that received no rows get exactly zero weight gradients
    empty = np.flatnonzero(ref_f["counts"] == 0)
    assert not np.any(got["dW1"][empty]) and not np.any(got["dW2"][empty])


def test_backward_is_deterministic():
    w = CASES["noisy-ragged-capacity"]
    inp = synth.make_inputs(w)
    dy = synth.make_dy(w)
    a, _ = run_backward(w, inp, dy)
    b, _ = run_backward(w, inp, dy)
    for k in a:
        assert np.array_equal(a[k].view(np.uint32), b[k].view(np.uint32)), k


def test_backward_zero_tokens():
    w = CASES["noise-free"].with_(T=0)
    inp = synth.make_inputs(w)
    cfg = dataclasses.replace(M.Config.from_workload(w), backward=1)
    layer = M.MoELayer(cfg, to_dev(inp), torch.device(DEV))
    x = torch.zeros(0, w.d, device=DEV)
    layer.forward_(x)
    g = layer.grads()
    for v in g.values():
        v.fill_(7.0)
    layer.backward_(x, torch.zeros(0, w.d, device=DEV))
    torch.cuda.synchronize()
    for k, v in g.items():
        if k != "dx":
            assert torch.all(v == 0), k


def test_backward_requires_flag():
    w = CASES["noise-free"]
    inp = to_dev(synth.make_inputs(w))
    layer = M.MoELayer(M.Config.from_workload(w), inp, torch.device(DEV))
    with pytest.raises(M.MoEError):
        layer.backward_(inp["x"], torch.zeros_like(inp["x"]))
    # the C ABI refuses too (the flag sizes the workspace and keeps the state)
    from sparsely_gated_mixture_gate_b200 import _lib
    import ctypes as C
    g = layer.grads()
    rc = _lib.load().moe_backward(C.byref(layer._c), M._ptr(inp["x"]), C.byref(layer._gp),
                                  C.byref(layer._ep), M._ptr(inp["x"]), M._ptr(layer.topk_idx),
                                  M._ptr(layer.topk_gate), M._ptr(layer.importance),
                                  M._ptr(layer.load), M._ptr(layer.counts), M._ptr(g["dx"]),
                                  C.byref(layer._mg), M._ptr(layer.ws), layer.ws.numel(),
                                  M._ptr(layer.status), None)
    assert rc == _lib.MOE_EINVAL


@pytest.mark.parametrize("graph", [False, True])
def test_train_host_batches_matches_device_path(graph):
    """The pipelined host-memory training path (direct calls, or one CUDA
    graph per buffer set) gives the same y, losses and dx, bit for bit, as
    forward_ + backward_ on device tensors, batch by batch."""
    w = CASES["noise-free"]
    inp = to_dev(synth.make_inputs(w))
    cfg = dataclasses.replace(M.Config.from_workload(w), backward=1)
    layer = M.MoELayer(cfg, inp, torch.device(DEV))
    xs = [synth.make_inputs(w.with_(seed=s), experts=False)["x"] for s in (1, 2, 3)]
    dys = [synth.make_dy(w.with_(seed=s)) for s in (4, 5, 6)]
    want = []
    for x, dy in zip(xs, dys):
        xd, dyd = x.to(DEV), dy.to(DEV)
        layer.forward_(xd)
        g = layer.backward_(xd, dyd)
        torch.cuda.synchronize()
        want.append((layer.y.cpu().clone(), layer.losses.cpu().clone(), g["dx"].cpu().clone()))
    pin = lambda t: t.contiguous().pin_memory()
    yh = [torch.empty(w.T, w.d).pin_memory() for _ in xs]
    lh = [torch.empty(layer.losses.numel()).pin_memory() for _ in xs]
    dxh = [torch.empty(w.T, w.d).pin_memory() for _ in xs]
    d2h = layer.train_host_batches([pin(x) for x in xs], [pin(d) for d in dys], yh, lh, dxh,
                                   graph=graph)
    d2h.synchronize()
    torch.cuda.synchronize()
    for i, (y, l, dx) in enumerate(want):
        assert torch.equal(yh[i], y), i
        assert torch.equal(lh[i], l), i
        assert torch.equal(dxh[i], dx), i


def test_train_graph_replay_matches_direct():
    """forward + backward replayed from one CUDA graph (MoELayer.train_graph_)
    give the direct calls' outputs and gradients bit for bit."""
    w = CASES["noisy-ragged-capacity"]
    inp = to_dev(synth.make_inputs(w))
    cfg = dataclasses.replace(M.Config.from_workload(w), backward=1)
    layer = M.MoELayer(cfg, inp, torch.device(DEV))
    x = inp["x"]
    dy = synth.make_dy(w).to(DEV)
    layer.forward_(x)
    g = layer.backward_(x, dy)
    torch.cuda.synchronize()
    want = {k: v.clone() for k, v in g.items()}
    want_y = layer.y.clone()
    for v in g.values():
        v.zero_()
    layer.y.zero_()
    layer.noise_seed_(w.seed)  # the same noise key as the direct step
    layer.train_graph_(x, dy)
    torch.cuda.synchronize()
    assert torch.equal(layer.y, want_y)
    for k, v in layer.grads().items():
        assert torch.equal(v, want[k]), k
    layer.release_graph()


def test_backward_uses_the_noise_of_its_forward(orc):
    """A layer's second training step (its forward advanced the noise key to
    seed + 1) gives the gradients the oracle computes with seed + 1: the gate
    backward reads the key its forward drew with."""
    w = CASES["lm-flat-512"]
    inp = synth.make_inputs(w)
    dy = synth.make_dy(w)
    dinp = to_dev(inp)
    cfg = dataclasses.replace(M.Config.from_workload(w), backward=1)
    layer = M.MoELayer(cfg, dinp, torch.device(DEV))
    layer.grads(intermediates=True)
    x = dinp["x"]
    layer.forward_(x)
    layer.backward_(x, dy.to(DEV))
    layer.forward_(x)
    g = layer.backward_(x, dy.to(DEV))
    torch.cuda.synchronize()
    assert M.status_bits(layer.status) == 0
    w1 = w.with_(seed=w.seed + 1)
    ref_f = orc.forward(w1.cfg(), np_inputs(inp))
    assert int((ref_f["near_tie"] < TIE).sum()) == 0
    assert np.array_equal(layer.topk_idx.cpu().numpy(), ref_f["topk_idx"])
    ref = orc.backward(w1.cfg(), np_inputs(inp), dy.numpy())
    assert rel_fro(g["dgate"].cpu().numpy(), ref["dgate"]) < 5e-3
    for gk, rk in (("dWg", "dWg"), ("dWn", "dWn"), ("dx", "dx")):
        assert rel_fro(g[gk].cpu().numpy(), ref[rk]) < 1e-2, gk
