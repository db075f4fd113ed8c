"""GPU parity: every stage of the CUDA path (through the C ABI) against the
oracle, element by element, on the same seeded inputs.

Tolerances: expert ids and the permutation bit-exact; gates, load,
importance and losses fp32 within 1e-5 relative; layer output within 1e-4
relative Frobenius for fp32 experts and 2e-2 for bf16 experts.  A token whose
kept logits come closer than 1e-5 (a near tie) is excluded together with
every expert it reaches on either side, and nothing is skipped: the rest of
the batch is compared (see parity_util).
"""
import numpy as np
import pytest
import torch

from parity_util import (TIE, assert_rel, check_routing, check_stats, rel_fro, touched_experts,
                         y_rows_to_compare)
from sparsely_gated_mixture_gate_b200 import build, synth
from sparsely_gated_mixture_gate_b200 import moe as M

pytestmark = pytest.mark.gpu
DEV = "cuda"


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


# ------------------------------------------------------------------ workloads
W = synth.WORKLOADS
V = synth.VARIANTS
SMALL = {
    "tiny-flat": W["tiny-flat"],
    "tiny-bias": V["tiny-bias"],
    "lm-flat-512": W["lm-flat"].with_(T=512),
    "lm-k1-nonoise": W["lm-flat"].with_(T=300, k=1, noise=0, n=96, d=64, f=64),
    "many-small": W["many-expert"].with_(T=384, n=1000, d=128, f=64),
    "switch-small": W["switch-top1"].with_(T=2048, d=256, n=64, f=512),
    "switch-skew-small": V["switch-skew"].with_(T=2048, d=256, n=64, f=512),
    "hier-small": W["hierarchical"].with_(T=256, d=64, n=8 * 16, hier_a=8, hier_b=16, f=128),
    "kn-equal": W["tiny-flat"].with_(T=33, n=3, k=3, d=16, f=24),
    "k8-n64": W["lm-flat"].with_(T=200, n=64, k=8, d=64, f=64),
    "flat-n8192": W["many-expert"].with_(T=96, n=8192, d=64, f=16),
    "one-token": W["lm-flat"].with_(T=1, n=16, k=2, d=64, f=64),
    "bf16-narrow": W["lm-flat"].with_(T=100, n=5, k=2, d=40, f=24),
    "hier-nonoise": W["hierarchical"].with_(T=256, d=64, n=8 * 16, hier_a=8, hier_b=16, f=128, noise=0),
    # sigmoid router with selection bias and shared expert, and its parts
    "deepseek-tiny": V["deepseek-tiny"],
    "deepseek-tiny-f32": V["deepseek-tiny-f32"],
    "deepseek-noshared": V["deepseek-tiny"].with_(shared_expert=0),
    "deepseek-512": V["deepseek-flat"].with_(T=512),
    "shared-noisy": W["lm-flat"].with_(T=200, n=32, k=2, d=64, f=64, shared_expert=1),
    "shared-passthrough": V["switch-skew"].with_(T=1024, d=128, n=16, f=128, shared_expert=1),
    # router z-loss and entropy (losses[8], [9]) on each kind of gate
    "stats-noisy": W["lm-flat"].with_(T=300, n=40, d=64, f=64, router_stats=1),
    "stats-switch": W["switch-top1"].with_(T=500, d=128, n=32, f=64, router_stats=1),
    "stats-sigmoid": V["deepseek-tiny"].with_(router_stats=1),
    "stats-hier": W["hierarchical"].with_(T=200, d=64, n=8 * 16, hier_a=8, hier_b=16, f=64,
                                          router_stats=1),
    # rows of at most 128 experts in tiles of 16+ rows: the routing kernel's
    # several-rows-per-warp instance (4 rows a warp at 64 experts and tiles of
    # 32+ rows, else 2), on each router
    "narrow-noisy-64": W["lm-flat"].with_(T=40000, n=64, k=2, d=32, f=32),
    "narrow-switch-64": W["switch-top1"].with_(T=40000, d=32, n=64, f=32),
    "narrow-switch-128-stats": W["switch-top1"].with_(T=40000, d=32, n=128, f=32, router_stats=1),
    "narrow-sigmoid-100": V["deepseek-tiny"].with_(T=20000, n=100, k=4, d=32, f=32),
    "narrow-noisy-96-stats": W["lm-flat"].with_(T=20000, n=96, k=3, d=32, f=32, router_stats=1),
}


GP = [pytest.param(0, id="fp32fma"), pytest.param(1, id="tf32x3")]


@pytest.mark.parametrize("gp", GP)
@pytest.mark.parametrize("name", list(SMALL))
def test_gate_matches_oracle(orc, name, gp):
    w = SMALL[name].with_(gate_precision=gp)
    inp = synth.make_inputs(w, experts=False)
    cfg = M.Config.from_workload(w)
    out = M.gate(cfg, inp["x"].to(DEV), to_dev(inp))
    torch.cuda.synchronize()
    assert M.status_bits(out["status"]) == 0
    ref = orc.gate_batch(w.cfg(), np_inputs(inp))
    idx = out["topk_idx"].cpu().numpy()
    tie = check_routing(idx, out["topk_gate"].cpu().numpy(), ref, name)
    u = ~touched_experts(w, tie, idx, ref["topk_idx"])
    load = out["load"].cpu().numpy()
    assert_rel(load[u], ref["load"][u], 1e-5, 1e-6 * w.T, f"{name} load")
    if w.noise and not w.hier_a:  # a near-tie swap moves the smoothed load by O(gap)
        assert_rel(load, ref["load"], 1e-5, 1e-6 * w.T, f"{name} load (all experts)")
    if w.router == 1:
        assert_rel(out["prob_sum"].cpu().numpy(), ref["prob_sum"], 1e-5, 1e-7 * w.T, f"{name} prob_sum")


# ------------------------------------------------------------------ dispatch (stage-wise)
DISPATCH = [
    # T, n, k, capacity factor, skew, invalid fraction, d
    (64, 8, 2, 0.0, 0.0, 0.0, 32),
    (1000, 37, 3, 0.0, 1.0, 0.0, 64),
    (1000, 37, 3, 1.0, 1.0, 0.0, 64),
    (4096, 256, 4, 0.0, 0.5, 0.0, 512),
    (777, 5, 5, 0.0, 0.0, 0.0, 16),
    (500, 1, 1, 0.0, 0.0, 0.0, 8),
    (0, 8, 2, 0.0, 0.0, 0.0, 32),
    (300, 16, 2, 0.0, 0.0, 0.05, 32),
    (32768, 128, 1, 1.25, 0.7, 0.0, 128),
    (65536, 4096, 4, 0.0, 1.1, 0.0, 64),
    (70000, 8192, 4, 0.5, 0.3, 0.0, 8),
]


@pytest.mark.parametrize("T,n,k,cf,skew,inv,d", DISPATCH)
def test_dispatch_matches_oracle(orc, T, n, k, cf, skew, inv, d):
    idx = synth.random_routing(T, k, n, device=DEV, skew=skew, invalid_frac=inv, seed=T + n).cpu()
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(5))
    cfg = M.Config(T=T, d=d, n=n, k=k, f=8, capacity_factor=cf)
    out = M.dispatch(cfg, x.to(DEV), idx.to(DEV))
    torch.cuda.synchronize()
    C = orc.capacity(T, k, n, cf)
    ref = orc.dispatch(idx.numpy(), n, C)
    assert np.array_equal(out["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(out["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(out["row_of"].cpu().numpy(), ref["row_of"])
    R = int(ref["offsets"][-1])
    assert np.array_equal(out["perm_token"][:R].cpu().numpy(), ref["perm_token"])
    xp = out["x_perm"][:R].cpu()
    want = x[torch.from_numpy(ref["perm_token"]).long()].bfloat16()
    assert torch.equal(xp.view(torch.int16), want.view(torch.int16))
    st = M.status_bits(out["status"])
    assert st == (M._lib.STATUS_BAD_INDEX if ref["n_invalid"] else 0)


# ------------------------------------------------------------------ combine (stage-wise)
@pytest.mark.parametrize("bf16", [True, False])
@pytest.mark.parametrize("passthrough", [0, 1])
def test_combine_matches_oracle(orc, bf16, passthrough):
    T, n, k, d = 1500, 12, 3, 96
    idx = synth.random_routing(T, k, n, skew=1.0, seed=3)
    C = 300
    ref_d = orc.dispatch(idx.numpy(), n, C)
    R = int(ref_d["offsets"][-1])
    g = torch.Generator().manual_seed(9)
    Y = torch.randn(max(T * k, 1), d, generator=g)
    Y = Y.bfloat16() if bf16 else Y
    gate = torch.rand(T, k, generator=g)
    x = torch.randn(T, d, generator=g)
    cfg = M.Config(T=T, d=d, n=n, k=k, f=8, expert_bf16=int(bf16), passthrough=passthrough)
    out = M.combine(cfg, Y.to(DEV), gate.to(DEV), torch.from_numpy(ref_d["row_of"]).to(DEV), x.to(DEV))
    torch.cuda.synchronize()
    want = orc.combine(Y[:max(R, 1)].double().numpy(), gate.numpy(), ref_d["row_of"], x.numpy(),
                       passthrough=bool(passthrough))
    assert_rel(out["y"].cpu().numpy(), want, 1e-6, 1e-6, "combine")
    assert (ref_d["row_of"] < 0).all(axis=1).any()  # the case covers fully dropped tokens


# ------------------------------------------------------------------ experts (stage-wise)
EXPERT = [
    # d, f, per-expert row counts, bf16
    (64, 128, [0, 1, 127, 128, 129, 300], True),
    (512, 1024, [200, 5, 256], True),
    (72, 136, [10, 140, 0, 3], True),
    (256, 64, [130] * 3 + [1], True),
    (32, 64, [3, 0, 17, 40], False),
    (72, 40, [5, 1, 0, 9], False),
]


def _expert_case(d, f, counts, bf16, seed=0):
    n = len(counts)
    S = sum(counts)
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if bf16 else torch.float32
    xp = torch.randn(max(S, 1), d, generator=g).to(dt)
    W1 = (torch.randn(n, f, d, generator=g) / d ** 0.5).to(dt)
    W2 = (torch.randn(n, d, f, generator=g) / f ** 0.5).to(dt)
    b1 = torch.randn(n, f, generator=g) * 0.1
    b2 = torch.randn(n, d, generator=g) * 0.1
    offsets = torch.tensor([0] + list(np.cumsum(counts)), dtype=torch.int32)
    return xp, W1, b1, W2, b2, offsets


def _bits(t):
    return synth.bf16_bits(t) if t.dtype == torch.bfloat16 else t.numpy()


@pytest.mark.parametrize("d,f,counts,bf16", EXPERT)
def test_expert_ffn_matches_oracle(orc, d, f, counts, bf16):
    n, S = len(counts), sum(counts)
    xp, W1, b1, W2, b2, offsets = _expert_case(d, f, counts, bf16)
    # T*k must cover the rows: use k = 1 and T = S
    cfg = M.Config(T=max(S, 1), d=d, n=n, k=1, f=f, expert_bf16=int(bf16))
    xpad = torch.zeros(max(S, 1), d, dtype=xp.dtype)
    xpad[:S] = xp[:S]
    out = M.expert_ffn(cfg, xpad.to(DEV), offsets.to(DEV),
                       dict(W1=W1.to(DEV), b1=b1.to(DEV), W2=W2.to(DEV), b2=b2.to(DEV)))
    torch.cuda.synchronize()
    assert M.status_bits(out["status"]) == 0
    got = out["y_perm"][:S].float().cpu().numpy()
    want = np.zeros((S, d))
    for e in range(n):
        for r in range(int(offsets[e]), int(offsets[e + 1])):
            want[r] = orc.expert_row(xp[r].float().numpy(), _bits(W1[e]), b1[e].numpy(), _bits(W2[e]),
                                     b2[e].numpy(), bf16=bf16)
    if S:
        tol = 1e-2 if bf16 else 1e-5
        assert rel_fro(got, want) < tol, rel_fro(got, want)
        for r in range(S):  # every row individually, so a masked/misplaced row cannot hide
            assert rel_fro(got[r], want[r]) < (3e-2 if bf16 else 1e-5), r


def test_expert_ffn_lm_size_sampled(orc):
    """LM-shaped sizes: 256 experts of 512 -> 1024 -> 512, ragged ~128 rows
    each; rows sampled across experts and tile positions."""
    n, d, f = 256, 512, 1024
    g = torch.Generator().manual_seed(11)
    counts = torch.poisson(torch.full((n,), 128.0), generator=g).int().tolist()
    counts[3] = 0
    counts[7] = 1
    counts[9] = 129
    xp, W1, b1, W2, b2, offsets = _expert_case(d, f, counts, True, seed=1)
    S = sum(counts)
    cfg = M.Config(T=S, d=d, n=n, k=1, f=f)
    out = M.expert_ffn(cfg, xp.to(DEV), offsets.to(DEV),
                       dict(W1=W1.to(DEV), b1=b1.to(DEV), W2=W2.to(DEV), b2=b2.to(DEV)))
    torch.cuda.synchronize()
    assert M.status_bits(out["status"]) == 0
    got = out["y_perm"].float().cpu().numpy()
    rng = np.random.default_rng(0)
    rows = sorted(set(rng.integers(0, S, 150).tolist()) | {int(offsets[8]), int(offsets[10]) - 1,
                                                              int(offsets[10]) + 128})
    off = offsets.numpy()
    for r in rows:
        e = int(np.searchsorted(off, r, side="right") - 1)
        want = orc.expert_row(xp[r].float().numpy(), _bits(W1[e]), b1[e].numpy(), _bits(W2[e]),
                              b2[e].numpy(), bf16=True)
        assert rel_fro(got[r], want) < 3e-2, (r, e)


SKEWED = [
    # one expert holds almost every row: its GEMM2 tiles land on CTAs that have
    # no GEMM1 tiles and wait for the counters of M-blocks computed elsewhere
    (256, 1024, [4000, 0, 3, 0]),
    # GEMM2 with more N-blocks than GEMM1, ragged tails
    (768, 256, [1, 2000, 0, 900, 5]),
    # fewer than 192 rows per expert on average, so GEMM2 tiles are interleaved
    # a few waves behind GEMM1's; one expert spans 313 M-blocks, more than
    # that lag, so its GEMM2 tiles wait on M-blocks finished moments before
    (128, 256, [40000] + [40] * 299),
]


@pytest.mark.parametrize("d,f,counts", SKEWED)
def test_expert_ffn_skewed_sampled(orc, d, f, counts):
    xp, W1, b1, W2, b2, offsets = _expert_case(d, f, counts, True, seed=5)
    n, S = len(counts), sum(counts)
    cfg = M.Config(T=S, d=d, n=n, k=1, f=f)
    out = M.expert_ffn(cfg, xp.to(DEV), offsets.to(DEV),
                       dict(W1=W1.to(DEV), b1=b1.to(DEV), W2=W2.to(DEV), b2=b2.to(DEV)))
    torch.cuda.synchronize()
    assert M.status_bits(out["status"]) == 0
    got = out["y_perm"].float().cpu().numpy()
    off = offsets.numpy()
    rng = np.random.default_rng(1)
    rows = set(rng.integers(0, S, 120).tolist())
    for e in range(n):  # first and last row of every expert and of every 128-row block
        for r0 in range(int(off[e]), int(off[e + 1]), 128):
            rows |= {r0, min(r0 + 127, int(off[e + 1]) - 1)}
    for r in sorted(rows):
        e = int(np.searchsorted(off, r, side="right") - 1)
        want = orc.expert_row(xp[r].float().numpy(), _bits(W1[e]), b1[e].numpy(), _bits(W2[e]),
                              b2[e].numpy(), bf16=True)
        assert rel_fro(got[r], want) < 3e-2, (r, e)


# ------------------------------------------------------------------ whole layer
def run_layer(w, inp):
    cfg = M.Config.from_workload(w)
    out = M.forward(cfg, inp["x"].to(DEV), to_dev(inp))
    torch.cuda.synchronize()
    return {k: v.cpu() for k, v in out.items()}


@pytest.mark.parametrize("gp", GP)
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_matches_oracle(orc, name, gp):
    w = SMALL[name].with_(gate_precision=gp)
    inp = synth.make_inputs(w)
    out = run_layer(w, inp)
    assert M.status_bits(out["status"]) == 0
    ref = orc.forward(w.cfg(), np_inputs(inp))
    o = {key: v.numpy() for key, v in out.items()}
    nt, nx = check_stats(orc, w, o, ref, name)
    tie = ref["near_tie"] < TIE
    touched = touched_experts(w, tie, o["topk_idx"], ref["topk_idx"])
    rows = y_rows_to_compare(w, tie, touched, o["topk_idx"], ref["topk_idx"])
    if nt:
        print(f"{name}: {nt} near-tie tokens, {nx} experts excluded, {rows.sum()} of {w.T} rows of y")
    if w.T:
        assert rows.sum() >= w.T // 2
    tol = 2e-2 if w.expert_bf16 else 1e-4
    err = rel_fro(o["y"][rows], ref["y"][rows])
    assert err < tol, err


@pytest.mark.parametrize("n,T,k", [(256, 8192, 8), (7, 1000, 3), (1, 5, 1), (300, 0, 2)])
def test_sel_bias_update_matches_oracle(orc, n, T, k):
    rng = np.random.default_rng(n + T)
    counts = rng.integers(0, 2 * max(T * k // max(n, 1), 1) + 1, n).astype(np.int32)
    if n > 1:
        counts[0] = (T * k) // n if (T * k) % n == 0 else counts[0]  # one exactly at the average
    bias = rng.normal(0, 1, n).astype(np.float32)
    gamma = 1e-3
    want = orc.sel_bias_update(counts, T, k, gamma, bias)
    cfg = M.Config(T=T, d=8, n=n, k=k, f=8, router=2, noise=0)
    b = torch.from_numpy(bias.copy()).to(DEV)
    M.sel_bias_update(cfg, torch.from_numpy(counts).to(DEV), gamma, b)
    torch.cuda.synchronize()
    assert np.array_equal(b.cpu().numpy().view(np.uint32), want.view(np.uint32))


def test_forward_is_deterministic():
    w = SMALL["lm-flat-512"]
    inp = synth.make_inputs(w)
    a = run_layer(w, inp)
    b = run_layer(w, inp)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_forward_zero_tokens():
    w = SMALL["tiny-flat"].with_(T=0)
    inp = synth.make_inputs(w)
    out = run_layer(w, inp)
    assert out["y"].numel() == 0
    assert torch.all(out["counts"] == 0)
    assert torch.all(out["losses"] == 0)


@pytest.mark.parametrize("w", [SMALL["lm-flat-512"], W["many-expert"].with_(T=64, d=64, f=64),
                               W["many-expert"].with_(T=64, d=64, f=64, noise=0)],
                         ids=["lm-flat-512", "n4096", "n4096-nonoise"])
def test_nonfinite_input_sets_status(w):
    inp = synth.make_inputs(w)
    inp["x"][5, 3] = float("nan")
    out = run_layer(w, inp)
    assert M.status_bits(out["status"]) & M._lib.STATUS_NONFINITE


def test_bad_expert_id_sets_status_and_is_ignored(orc):
    idx = torch.tensor([[0, 9], [1, -2], [2, 0]], dtype=torch.int32)
    cfg = M.Config(T=3, d=8, n=3, k=2, f=8)
    out = M.dispatch(cfg, torch.ones(3, 8, device=DEV), idx.to(DEV))
    torch.cuda.synchronize()
    assert M.status_bits(out["status"]) == M._lib.STATUS_BAD_INDEX
    ref = orc.dispatch(idx.numpy(), 3, 2**62)
    assert np.array_equal(out["row_of"].cpu().numpy(), ref["row_of"])


# ------------------------------------------------------------------ balance losses (stage-wise)
@pytest.mark.parametrize("router,T,n,k,cf", [(0, 3000, 64, 4, 0.0), (0, 5000, 1000, 2, 1.0),
                                             (1, 4096, 128, 1, 1.25), (0, 0, 16, 2, 0.0)])
def test_balance_losses_matches_oracle(orc, router, T, n, k, cf):
    idx = synth.random_routing(T, k, n, skew=0.9, seed=n)
    g = torch.Generator().manual_seed(4)
    gate = torch.rand(T, k, generator=g)
    gate = gate / gate.sum(1, keepdim=True) if T else gate
    C = orc.capacity(T, k, n, cf)
    counts = orc.dispatch(idx.numpy(), n, C)["counts"]
    load = (torch.rand(n, generator=g) * T / n * 2).numpy().astype(np.float32)
    psum = (torch.rand(n, generator=g) * T / n).numpy().astype(np.float32) if router else None
    cfg = M.Config(T=T, d=8, n=n, k=k, f=8, router=router, noise=0 if router else 1, capacity_factor=cf)
    out = M.balance_losses(cfg, idx.to(DEV), gate.to(DEV), torch.from_numpy(counts).to(DEV),
                           torch.from_numpy(load).to(DEV),
                           torch.from_numpy(psum).to(DEV) if psum is not None else None)
    torch.cuda.synchronize()
    imp_ref, losses_ref = orc.balance(n, idx.numpy(), gate.double().numpy(), counts, load.astype(np.float64),
                                      None if psum is None else psum.astype(np.float64), C, router)
    assert_rel(out["importance"].cpu().numpy(), imp_ref, 1e-5, 1e-6, "importance")
    losses = out["losses"].cpu().numpy()
    assert_rel(losses[:8], losses_ref, 1e-5, 1e-7, "losses")
    assert np.all(losses[8:] == 0.0)  # router statistics come from moe_forward only


def test_pipelined_host_batches_match_device_calls():
    """The overlapped host-memory path returns, batch by batch, exactly what
    the device-resident call computes (double buffers never mix batches)."""
    w = SMALL["lm-flat-512"]
    inp = synth.make_inputs(w)
    cfg = M.Config.from_workload(w)
    layer = M.MoELayer(cfg, to_dev(inp), torch.device(DEV))
    g = torch.Generator().manual_seed(21)
    xs = [torch.randn(w.T, w.d, generator=g).pin_memory() for _ in range(5)]
    ys = [torch.empty(w.T, w.d).pin_memory() for _ in range(5)]
    ls = [torch.empty(layer.losses.numel()).pin_memory() for _ in range(5)]
    layer.forward_host_batches(xs, ys, ls)
    torch.cuda.synchronize()
    for i in range(5):
        layer.noise_seed_(w.seed + i)  # batch i drew its noise with key seed + i
        layer.forward_(xs[i].to(DEV))
        torch.cuda.synchronize()
        assert torch.equal(ys[i], layer.y.cpu()), i
        assert torch.equal(ls[i], layer.losses.cpu()), i


def test_forward_graph_replay_matches_direct():
    """The CUDA-graph replay of moe_forward (MoELayer.forward_graph_) gives the
    direct call's outputs bit for bit, and follows new contents of the same
    input buffer."""
    for name in ("lm-flat-512", "deepseek-tiny", "switch-skew-small"):
        w = SMALL[name]
        inp = synth.make_inputs(w)
        dinp = to_dev(inp)
        layer = M.MoELayer(M.Config.from_workload(w), dinp, torch.device(DEV))
        x = dinp["x"]
        x2 = synth.make_inputs(w.with_(seed=w.seed + 7), experts=False)["x"].to(DEV)
        outs = []
        for step, src in enumerate((x.clone(), x2)):
            x.copy_(src)
            layer.noise_seed_(w.seed + step)
            layer.forward_(x)
            torch.cuda.synchronize()
            want = {k: v.clone() for k, v in layer.outputs().items()}
            layer.y.zero_()
            layer.noise_seed_(w.seed + step)
            layer.forward_graph_(x)
            torch.cuda.synchronize()
            got = layer.outputs()
            for k in ("y", "topk_idx", "topk_gate", "importance", "load", "counts", "losses"):
                assert torch.equal(got[k], want[k]), (name, k)
            outs.append(want["y"])
        assert not torch.equal(outs[0], outs[1])
        layer.release_graph()


def test_forward_host_batches_with_graphs_matches_direct():
    """The pipelined host path with a CUDA graph per buffer set gives each
    batch's y and losses bit for bit as direct device calls."""
    w = SMALL["lm-flat-512"]
    dinp = to_dev(synth.make_inputs(w))
    layer = M.MoELayer(M.Config.from_workload(w), dinp, torch.device(DEV))
    xs = [synth.make_inputs(w.with_(seed=s), experts=False)["x"] for s in (11, 12, 13)]
    want = []
    for x in xs:
        layer.forward_(x.to(DEV))
        torch.cuda.synchronize()
        want.append((layer.y.cpu().clone(), layer.losses.cpu().clone()))
    yh = [torch.empty(w.T, w.d).pin_memory() for _ in xs]
    lh = [torch.empty(layer.losses.numel()).pin_memory() for _ in xs]
    layer.noise_seed_(w.seed)  # the same keys as the direct calls above
    d2h = layer.forward_host_batches([x.contiguous().pin_memory() for x in xs], yh, lh, graph=True)
    d2h.synchronize()
    torch.cuda.synchronize()
    for i, (y, l) in enumerate(want):
        assert torch.equal(yh[i], y), i
        assert torch.equal(lh[i], l), i
    layer.release_graph()


def test_noise_is_redrawn_every_step(orc):
    """The noisy gate draws new noise every time it runs ("極大規模神經網路：
    稀疏門控專家混合層", Noisy Top-K 門控): step s of a layer uses noise key
    seed + s, whether the step is a direct call or a CUDA graph replay, and
    equals, bit for bit, a fresh layer configured with that seed; the oracle
    with that seed gives the same routing."""
    w = SMALL["lm-flat-512"]
    inp = synth.make_inputs(w)
    dinp = to_dev(inp)
    layer = M.MoELayer(M.Config.from_workload(w), dinp, torch.device(DEV))
    x = dinp["x"]
    keys = ("y", "topk_idx", "topk_gate", "importance", "load", "counts", "losses")
    steps = []
    for call in (layer.forward_, layer.forward_graph_, layer.forward_graph_, layer.forward_):
        call(x)
        torch.cuda.synchronize()
        steps.append({k: v.cpu().clone() for k, v in layer.outputs().items()})
    layer.release_graph()
    for s, got in enumerate(steps):
        fresh = run_layer(w.with_(seed=w.seed + s), inp)
        for k in keys:
            assert torch.equal(got[k], fresh[k]), (s, k)
    assert not torch.equal(steps[1]["topk_gate"], steps[2]["topk_gate"])
    assert not torch.equal(steps[1]["load"], steps[2]["load"])
    ref = orc.gate_batch(w.with_(seed=w.seed + 2).cfg(), np_inputs(synth.make_inputs(w, experts=False)))
    check_routing(steps[2]["topk_idx"].numpy(), steps[2]["topk_gate"].numpy(), ref, "step 2")
    # with resampling off every step draws with cfg.seed
    fixed = M.MoELayer(M.Config.from_workload(w), dinp, torch.device(DEV), resample_noise=False)
    fixed.forward_(x)
    fixed.forward_(x)
    torch.cuda.synchronize()
    assert torch.equal(fixed.y.cpu(), steps[0]["y"])


@pytest.mark.parametrize("name", ["lm-flat-512", "hier-small"])
def test_shard_with_token_base_draws_the_batch_noise(name):
    """A data-parallel shard of a batch (its tokens, token_base = the index
    of its first token) routes exactly as those tokens do in the whole batch:
    the noise counter runs over the batch's token indices."""
    import dataclasses
    w = SMALL[name]
    inp = to_dev(synth.make_inputs(w, experts=False))
    x = inp["x"]
    whole = M.gate(M.Config.from_workload(w), x, inp)
    h = w.T // 2 + 3
    cfg = dataclasses.replace(M.Config.from_workload(w.with_(T=w.T - h)), token_base=h)
    part = M.gate(cfg, x[h:].contiguous(), inp)
    torch.cuda.synchronize()
    assert torch.equal(part["topk_idx"], whole["topk_idx"][h:])
    assert torch.equal(part["topk_gate"], whole["topk_gate"][h:])
    # and without the base the shard draws other noise
    other = M.gate(M.Config.from_workload(w.with_(T=w.T - h)), x[h:].contiguous(), inp)
    torch.cuda.synchronize()
    assert not torch.equal(other["topk_gate"], whole["topk_gate"][h:])


def test_wide_gate_tiling_routes_alike():
    """Every logit is one fp32 FMA chain over d in order, whatever column tile
    of the gate GEMM it falls in, and the routing kernel's result does not
    depend on how many columns share a row.  Run the same 2044 experts as a
    gate of 2044 columns and of 2048, where the four extra experts carry a
    bias of -1e30 (never kept, never a threshold): the routing, the gates and
    the smoothed Load of the 2044 must agree exactly."""
    w = W["many-expert"].with_(T=1000, d=256, n=2048, k=4)
    inp = to_dev(synth.make_inputs(w, experts=False))
    inp["bg"][2044:] = -1e30
    narrow = {k: (v[..., :2044].contiguous() if k in ("Wg", "Wn", "bg") else v)
              for k, v in inp.items()}
    wide = M.gate(M.Config.from_workload(w), inp["x"], inp)
    own = M.gate(M.Config.from_workload(w.with_(n=2044)), inp["x"], narrow)
    torch.cuda.synchronize()
    assert M.status_bits(wide["status"]) == 0 and M.status_bits(own["status"]) == 0
    assert int(wide["topk_idx"].max()) < 2044
    assert torch.equal(wide["topk_idx"], own["topk_idx"])
    assert torch.equal(wide["topk_gate"], own["topk_gate"])
    assert torch.equal(wide["load"][:2044], own["load"])
