"""Pins of the oracle's dispatch, expert and whole-layer results (CPU only).

Hand-computed cases, numpy / torch library routines (stable argsort,
bincount, matmul of a plain MLP), a dense soft-MoE brute force over every
expert, invariants the pages imply and the zero-noise limit of the load.
"""
import math

import numpy as np
import pytest
import torch

from sparsely_gated_mixture_gate_b200 import synth


# ------------------------------------------------------------------ dispatch
def test_dispatch_hand_capacity(orc):
    """3 tokens, all on expert 0, capacity 1: only token 0 is kept."""
    idx = np.array([[0], [0], [0]], np.int32)
    r = orc.dispatch(idx, 2, 1)
    assert list(r["counts"]) == [3, 0]
    assert list(r["offsets"]) == [0, 1, 1]
    assert list(r["row_of"].ravel()) == [0, -1, -1]
    assert list(r["perm_token"]) == [0]


def test_dispatch_matches_stable_argsort(orc):
    rng = np.random.default_rng(8)
    for trial in range(20):
        T, n = int(rng.integers(0, 300)), int(rng.integers(1, 50))
        k = int(rng.integers(1, min(n, 6) + 1))
        idx = np.stack([rng.permutation(n)[:k] for _ in range(T)]).astype(np.int32).reshape(T, k)
        C = int(rng.integers(1, 12)) if trial % 2 else 2**62
        r = orc.dispatch(idx, n, C)
        flat = idx.ravel()
        assert np.array_equal(r["counts"], np.bincount(flat, minlength=n))
        order = np.argsort(flat, kind="stable")          # expert-major, token order inside
        kept_rows = []
        for e in range(n):
            pos = order[flat[order] == e][: min(C, (flat == e).sum())]
            kept_rows.extend(pos.tolist())
        assert np.array_equal(r["perm_token"] * k + r["perm_slot"], np.array(kept_rows, dtype=np.int64))
        # row_of is the inverse map on kept slots; every kept row used once
        ro = r["row_of"].ravel()
        kept = ro >= 0
        assert sorted(ro[kept].tolist()) == list(range(int(r["offsets"][-1])))
        assert np.array_equal(r["perm_token"][ro[kept]] * k + r["perm_slot"][ro[kept]], np.nonzero(kept)[0])
        assert kept.sum() == np.minimum(r["counts"].astype(np.int64), C).sum()


def test_dispatch_ignores_invalid_ids(orc):
    idx = np.array([[0, -1], [5, 1], [1, 0]], np.int32)
    r = orc.dispatch(idx, 2, 2**62)
    assert r["n_invalid"] == 2
    assert list(r["counts"]) == [2, 2]
    assert list(r["row_of"].ravel()) == [0, -1, -1, 2, 3, 1]


# ------------------------------------------------------------------ expert
def _mlp_numpy(x, W1, b1, W2, b2):
    return np.maximum(x @ W1.T + b1, 0.0) @ W2.T + b2


def test_expert_fp32_is_plain_mlp(orc):
    rng = np.random.default_rng(9)
    d, f = 12, 20
    x = rng.standard_normal(d).astype(np.float32)
    W1 = rng.standard_normal((f, d)).astype(np.float32)
    W2 = rng.standard_normal((d, f)).astype(np.float32)
    b1 = rng.standard_normal(f).astype(np.float32)
    b2 = rng.standard_normal(d).astype(np.float32)
    y = orc.expert_row(x, W1, b1, W2, b2, bf16=False)
    want = _mlp_numpy(*(a.astype(np.float64) for a in (x, W1, b1, W2, b2)))
    assert y == pytest.approx(want, rel=1e-12, abs=1e-12)


def test_expert_bf16_rounds_activations(orc):
    rng = np.random.default_rng(10)
    d, f = 16, 32
    x = torch.from_numpy(rng.standard_normal(d).astype(np.float32))
    W1 = torch.from_numpy(rng.standard_normal((f, d)).astype(np.float32)).bfloat16()
    W2 = torch.from_numpy(rng.standard_normal((d, f)).astype(np.float32)).bfloat16()
    b1 = torch.from_numpy(rng.standard_normal(f).astype(np.float32))
    b2 = torch.from_numpy(rng.standard_normal(d).astype(np.float32))
    y = orc.expert_row(x.numpy(), synth.bf16_bits(W1), b1.numpy(), synth.bf16_bits(W2), b2.numpy(), bf16=True)
    # library: torch's bf16 rounding of x and of the hidden layer, fp64 matmuls
    xb = x.bfloat16().double()
    h = torch.relu(xb @ W1.double().T + b1.double()).float().bfloat16().double()
    want = (h @ W2.double().T + b2.double()).numpy()
    assert y == pytest.approx(want, rel=1e-12, abs=1e-12)


# ------------------------------------------------------------------ whole layer
def _np_inputs(inp):
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif v.dtype == torch.bfloat16:
            out[k] = synth.bf16_bits(v)
        else:
            out[k] = v.cpu().numpy()
    return out


def _fwd(orc, w, inp):
    return orc.forward(w.cfg(), _np_inputs(inp))


@pytest.fixture(scope="module")
def tiny():
    w = synth.WORKLOADS["tiny-flat"]
    return w, synth.make_inputs(w)


def test_tiny_invariants(orc, tiny):
    w, inp = tiny
    o = _fwd(orc, w, inp)
    T, k, n = w.T, w.k, w.n
    assert o["topk_gate"].sum(1) == pytest.approx(np.ones(T), abs=1e-15 * k)
    assert o["importance"].sum() == pytest.approx(T, rel=1e-13)
    assert o["counts"].sum() == T * k
    for t in range(T):
        assert len(set(o["topk_idx"][t].tolist())) == k
    assert o["losses"][0] == pytest.approx(0.1 * o["losses"][5])
    assert o["losses"][1] == pytest.approx(0.1 * o["losses"][6])
    assert o["losses"][4] == 0.0 and o["losses"][7] == 0.0
    # load is a sum of probabilities: bounded by T per expert, positive
    assert np.all(o["load"] > 0) and np.all(o["load"] <= T)


def _dense_soft_moe(inp, gates_dense, bf16):
    """sum_i G_i E_i(x) over EVERY expert (the soft-routing form), by library
    matmuls; unselected experts carry G_i = 0."""
    x = inp["x"].double()
    W1, W2 = inp["W1"], inp["W2"]
    if bf16:
        x = inp["x"].bfloat16().double()
    y = torch.zeros_like(x)
    for e in range(W1.shape[0]):
        h = torch.relu(x @ W1[e].double().T + inp["b1"][e].double())
        if bf16:
            h = h.float().bfloat16().double()
        y += torch.from_numpy(gates_dense[:, e])[:, None] * (h @ W2[e].double().T + inp["b2"][e].double())
    return y.numpy()


@pytest.mark.parametrize("name", ["tiny-flat", "tiny-bias"])
def test_sparse_equals_dense_bruteforce(orc, name):
    w = synth.WORKLOADS.get(name) or synth.VARIANTS[name]
    inp = synth.make_inputs(w)
    o = _fwd(orc, w, inp)
    G = np.zeros((w.T, w.n))
    for t in range(w.T):
        G[t, o["topk_idx"][t]] = o["topk_gate"][t]
    want = _dense_soft_moe(inp, G, bf16=False)
    np.testing.assert_allclose(o["y"], want, rtol=1e-9, atol=1e-9)


def test_sparse_equals_dense_bruteforce_bf16(orc):
    w = synth.WORKLOADS["lm-flat"].with_(T=48, n=16, k=3, d=64, f=128)
    inp = synth.make_inputs(w)
    o = _fwd(orc, w, inp)
    G = np.zeros((w.T, w.n))
    for t in range(w.T):
        G[t, o["topk_idx"][t]] = o["topk_gate"][t]
    want = _dense_soft_moe(inp, G, bf16=True)
    np.testing.assert_allclose(o["y"], want, rtol=1e-9, atol=1e-9)


def test_single_expert_is_plain_mlp(orc):
    """n = 1, k = 1, no noise: the layer is E(x) (gate = 1)."""
    w = synth.WORKLOADS["tiny-flat"].with_(n=1, k=1, noise=0, bias_var=0.2)
    inp = synth.make_inputs(w)
    o = _fwd(orc, w, inp)
    assert np.all(o["topk_gate"] == 1.0)
    a = {k: v.double().numpy() for k, v in inp.items() if v is not None}
    want = _mlp_numpy(a["x"], a["W1"][0], a["b1"][0], a["W2"][0], a["b2"][0])
    np.testing.assert_allclose(o["y"], want, rtol=1e-12, atol=1e-12)


def test_zero_noise_limit_load_equals_counts(orc):
    """With Softplus(x W_noise) ~ 1e-14 the noise cannot change the top k and
    P(x,i) becomes the indicator of being kept: Load == counts exactly."""
    w = synth.WORKLOADS["tiny-flat"]
    inp = synth.make_inputs(w)
    inp["x"] = inp["x"].abs() + 0.1
    inp["Wn"] = torch.full_like(inp["Wn"], -40.0 / w.d * 8)
    o = _fwd(orc, w, inp)
    assert np.array_equal(o["load"], o["counts"].astype(np.float64))
    assert o["load"].sum() == w.T * w.k


def test_switch_aux_closed_forms(orc):
    """All tokens have logits (ln 3, 0): every token goes to expert 0 with
    p = (3/4, 1/4), so f = (1, 0), P = (3/4, 1/4), N sum f P = 2 * 3/4."""
    T = 10
    w = synth.Workload("sw", T=T, d=1, n=2, k=1, f=4, router=1, noise=0, expert_bf16=0)
    inp = synth.make_inputs(w)
    inp["x"] = torch.ones(T, 1)
    inp["Wg"] = torch.tensor([[math.log(3.0), 0.0]])
    o = _fwd(orc, w, inp)
    assert np.all(o["topk_idx"] == 0)
    assert o["topk_gate"] == pytest.approx(np.full((T, 1), 0.75), rel=1e-7)
    assert o["prob_sum"] == pytest.approx([0.75 * T, 0.25 * T], rel=1e-7)
    assert o["losses"][2] == pytest.approx(1.5, rel=1e-7)
    assert o["losses"][3] == pytest.approx(0.015, rel=1e-7)
    # uniform router: W_r = 0 -> all logits tie, lower index wins: f = (1,0),
    # P = (1/2, 1/2) -> N sum f P = 1
    inp["Wg"] = torch.zeros(1, 2)
    o = _fwd(orc, w, inp)
    assert o["losses"][2] == pytest.approx(1.0, rel=1e-15)


def test_capacity_overflow_passes_through(orc):
    """3 tokens, every one routed to expert 0, C = ceil(3*1*0.5/2) = 1:
    tokens 1 and 2 overflow and leave the layer unchanged (y = x)."""
    w = synth.Workload("cap", T=3, d=2, n=2, k=1, f=4, noise=0, expert_bf16=0,
                       capacity_factor=0.5, passthrough=1, bias_var=0.3)
    inp = synth.make_inputs(w)
    inp["x"] = torch.tensor([[1.0, 2.0], [0.5, -1.0], [2.0, 0.0]])
    inp["Wg"] = torch.tensor([[1.0, 0.0], [0.0, 0.0]])
    o = _fwd(orc, w, inp)
    assert list(o["topk_idx"].ravel()) == [0, 0, 0]
    assert list(o["row_of"].ravel()) == [0, -1, -1]
    a = {k: v.double().numpy() for k, v in inp.items() if v is not None}
    assert o["y"][0] == pytest.approx(_mlp_numpy(a["x"][0], a["W1"][0], a["b1"][0], a["W2"][0], a["b2"][0]))
    assert list(o["y"][1]) == [0.5, -1.0]
    assert list(o["y"][2]) == [2.0, 0.0]
    assert o["losses"][4] == pytest.approx(2 / 3)
    assert o["losses"][7] == 2.0
    # without pass-through the overflowed tokens get 0
    o = orc.forward(dict(w.cfg(), passthrough=0), _np_inputs(inp))
    assert list(o["y"][1]) == [0.0, 0.0]


def test_hierarchical_structure_and_zero_noise(orc):
    w = synth.Workload("h", T=40, d=16, n=4 * 6, k=4, f=8, hier_a=4, hier_b=6, hier_k1=2, hier_k2=2,
                       expert_bf16=0)
    inp = synth.make_inputs(w)
    o = _fwd(orc, w, inp)
    idx, g = o["topk_idx"], o["topk_gate"]
    assert g.sum(1) == pytest.approx(np.ones(w.T), abs=1e-14)
    for t in range(w.T):
        groups = idx[t] // w.hier_b
        # slots 0,1 come from the first chosen group, slots 2,3 from the second
        assert groups[0] == groups[1] and groups[2] == groups[3] and groups[0] != groups[2]
        assert len(set(idx[t].tolist())) == 4
    assert o["importance"].sum() == pytest.approx(w.T, rel=1e-13)
    assert o["counts"].sum() == w.T * w.k
    # zero-noise limit: Load_p(i) = |X_i| and Load_i(X_i)_j = count(i,j), so
    # Load_p(i) Load_i(j) / |X_i| = count(i,j)
    inp["x"] = inp["x"].abs() + 0.1
    inp["Wn"] = torch.full_like(inp["Wn"], -40.0)
    inp["Wn2"] = torch.full_like(inp["Wn2"], -40.0)
    o = _fwd(orc, w, inp)
    np.testing.assert_allclose(o["load"], o["counts"].astype(np.float64), rtol=1e-12)


def test_combine_hand(orc):
    """y_0 = 1/4 (1,2) + 3/4 (5,6) = (4,5); token 1 has no kept slot and
    passes through (9,8), or gets 0 without pass-through."""
    Y = np.array([[1.0, 2.0], [3.0, 4.0], [5.0, 6.0]])
    gate = np.array([[0.25, 0.75], [1.0, 0.0]])
    row_of = np.array([[0, 2], [-1, -1]], np.int32)
    x = np.array([[0.0, 0.0], [9.0, 8.0]], np.float32)
    y = orc.combine(Y, gate, row_of, x, passthrough=True)
    assert y.tolist() == [[4.0, 5.0], [9.0, 8.0]]
    y = orc.combine(Y, gate, row_of, x, passthrough=False)
    assert y.tolist() == [[4.0, 5.0], [0.0, 0.0]]


def test_balance_hand(orc):
    """idx (0,0,1), gates (1/2,1/2,1): Importance = (1,1) -> CV^2 = 0;
    Load = (2,0) -> mean 1, population variance 1 -> CV^2 = 1, L_load = 0.1;
    counts (2,1) with C = 1: one slot dropped of 3."""
    imp, losses = orc.balance(2, [[0], [0], [1]], [[0.5], [0.5], [1.0]], [2, 1], [2.0, 0.0], C=1)
    assert imp.tolist() == [1.0, 1.0]
    assert losses[0] == 0.0 and losses[5] == 0.0
    assert losses[1] == pytest.approx(0.1) and losses[6] == pytest.approx(1.0)
    assert losses[4] == pytest.approx(1 / 3) and losses[7] == 1.0
    assert losses[2] == 0.0  # noisy-gate router: no Switch loss
    # Switch: f = (2/3, 1/3), P = (0.6, 0.4) -> 2 * (0.4 + 0.4/3)
    imp, losses = orc.balance(2, [[0], [0], [1]], [[0.5], [0.5], [1.0]], [2, 1], [2.0, 1.0],
                              prob_sum=[1.8, 1.2], router=1, alpha=0.01)
    assert losses[2] == pytest.approx(2 * (2 / 3 * 0.6 + 1 / 3 * 0.4))
    assert losses[3] == pytest.approx(0.01 * losses[2])


def test_gate_batch_matches_forward(orc, tiny):
    w, inp = tiny
    o = _fwd(orc, w, inp)
    g = orc.gate_batch(w.cfg(), _np_inputs(inp))
    assert np.array_equal(g["topk_idx"], o["topk_idx"])
    assert np.array_equal(g["topk_gate"], o["topk_gate"])
    assert np.array_equal(g["load"], o["load"])


def test_gate_tokens_is_gate_batch_restricted(orc, tiny):
    """The gate of a token does not depend on the other tokens of the batch:
    a token list gives the same rows as the whole batch."""
    w, inp = tiny
    npin = _np_inputs(inp)
    full = orc.gate_batch(w.cfg(), npin)
    toks = np.array([5, 0, 63, 17], np.int32)
    part = orc.gate_tokens(w.cfg(), npin, toks)
    assert np.array_equal(part["topk_idx"], full["topk_idx"][toks])
    assert np.array_equal(part["topk_gate"], full["topk_gate"][toks])
    hw = synth.Workload("h", T=30, d=16, n=4 * 6, k=4, f=8, hier_a=4, hier_b=6, hier_k1=2, hier_k2=2,
                        expert_bf16=0)
    hin = _np_inputs(synth.make_inputs(hw))
    hf = orc.gate_batch(hw.cfg(), hin)
    hp = orc.gate_tokens(hw.cfg(), hin, [29, 3])
    assert np.array_equal(hp["topk_idx"], hf["topk_idx"][[29, 3]])
