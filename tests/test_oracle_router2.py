"""Pins of the oracle's sigmoid router (router 2), its selection bias and the
shared expert ("MoE 稀疏架构深度解析", §5.2 shared expert, §6.2 sigmoid scores
normalised over the top K, §6.3 auxiliary-loss-free selection bias).

Values here are fixed by hand or by mathematics the test states, not by the
oracle's own code: sigmoid(0) = 1/2 and sigmoid(ln 3) = 3/4 make exact gates,
the bias-update rule is a sign rule on integers, a dense evaluation of every
expert pins the sparse path, and n = 1 with the shared expert equal to the
routed one must give twice one expert."""
import math

import numpy as np
import pytest

from oracle import oracle as O


def _row(h, k, sel_bias=None):
    x = np.array([1.0], np.float32)
    Wg = np.array([h], np.float32)  # d = 1: c = h
    return O.gate_row(x, Wg, k, router=2, noise=False, sel_bias=sel_bias)


def test_sigmoid_gates_by_hand():
    # h = (ln 3, 0, 2, -1); the bias lifts expert 1 above everything and sinks
    # expert 2: scores (ln 3, 5, -1, -1) -> keep 1, 0.  The gates use the
    # logits without the bias: sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4, so
    # g = (1/2, 3/4) / (5/4) = (0.4, 0.6).
    r = _row([math.log(3.0), 0.0, 2.0, -1.0], 2, sel_bias=np.array([0, 5, -3, 0], np.float32))
    assert r["idx"].tolist() == [1, 0]
    assert r["gates"] == pytest.approx([0.4, 0.6], abs=1e-7)


def test_bias_changes_selection_not_gates():
    h = [math.log(3.0), 0.0, 2.0, -1.0]
    r0 = _row(h, 2)  # no bias: keep 2 (h = 2) and 0 (h = ln 3)
    assert r0["idx"].tolist() == [2, 0]
    # sigmoid(2) = e^2 / (1 + e^2); with sigmoid(ln 3) = 3/4
    s2 = math.exp(2.0) / (1.0 + math.exp(2.0))
    assert r0["gates"] == pytest.approx([s2 / (s2 + 0.75), 0.75 / (s2 + 0.75)], abs=1e-7)
    # a bias that keeps the same pair changes nothing in the gates
    r1 = _row(h, 2, sel_bias=np.array([0.5, -1, 0.1, 0], np.float32))
    assert r1["idx"].tolist() == [2, 0]
    assert r1["gates"] == pytest.approx(r0["gates"], abs=0)


def test_bias_tie_goes_to_lower_index():
    # scores 1 + 0 and 0 + 1 are equal: the lower index wins; k = 1 gives gate 1
    r = _row([1.0, 0.0], 1, sel_bias=np.array([0.0, 1.0], np.float32))
    assert r["idx"].tolist() == [0]
    assert r["gates"][0] == 1.0


def test_gates_sum_to_one():
    rng = np.random.default_rng(3)
    for _ in range(20):
        n = int(rng.integers(2, 40))
        k = int(rng.integers(1, min(n, 8) + 1))
        r = _row(rng.normal(0, 3, n), k, sel_bias=rng.normal(0, 1, n).astype(np.float32))
        assert r["gates"].sum() == pytest.approx(1.0, abs=1e-12)
        assert (r["gates"] > 0).all()


def test_bias_update_sign_rule():
    # T = 3 tokens, k = 4 slots: 12 slots over n = 4 experts, average 3
    b = O.sel_bias_update([5, 1, 3, 3], 3, 4, 0.25, [0.5, 0.5, 0.5, 0.5])
    assert b.tolist() == [0.25, 0.75, 0.5, 0.5]
    # the comparison is exact on integers: 7 slots over n = 3 (average 7/3)
    b = O.sel_bias_update([3, 2, 2], 7, 1, 1.0, [0.0, 0.0, 0.0])
    assert b.tolist() == [-1.0, 1.0, 1.0]


def _mlp(x, W1, b1, W2, b2):
    h = np.maximum(W1.astype(np.float64) @ x + b1, 0.0)
    return W2.astype(np.float64) @ h + b2


def test_dense_brute_force_with_shared_expert():
    """Every expert evaluated on every token, unselected ones weighted 0, plus
    the shared expert: equal to the sparse forward (fp32 experts)."""
    rng = np.random.default_rng(7)
    T, d, n, k, f = 24, 8, 6, 3, 16
    inp = dict(
        x=rng.normal(0, 1, (T, d)).astype(np.float32),
        Wg=rng.normal(0, 1, (d, n)).astype(np.float32),
        bg=None, Wn=None,
        W1=(rng.normal(0, 1, (n, f, d)) / math.sqrt(d)).astype(np.float32),
        b1=rng.normal(0, 0.1, (n, f)).astype(np.float32),
        W2=(rng.normal(0, 1, (n, d, f)) / math.sqrt(f)).astype(np.float32),
        b2=rng.normal(0, 0.1, (n, d)).astype(np.float32),
        sel_bias=rng.normal(0, 1, n).astype(np.float32),
        W1s=(rng.normal(0, 1, (f, d)) / math.sqrt(d)).astype(np.float32),
        b1s=rng.normal(0, 0.1, f).astype(np.float32),
        W2s=(rng.normal(0, 1, (d, f)) / math.sqrt(f)).astype(np.float32),
        b2s=rng.normal(0, 0.1, d).astype(np.float32),
    )
    out = O.forward(dict(T=T, d=d, n=n, k=k, f=f, router=2, noise=0, shared_expert=1), inp)
    for t in range(T):
        h = inp["x"][t].astype(np.float64) @ inp["Wg"].astype(np.float64)
        score = (h + inp["sel_bias"]).astype(np.float32)
        kept = sorted(range(n), key=lambda i: (-score[i], i))[:k]
        sig = 1.0 / (1.0 + np.exp(-h))
        G = np.zeros(n)
        G[kept] = sig[kept] / sig[kept].sum()
        want = sum(G[i] * _mlp(inp["x"][t], inp["W1"][i], inp["b1"][i], inp["W2"][i], inp["b2"][i])
                   for i in range(n))
        want = want + _mlp(inp["x"][t], inp["W1s"], inp["b1s"], inp["W2s"], inp["b2s"])
        assert out["topk_idx"][t].tolist() == kept
        assert np.allclose(out["y"][t], want, rtol=1e-10, atol=1e-10), t
    # no noise: the smoothed load is the count of selections
    assert np.array_equal(out["load"], out["counts"].astype(np.float64))


def test_single_expert_plus_identical_shared_expert_doubles():
    rng = np.random.default_rng(2)
    T, d, f = 5, 8, 8
    W1 = rng.normal(0, 0.3, (1, f, d)).astype(np.float32)
    W2 = rng.normal(0, 0.3, (1, d, f)).astype(np.float32)
    b1 = rng.normal(0, 0.1, (1, f)).astype(np.float32)
    b2 = rng.normal(0, 0.1, (1, d)).astype(np.float32)
    inp = dict(x=rng.normal(0, 1, (T, d)).astype(np.float32),
               Wg=rng.normal(0, 1, (d, 1)).astype(np.float32), W1=W1, b1=b1, W2=W2, b2=b2,
               W1s=W1[0], b1s=b1[0], W2s=W2[0], b2s=b2[0])
    out = O.forward(dict(T=T, d=d, n=1, k=1, f=f, router=2, noise=0, shared_expert=1), inp)
    assert np.all(out["topk_gate"] == 1.0)  # one kept expert: s / s
    for t in range(T):
        one = O.expert_row(inp["x"][t], W1[0], b1[0], W2[0], b2[0], bf16=False)
        assert np.allclose(out["y"][t], 2.0 * one, rtol=1e-12, atol=1e-12)


def test_router2_rejects_noise():
    with pytest.raises(ValueError):
        O.gate_batch(dict(T=2, d=1, n=2, k=1, f=8, router=2, noise=1),
                     dict(x=np.ones((2, 1), np.float32), Wg=np.ones((1, 2), np.float32),
                          Wn=np.ones((1, 2), np.float32)))
