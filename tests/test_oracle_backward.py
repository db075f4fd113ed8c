"""Pins of the oracle's backward pass.

The forward pass is pinned elsewhere (pages' worked examples, closed forms,
library routines, brute force); here the gradients are pinned to it by
central finite differences of

    L = sum(dy * y) + losses[0] + losses[1] + losses[3]

with fp32 experts (the bf16 path's roundings make L piecewise constant at the
scale of a difference step).  The pages say which paths carry a gradient: the
kept gates are smooth in the logits ("極大規模神經網路：稀疏門控專家混合層",
常見問題), dropped experts get none (reading note, 缺点与局限性), and the noise
lets the load loss reach the gate through Phi (reading note, Noisy Top-K
Gating).  A step that flips a top-k choice or a capacity drop makes L jump;
such entries are detected (routing compared at both ends) and skipped.

Closed forms pin the CV^2 derivative, and torch autograd of a plain MLP (a
library derivative, n = k = 1 so that the layer is one expert) pins the
expert backward.  The bf16 rounding points are pinned against the fp32
gradient of the same bf16-representable weights."""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O

LOSS_IDX = (0, 1, 3)


def _loss(cfg, inp, dy):
    out = O.forward(cfg, inp)
    return float(np.sum(dy * out["y"]) + sum(out["losses"][i] for i in LOSS_IDX)), out


def _inputs(rng, T, d, n, f, *, noise=True, router=0, shared=False, bias=True):
    inp = dict(
        x=rng.normal(0, 1, (T, d)).astype(np.float32),
        Wg=rng.normal(0, 0.7, (d, n)).astype(np.float32),
        bg=rng.normal(0, 0.3, n).astype(np.float32) if bias else None,
        Wn=rng.normal(0, 0.4, (d, n)).astype(np.float32) if noise else None,
        W1=(rng.normal(0, 1, (n, f, d)) / math.sqrt(d)).astype(np.float32),
        b1=rng.normal(0, 0.2, (n, f)).astype(np.float32),
        W2=(rng.normal(0, 1, (n, d, f)) / math.sqrt(f)).astype(np.float32),
        b2=rng.normal(0, 0.2, (n, d)).astype(np.float32),
    )
    if router == 2:
        inp["sel_bias"] = rng.normal(0, 0.5, n).astype(np.float32)
    if shared:
        inp.update(W1s=(rng.normal(0, 1, (f, d)) / math.sqrt(d)).astype(np.float32),
                   b1s=rng.normal(0, 0.2, f).astype(np.float32),
                   W2s=(rng.normal(0, 1, (d, f)) / math.sqrt(f)).astype(np.float32),
                   b2s=rng.normal(0, 0.2, d).astype(np.float32))
    return inp


GRAD_OF = dict(x="dx", Wg="dWg", bg="dbg", Wn="dWn", W1="dW1", b1="db1", W2="dW2", b2="db2",
               W1s="dW1s", b1s="db1s", W2s="dW2s", b2s="db2s")


def _check_fd(cfg, inp, dy, names, rng, per=10, step=2e-3, rtol=2e-3):
    g = O.backward(cfg, inp, dy)
    _, base = _loss(cfg, inp, dy)
    checked = skipped = 0
    for name in names:
        arr = inp[name]
        an = g[GRAD_OF[name]]
        scale = float(np.abs(an).max()) + 1e-12
        flat = rng.choice(arr.size, size=min(per, arr.size), replace=False)
        for i in flat:
            pos = np.unravel_index(int(i), arr.shape)
            v0 = arr[pos]
            h = np.float32(step * max(1.0, abs(float(v0))))
            vp, vm = np.float32(v0 + h), np.float32(v0 - h)
            arr[pos] = vp
            lp, op = _loss(cfg, inp, dy)
            arr[pos] = vm
            lm, om = _loss(cfg, inp, dy)
            arr[pos] = v0
            same = all(np.array_equal(o["topk_idx"], base["topk_idx"]) and
                       np.array_equal(o["row_of"], base["row_of"]) for o in (op, om))
            if not same:
                skipped += 1
                continue
            fd = (lp - lm) / (float(vp) - float(vm))
            assert abs(fd - an[pos]) <= rtol * (abs(an[pos]) + 0.05 * scale) + 1e-9, \
                (name, pos, fd, an[pos], scale)
            checked += 1
    assert checked >= 0.8 * (checked + skipped), (checked, skipped)
    return g


def test_cv2_grad_closed_form_and_differences():
    # [1, 2, 3]: mean 2, var 2/3, CV^2 = 1/6; dCV^2/dv = (v - 2 - 1/3) / 6
    assert O.cv2_grad([1, 2, 3]) == pytest.approx([-2 / 9, -1 / 18, 1 / 9], abs=1e-15)
    rng = np.random.default_rng(0)
    v = rng.uniform(0.5, 3, 9)
    g = O.cv2_grad(v)
    for i in range(v.size):
        e = np.zeros_like(v); e[i] = 1e-6
        fd = (O.cv2(v + e) - O.cv2(v - e)) / 2e-6
        assert g[i] == pytest.approx(fd, rel=1e-6, abs=1e-9)
    # a scale change leaves CV^2 alone: the gradient is orthogonal to v
    assert float(np.dot(g, v)) == pytest.approx(0.0, abs=1e-12)
    assert np.all(O.cv2_grad(np.zeros(4)) == 0)


def test_noisy_topk_with_capacity_and_passthrough():
    rng = np.random.default_rng(11)
    T, d, n, k, f = 14, 6, 5, 2, 8
    inp = _inputs(rng, T, d, n, f)
    cfg = dict(T=T, d=d, n=n, k=k, f=f, router=0, noise=1, seed=5, capacity_factor=0.8,
               passthrough=1, w_importance=0.4, w_load=0.6)
    dy = rng.normal(0, 1, (T, d)).astype(np.float32)
    out = O.forward(cfg, inp)
    assert (out["row_of"] < 0).any()  # the capacity limit drops slots
    g = _check_fd(cfg, inp, dy, ["x", "Wg", "bg", "Wn", "W1", "b1", "W2", "b2"], rng)
    # the load loss reaches the noise weights
    assert np.abs(g["dWn"]).max() > 0


def test_load_loss_alone_reaches_gate_through_phi():
    # dy = 0 and no importance weight: the only gradient is the load loss's
    rng = np.random.default_rng(4)
    T, d, n, k, f = 10, 5, 6, 2, 8
    inp = _inputs(rng, T, d, n, f)
    cfg = dict(T=T, d=d, n=n, k=k, f=f, router=0, noise=1, seed=1, w_importance=0.0, w_load=1.0)
    dy = np.zeros((T, d), np.float32)
    g = _check_fd(cfg, inp, dy, ["x", "Wg", "bg", "Wn"], rng)
    assert np.abs(g["dW1"]).max() == 0 and np.abs(g["dW2"]).max() == 0
    assert np.abs(g["dbg"]).max() > 0


def test_noise_free_gate_and_k_equals_n():
    rng = np.random.default_rng(5)
    T, d, n, k, f = 9, 5, 4, 2, 8
    inp = _inputs(rng, T, d, n, f, noise=False)
    cfg = dict(T=T, d=d, n=n, k=k, f=f, router=0, noise=0, w_importance=0.5, w_load=0.5)
    dy = rng.normal(0, 1, (T, d)).astype(np.float32)
    _check_fd(cfg, inp, dy, ["x", "Wg", "bg", "W1", "b2"], rng)
    # k = n: every expert kept, the gate is the full softmax, kth_excluding of
    # a kept expert does not exist (P = 1): still differentiable
    inp = _inputs(rng, T, d, n, f)
    cfg = dict(T=T, d=d, n=n, k=n, f=f, router=0, noise=1, seed=3, w_importance=0.5, w_load=0.5)
    _check_fd(cfg, inp, dy, ["x", "Wg", "Wn", "W2"], rng)


def test_switch_router_with_aux_loss_and_capacity():
    rng = np.random.default_rng(8)
    T, d, n, f = 16, 6, 4, 8
    inp = _inputs(rng, T, d, n, f, noise=False, router=1)
    cfg = dict(T=T, d=d, n=n, k=1, f=f, router=1, noise=0, capacity_factor=1.0, passthrough=1,
               w_importance=0.3, w_load=0.0, alpha=0.7)
    dy = rng.normal(0, 1, (T, d)).astype(np.float32)
    assert (O.forward(cfg, inp)["row_of"] < 0).any()
    _check_fd(cfg, inp, dy, ["x", "Wg", "bg", "W1", "b1", "W2"], rng)


def test_sigmoid_router_with_bias_and_shared_expert():
    rng = np.random.default_rng(9)
    T, d, n, k, f = 12, 6, 6, 3, 8
    inp = _inputs(rng, T, d, n, f, noise=False, router=2, shared=True)
    cfg = dict(T=T, d=d, n=n, k=k, f=f, router=2, noise=0, shared_expert=1, w_importance=0.2,
               w_load=0.0)
    dy = rng.normal(0, 1, (T, d)).astype(np.float32)
    _check_fd(cfg, inp, dy, ["x", "Wg", "bg", "W1", "W2", "W1s", "b1s", "W2s", "b2s"], rng)


def test_single_expert_matches_torch_autograd():
    """n = k = 1: the layer is y = E(x) (gate 1 for any logit), so the
    expert gradients are those of a plain MLP, taken by torch autograd."""
    rng = np.random.default_rng(2)
    T, d, f = 7, 5, 9
    inp = _inputs(rng, T, d, 1, f, noise=False)
    cfg = dict(T=T, d=d, n=1, k=1, f=f, router=0, noise=0, w_importance=0.0, w_load=0.0)
    dy = rng.normal(0, 1, (T, d)).astype(np.float32)
    g = O.backward(cfg, inp, dy)
    x = torch.tensor(inp["x"], dtype=torch.float64, requires_grad=True)
    W1 = torch.tensor(inp["W1"][0], dtype=torch.float64, requires_grad=True)
    b1 = torch.tensor(inp["b1"][0], dtype=torch.float64, requires_grad=True)
    W2 = torch.tensor(inp["W2"][0], dtype=torch.float64, requires_grad=True)
    b2 = torch.tensor(inp["b2"][0], dtype=torch.float64, requires_grad=True)
    y = torch.nn.functional.linear(torch.relu(torch.nn.functional.linear(x, W1, b1)), W2, b2)
    (y * torch.tensor(dy, dtype=torch.float64)).sum().backward()
    for a, b in ((g["dx"], x), (g["dW1"][0], W1), (g["db1"][0], b1), (g["dW2"][0], W2),
                 (g["db2"][0], b2)):
        assert np.allclose(a, b.grad.numpy(), rtol=1e-12, atol=1e-12)
    # one kept expert: the gate is identically 1, no gradient reaches W_g
    assert np.abs(g["dWg"]).max() < 1e-12


def _to_bf16_bits(a):
    t = torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16), t.float().numpy()


def test_bf16_rounding_points_track_fp32_gradient():
    """The mixed-precision backward rounds only activation gradients to bf16:
    with bf16-representable weights it stays within bf16 error of the fp32
    backward, and exactly equal where nothing is rounded (the gate's dlogits
    for dy = 0)."""
    rng = np.random.default_rng(6)
    T, d, n, k, f = 16, 16, 4, 2, 32
    inp = _inputs(rng, T, d, n, f)
    inp["x"] = _to_bf16_bits(inp["x"])[1]
    b = dict(inp)
    for w in ("W1", "W2"):
        bits, vals = _to_bf16_bits(inp[w])
        b[w] = bits
        inp[w] = vals
    cfg = dict(T=T, d=d, n=n, k=k, f=f, router=0, noise=1, seed=2, w_importance=0.3, w_load=0.3)
    dy = rng.normal(0, 1, (T, d)).astype(np.float32)
    g32 = O.backward(cfg, inp, dy)
    g16 = O.backward(dict(cfg, expert_bf16=1), b, dy)
    for key in ("dx", "dW1", "db1", "dW2", "db2", "dgate", "dlogits", "dWg"):
        ref = g32[key]
        err = np.abs(g16[key] - ref).max() / (np.abs(ref).max() + 1e-30)
        assert err < 2e-2, (key, err)
        assert err > 0 or key in ("dWg",), key  # something was rounded
    z = np.zeros_like(dy)
    assert np.array_equal(O.backward(cfg, inp, z)["dlogits"],
                          O.backward(dict(cfg, expert_bf16=1), b, z)["dlogits"])


def test_hierarchical_with_a_shared_expert_rejected():
    """The hierarchical layer's backward covers routed experts only (the pages'
    hierarchical layer has no shared expert)."""
    with pytest.raises(ValueError):
        O.backward(dict(T=2, d=4, n=4, k=1, f=8, hier_a=2, hier_b=2, hier_k1=1, hier_k2=1,
                        shared_expert=1),
                   dict(x=np.zeros((2, 4), np.float32), Wg=np.zeros((4, 2), np.float32),
                        Wn=np.zeros((4, 2), np.float32), Wg2=np.zeros((2, 4, 2), np.float32),
                        Wn2=np.zeros((2, 4, 2), np.float32), W1=np.zeros((4, 8, 4), np.float32),
                        W2=np.zeros((4, 4, 8), np.float32), W1s=np.zeros((8, 4), np.float32),
                        W2s=np.zeros((4, 8), np.float32)),
                   np.zeros((2, 4), np.float32))


def test_expert_backward_is_the_layer_backward_of_one_expert():
    """The per-expert entry point, applied to the rows the layer routed to each
    expert with their gates, gives the layer backward's dW1..db2 and dgate
    (the whole-layer backward is pinned above)."""
    rng = np.random.default_rng(12)
    T, d, n, k, f = 20, 8, 4, 2, 16
    inp = _inputs(rng, T, d, n, f)
    for bf16 in (0, 1):
        cfg = dict(T=T, d=d, n=n, k=k, f=f, router=0, noise=1, seed=4, capacity_factor=0.8,
                   expert_bf16=bf16)
        e_inp = dict(inp)
        if bf16:
            for w in ("W1", "W2"):
                e_inp[w] = _to_bf16_bits(inp[w])[0]
        dy = rng.normal(0, 1, (T, d)).astype(np.float32)
        out = O.forward(cfg, e_inp)
        g = O.backward(cfg, e_inp, dy)
        for e in range(n):
            rows = [(t, j) for t in range(T) for j in range(k)
                    if out["topk_idx"][t, j] == e and out["row_of"][t, j] >= 0]
            toks = np.array([t for t, _ in rows], np.int64)
            gates = np.array([out["topk_gate"][t, j] for t, j in rows])
            r = O.expert_backward(inp["x"][toks], gates, dy[toks], e_inp["W1"][e], inp["b1"][e],
                                  e_inp["W2"][e], inp["b2"][e], bf16=bool(bf16))
            for key in ("dW1", "db1", "dW2", "db2"):
                assert np.allclose(r[key], g[key][e], rtol=1e-12, atol=1e-12), (bf16, e, key)
            for (t, j), dg in zip(rows, r["dgate"]):
                assert dg == pytest.approx(g["dgate"][t, j], rel=1e-12, abs=1e-12)


@pytest.mark.parametrize("router", [0, 1, 2])
def test_zloss_and_entropy_terms(router):
    """With weights on the router z-loss and the gate entropy the backward's
    loss is L + w_z losses[8] - w_entropy losses[9]: central differences of the
    forward (router_stats on) pin their gradients, alone (dy = 0, no other
    loss) and together with everything else."""
    rng = np.random.default_rng(30 + router)
    T, d, n, f = 10, 5, 5, 8
    k = 1 if router == 1 else 2
    inp = _inputs(rng, T, d, n, f, noise=(router == 0), router=router)
    base = dict(T=T, d=d, n=n, k=k, f=f, router=router, noise=int(router == 0), seed=2,
                router_stats=1, w_z=0.7, w_entropy=1.3)

    def loss(cfg, inp, dy):
        out = O.forward(cfg, inp)
        return float(np.sum(dy * out["y"]) + out["losses"][0] + out["losses"][1] +
                     out["losses"][3] + cfg["w_z"] * out["losses"][8] -
                     cfg["w_entropy"] * out["losses"][9]), out

    for cfg, dy in ((dict(base, w_importance=0.0, w_load=0.0, alpha=0.0),
                     np.zeros((T, d), np.float32)),
                    (dict(base, w_importance=0.3, w_load=0.4, alpha=0.5),
                     rng.normal(0, 1, (T, d)).astype(np.float32))):
        g = O.backward(cfg, inp, dy)
        _, ref_out = loss(cfg, inp, dy)
        for name in ("Wg", "bg", "x"):
            arr = inp[name]
            an = g[GRAD_OF[name]]
            scale = float(np.abs(an).max()) + 1e-12
            for i in rng.choice(arr.size, size=min(8, arr.size), replace=False):
                pos = np.unravel_index(int(i), arr.shape)
                v0 = arr[pos]
                h = np.float32(2e-3 * max(1.0, abs(float(v0))))
                arr[pos] = np.float32(v0 + h); lp, op = loss(cfg, inp, dy)
                arr[pos] = np.float32(v0 - h); lm, om = loss(cfg, inp, dy)
                arr[pos] = v0
                if not (np.array_equal(op["topk_idx"], ref_out["topk_idx"]) and
                        np.array_equal(om["topk_idx"], ref_out["topk_idx"])):
                    continue
                fd = (lp - lm) / (float(np.float32(v0 + h)) - float(np.float32(v0 - h)))
                assert abs(fd - an[pos]) <= 2e-3 * (abs(an[pos]) + 0.05 * scale) + 1e-9, \
                    (router, name, pos, fd, an[pos])


# ------------------------------------------------------------------ hierarchical layer
GRAD_OF.update(Wg2="dWg2", bg2="dbg2", Wn2="dWn2")


def _hier_inputs(rng, T, d, a, b, f, *, noise=True):
    n = a * b
    inp = _inputs(rng, T, d, a, f, noise=noise)           # the primary gate over a groups
    inp.update(
        Wg2=rng.normal(0, 0.7, (a, d, b)).astype(np.float32),
        bg2=rng.normal(0, 0.3, (a, b)).astype(np.float32),
        Wn2=rng.normal(0, 0.4, (a, d, b)).astype(np.float32) if noise else None,
        W1=(rng.normal(0, 1, (n, f, d)) / math.sqrt(d)).astype(np.float32),
        b1=rng.normal(0, 0.2, (n, f)).astype(np.float32),
        W2=(rng.normal(0, 1, (n, d, f)) / math.sqrt(f)).astype(np.float32),
        b2=rng.normal(0, 0.2, (n, d)).astype(np.float32))
    return inp


def _hier_cfg(T, d, a, b, f, **kw):
    return dict(T=T, d=d, n=a * b, k=4, f=f, hier_a=a, hier_b=b, hier_k1=2, hier_k2=2, **kw)


def test_hierarchical_noisy_with_capacity_and_passthrough():
    """Both gate levels, the product-form load and the experts ("Outrageously
    Large Neural Networks" reading note, 分层 MoE): every gradient against
    central differences of the forward loss, capacity drops included."""
    rng = np.random.default_rng(21)
    T, d, a, b, f = 14, 5, 3, 4, 6
    inp = _hier_inputs(rng, T, d, a, b, f)
    cfg = _hier_cfg(T, d, a, b, f, router=0, noise=1, seed=3, capacity_factor=0.9, passthrough=1,
                    w_importance=0.5, w_load=0.7)
    dy = rng.normal(0, 1, (T, d)).astype(np.float32)
    assert (O.forward(cfg, inp)["row_of"] < 0).any()
    g = _check_fd(cfg, inp, dy, ["x", "Wg", "bg", "Wn", "Wg2", "bg2", "Wn2", "W1", "b1", "W2", "b2"],
                  rng, per=8)
    assert np.abs(g["dWn2"]).max() > 0 and np.abs(g["dbg2"]).max() > 0


def test_hierarchical_load_loss_reaches_both_levels():
    """dy = 0, no importance weight: the only gradient is the load loss of
    Load(i b + j) = Load_p_i Load_i_j / |X_i|, reaching the primary gate and
    each group's gate through Phi."""
    rng = np.random.default_rng(22)
    T, d, a, b, f = 12, 4, 3, 3, 4
    inp = _hier_inputs(rng, T, d, a, b, f)
    cfg = _hier_cfg(T, d, a, b, f, router=0, noise=1, seed=9, w_importance=0.0, w_load=1.0)
    dy = np.zeros((T, d), np.float32)
    g = _check_fd(cfg, inp, dy, ["x", "Wg", "bg", "Wn", "Wg2", "bg2", "Wn2"], rng, per=8)
    assert np.abs(g["dW1"]).max() == 0
    assert np.abs(g["dbg"]).max() > 0 and np.abs(g["dbg2"]).max() > 0


def test_hierarchical_noise_free_and_router_statistics():
    rng = np.random.default_rng(23)
    T, d, a, b, f = 10, 5, 4, 3, 6
    inp = _hier_inputs(rng, T, d, a, b, f, noise=False)
    cfg = _hier_cfg(T, d, a, b, f, router=0, noise=0, w_importance=0.6, w_load=0.4, router_stats=1,
                    w_z=0.05, w_entropy=0.2)
    dy = rng.normal(0, 1, (T, d)).astype(np.float32)

    def loss(cfg_, inp_, dy_):
        out = O.forward(cfg_, inp_)
        L = float(np.sum(dy_ * out["y"]) + sum(out["losses"][i] for i in LOSS_IDX)
                   + cfg_["w_z"] * out["losses"][8] - cfg_["w_entropy"] * out["losses"][9])
        return L, out
    g = O.backward(cfg, inp, dy)
    _, base = loss(cfg, inp, dy)
    checked = 0
    for name in ("x", "Wg", "bg", "Wg2", "bg2"):
        arr = inp[name]
        for i in rng.choice(arr.size, size=min(6, arr.size), replace=False):
            pos = np.unravel_index(int(i), arr.shape)
            v0 = arr[pos]
            h = np.float32(2e-3 * max(1.0, abs(float(v0))))
            arr[pos] = v0 + h
            lp, op = loss(cfg, inp, dy)
            arr[pos] = v0 - h
            lm, om = loss(cfg, inp, dy)
            arr[pos] = v0
            if not all(np.array_equal(o["topk_idx"], base["topk_idx"]) for o in (op, om)):
                continue
            fd = (lp - lm) / (float(np.float32(v0 + h)) - float(np.float32(v0 - h)))
            an = g[GRAD_OF[name]][pos]
            assert abs(fd - an) <= 2e-3 * (abs(an) + 0.05 * np.abs(g[GRAD_OF[name]]).max()) + 1e-9, \
                (name, pos, fd, an)
            checked += 1
    assert checked >= 20
