"""Full-size parity: every workload at its real size, through the fused
moe_forward in the launch configuration the bench times.

The oracle cannot run whole batches of the large workloads in seconds, so:
  - sampled tokens: routing (ids bit-exact outside near ties, gates 1e-5) and
    the layer output (2e-2 relative) from the oracle's own gate and experts;
  - the LM-shaped workload (the bench workload): the oracle's gate over the
    whole batch, so load, importance, counts and losses are compared too;
  - the Switch workloads: the oracle's gate and dispatch over the whole batch
    (capacity decisions depend on every token);
  - everything else: properties that hold at any size.
"""
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


def _host(inp, keys):
    out = {}
    for k in keys:
        v = inp.get(k)
        out[k] = None if v is None else v.detach().cpu().numpy()
    return out


def _bits(t):
    return synth.bf16_bits(t) if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / max(np.linalg.norm(b), 1e-30))


def _sample(T, m=40, seed=0):
    rng = np.random.default_rng(seed)
    return np.array(sorted(set(rng.integers(0, T, m).tolist()) | {0, T - 1}), np.int32)


def _expert_sum(orc, w, inp, t, idx_row, gate_row, kept):
    x = inp["x"][t].detach().cpu().numpy()
    y = np.zeros(w.d)
    for j, e in enumerate(idx_row):
        if not kept[j]:
            continue
        e = int(e)
        y += gate_row[j] * orc.expert_row(x, _bits(inp["W1"][e]), inp["b1"][e].cpu().numpy(),
                                          _bits(inp["W2"][e]), inp["b2"][e].cpu().numpy(),
                                          bf16=bool(w.expert_bf16))
    if not any(kept) and w.passthrough:
        y = x.astype(np.float64)
    if w.shared_expert:  # the always-active expert, weight 1
        y = y + orc.expert_row(x, _bits(inp["W1s"]), inp["b1s"].cpu().numpy(), _bits(inp["W2s"]),
                               inp["b2s"].cpu().numpy(), bf16=bool(w.expert_bf16))
    return y


CASES = ["lm-flat", "many-expert", "hierarchical", "switch-top1", "switch-skew", "deepseek-flat"]


@pytest.mark.parametrize("gp", [pytest.param(0, id="fp32fma"), pytest.param(1, id="tf32x3")])
@pytest.mark.parametrize("name", CASES)
def test_fullsize(orc, name, gp):
    w = (synth.WORKLOADS.get(name) or synth.VARIANTS[name]).with_(gate_precision=gp)
    torch.manual_seed(0)
    inp = synth.make_inputs(w, device=DEV)
    cfg = M.Config.from_workload(w)
    layer = M.MoELayer(cfg, inp, DEV)
    layer.forward_(inp["x"])
    torch.cuda.synchronize()
    out = {k: v.cpu() for k, v in layer.outputs().items()}
    assert M.status_bits(out["status"]) == 0
    T, k, n = w.T, w.k, w.n
    idx = out["topk_idx"].numpy()
    gate = out["topk_gate"].numpy()
    counts = out["counts"].numpy()

    # ---- properties at any size
    assert counts.sum() == T * k
    assert np.array_equal(np.bincount(idx.ravel(), minlength=n), counts)
    if w.router in (0, 2):
        assert np.allclose(gate.sum(1), 1.0, atol=2e-6 * k)
    assert out["importance"].sum().item() == pytest.approx(float(gate.sum()), rel=1e-5)
    load = out["load"].numpy()
    assert np.all(load >= 0) and np.all(load <= T * (1 + 1e-6))
    losses = out["losses"].numpy()
    assert losses[0] == pytest.approx(w.w_importance * losses[5], rel=1e-6)
    assert losses[1] == pytest.approx(w.w_load * losses[6], rel=1e-6)
    C = orc.capacity(T, k, n, w.capacity_factor)
    assert losses[7] == np.maximum(counts.astype(np.int64) - C, 0).sum()

    gate_keys = ["x", "Wg", "bg", "Wn", "Wg2", "bg2", "Wn2", "sel_bias"]
    ginp = _host(inp, gate_keys)
    toks = _sample(T)

    full_ref = None
    if name == "lm-flat" or w.router == 1:
        full_ref = orc.gate_batch(w.cfg(), ginp)     # seconds for these sizes
        ref = {key: (v[toks] if key in ("topk_idx", "topk_gate", "near_tie") else v)
               for key, v in full_ref.items()}
    else:
        ref = orc.gate_tokens(w.cfg(), ginp, toks)

    ok = ref["near_tie"] >= TIE
    print(f"{name}: {int((~ok).sum())} near-tie tokens of {len(toks)} sampled")
    assert np.array_equal(idx[toks][ok], ref["topk_idx"][ok])
    g_ok = gate[toks][ok]
    assert np.allclose(g_ok, ref["topk_gate"][ok], rtol=1e-5, atol=1e-7)

    if full_ref is not None:
        tie_all = full_ref["near_tie"] < TIE
        near = int(tie_all.sum())
        print(f"{name}: {near} near-tie tokens of {T}")
        # load is insensitive to a near-tie swap (the two thresholds coincide)
        assert np.allclose(load, full_ref["load"], rtol=1e-5, atol=1e-6 * T)
        if w.router == 1:
            assert np.allclose(layer.outputs()["load"].cpu().numpy(), full_ref["load"], rtol=1e-5)
        # importance / counts of experts that no near-tie token touches
        touched = np.zeros(n, bool)
        for t in np.nonzero(tie_all)[0]:
            touched[idx[t]] = True
            touched[full_ref["topk_idx"][t]] = True
        ref_counts = np.bincount(full_ref["topk_idx"].ravel(), minlength=n)
        assert np.array_equal(counts[~touched], ref_counts[~touched])
        imp_ref, losses_ref = orc.balance(n, full_ref["topk_idx"], full_ref["topk_gate"], ref_counts,
                                          full_ref["load"], full_ref["prob_sum"], C, w.router,
                                          w.w_importance, w.w_load, w.alpha)
        imp = out["importance"].numpy()
        assert np.allclose(imp[~touched], imp_ref[~touched], rtol=1e-5, atol=1e-6)
        if near == 0:
            assert np.allclose(losses[:8], losses_ref, rtol=1e-5, atol=1e-7)

    # ---- the layer output of the sampled tokens
    kept_all = None
    skip_tok = np.zeros(T, bool)
    if w.capacity_factor > 0:
        # an expert that no near-tie token touches receives the same tokens in
        # the same order on both sides, so its capacity cut is identical
        d = orc.dispatch(full_ref["topk_idx"], n, C)
        assert np.array_equal(counts[~touched], d["counts"][~touched])
        kept_all = d["row_of"] >= 0
        for t in range(T):
            if touched[full_ref["topk_idx"][t]].any() or touched[idx[t]].any():
                skip_tok[t] = True
        if near == 0:
            assert losses[7] == (~kept_all).sum()
    y = out["y"].numpy()
    checked = 0
    for r, t in enumerate(toks):
        if not ok[r] or skip_tok[t]:
            continue
        kept = kept_all[t] if kept_all is not None else [True] * k
        want = _expert_sum(orc, w, inp, int(t), ref["topk_idx"][r], ref["topk_gate"][r], kept)
        err = _rel(y[t], want)
        assert err < 2e-2, (t, err)
        checked += 1
    assert checked >= len(toks) // 2


# ------------------------------------------------------------------ backward
@pytest.mark.parametrize("name", ["lm-flat", "deepseek-flat", "hierarchical"])
def test_fullsize_backward(orc, name):
    """The training step the bench times (forward + moe_backward) at full size.
    The oracle routes the whole batch (its own gate), then computes the
    weight and bias gradients of sampled experts from the rows it routed to
    them and dL/dgate of their tokens; the gate's gradients depend on
    whole-batch sums and are covered by the small parity cases."""
    import dataclasses
    w = synth.WORKLOADS.get(name) or synth.VARIANTS[name]
    inp = synth.make_inputs(w, device=DEV)
    dy = synth.make_dy(w, device=DEV)
    cfg = dataclasses.replace(M.Config.from_workload(w), backward=1)
    layer = M.MoELayer(cfg, inp, DEV)
    layer.forward_(inp["x"])
    layer.grads(intermediates=True)
    g = layer.backward_(inp["x"], dy)
    torch.cuda.synchronize()
    assert M.status_bits(layer.status) == 0
    host = _host(inp, ["x", "Wg", "bg", "Wn", "sel_bias", "Wg2", "bg2", "Wn2"])
    ref = orc.gate_batch(w.cfg(), host)
    tie = ref["near_tie"] < TIE
    idx = layer.topk_idx.cpu().numpy()
    assert np.array_equal(idx[~tie], ref["topk_idx"][~tie])
    # an expert a near-tie token reaches on either side may hold a row the
    # other side does not
    tie_experts = set(idx[tie].ravel().tolist()) | set(ref["topk_idx"][tie].ravel().tolist())
    x = host["x"]
    dyh = dy.cpu().numpy()
    dgate = g["dgate"].cpu().numpy()
    counts = np.bincount(ref["topk_idx"].ravel(), minlength=w.n)
    rng = np.random.default_rng(3)
    experts = sorted({int(np.argmax(counts)), int(np.argmin(counts))} |
                     set(rng.integers(0, w.n, 4).tolist()))
    checked = 0
    for e in experts:
        slots = np.argwhere(ref["topk_idx"] == e)  # (token, slot), token order
        if e in tie_experts:
            continue  # a near tie could move a row in or out of this expert
        toks = slots[:, 0]
        gates = ref["topk_gate"][slots[:, 0], slots[:, 1]]
        r = orc.expert_backward(x[toks], gates, dyh[toks], _bits(inp["W1"][e]),
                                inp["b1"][e].cpu().numpy(), _bits(inp["W2"][e]),
                                inp["b2"][e].cpu().numpy(), bf16=True)
        for key in ("dW1", "db1", "dW2", "db2"):
            got = g[key][e].cpu().numpy()
            if not np.any(r[key]) and not np.any(got):
                continue
            assert _rel(got, r[key]) < 1e-2, (name, e, key, _rel(got, r[key]))
        if len(toks):
            assert _rel(dgate[slots[:, 0], slots[:, 1]], r["dgate"]) < 5e-3, (name, e)
        checked += 1
    assert checked >= 3
