"""Comparison helpers shared by the GPU parity tests (no GPU code here).

Near ties.  A token whose k-th and (k+1)-th logits (or any two of its kept
logits) are closer than TIE may legitimately be routed differently by the
kernel and the oracle: both choices are correct to fp32 rounding.  Such a
token is excluded, and so is every expert it reaches on either side
(for the hierarchical gate, every expert of those groups: a token moving
between groups changes the group's token count and so each of its experts'
load).  On the rest the comparison is exact for integers and within the
stated tolerances for floats.  The losses are whole-batch functions of the
routing, so with near ties present they are checked against the oracle's
balancing formulas applied to the kernel's own routing (which agrees with
the oracle's wherever the choice is unique).
"""
import numpy as np

TIE = 1e-5


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def assert_rel(got, want, rtol, atol=0.0, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, f"{what}: shape {got.shape} vs {want.shape}"
    err = np.abs(got - want)
    bad = err > atol + rtol * np.abs(want)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} off; worst {err.max():.3e} " \
                          f"at {np.unravel_index(np.argmax(err), err.shape)}"


def touched_experts(w, tie, gpu_idx, ref_idx):
    """Experts reached by a near-tie token on either side (whole groups for
    the hierarchical gate)."""
    n = w.n
    touched = np.zeros(n, bool)
    for t in np.nonzero(tie)[0]:
        g = np.asarray(gpu_idx[t])
        touched[g[(g >= 0) & (g < n)]] = True
        touched[np.asarray(ref_idx[t])] = True
    if w.hier_a:
        grp = touched.reshape(w.hier_a, w.hier_b).any(axis=1)
        touched = np.repeat(grp, w.hier_b)
    return touched


def check_routing(idx, gate, ref, what=""):
    """Expert ids bit-exact and gates within 1e-5 on the tokens without a
    near tie; returns the near-tie mask."""
    tie = np.asarray(ref["near_tie"]) < TIE
    ok = ~tie
    assert np.array_equal(idx[ok], ref["topk_idx"][ok]), f"{what}: expert ids differ"
    assert_rel(gate[ok], ref["topk_gate"][ok], 1e-5, 1e-7, f"{what} gates")
    return tie


def check_stats(orc, w, out, ref, what=""):
    """Counts, importance, load and losses of a whole batch against the
    oracle's (ref holds topk_idx, topk_gate, near_tie, load, prob_sum and,
    from a whole-layer run, importance, counts and losses).  Returns the
    number of near-tie tokens and of excluded experts."""
    T, n, k = w.T, w.n, w.k
    idx = np.asarray(out["topk_idx"])
    gate = np.asarray(out["topk_gate"], np.float64)
    tie = check_routing(idx, gate, ref, what)
    touched = touched_experts(w, tie, idx, ref["topk_idx"])
    u = ~touched
    counts = np.asarray(out["counts"])
    ref_counts = np.bincount(ref["topk_idx"].ravel(), minlength=n)
    assert np.array_equal(counts[u], ref_counts[u]), f"{what}: counts differ"
    C = orc.capacity(T, k, n, w.capacity_factor)
    if "importance" in ref:
        ref_imp = ref["importance"]
        ref_losses = ref["losses"]
    else:
        ref_imp, ref_losses = orc.balance(n, ref["topk_idx"], ref["topk_gate"], ref_counts,
                                          ref["load"], ref["prob_sum"], C, w.router,
                                          w.w_importance, w.w_load, w.alpha)
    imp = np.asarray(out["importance"], np.float64)
    assert_rel(imp[u], ref_imp[u], 1e-5, 1e-6, f"{what} importance")
    load = np.asarray(out["load"], np.float64)
    assert_rel(load[u], ref["load"][u], 1e-5, 1e-6 * max(T, 1), f"{what} load")
    if w.noise and not w.hier_a:
        # the smoothed load moves by O(gap) under a near-tie swap: all experts
        assert_rel(load, ref["load"], 1e-5, 1e-6 * max(T, 1), f"{what} load (all experts)")
    losses = np.asarray(out["losses"], np.float64)
    if not tie.any():
        assert_rel(losses[:8], ref_losses[:8], 1e-5, 1e-7, f"{what} losses")
    else:
        psum = ref["prob_sum"] if w.router == 1 else None
        _, own = orc.balance(n, idx, gate, counts, load, psum, C, w.router, w.w_importance,
                             w.w_load, w.alpha)
        assert_rel(losses[:8], own, 1e-5, 1e-7, f"{what} losses (on the kernel's routing)")
    if len(ref_losses) > 8 and len(losses) > 8:
        assert_rel(losses[8:], ref_losses[8:], 1e-5, 1e-7, f"{what} router statistics")
    return int(tie.sum()), int(touched.sum())


def y_rows_to_compare(w, tie, touched, gpu_idx, ref_idx):
    """Tokens whose layer output is comparable: no near tie and, with a
    capacity limit, none of their experts excluded (an excluded expert's
    capacity cut can differ)."""
    ok = ~tie
    if w.capacity_factor > 0 and touched.any():
        for t in np.nonzero(ok)[0]:
            if touched[ref_idx[t]].any() or touched[np.clip(gpu_idx[t], 0, w.n - 1)].any():
                ok[t] = False
    return ok


def host_arrays(inp, keys):
    """numpy copies of the named inputs (None stays None)."""
    return {key: (None if inp.get(key) is None else inp[key].detach().cpu().numpy()) for key in keys}


def weight_bits(t):
    """bf16 tensor -> uint16 bit patterns; fp32 -> numpy."""
    import torch
    if t.dtype == torch.bfloat16:
        return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")
    return t.detach().cpu().numpy()


def expert_sum(orc, w, inp, t, idx_row, gate_row, kept):
    """The oracle's layer output for token t from a given routing: the
    gate-weighted sum of its kept experts' outputs, the pass-through of a
    fully dropped token, and the shared expert (weights from inp, which may
    live on the GPU; only the rows needed are copied)."""
    x = inp["x"][t].detach().cpu().numpy()
    y = np.zeros(w.d)
    for j, e in enumerate(idx_row):
        if not kept[j]:
            continue
        e = int(e)
        y += gate_row[j] * orc.expert_row(x, weight_bits(inp["W1"][e]), inp["b1"][e].cpu().numpy(),
                                          weight_bits(inp["W2"][e]), inp["b2"][e].cpu().numpy(),
                                          bf16=bool(w.expert_bf16))
    if not any(kept) and w.passthrough:
        y = x.astype(np.float64)
    if w.shared_expert:
        y = y + orc.expert_row(x, weight_bits(inp["W1s"]), inp["b1s"].cpu().numpy(),
                               weight_bits(inp["W2s"]), inp["b2s"].cpu().numpy(),
                               bf16=bool(w.expert_bf16))
    return y
