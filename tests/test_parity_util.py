"""The GPU tests' comparison helpers, checked on the CPU with the oracle's own
results: they accept the oracle's output, accept a routing that differs only
at a near tie, and reject planted mistakes in every compared quantity."""
import numpy as np
import pytest
import torch

from parity_util import check_stats, touched_experts, y_rows_to_compare
from sparsely_gated_mixture_gate_b200 import synth

W = synth.WORKLOADS


def _np(inp):
    return {key: (None if v is None else (synth.bf16_bits(v) if v.dtype == torch.bfloat16 else v.numpy()))
            for key, v in inp.items()}


def _as_kernel_output(ref):
    """The oracle's whole-layer result in the kernel's output types."""
    return dict(topk_idx=ref["topk_idx"].copy(), topk_gate=ref["topk_gate"].astype(np.float32),
                counts=ref["counts"].copy(), importance=ref["importance"].astype(np.float32),
                load=ref["load"].astype(np.float32), losses=ref["losses"].astype(np.float32),
                y=ref["y"].astype(np.float32))


def _case(orc, w):
    inp = synth.make_inputs(w)
    return w, orc.forward(w.cfg(), _np(inp))


def test_accepts_the_oracle_and_rejects_planted_mistakes(orc):
    w, ref = _case(orc, W["lm-flat"].with_(T=64, n=16, d=32, f=32, k=2))
    out = _as_kernel_output(ref)
    assert check_stats(orc, w, out, ref) == (0, 0)
    for key, change in (("counts", lambda a: a.__setitem__(3, a[3] + 1)),
                        ("importance", lambda a: a.__setitem__(2, a[2] * (1 + 1e-4))),
                        ("load", lambda a: a.__setitem__(5, a[5] + 1e-2)),
                        ("losses", lambda a: a.__setitem__(1, a[1] * (1 + 1e-4))),
                        ("topk_gate", lambda a: a.__setitem__((7, 0), a[7, 0] * (1 + 1e-4))),
                        ("topk_idx", lambda a: a.__setitem__((4, 1), (a[4, 1] + 1) % w.n))):
        bad = {k: v.copy() for k, v in out.items()}
        change(bad[key])
        with pytest.raises(AssertionError):
            check_stats(orc, w, bad, ref)


def test_near_tie_flip_excludes_its_experts(orc):
    """A token with a near tie that the kernel routed the other way: its two
    experts are excluded from counts / importance / load, the losses are
    checked on the kernel's routing, the rest must still match."""
    w, ref = _case(orc, W["lm-flat"].with_(T=64, n=16, d=32, f=32, k=2, noise=0))
    out = _as_kernel_output(ref)
    t, old = 10, int(ref["topk_idx"][10, 1])
    new = next(e for e in range(w.n) if e not in ref["topk_idx"][10])
    ref = dict(ref, near_tie=ref["near_tie"].copy())
    ref["near_tie"][t] = 1e-6
    out["topk_idx"][t, 1] = new
    out["counts"][old] -= 1
    out["counts"][new] += 1
    g = float(out["topk_gate"][t, 1])
    out["importance"][old] -= g
    out["importance"][new] += g
    out["load"][old] -= 1  # noise off: the load is the count of selections
    out["load"][new] += 1
    C = orc.capacity(w.T, w.k, w.n, 0.0)
    _, own = orc.balance(w.n, out["topk_idx"], out["topk_gate"].astype(np.float64), out["counts"],
                         out["load"].astype(np.float64), None, C, 0)
    out["losses"][:8] = own
    nt, nx = check_stats(orc, w, out, ref)
    assert nt == 1 and nx == len({old, new} | set(ref["topk_idx"][t].tolist()))
    # ... but a mistake on an expert no tie touches still fails
    bad = {k: v.copy() for k, v in out.items()}
    free = next(e for e in range(w.n) if e not in (old, new) and e not in ref["topk_idx"][t])
    bad["importance"][free] += 1e-3
    with pytest.raises(AssertionError):
        check_stats(orc, w, bad, ref)


def test_hierarchical_exclusion_covers_whole_groups():
    w = W["hierarchical"].with_(T=4, n=4 * 8, hier_a=4, hier_b=8)
    tie = np.array([False, True, False, False])
    gpu = np.array([[0, 1, 8, 9]] * 4, np.int32)
    ref = gpu.copy()
    ref[1] = [0, 1, 16, 17]
    touched = touched_experts(w, tie, gpu, ref)
    assert touched.reshape(4, 8).all(axis=1).tolist() == [True, True, True, False]


def test_capacity_rows_skip_tokens_on_excluded_experts():
    w = W["switch-top1"].with_(T=4, n=4)
    tie = np.array([True, False, False, False])
    gpu = np.array([[0], [0], [2], [3]], np.int32)
    ref = np.array([[1], [0], [2], [3]], np.int32)
    touched = touched_experts(w, tie, gpu, ref)
    rows = y_rows_to_compare(w, tie, touched, gpu, ref)
    assert rows.tolist() == [False, False, True, True]
