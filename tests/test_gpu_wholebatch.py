"""Whole-batch statistics at the shapes of the two largest workloads.

The many-expert layer (4096 experts, d_model 512, FFN 512 -> 1024 -> 512,
k = 4, per-expert logit bias of variance 0.5 to skew the load) and the
hierarchical layer (64 groups of 128 experts, top 2 at each level), each on a
batch the oracle finishes in seconds (2048 and 8192 tokens), run through the
fused moe_forward exactly as the benchmark runs it.  The oracle gates the
whole batch, so counts, Importance, the smoothed Load (for the hierarchical
layer the product form of the two levels), L_importance, L_load and the other
loss entries are compared for the whole batch ("極大規模神經網路：稀疏門控專家混合層",
負載平衡損失; "Outrageously Large Neural Networks" reading note, 分层 MoE), and
the layer output of sampled tokens from the oracle's own experts.
"""
import numpy as np
import pytest
import torch

from parity_util import (TIE, check_stats, expert_sum, host_arrays, rel_fro, touched_experts,
                         y_rows_to_compare)
from sparsely_gated_mixture_gate_b200 import build, synth
from sparsely_gated_mixture_gate_b200 import moe as M

pytestmark = pytest.mark.gpu
DEV = "cuda"

W = synth.WORKLOADS
CASES = {
    "many-expert-2048": W["many-expert"].with_(T=2048),
    "hierarchical-8192": W["hierarchical"].with_(T=8192),
}
GATE_KEYS = ["x", "Wg", "bg", "Wn", "Wg2", "bg2", "Wn2", "sel_bias"]
_REF = {}


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def _oracle_gate(orc, name, w, inp):
    """The oracle's gate over the whole batch (independent of the kernel's
    gate precision, so computed once per shape)."""
    if name not in _REF:
        _REF[name] = orc.gate_batch(w.cfg(), host_arrays(inp, GATE_KEYS))
    return _REF[name]


@pytest.mark.parametrize("gp", [pytest.param(0, id="fp32fma"), pytest.param(1, id="tf32x3")])
@pytest.mark.parametrize("name", list(CASES))
def test_wholebatch_statistics(orc, name, gp):
    w = CASES[name].with_(gate_precision=gp)
    inp = synth.make_inputs(w, device=DEV)
    layer = M.MoELayer(M.Config.from_workload(w), inp, DEV)
    layer.forward_(inp["x"])
    torch.cuda.synchronize()
    out = {key: v.cpu().numpy() for key, v in layer.outputs().items()}
    assert M.status_bits(layer.status) == 0
    ref = _oracle_gate(orc, name, w, inp)
    nt, nx = check_stats(orc, w, out, ref, name)
    print(f"{name}: {nt} near-tie tokens, {nx} experts excluded; "
          f"L_importance {out['losses'][0]:.6g}, L_load {out['losses'][1]:.6g}")
    # the skew of the many-expert layer is real: a spread of expert loads
    if w.logit_bias_var > 0:
        assert out["counts"].max() > 4 * max(out["counts"].mean(), 1)

    # the layer output of sampled tokens, from the oracle's routing and experts
    tie = ref["near_tie"] < TIE
    touched = touched_experts(w, tie, out["topk_idx"], ref["topk_idx"])
    rows = y_rows_to_compare(w, tie, touched, out["topk_idx"], ref["topk_idx"])
    rng = np.random.default_rng(7)
    toks = sorted(set(rng.integers(0, w.T, 24).tolist()) | {0, w.T - 1})
    checked = 0
    for t in toks:
        if not rows[t]:
            continue
        want = expert_sum(orc, w, inp, t, ref["topk_idx"][t], ref["topk_gate"][t], [True] * w.k)
        err = rel_fro(out["y"][t], want)
        assert err < 2e-2, (t, err)
        checked += 1
    assert checked >= len(toks) // 2
