"""The expert-parallel layer's exchanges on CPU ranks (gloo).

Two processes, each with its own shard of the batch and half of the experts,
run ExpertParallelMoE.forward with the oracle standing in for the CUDA steps
(OracleSteps below: test infrastructure, never the product path).  What this
checks is the part that is the same on GPUs: the counts and rows exchanged,
the regrouping by local expert and back, the reverse exchange, the combine
on the right rows, the statistics summed over the ranks.  Without a capacity
limit the result must equal the oracle's layer on the whole batch; with one,
each shard cuts at its own capacity (ceil(T_r k cf / n)).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparsely_gated_mixture_gate_b200 import synth
from sparsely_gated_mixture_gate_b200.expert_parallel import ExpertParallelMoE, regroup_index
from sparsely_gated_mixture_gate_b200 import moe as M

W = synth.WORKLOADS
CASES = {
    "noisy": W["lm-flat"].with_(T=96, d=32, n=8, k=2, f=32),
    "switch-capacity": synth.VARIANTS["switch-skew"].with_(T=120, d=32, n=8, f=32),
    "fp32-uneven": W["tiny-flat"].with_(T=70, n=8, k=3),
    "sigmoid": synth.VARIANTS["deepseek-tiny"].with_(shared_expert=0, T=80, n=8, k=2),
}
SPLITS = {"noisy": [40, 56], "switch-capacity": [60, 60], "fp32-uneven": [1, 69], "sigmoid": [33, 47]}


def _np(t):
    if t is None:
        return None
    return synth.bf16_bits(t) if t.dtype == torch.bfloat16 else t.numpy()


class OracleSteps:
    """The layer's steps computed by the oracle on the CPU, with float64 rows
    (the exchanges move any row type as 32-bit words)."""

    def __init__(self, orc, w, full):
        self.orc, self.w = orc, w
        self.gin = {k: _np(full.get(k)) for k in ("x", "Wg", "bg", "Wn", "sel_bias")}

    def gate(self, cfg, x, params):
        toks = np.arange(cfg.token_base, cfg.token_base + cfg.T, dtype=np.int32)
        r = self.orc.gate_tokens(self.w.cfg(), self.gin, toks)
        return dict(topk_idx=torch.from_numpy(r["topk_idx"]), topk_gate=torch.from_numpy(r["topk_gate"]),
                    load=torch.from_numpy(r["load"]), prob_sum=torch.from_numpy(r["prob_sum"]))

    def dispatch(self, cfg, x, idx):
        C = self.orc.capacity(cfg.T, cfg.k, cfg.n, cfg.capacity_factor)
        r = self.orc.dispatch(idx.numpy(), cfg.n, C)
        xp = torch.zeros(max(cfg.T * cfg.k, 1), cfg.d, dtype=torch.float64)
        R = int(r["offsets"][-1])
        xp[:R] = x.double()[torch.from_numpy(r["perm_token"]).long()]
        return dict(counts=torch.from_numpy(r["counts"]), offsets=torch.from_numpy(r["offsets"]),
                    row_of=torch.from_numpy(r["row_of"]), x_perm=xp)

    def gather_rows(self, src, index):
        return src[index.long()]

    def expert_ffn(self, cfg, rows, offsets, params):
        y = torch.zeros(rows.shape[0], cfg.d, dtype=torch.float64)
        off = offsets.numpy()
        for e in range(cfg.n):
            for r in range(int(off[e]), int(off[e + 1])):
                y[r] = torch.from_numpy(self.orc.expert_row(
                    rows[r].float().numpy(), _np(params["W1"][e]), params["b1"][e].numpy(),
                    _np(params["W2"][e]), params["b2"][e].numpy(), bf16=bool(self.w.expert_bf16)))
        return y

    def combine(self, cfg, y_perm, gate, row_of, x):
        R = int((row_of >= 0).sum())
        return torch.from_numpy(self.orc.combine(y_perm[:max(R, 1)].numpy(), gate.numpy(), row_of.numpy(),
                                                 x.numpy(), passthrough=bool(cfg.passthrough)))

    def importance(self, cfg, idx, gate, counts, load, prob_sum):
        imp, _ = self.orc.balance(cfg.n, idx.numpy(), gate.numpy(), counts.numpy(), load.numpy())
        return torch.from_numpy(imp)

    def totals(self, cfg, importance, load, counts, prob_sum, dropped):
        imp, ld = importance.double().numpy(), load.double().numpy()
        aux = 0.0
        if cfg.router == 1:
            aux = cfg.n * float(np.sum(counts.numpy() / cfg.T * prob_sum.double().numpy() / cfg.T))
        dr = float(dropped[0])
        ci, cl = self.orc.cv2(imp), self.orc.cv2(ld)
        return torch.tensor([cfg.w_importance * ci, cfg.w_load * cl, aux, cfg.alpha * aux,
                             dr / (cfg.T * cfg.k), ci, cl, dr, 0.0, 0.0], dtype=torch.float64)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, case, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import oracle as orc
        w = CASES[case]
        full = synth.make_inputs(w)
        splits = SPLITS[case]
        base = sum(splits[:rank])
        m = w.n // world
        params = {k: full[k] for k in ("Wg", "bg", "Wn", "sel_bias")}
        params.update({k: full[k][rank * m:(rank + 1) * m] for k in ("W1", "b1", "W2", "b2")})
        cfg = M.Config.from_workload(w.with_(T=splits[rank]))
        layer = ExpertParallelMoE(cfg, params, steps=OracleSteps(orc, w, full), device="cpu")
        assert layer.cfg.token_base == base and layer.T_all == w.T
        out = layer.forward(full["x"][base:base + splits[rank]].contiguous())
        torch.save({k: (v if not torch.is_tensor(v) else v.clone()) for k, v in out.items()},
                   os.path.join(outdir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def _run(case, tmp_path):
    mp.start_processes(_worker, args=(2, _free_port(), case, str(tmp_path)), nprocs=2,
                       start_method="spawn")
    return [torch.load(os.path.join(tmp_path, f"rank{r}.pt")) for r in range(2)]


@pytest.mark.parametrize("case", list(CASES))
def test_two_ranks_match_the_oracle(orc, case, tmp_path):
    w = CASES[case]
    outs = _run(case, tmp_path)
    y = torch.cat([o["y"] for o in outs]).numpy()
    idx = torch.cat([o["topk_idx"] for o in outs]).numpy()
    gate = torch.cat([o["topk_gate"] for o in outs]).numpy()
    full = synth.make_inputs(w)
    npin = {k: _np(v) for k, v in full.items()}
    splits = SPLITS[case]
    # rows really crossed: some of each rank's rows went to the other rank's experts
    assert all(o["rows_sent"] > 0 for o in outs)
    if w.capacity_factor <= 0:
        ref = orc.forward(w.cfg(), npin)                      # the layer on the whole batch
        assert np.array_equal(idx, ref["topk_idx"])
        np.testing.assert_allclose(gate, ref["topk_gate"], rtol=1e-12)
        np.testing.assert_allclose(y, ref["y"], rtol=1e-10, atol=1e-12)
        counts_ref, imp_ref, load_ref, losses_ref = ref["counts"], ref["importance"], ref["load"], ref["losses"]
    else:
        # each shard cuts at its own capacity: the reference composed from the
        # oracle's whole-batch gate and per-shard dispatches
        g = orc.gate_batch(w.cfg(), npin)
        assert np.array_equal(idx, g["topk_idx"])
        y_ref, dropped, base = [], 0, 0
        for T_r in splits:
            sl = slice(base, base + T_r)
            C = orc.capacity(T_r, w.k, w.n, w.capacity_factor)
            dd = orc.dispatch(g["topk_idx"][sl], w.n, C)
            dropped += int(np.maximum(dd["counts"].astype(np.int64) - C, 0).sum())
            Y = np.zeros((max(len(dd["perm_token"]), 1), w.d))
            for r, t in enumerate(dd["perm_token"]):
                e = int(g["topk_idx"][base + t][dd["perm_slot"][r]])
                Y[r] = orc.expert_row(npin["x"][base + t], npin["W1"][e], npin["b1"][e], npin["W2"][e],
                                      npin["b2"][e], bf16=bool(w.expert_bf16))
            y_ref.append(orc.combine(Y, g["topk_gate"][sl], dd["row_of"], npin["x"][sl],
                                     passthrough=bool(w.passthrough)))
            base += T_r
        np.testing.assert_allclose(y, np.concatenate(y_ref), rtol=1e-10, atol=1e-12)
        counts_ref = np.bincount(g["topk_idx"].ravel(), minlength=w.n)
        imp_ref, losses_ref = orc.balance(w.n, g["topk_idx"], g["topk_gate"], counts_ref, g["load"],
                                          g["prob_sum"], 2**62, w.router, w.w_importance, w.w_load,
                                          w.alpha)
        load_ref = g["load"]
        losses_ref = np.array(losses_ref)
        losses_ref[4] = dropped / (w.T * w.k)
        losses_ref[7] = dropped
        assert dropped > 0
    for o in outs:  # every rank holds the whole batch's statistics
        assert np.array_equal(o["counts"].numpy(), counts_ref)
        np.testing.assert_allclose(o["importance"].numpy(), imp_ref, rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(o["load"].numpy(), load_ref, rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(o["losses"].numpy()[:8], np.asarray(losses_ref)[:8], rtol=1e-5,
                                   atol=1e-7)


def test_regroup_index_is_expert_major_and_invertible():
    rng = np.random.default_rng(0)
    for R, m in [(1, 1), (2, 3), (4, 5), (3, 1)]:
        cnt = rng.integers(0, 4, size=(R, m))
        cnt[0, 0] = 0
        g2r, r2g, off = regroup_index(cnt)
        total = int(cnt.sum())
        assert sorted(g2r.tolist()) == list(range(total))
        assert np.array_equal(g2r[r2g], np.arange(total))
        # received rows carry (rank, expert, i) in the exchange's order
        tags = [(s, j, i) for s in range(R) for j in range(m) for i in range(cnt[s, j])]
        grouped = [tags[r] for r in g2r]
        assert grouped == sorted(grouped, key=lambda t: (t[1], t[0], t[2]))
        assert list(off) == [0] + list(np.cumsum(cnt.sum(axis=0)))
