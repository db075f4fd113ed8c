"""Expert-parallel forward of the Sparsely-Gated MoE layer over the ranks of a
torch.distributed process group.

The pages' multi-device scheme ("MoE 稀疏架构深度解析" §7.1; the reading note
"Outrageously Large Neural Networks", 工程优化): the gate and every per-token
step run data-parallel, each rank on its own shard of the batch; the experts
are spread over the ranks; two all-to-all exchanges per layer carry each kept
(token, slot) row to the rank that holds its expert and the expert's output
back.  Rank r holds experts [r*m, (r+1)*m), m = n / R: contiguous blocks, so
the dispatch's expert-sorted rows are already grouped by destination rank.

One forward, on every rank, in this order (the same collectives on every
rank, in the same order):
  1. gate (moe_gate) on the rank's tokens, token_base = the index of the
     shard's first token in the batch, so every token draws the noise it
     would draw in the whole batch;
  2. dispatch (moe_dispatch): per-expert counts and the kept rows sorted by
     expert; capacity, when set, is the shard's own, C = ceil(T_r k cf / n)
     (the batch a device sees is its shard);
  3. the kept row counts per expert go to the experts' ranks (all-to-all of
     m integers between every pair of ranks);
  4. the rows follow (all-to-all with those split sizes, bf16 rows moved as
     int32 pairs), and the received rows are regrouped by local expert
     (moe_gather_rows with an index built on the host from the counts);
  5. the rank's experts run on their rows (moe_expert_ffn);
  6. the outputs go back to the received order (moe_gather_rows, inverse
     index) and to the ranks they came from (the reverse all-to-all);
  7. combine (moe_combine) on the rank's tokens;
  8. statistics of the whole batch: the shard's Importance (moe_balance_losses),
     Load, counts, Switch probability sums and dropped slots summed over the
     ranks (all-reduce), then the losses (moe_balance_from_totals).

Flat layers (noisy top-k, Switch, sigmoid router) without a shared expert.
Transport: with the NCCL backend the collectives run on the CUDA tensors;
with any other backend (gloo) the rows are staged through host memory.  The
compute steps are the CUDA library's (CudaSteps); the class only moves rows
and bookkeeping, so the CPU tests can run the same exchanges with other
steps.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch
import torch.distributed as dist

from . import moe as M


class CudaSteps:
    """The layer's steps, each one C-ABI call of the CUDA library."""

    def gate(self, cfg, x, params):
        return M.gate(cfg, x, params)

    def dispatch(self, cfg, x, idx):
        return M.dispatch(cfg, x, idx)

    def gather_rows(self, src, index):
        return M.gather_rows(src, index)

    def expert_ffn(self, cfg, rows, offsets, params):
        return M.expert_ffn(cfg, rows, offsets, params)["y_perm"]

    def combine(self, cfg, y_perm, gate, row_of, x):
        return M.combine(cfg, y_perm, gate, row_of, x)["y"]

    def importance(self, cfg, idx, gate, counts, load, prob_sum):
        return M.balance_losses(cfg, idx, gate, counts, load, prob_sum)["importance"]

    def totals(self, cfg, importance, load, counts, prob_sum, dropped):
        return M.balance_from_totals(cfg, importance, load, counts, prob_sum, dropped)


def regroup_index(cnt: np.ndarray):
    """cnt[s][j]: rows received from rank s for local expert j, in the order
    the exchange delivers them (rank by rank, expert by expert inside a
    rank).  Returns (to_grouped, to_received, offsets): grouped row g is
    received row to_grouped[g] (experts contiguous, ranks in order inside an
    expert), received row r is grouped row to_received[r], and offsets[j] is
    the first grouped row of local expert j (offsets[m] = all rows)."""
    R, m = cnt.shape
    flat = cnt.reshape(-1).astype(np.int64)             # blocks (s, j), received order
    total = int(flat.sum())
    r_start = np.concatenate([[0], np.cumsum(flat)[:-1]])
    per_expert = cnt.sum(axis=0).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(per_expert)]).astype(np.int32)
    # grouped start of block (s, j): expert j's first row + rows of ranks before s
    before = np.cumsum(cnt, axis=0) - cnt               # [s][j]: rows of ranks < s for expert j
    g_start = (offsets[:-1][None, :] + before).reshape(-1).astype(np.int64)
    block = np.repeat(np.arange(R * m), flat)
    within = np.arange(total, dtype=np.int64) - np.repeat(r_start, flat)
    to_received = (g_start[block] + within).astype(np.int32)   # received row -> grouped row
    to_grouped = np.empty(total, np.int32)
    to_grouped[to_received] = np.arange(total, dtype=np.int32)
    return to_grouped, to_received, offsets


class ExpertParallelMoE:
    """The flat layer with its n experts spread over the R ranks of `group`.

    cfg: the layer as on one device, with T the number of tokens of THIS
    rank's shard.  params: the gate weights (replicated: Wg, Wn, bg,
    sel_bias) and this rank's experts only: W1 [m][f][d], W2 [m][d][f],
    b1 [m][f], b2 [m][d], m = n / R.  token_base: index of the shard's first
    token in the batch (default: the sum of the lower ranks' token counts).
    steps: the compute steps (default: the CUDA library)."""

    def __init__(self, cfg: M.Config, params: dict, group=None, token_base: Optional[int] = None,
                 steps=None, device=None):
        if cfg.hier_a or cfg.shared_expert:
            raise M.MoEError("the expert-parallel layer covers flat layers without a shared expert")
        self.group = group
        self.R = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if cfg.n % self.R:
            raise M.MoEError(f"n = {cfg.n} experts do not split over {self.R} ranks")
        self.m = cfg.n // self.R
        self.params = params
        self.steps = steps or CudaSteps()
        self.device = torch.device(device) if device is not None else params["Wg"].device
        self.nccl = dist.get_backend(group) == "nccl"
        # every rank's token count: the batch size and the default token base
        Ts = self._all_gather_int(cfg.T)
        self.T_all = int(sum(Ts))
        base = int(sum(Ts[:self.rank])) if token_base is None else int(token_base)
        self.cfg = dataclasses.replace(cfg, token_base=base)
        self.cfg_batch = dataclasses.replace(cfg, T=self.T_all, token_base=0)

    # ------------------------------------------------------------ transport
    def _comm(self, t: torch.Tensor) -> torch.Tensor:
        """A tensor the backend can exchange: device tensors for NCCL, host
        tensors otherwise."""
        return t if (self.nccl or not t.is_cuda) else t.cpu()

    def _back(self, t: torch.Tensor) -> torch.Tensor:
        return t.to(self.device) if t.device != self.device else t

    def _all_gather_int(self, v: int):
        t = torch.tensor([v], dtype=torch.int64,
                         device=self.device if dist.get_backend(self.group) == "nccl" else "cpu")
        out = [torch.zeros_like(t) for _ in range(self.R)]
        dist.all_gather(out, t, group=self.group)
        return [int(o.item()) for o in out]

    def _all_to_all(self, send: torch.Tensor, send_splits, recv_splits, cols: int, dtype):
        recv = torch.empty(int(sum(recv_splits)), cols, dtype=dtype,
                           device=send.device if (self.nccl or not send.is_cuda) else "cpu")
        dist.all_to_all_single(recv, self._comm(send), [int(v) for v in recv_splits],
                               [int(v) for v in send_splits], group=self.group)
        return self._back(recv)

    @staticmethod
    def _as_i32(rows: torch.Tensor) -> torch.Tensor:
        """bf16 / fp32 rows as int32 words (the exchange moves bits)."""
        return rows.contiguous().view(torch.int32)

    # ------------------------------------------------------------ forward
    def forward(self, x: torch.Tensor) -> dict:
        cfg, R, m, st = self.cfg, self.R, self.m, self.steps
        T, k, n, d = cfg.T, cfg.k, cfg.n, cfg.d
        # 1-2: gate and dispatch of the shard
        g = st.gate(cfg, x, self.params)
        disp = st.dispatch(cfg, x, g["topk_idx"])
        edt = disp["x_perm"].dtype                                # the expert rows' type
        offsets = disp["offsets"].cpu().numpy().astype(np.int64)
        counts_h = disp["counts"].cpu().numpy().astype(np.int64)
        kept = np.diff(offsets)                                   # kept rows per expert
        send_splits = kept.reshape(R, m).sum(axis=1)              # rows to every rank
        # 3: kept counts per expert to the experts' ranks
        kc = torch.from_numpy(kept.astype(np.int32)).view(n, 1)
        kc = kc.to(self.device) if self.nccl else kc
        cnt = self._all_to_all(kc, [m] * R, [m] * R, 1, torch.int32).view(R, m).cpu().numpy()
        recv_splits = cnt.sum(axis=1)
        # 4: rows to the experts' ranks, regrouped by local expert
        R_kept = int(offsets[-1])
        x_perm = disp["x_perm"][:R_kept]
        words = x_perm.element_size() * d // 4
        recv = self._all_to_all(self._as_i32(x_perm).view(R_kept, words), send_splits, recv_splits,
                                words, torch.int32).view(edt)
        to_grouped, to_received, off_local = regroup_index(cnt)
        S_recv = int(off_local[-1])
        dev = recv.device
        grouped = torch.zeros(max(S_recv, 1), d, dtype=edt, device=dev)
        if S_recv:
            grouped[:S_recv] = st.gather_rows(recv, torch.from_numpy(to_grouped).to(dev))
        # 5: this rank's experts
        cfg_local = dataclasses.replace(cfg, T=max(S_recv, 1), k=1, n=m, capacity_factor=0.0,
                                        token_base=0)
        y_grouped = st.expert_ffn(cfg_local, grouped, torch.from_numpy(off_local).to(dev),
                                  self.params)
        # 6: back to the received order and to the ranks the rows came from
        ydt = y_grouped.dtype
        y_recv = (st.gather_rows(y_grouped[:max(S_recv, 1)], torch.from_numpy(to_received).to(dev))
                  if S_recv else torch.zeros(0, d, dtype=ydt, device=dev))
        ywords = y_recv.element_size() * d // 4
        y_back = self._all_to_all(self._as_i32(y_recv).view(S_recv, ywords), recv_splits,
                                  send_splits, ywords, torch.int32).view(ydt)
        y_perm = torch.zeros(max(T * k, 1), d, dtype=ydt, device=dev)
        y_perm[:R_kept] = y_back
        # 7: combine the shard's tokens
        y = st.combine(cfg, y_perm, g["topk_gate"], disp["row_of"], x)
        # 8: statistics of the whole batch
        sw = cfg.router == M._lib.ROUTER_SWITCH
        psum = g["prob_sum"] if sw else None
        imp = st.importance(cfg, g["topk_idx"], g["topk_gate"], disp["counts"], g["load"], psum)
        C = M.capacity(cfg) if cfg.capacity_factor > 0 else None
        dropped = float(np.maximum(counts_h - C, 0).sum()) if C is not None else 0.0
        fl = torch.cat([imp.float().reshape(-1), g["load"].float().reshape(-1),
                        (psum if psum is not None else torch.zeros_like(g["load"])).float().reshape(-1),
                        torch.tensor([dropped], dtype=torch.float32, device=imp.device)])
        fl = self._comm(fl)
        dist.all_reduce(fl, op=dist.ReduceOp.SUM, group=self.group)
        ci = self._comm(disp["counts"].to(torch.int32).clone())
        dist.all_reduce(ci, op=dist.ReduceOp.SUM, group=self.group)
        fl, ci = self._back(fl), self._back(ci)
        importance, load, psum_g, dropped_g = fl[:n], fl[n:2 * n], fl[2 * n:3 * n], fl[3 * n:]
        losses = st.totals(self.cfg_batch, importance, load, ci, psum_g if sw else None, dropped_g)
        return dict(y=y, topk_idx=g["topk_idx"], topk_gate=g["topk_gate"], importance=importance,
                    load=load, counts=ci, losses=losses, rows_sent=R_kept, rows_received=S_recv)
