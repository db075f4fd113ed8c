"""The expert-parallel layer with the CUDA steps.

Two processes on the one GPU, gloo between them (rows staged through host
memory; no kernel of one process waits on the other's), each with its own
shard of the batch and half of the experts; and one process alone over NCCL
(its exchanges are local).  Every row is computed by the same kernels as in
the single-device layer and rows do not interact in them, so the tokens'
expert ids, gates and outputs must equal, bit for bit, those of moe_forward
on the whole batch (with a capacity limit: on each shard, as each shard cuts
at its own capacity); the statistics summed over the ranks within 1e-5.
Not measured on more than one GPU.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparsely_gated_mixture_gate_b200 import build, synth
from sparsely_gated_mixture_gate_b200 import moe as M
from sparsely_gated_mixture_gate_b200.expert_parallel import ExpertParallelMoE

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
CASES = {
    "noisy": W["lm-flat"].with_(T=512, d=256, n=64, k=4, f=512),
    "switch-capacity": synth.VARIANTS["switch-skew"].with_(T=1024, d=256, n=32, f=512),
    "sigmoid": synth.VARIANTS["deepseek-flat"].with_(T=384, shared_expert=0, n=32, f=256),
}
SPLITS = {"noisy": [200, 312], "switch-capacity": [512, 512], "sigmoid": [384 // 2, 384 // 2]}


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, backend, case, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group(backend, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        w = CASES[case]
        full = synth.make_inputs(w, device="cuda")
        splits = SPLITS[case] if world == 2 else [w.T]
        base = sum(splits[:rank])
        m = w.n // world
        params = {k: full[k] for k in ("Wg", "bg", "Wn", "sel_bias")}
        params.update({k: full[k][rank * m:(rank + 1) * m].contiguous() for k in ("W1", "b1", "W2", "b2")})
        cfg = M.Config.from_workload(w.with_(T=splits[rank]))
        layer = ExpertParallelMoE(cfg, params)
        out = layer.forward(full["x"][base:base + splits[rank]].contiguous())
        torch.cuda.synchronize()
        torch.save({k: (v.cpu() if torch.is_tensor(v) else v) for k, v in out.items()},
                   os.path.join(outdir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("backend,world", [("gloo", 2), ("nccl", 1)])
def test_expert_parallel_equals_the_single_device_layer(case, backend, world, tmp_path):
    mp.start_processes(_worker, args=(world, _free_port(), backend, case, str(tmp_path)),
                       nprocs=world, start_method="spawn")
    outs = [torch.load(os.path.join(tmp_path, f"rank{r}.pt")) for r in range(world)]
    w = CASES[case]
    full = synth.make_inputs(w, device="cuda")
    splits = SPLITS[case] if world == 2 else [w.T]
    if w.capacity_factor > 0:  # every shard cuts at its own capacity: the shard's own layer
        refs, base = [], 0
        for T_r in splits:
            import dataclasses
            cfg = dataclasses.replace(M.Config.from_workload(w.with_(T=T_r)), token_base=base)
            layer = M.MoELayer(cfg, full, torch.device("cuda"))
            layer.forward_(full["x"][base:base + T_r].contiguous())
            torch.cuda.synchronize()
            refs.append({k: v.cpu().clone() for k, v in layer.outputs().items()})
            base += T_r
        ref_cat = {k: torch.cat([r[k] for r in refs]) for k in ("y", "topk_idx", "topk_gate")}
    else:
        layer = M.MoELayer(M.Config.from_workload(w), full, torch.device("cuda"))
        layer.forward_(full["x"])
        torch.cuda.synchronize()
        ref_cat = {k: v.cpu() for k, v in layer.outputs().items()}
        for o in outs:
            assert torch.equal(o["counts"], ref_cat["counts"])
            np.testing.assert_allclose(o["importance"].numpy(), ref_cat["importance"].numpy(),
                                       rtol=1e-5, atol=1e-6)
            np.testing.assert_allclose(o["load"].numpy(), ref_cat["load"].numpy(), rtol=1e-5,
                                       atol=1e-6 * w.T)
            np.testing.assert_allclose(o["losses"].numpy()[:8], ref_cat["losses"].numpy()[:8],
                                       rtol=1e-5, atol=1e-7)
    for key in ("topk_idx", "topk_gate", "y"):
        got = torch.cat([o[key] for o in outs])
        assert torch.equal(got, ref_cat[key]), key
    if world == 2:
        assert all(o["rows_sent"] > 0 and o["rows_received"] > 0 for o in outs)
