"""The bench line's routing report: the load histogram summary, the losses
and the drop rate, read from a layer's outputs (a stand-in layer on the CPU)."""
import os
import sys
import types

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def _layer(counts, losses):
    return types.SimpleNamespace(counts=torch.tensor(counts, dtype=torch.int32),
                                 losses=torch.tensor(losses, dtype=torch.float32))


def test_routing_report_noisy():
    import bench
    w = types.SimpleNamespace(router=0)
    losses = [0.5, 0.25, 0.0, 0.0, 0.125, 5.0, 2.5, 3.0, 0.0, 0.0]
    rep = bench.routing_report(w, _layer([0, 2, 4, 6], losses))
    assert rep["counts"] == {"experts": 4, "min": 0, "max": 6, "mean": 3.0,
                             "std": round(5.0 ** 0.5, 3), "max_over_mean": 2.0, "empty_experts": 1}
    assert rep["L_importance"] == 0.5 and rep["L_load"] == 0.25
    assert rep["cv2_importance"] == 5.0 and rep["cv2_load"] == 2.5
    assert rep["drop_rate"] == 0.125 and rep["dropped_slots"] == 3
    assert "L_aux" not in rep


def test_routing_report_switch_and_empty():
    import bench
    w = types.SimpleNamespace(router=1)
    losses = [0.0, 0.0, 1.5, 0.015, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0]
    rep = bench.routing_report(w, _layer([0, 0], losses))
    assert rep["counts"]["mean"] == 0.0 and rep["counts"]["max_over_mean"] is None
    assert rep["counts"]["empty_experts"] == 2
    assert rep["switch_aux"] == 1.5 and abs(rep["L_aux"] - 0.015) < 1e-9
