"""A forward captured into a CUDA graph and replayed gives the same bits as
the same forward launched from the host, reads its input at replay time, and
its stage events (external records) still time the replay."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import mixture_experts_layer_37_b200 as M
import workloads as W
from gpu_common import SMALL_WORKLOADS, to_dev, weights_dev

pytestmark = pytest.mark.gpu

GRAPH_CASES = [
    SMALL_WORKLOADS[0],  # SwiGLU, ragged, drops
    SMALL_WORKLOADS[1],  # GELU + bias, k=3
    SMALL_WORKLOADS[6],  # 16 experts: tensor-core router
]

OUT_KEYS = ("out", "topk_idx", "topk_w", "counts", "offsets", "slot", "f", "p", "l_aux")


def _snapshot(outputs):
    return {k: outputs[k].clone() for k in OUT_KEYS}


@pytest.mark.parametrize("wl", GRAPH_CASES, ids=lambda w: w.name)
def test_graph_replay_is_bitwise_eager(wl):
    cfg = M.MoEConfig.of(wl)
    inp = W.make_inputs(wl)
    wd = weights_dev(wl, inp)
    x = to_dev(inp["x"])
    inp2 = W.make_inputs(wl, seed=wl.seed + 77, with_experts=False)
    x2 = to_dev(inp2["x"])

    eager = M.MoELayer(cfg, wd)
    ref1 = _snapshot(eager.forward(x))
    ref2 = _snapshot(eager.forward(x2))
    torch.cuda.synchronize()

    layer = M.MoELayer(cfg, wd)
    buf = x.clone()
    layer.capture(buf)
    for _ in range(2):
        layer.replay()
    torch.cuda.synchronize()
    layer.check()
    got = _snapshot(layer.outputs)
    for k in OUT_KEYS:
        assert torch.equal(got[k], ref1[k]), k
    # the replay reads the buffer as it is now
    buf.copy_(x2)
    layer.replay()
    torch.cuda.synchronize()
    got = _snapshot(layer.outputs)
    for k in OUT_KEYS:
        assert torch.equal(got[k], ref2[k]), k


def test_profiled_events_time_a_graph_replay():
    wl = SMALL_WORKLOADS[0]
    cfg = M.MoEConfig.of(wl)
    inp = W.make_inputs(wl)
    wd = weights_dev(wl, inp)
    x = to_dev(inp["x"])
    layer = M.MoELayer(cfg, wd)
    ref = layer.forward(x)["out"].clone()
    n = M.moe_forward_launch_count(cfg)
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n + 1)]
    for e in evs:
        e.record()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        M.moe_forward_profiled(cfg, wd, x, layer.outputs, layer.ws, evs)
    layer.outputs["out"].zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(layer.outputs["out"], ref)
    stages = [evs[i].elapsed_time(evs[i + 1]) for i in range(n)]
    assert all(np.isfinite(s) and s >= 0.0 for s in stages), stages
    assert sum(stages) > 0.0
