"""moe_pipeline_*: each step's host results equal moe_forward on the same
batch bit for bit, whatever the depth and with steps in flight together."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import mixture_experts_layer_37_b200 as M
import workloads as W
from gpu_common import SMALL_WORKLOADS, to_dev, weights_dev

pytestmark = pytest.mark.gpu


def _pinned(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()
    return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()


@pytest.mark.parametrize("depth", [1, 2, 3])
@pytest.mark.parametrize("wl", [SMALL_WORKLOADS[0], SMALL_WORKLOADS[3], SMALL_WORKLOADS[6]], ids=lambda w: w.name)
def test_pipeline_steps_equal_forward(wl, depth):
    cfg = M.MoEConfig.of(wl)
    inp = W.make_inputs(wl)
    wd = weights_dev(wl, inp)
    steps = 6
    xs = [inp["x"]] + [W.make_inputs(wl, seed=wl.seed + 1000 + i, with_experts=False)["x"] for i in range(steps - 1)]
    layer = M.MoELayer(cfg, wd)
    want = []
    for x in xs:
        o = layer.forward(to_dev(x))
        want.append((o["out"].cpu().clone(), o["l_aux"].cpu().clone()))
    torch.cuda.synchronize()

    x_host = [_pinned(x) for x in xs]
    out_host = [torch.empty_like(x).pin_memory() for x in x_host]
    l_host = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in xs]
    with M.Pipeline(cfg, wd, depth=depth) as pipe:
        tickets = [pipe.submit(x_host[i], out_host[i], l_host[i]) for i in range(steps)]
        assert tickets == list(range(steps))
        pipe.wait(0)
        assert torch.equal(out_host[0], want[0][0]) and torch.equal(l_host[0], want[0][1])
        pipe.wait()
        pipe.check()
        for i in range(steps):
            assert torch.equal(out_host[i], want[i][0]), f"step {i} output"
            assert torch.equal(l_host[i], want[i][1]), f"step {i} l_aux"
        with pytest.raises(M.MoEError):
            pipe.wait(steps)  # not submitted


def test_pipeline_empty_batch():
    wl = W.Workload("empty", T=0, d=128, ffn=128, E=4, k=2, act="swiglu", dtype="bf16", capacity_factor=1.0)
    cfg = M.MoEConfig.of(wl)
    inp = W.make_inputs(wl)
    wd = weights_dev(wl, inp)
    l_host = torch.full((1,), 7.0, dtype=torch.float32).pin_memory()
    empty = torch.empty((0, 128), dtype=torch.bfloat16).pin_memory()
    with M.Pipeline(cfg, wd) as pipe:
        pipe.submit(empty, empty, l_host)
        pipe.wait()
        pipe.check()
    assert float(l_host[0]) == 0.0
