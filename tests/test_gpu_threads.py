"""Forwards issued from several host threads at once, each on its own stream
and workspace, give the same bits as one forward issued alone (the library's
per-device one-time setup is safe under concurrent first calls)."""
from __future__ import annotations

import threading

import pytest
import torch

import mixture_experts_layer_37_b200 as M
import workloads as W
from gpu_common import SMALL_WORKLOADS, to_dev, weights_dev

pytestmark = pytest.mark.gpu


def test_concurrent_host_threads():
    cases = [SMALL_WORKLOADS[0], SMALL_WORKLOADS[1], SMALL_WORKLOADS[6], SMALL_WORKLOADS[3]]
    prepared = []
    for wl in cases:
        inp = W.make_inputs(wl)
        prepared.append((M.MoEConfig.of(wl), weights_dev(wl, inp), to_dev(inp["x"])))
    # references, one at a time
    refs = []
    for cfg, wd, x in prepared:
        o = M.MoELayer(cfg, wd).forward(x)
        torch.cuda.synchronize()
        refs.append(o["out"].clone())
    results = [None] * len(prepared)
    errors = []

    def work(i):
        try:
            cfg, wd, x = prepared[i]
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                layer = M.MoELayer(cfg, wd)
                for _ in range(3):
                    o = layer.forward(x, stream=stream)
            stream.synchronize()
            layer.check(stream)
            results[i] = o["out"].clone()
        except Exception as exc:  # reported below
            errors.append(exc)

    threads = [threading.Thread(target=work, args=(i,)) for i in range(len(prepared))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    for i, ref in enumerate(refs):
        assert results[i] is not None and torch.equal(results[i], ref), f"case {i}"
