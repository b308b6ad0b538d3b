"""INT8 routed-expert weights (per-expert, per-output-column scales): the
quantiser's codes and scales bit for bit against the oracle's (the codes are
integers decided in fp32 on both sides), and the layer on INT8 weights
against the oracle's layer on the dequantised weights."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import mixture_experts_layer_37_b200 as M
import workloads as W
from oracle import moe_oracle as O
from gpu_common import SMALL_WORKLOADS, to_dev
from test_gpu_parity import _check_workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,which", [("decode_t64_e64", "w_gate"), ("decode_t64_e64", "w_down"),
                                        ("flat_gelu_t8192", "w2")])
def test_quantize_codes_and_scales_exact(name, which):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    w = inp[which]
    cfg = M.MoEConfig.of(wl)
    q, s = M.moe_quantize_int8(cfg, to_dev(w))
    torch.cuda.synchronize()
    qg, sg = q.cpu().numpy(), s.cpu().numpy()
    for e in range(min(wl.E, 8)):
        qo, so = O.quantize_int8(O.to_f64(w[e], wl.dtype).astype(np.float32))
        np.testing.assert_array_equal(sg[e].view(np.uint32), so.view(np.uint32))
        np.testing.assert_array_equal(qg[e], qo)


def test_quantize_edge_columns():
    """A zero column, a column of equal magnitudes, and values halfway between codes."""
    cfg = M.MoEConfig(T=8, d=64, ffn=64, E=1, k=1)
    w = np.zeros((1, 64, 64), dtype=np.float32)
    w[0, :, 1] = 3.0
    w[0, :, 2] = (np.arange(64, dtype=np.float32) - 31.5) / 127.0 * 2.0   # codes at x.5 of the grid
    w[0, 0, 3] = -5.0
    bits = (w.view(np.uint32) >> 16).astype(np.uint16)                     # bf16 bit patterns (exact here)
    q, s = M.moe_quantize_int8(cfg, to_dev(bits))
    torch.cuda.synchronize()
    qo, so = O.quantize_int8(O.to_f64(bits[0], "bf16").astype(np.float32))
    np.testing.assert_array_equal(s.cpu().numpy()[0].view(np.uint32), so.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy()[0], qo)
    assert (q.cpu().numpy()[0][:, 0] == 0).all() and float(s[0, 0]) == 0.0


INT8_CASES = [W.WORKLOADS["decode_t64_e64"].with_(weights="int8")] + \
    [w.with_(weights="int8") for w in SMALL_WORKLOADS if w.dtype == "bf16" and w.name in
     ("ragged_swiglu", "drops_gelu_k3", "single_token", "zipf_heavy_drops", "shared2_swiglu_pad")]


@pytest.mark.parametrize("wl", INT8_CASES, ids=lambda w: w.name)
def test_int8_layer_parity(wl):
    _check_workload(wl, full_size=wl.T > 4096)
