"""The two warp-MMA routers against each other and against the oracle.

The resident-weight router (router_v2.cu: weight slices held across a CTA
cluster, tokens streamed by TMA, partial sums exchanged through distributed
shared memory) computes every logit with the same sequence of tensor-core
steps as the slab-staged router (router.cu), so their logits must agree bit
for bit on every shape: E not a multiple of 8, more than 32 experts (two
experts per lane in the finish), clusters of 2, 4 and 8 CTAs (expert splits
for small batches), d with a half block pair at the end (d % 128 == 64), a
ragged last tile, one token.  Their softmax sums differ only in summation
order, so probabilities and weights agree within 1e-6; selections and the
dispatch that follows are compared bit for bit, and both against the oracle
within the fp32 accumulation bound."""
import dataclasses

import numpy as np
import pytest
import torch

import mixture_experts_layer_37_b200 as M
import workloads as W
from oracle import moe_oracle as O
from gpu_common import logit_error_bound, rel_close, to_dev, weights_dev

pytestmark = pytest.mark.gpu

CASES = [
    W.Workload("r_e6", T=1000, d=256, ffn=64, E=6, k=2, act="swiglu", dtype="bf16", capacity_factor=1.0, seed=401),
    W.Workload("r_e8_t1", T=1, d=128, ffn=64, E=8, k=2, act="swiglu", dtype="bf16", capacity_factor=1.0, seed=402),
    W.Workload("r_e16_half_pair", T=777, d=4160, ffn=64, E=16, k=3, act="swiglu", dtype="bf16",
               capacity_factor=1.0, seed=403),
    W.Workload("r_e24", T=300, d=192, ffn=64, E=24, k=4, act="swiglu", dtype="bf16", capacity_factor=1.0, seed=404),
    W.Workload("r_e40", T=513, d=320, ffn=64, E=40, k=5, act="swiglu", dtype="bf16", capacity_factor=1.0, seed=405),
    W.Workload("r_e64_big_d", T=1000, d=4096, ffn=64, E=64, k=8, act="swiglu", dtype="bf16", capacity_factor=1.0,
               seed=406),
    W.Workload("r_e32_zipf_pad", T=2049, d=512, ffn=64, E=32, k=2, act="swiglu", dtype="bf16", capacity_factor=1.0,
               zipf_router_bias=True, pad_fraction=0.2, seed=407),
    W.WORKLOADS["llama4moe_t4096"].with_(ffn=64, name="r_llama4moe_router"),
    W.WORKLOADS["decode_t64_e64"].with_(ffn=64, name="r_decode_router"),
    W.WORKLOADS["longctx_zipf_t32768"].with_(ffn=64, name="r_longctx_router"),
]


def _route(cfg, wl, x, wd, tm, logits_in=None):
    T, E, k = wl.T, wl.E, wl.k
    ws = M.Workspace(cfg)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    lo = torch.empty((T, E), dtype=torch.float32, device="cuda")
    pr = torch.empty((T, E), dtype=torch.float32, device="cuda")
    M.moe_router_topk(cfg, x, wd["w_router"], wd.get("router_bias"), logits_in, idx, tw, lo, pr, ws, token_mask=tm)
    torch.cuda.synchronize()
    assert M.moe_check_device_status(ws)[0] == M.MOE_OK
    return idx.cpu().numpy(), tw.cpu().numpy(), lo.cpu().numpy(), pr.cpu().numpy()


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_resident_router_equals_staged_router(wl):
    inp = W.make_inputs(wl)
    wd = weights_dev(wl, inp)
    x = to_dev(inp["x"])
    tm = None if inp.get("token_mask") is None else to_dev(inp["token_mask"])
    v2 = _route(M.MoEConfig.of(wl, router_kernel="warp_mma"), wl, x, wd, tm)
    st = _route(M.MoEConfig.of(wl, router_kernel="warp_mma_staged"), wl, x, wd, tm)
    assert np.array_equal(v2[2].view(np.int32), st[2].view(np.int32)), "logits differ between the warp routers"
    assert np.array_equal(v2[0], st[0])
    assert rel_close(v2[1], st[1], rtol=1e-6, atol=1e-30)[0]
    assert rel_close(v2[3], st[3], rtol=1e-6, atol=1e-30)[0]
    # against the oracle: logits within the fp32 accumulation bound
    r = O.route(wl, inp)
    toks = np.arange(wl.T) if wl.T <= 4096 else np.random.default_rng(5).choice(wl.T, 4096, replace=False)
    err = np.abs(v2[2][toks].astype(np.float64) - r["logits64"][toks])
    assert (err <= logit_error_bound(wl, inp, toks)).all()
    # fed logits: both selection paths give the oracle's indices
    feed = to_dev(r["logits"].astype(np.float32))
    for router in ("warp_mma", "warp_mma_staged"):
        got = _route(M.MoEConfig.of(wl, router_kernel=router), wl, x, wd, tm, logits_in=feed)
        assert np.array_equal(got[0], r["idx"])
        assert rel_close(got[1], r["w"])[0] and rel_close(got[3], r["p"])[0]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_resident_router_forward_equals_staged(wl):
    """Whole forwards (fused dispatch scan, statistics) on both warp routers:
    routing, counts, offsets, slots bit for bit; statistics within 1e-6, the
    layer output within one bf16 rounding; each router's second launch on the
    same workspace repeats its first bit for bit (its counters return to zero)."""
    inp = W.make_inputs(wl)
    wd = weights_dev(wl, inp)
    x = to_dev(inp["x"])
    tm = None if inp.get("token_mask") is None else to_dev(inp["token_mask"])
    outs = []
    for router in ("warp_mma", "warp_mma_staged"):
        # routing weights applied in the combine (one rounding per output), so that
        # last-bit differences of the weights move an output by one rounding at most
        cfg = dataclasses.replace(M.MoEConfig.of(wl, router_kernel=router), weighting="combine")
        layer = M.MoELayer(cfg, wd)
        o = layer.forward(x, token_mask=tm)
        layer.check()
        outs.append({n: v.clone().cpu() for n, v in o.items()})
        o2 = layer.forward(x, token_mask=tm)  # a second launch on the same workspace: counters back to zero
        layer.check()
        for n in ("topk_idx", "counts", "offsets", "slot", "out"):
            assert torch.equal(o2[n].cpu(), outs[-1][n]), f"{router}: {n} differs on the second launch"
    a, b = outs
    R = int(a["offsets"][-1])
    for n in ("topk_idx", "counts", "offsets", "slot"):
        assert torch.equal(a[n], b[n]), n
    assert torch.equal(a["src_assign"][:R], b["src_assign"][:R])
    # the combine weights differ in their last fp32 bits (softmax summation
    # order), so a bf16 output may round one unit in the last place apart
    # (and near-zero outputs, sums that cancel, by a little more: an absolute floor)
    oa, ob = a["out"].double(), b["out"].double()
    floor = 1e-4 * float(oa.abs().max())
    assert ((oa - ob).abs() <= 2.0 ** -7 * torch.maximum(oa.abs(), ob.abs()) + floor).all()
    for n in ("f", "p", "l_aux"):
        assert rel_close(a[n].numpy(), b[n].numpy(), rtol=1e-6, atol=1e-30)[0], n
