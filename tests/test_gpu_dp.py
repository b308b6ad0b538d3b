"""Data-parallel shards of one batch, emulated on one GPU: every shard runs
moe_dp_route, the counts and probability sums are stacked in rank order (the
all-gather), and every shard runs moe_dp_finish.  The concatenated results
must equal one moe_forward over the whole batch bit for bit (routing, drops,
layer output), with the whole batch's statistics; and the layer output must
match the oracle."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_37_b200 as M
import workloads as W
from oracle import moe_oracle as O
from gpu_common import host_f64, mask_dev, out_close, rel_close, sample_tokens, to_dev, weights_dev

pytestmark = pytest.mark.gpu

CASES = [
    (W.Workload("dp_zipf_drops", T=1000, d=128, ffn=192, E=16, k=2, act="swiglu", dtype="bf16",
                capacity_factor=0.6, zipf_router_bias=True, seed=301, w_std=0.05), [0, 300, 301, 777, 1000]),
    (W.Workload("dp_gelu_k3", T=600, d=192, ffn=256, E=5, k=3, act="gelu_bias", dtype="bf16",
                capacity_factor=0.9, seed=302), [0, 333, 600]),
    (W.WORKLOADS["longctx_zipf_t32768"], [0, 8192, 16384, 24576, 32768]),
    (W.Workload("dp_shared_pad", T=900, d=128, ffn=192, E=8, k=2, act="swiglu", dtype="bf16",
                capacity_factor=0.8, n_shared=1, pad_fraction=0.2, seed=303), [0, 450, 451, 900]),
]


PARAMS = [(wl, b, "auto") for wl, b in CASES] + [(wl, b, "tcgen05") for wl, b in CASES if wl.E % 8 == 0]


@pytest.mark.parametrize("wl,bounds,router", PARAMS,
                         ids=[f"{w.name}-{len(b) - 1}-{r}" for w, b, r in PARAMS])
def test_dp_shards_equal_whole_batch(wl, bounds, router):
    inp = W.make_inputs(wl)
    wd = weights_dev(wl, inp)
    x = to_dev(inp["x"])
    cfg = M.MoEConfig.of(wl, router)
    mask = mask_dev(inp)
    whole = M.MoELayer(cfg, wd).forward(x, token_mask=mask)
    torch.cuda.synchronize()
    world = len(bounds) - 1
    shards = []
    for r in range(world):
        t0, t1 = bounds[r], bounds[r + 1]
        c = M.MoEConfig(T=t1 - t0, d=wl.d, ffn=wl.ffn, E=wl.E, k=wl.k, dtype=wl.dtype, act=wl.act,
                        capacity_factor=wl.capacity_factor, aux_alpha=wl.aux_alpha, router_kernel=router,
                        n_shared=wl.n_shared)
        o = M.allocate_outputs(c)
        o["src_assign"] = torch.empty(max(M.moe_dp_max_rows(c, wl.T), 1), dtype=torch.int32, device="cuda")
        ws = M.Workspace(c, nbytes=M.moe_dp_workspace_size(c, wl.T))
        lc = torch.zeros(wl.E, dtype=torch.int32, device="cuda")
        lp = torch.zeros(wl.E, dtype=torch.float64, device="cuda")
        lr = torch.zeros(1, dtype=torch.int32, device="cuda")
        M.moe_dp_route(c, wl.T, wd, x[t0:t1], o, lc, lp, ws, token_mask=None if mask is None else mask[t0:t1],
                       local_real=lr)
        shards.append((c, o, ws, lc, lp, t0, t1, lr))
    all_counts = torch.stack([s[3] for s in shards])
    all_psum = torch.stack([s[4] for s in shards])
    all_real = torch.cat([s[7] for s in shards])
    assert all_real.sum().item() == (wl.T if mask is None else int(mask.sum().item()))
    for r, (c, o, ws, _, _, t0, t1, _) in enumerate(shards):
        M.moe_dp_finish(c, wl.T, all_counts, all_psum, world, r, wd, x[t0:t1], o, ws, all_real=all_real)
    torch.cuda.synchronize()
    for _, _, ws, *_ in shards:
        assert M.moe_check_device_status(ws)[0] == M.MOE_OK
    cat = lambda n: torch.cat([s[1][n] for s in shards]).cpu()  # noqa: E731
    assert torch.equal(cat("topk_idx"), whole["topk_idx"].cpu())
    assert torch.equal(cat("slot") >= 0, whole["slot"].cpu() >= 0)
    assert (whole["slot"] < 0).any(), "the case must exercise drops"
    assert torch.equal(cat("out").view(torch.int16), whole["out"].cpu().view(torch.int16)), "layer output differs"
    for c, o, *_ in shards:
        assert torch.equal(o["counts"].cpu(), whole["counts"].cpu())
        assert torch.equal(o["f"].cpu(), whole["f"].cpu())
        assert rel_close(o["p"].cpu().numpy(), whole["p"].cpu().numpy(), rtol=1e-6)[0]
        assert rel_close(o["l_aux"].cpu().numpy(), whole["l_aux"].cpu().numpy(), rtol=1e-6)[0]
    # and against the oracle (logits computed on the GPU, so compare where routing agrees)
    r_or = O.route(wl, inp)
    toks = np.arange(wl.T) if wl.T <= 2048 else sample_tokens(wl, r_or, n_random=128, per_expert=4)
    agree = (whole["topk_idx"].cpu().numpy() == r_or["idx"]).all(axis=1) & \
            ((whole["slot"].cpu().numpy() >= 0) == (r_or["slot"] >= 0)).all(axis=1)
    toks = toks[agree[toks]]
    ref = O.forward(wl, inp, routing=r_or, tokens=toks)
    if mask is not None:
        assert (mask == 0).any(), "the case must exercise padding"
    ok, e_, s_ = out_close(host_f64(cat("out"))[toks], ref["out"], wl.dtype)
    assert ok, f"max err {e_} vs scale {s_}"
