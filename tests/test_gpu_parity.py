"""GPU parity: every stage of the CUDA path against the CPU oracle, through the
C ABI, on the five benchmark workloads at full size and on small cases that
span several tiles, ragged tails, drops, k = E, E = 1, T = 1 and fp32.

Inputs come from the seeded generator; expected values come only from the
oracle.  Where both sides must take a discrete decision on identical values
(top-k, capacity ranks), the oracle's fp32 logits are fed to both."""
import dataclasses

import numpy as np
import pytest
import torch

import mixture_experts_layer_37_b200 as M
import workloads as W
from oracle import moe_oracle as O
from gpu_common import (SMALL_WORKLOADS, expert_rows_ref, host_f64, logit_error_bound, mask_dev, out_close, rel_close,
                        sample_tokens, to_dev, weights_dev)

pytestmark = pytest.mark.gpu

FULL = ["tiny_f32", "llama4moe_t4096", "flat_gelu_t8192", "longctx_zipf_t32768", "decode_t64_e64"]


def _cfg(wl, router="auto", gemm="auto"):
    return M.MoEConfig.of(wl, router, gemm)


def _check_workload(wl, full_size: bool, router: str = "auto", gemm: str = "auto"):
    # The tcgen05 router refuses fed logits (it has no GEMM-free path), so the
    # fed-logit steps 1, 7 and 8 run the warp router's selection; steps 2 and 9
    # (the router's own GEMM) run the kernel asked for.
    cfg = _cfg(wl, router, gemm)
    cfg_feed = _cfg(wl, "warp_mma" if router == "tcgen05" else router, gemm)
    T, E, k, d = wl.T, wl.E, wl.k, wl.d
    inp = W.make_inputs(wl)
    r = O.route(wl, inp)
    feed = r["logits"].astype(np.float32)
    wd = weights_dev(wl, inp)
    if wl.weights == "int8":
        wd = M.quantize_expert_weights(cfg, wd)
    x = to_dev(inp["x"])
    ws = M.Workspace(cfg)
    dev = lambda a: to_dev(np.ascontiguousarray(a))  # noqa: E731
    R = int(r["offsets"][-1])
    rows_cap = M.moe_max_rows(cfg)
    tm = mask_dev(inp)
    real = np.ones(T, dtype=bool) if tm is None else inp["token_mask"] != 0

    # ---- 1. router + softmax + top-k with identical logits: bit-exact indices
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    probs = torch.empty((T, E), dtype=torch.float32, device="cuda")
    M.moe_router_topk(cfg_feed, x, wd["w_router"], wd.get("router_bias"), dev(feed), idx, tw, None, probs, ws,
                      token_mask=tm)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), r["idx"]), "top-k indices differ on identical logits"
    ok, worst = rel_close(tw.cpu().numpy(), r["w"])
    assert ok, f"top-k weights rel err {worst}"
    ok, worst = rel_close(probs.cpu().numpy(), r["p"])
    assert ok, f"router probabilities rel err {worst}"

    # ---- 2. router GEMM on the GPU: logits within the fp32 accumulation bound;
    #         the chosen experts are the top-k of the GPU's own logits, and equal
    #         the oracle's wherever the oracle's k-th / (k+1)-th gap exceeds the bound
    lo = torch.empty((T, E), dtype=torch.float32, device="cuda")
    M.moe_router_topk(cfg, x, wd["w_router"], wd.get("router_bias"), None, idx, tw, lo, probs, ws, token_mask=tm)
    torch.cuda.synchronize()
    lg = lo.cpu().numpy().astype(np.float64)
    gi = idx.cpu().numpy()
    assert (gi[~real] == -1).all() and (tw.cpu().numpy()[~real] == 0).all(), "padding selected an expert"
    # the GPU's probabilities and weights are the softmax / renormalisation of its own logits
    pg = probs.cpu().numpy().astype(np.float64)
    z = np.exp(lg - lg.max(axis=1, keepdims=True))
    assert rel_close(pg, z / z.sum(axis=1, keepdims=True), rtol=1e-5, atol=1e-12)[0]
    sel = np.take_along_axis(pg[real], gi[real].astype(np.int64), axis=1)
    assert rel_close(tw.cpu().numpy()[real], sel / sel.sum(axis=1, keepdims=True), rtol=1e-5)[0]
    toks = np.arange(T) if T <= 8192 else np.random.default_rng(1).choice(T, 8192, replace=False)
    bound = logit_error_bound(wl, inp, toks)
    err = np.abs(lg[toks] - r["logits64"][toks])
    assert (err <= bound).all(), f"router logits error {err.max()} above bound"
    for t in np.nonzero(real)[0]:
        sel = set(gi[t].tolist())
        for j, e in enumerate(gi[t]):
            for u in range(E):
                if u not in sel:
                    assert lg[t, e] > lg[t, u] or (lg[t, e] == lg[t, u] and e < u)
            if j:
                pe = gi[t, j - 1]
                assert lg[t, pe] > lg[t, e] or (lg[t, pe] == lg[t, e] and pe < e)
    srt = np.sort(r["logits64"], axis=1)[:, ::-1]
    gap = srt[:, k - 1] - (srt[:, k] if k < E else -np.inf)
    full_bound = logit_error_bound(wl, inp, np.arange(T)) if T <= 8192 else None
    margin = 2 * (full_bound.max(axis=1) if full_bound is not None else bound.max())
    clear = (gap > margin) & real
    assert np.array_equal(np.sort(gi[clear], axis=1), np.sort(r["idx"][clear], axis=1))

    # ---- 3. dispatch with identical indices: bit-exact counts/offsets/slots/permutation, exact row copies
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    slot = torch.empty((T, k), dtype=torch.int32, device="cuda")
    src = torch.full((max(rows_cap, 1),), -7, dtype=torch.int32, device="cuda")
    xp = torch.zeros((max(rows_cap, 1), d), dtype=cfg.torch_dtype, device="cuda")
    M.moe_dispatch(cfg, x, dev(r["idx"]), counts, offsets, slot, src, xp, ws)
    torch.cuda.synchronize()
    assert np.array_equal(counts.cpu().numpy(), r["counts"])
    assert np.array_equal(offsets.cpu().numpy(), r["offsets"])
    assert np.array_equal(slot.cpu().numpy(), r["slot"])
    assert np.array_equal(src.cpu().numpy()[:R], r["src_assign"])
    xin = inp["x"]
    xp_np = xp.cpu().view(torch.int16 if wl.dtype == "bf16" else torch.int32).numpy()[:R]
    want = xin[r["src_assign"] // k].view(np.int16 if wl.dtype == "bf16" else np.int32)
    assert np.array_equal(xp_np, want), "x_perm rows are not exact copies"

    # ---- 4. expert FFNs on the oracle's sorted rows
    if R > 0:
        xperm_ref = np.zeros((max(rows_cap, 1), d), dtype=xin.dtype)
        xperm_ref[:R] = xin[r["src_assign"] // k]
        y = torch.zeros((max(rows_cap, 1), d), dtype=cfg.torch_dtype, device="cuda")
        M.moe_expert_ffn(cfg, wd, dev(xperm_ref), dev(r["offsets"]), y, ws)
        torch.cuda.synchronize()
        if R <= 4096:
            rows = np.arange(R)
        else:
            # 512 random rows plus the first and last 64 kept rows of every expert
            rng = np.random.default_rng(2)
            rows = set(rng.choice(R, 512, replace=False).tolist())
            for e in range(E):
                o0, o1 = int(r["offsets"][e]), int(r["offsets"][e + 1])
                rows.update(range(o0, min(o1, o0 + 64)))
                rows.update(range(max(o0, o1 - 64), o1))
            rows = np.array(sorted(rows))
        yref = expert_rows_ref(wl, inp, r, rows)
        ok, e_, s_ = out_close(host_f64(y)[rows], yref, wl.dtype)
        assert ok, f"expert FFN max err {e_} vs scale {s_}"
        st, site = M.moe_check_device_status(ws)
        assert st == M.MOE_OK, f"device status {st} site {site:#x}"

    # ---- 5. combine on identical synthetic expert rows
    ysyn = W.normal(wl.seed + 17, 20, (max(rows_cap, 1), d), 1.0, wl.dtype)
    w32 = r["w"].astype(np.float32)
    out = torch.empty((T, d), dtype=cfg.torch_dtype, device="cuda")
    M.moe_combine(cfg, dev(ysyn), dev(r["slot"]), dev(w32), out)
    torch.cuda.synchronize()
    ctoks = np.arange(T) if T <= 4096 else np.random.default_rng(3).choice(T, 4096, replace=False)
    yrow = {}
    ys64 = O.to_f64(ysyn, wl.dtype)
    for t in ctoks:
        for j in range(k):
            if r["slot"][t, j] >= 0:
                yrow[int(t) * k + j] = ys64[r["slot"][t, j]]
    cref = O.combine(yrow, r["slot"], w32.astype(np.float64), T, d, ctoks)
    ok, e_, s_ = out_close(host_f64(out)[ctoks], cref, wl.dtype)
    assert ok, f"combine max err {e_} vs scale {s_}"
    dropped_all = (r["slot"] < 0).all(axis=1)
    if dropped_all.any():
        assert (host_f64(out)[dropped_all] == 0).all()

    # ---- 6. aux statistics from identical counts and probabilities
    f = torch.empty(E, dtype=torch.float32, device="cuda")
    p = torch.empty(E, dtype=torch.float32, device="cuda")
    la = torch.empty(1, dtype=torch.float32, device="cuda")
    p32 = r["p"].astype(np.float32)
    M.moe_aux_stats(cfg, dev(r["counts"]), dev(p32), f, p, la)
    torch.cuda.synchronize()
    fr, pr, lr = O.aux_stats(r["counts"], p32.astype(np.float64), T, k, wl.aux_alpha)
    assert rel_close(f.cpu().numpy(), fr)[0] and rel_close(p.cpu().numpy(), pr)[0]
    assert rel_close(la.cpu().numpy(), [lr])[0]

    # ---- 7. whole forward, logits fed: bit-exact routing/dispatch, outputs within tolerance
    layer = M.MoELayer(cfg, wd)
    layer_feed = M.MoELayer(cfg_feed, wd)
    o = layer_feed.forward(x, logits_in=dev(feed), token_mask=tm)
    layer_feed.check()
    assert np.array_equal(o["topk_idx"].cpu().numpy(), r["idx"])
    assert np.array_equal(o["counts"].cpu().numpy(), r["counts"])
    assert np.array_equal(o["offsets"].cpu().numpy(), r["offsets"])
    assert np.array_equal(o["slot"].cpu().numpy(), r["slot"])
    assert np.array_equal(o["src_assign"].cpu().numpy()[:R], r["src_assign"])
    assert rel_close(o["topk_w"].cpu().numpy(), r["w"])[0]
    assert rel_close(o["f"].cpu().numpy(), r["f"])[0]
    assert rel_close(o["p"].cpu().numpy(), r["p_mean"])[0]
    assert rel_close(o["l_aux"].cpu().numpy(), [r["l_aux"]])[0]
    toks = np.arange(T) if not full_size or T <= 4096 else sample_tokens(wl, r)
    ref = O.forward(wl, inp, routing=r, tokens=toks)
    got = host_f64(o["out"])[toks]
    ok, e_, s_ = out_close(got, ref["out"], wl.dtype)
    assert ok, f"layer output max err {e_} vs scale {s_}"
    first = {n: v.clone() for n, v in o.items()}

    # ---- 7b. bf16 with native weights: the forward weights each expert row in the
    #          second GEMM's epilogue; with the weights applied in the combine
    #          instead, routing is the same bit for bit and the output is within
    #          the same tolerance (only the rounding order differs)
    if wl.dtype == "bf16" and wl.weights == "native":
        lc = M.MoELayer(dataclasses.replace(cfg_feed, weighting="combine"), wd)
        oc = lc.forward(x, logits_in=dev(feed), token_mask=tm)
        lc.check()
        for n in ("topk_idx", "topk_w", "counts", "offsets", "slot", "f", "p", "l_aux"):
            assert torch.equal(oc[n].cpu(), o[n].cpu()), f"{n} depends on the weighting order"
        ok, e_, s_ = out_close(host_f64(oc["out"])[toks], ref["out"], wl.dtype)
        assert ok, f"layer output (weights in the combine) max err {e_} vs scale {s_}"
        del lc, oc

    # ---- 8. determinism: a second run is bit-identical
    o2 = layer_feed.forward(x, logits_in=dev(feed), token_mask=tm)
    torch.cuda.synchronize()
    for n, v in first.items():
        a, b = v.cpu(), o2[n].cpu()
        if n == "src_assign":
            a, b = a[:R], b[:R]
        assert torch.equal(a, b), f"{n} differs between two identical runs"

    # ---- 9. whole forward with the GPU's own router: same outputs where routing agrees
    o3 = layer.forward(x, token_mask=tm)
    layer.check()
    gi = o3["topk_idx"].cpu().numpy()
    gs = o3["slot"].cpu().numpy()
    agree = (gi == r["idx"]).all(axis=1) & ((gs >= 0) == (r["slot"] >= 0)).all(axis=1)
    assert agree.mean() >= 0.99, f"routing agrees on only {agree.mean():.4f} of tokens"
    tt = toks[agree[toks]]
    ok, e_, s_ = out_close(host_f64(o3["out"])[tt], ref["out"][agree[toks]], wl.dtype)
    assert ok, f"layer output (GPU router) max err {e_} vs scale {s_}"
    assert rel_close(o3["p"].cpu().numpy(), r["p_mean"], rtol=1e-4)[0]


@pytest.mark.parametrize("name", FULL)
def test_benchmark_workload_parity(name):
    _check_workload(W.WORKLOADS[name], full_size=True)


@pytest.mark.parametrize("wl", SMALL_WORKLOADS, ids=lambda w: w.name)
def test_small_workload_parity(wl):
    _check_workload(wl, full_size=False)


# the tensor-core router on every workload shape it takes (E % 8 == 0, bf16):
# 128-token tiles with a ragged last tile, one token, E from 8 to 64
TC_ROUTER_CASES = [w for w in SMALL_WORKLOADS if w.dtype == "bf16" and w.E % 8 == 0] + \
    [W.WORKLOADS[n] for n in ("llama4moe_t4096", "longctx_zipf_t32768", "decode_t64_e64")]


@pytest.mark.parametrize("wl", TC_ROUTER_CASES, ids=lambda w: w.name)
def test_tcgen05_router_parity(wl):
    _check_workload(wl, full_size=wl.T > 4096, router="tcgen05")


# both expert-GEMM kernels on every bf16 shape: ragged experts, drops, one
# expert, k = E, a single token, 16 experts; the pair kernel's 128-row tail
# tiles appear wherever an expert's rows end within 128 of a 256 boundary
GEMM_CASES = [(w, g) for w in SMALL_WORKLOADS if w.dtype == "bf16" for g in ("one_cta", "cta_pair")] + \
    [(W.WORKLOADS["llama4moe_t4096"], "cta_pair"), (W.WORKLOADS["llama4moe_t4096"], "one_cta"),
     (W.WORKLOADS["flat_gelu_t8192"], "one_cta"), (W.WORKLOADS["decode_t64_e64"], "cta_pair")]


@pytest.mark.parametrize("wl,gemm", GEMM_CASES, ids=[f"{w.name}-{g}" for w, g in GEMM_CASES])
def test_gemm_kernel_parity(wl, gemm):
    _check_workload(wl, full_size=wl.T > 4096, gemm=gemm)


@pytest.mark.parametrize("wl", [w for w in SMALL_WORKLOADS if w.dtype == "bf16"] + [W.WORKLOADS["llama4moe_t4096"]],
                         ids=lambda w: w.name)
def test_gemm_kernels_agree_bitwise(wl):
    """The one-CTA and the CTA-pair kernels give the same bits: each output is
    the same fp32 tensor-core sum over K, rounded once."""
    inp = W.make_inputs(wl)
    r = O.route(wl, inp)
    wd = weights_dev(wl, inp)
    R = int(r["offsets"][-1])
    outs = []
    for g in ("one_cta", "cta_pair"):
        cfg = _cfg(wl, gemm=g)
        rows_cap = M.moe_max_rows(cfg)
        xperm = np.zeros((max(rows_cap, 1), wl.d), dtype=inp["x"].dtype)
        xperm[:R] = inp["x"][r["src_assign"] // wl.k]
        y = torch.zeros((max(rows_cap, 1), wl.d), dtype=cfg.torch_dtype, device="cuda")
        ws = M.Workspace(cfg)
        M.moe_expert_ffn(cfg, wd, to_dev(xperm), to_dev(r["offsets"]), y, ws)
        torch.cuda.synchronize()
        assert M.moe_check_device_status(ws)[0] == M.MOE_OK
        outs.append(y[:R].cpu())
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


def test_empty_batch():
    cfg = M.MoEConfig(T=0, d=128, ffn=128, E=4, k=2)
    wl = W.Workload("empty", T=0, d=128, ffn=128, E=4, k=2, act="swiglu", dtype="bf16", capacity_factor=1.0)
    inp = W.make_inputs(wl)
    layer = M.MoELayer(cfg, weights_dev(wl, inp))
    o = layer.forward(torch.empty((0, 128), dtype=torch.bfloat16, device="cuda"))
    layer.check()
    assert o["offsets"].cpu().tolist() == [0] * 5 and o["counts"].cpu().tolist() == [0] * 4
    assert float(o["l_aux"].cpu()[0]) == 0.0 and (o["f"].cpu() == 0).all() and (o["p"].cpu() == 0).all()


def test_hostio_matches_device_path():
    wl = SMALL_WORKLOADS[0]
    cfg = _cfg(wl)
    inp = W.make_inputs(wl)
    wd = weights_dev(wl, inp)
    layer = M.MoELayer(cfg, wd)
    x = to_dev(inp["x"])
    ref = layer.forward(x)["out"].clone()
    x_host = torch.from_numpy(inp["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    out_host = torch.empty((wl.T, wl.d), dtype=torch.bfloat16).pin_memory()
    l_host = torch.empty(1, dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(x)
    M.moe_forward_hostio(cfg, wd, x_host, x_dev, layer.outputs, out_host, l_host, layer.ws)
    torch.cuda.synchronize()
    assert torch.equal(out_host, ref.cpu())
    assert float(l_host[0]) == float(layer.outputs["l_aux"].cpu()[0])


def test_bounded_wait_gives_up_and_context_survives():
    """A wait on a flag nothing sets gives up after its limit, the status word
    reports MOE_ERR_TIMEOUT, and the context still runs a correct forward."""
    wl = SMALL_WORKLOADS[5]
    cfg = _cfg(wl)
    ws = M.Workspace(cfg)
    M.moe_selftest_bounded_wait(ws, 50)
    st, site = M.moe_check_device_status(ws)
    assert st == M.MOE_ERR_TIMEOUT and site in (0x201, 0x202)
    st, _ = M.moe_check_device_status(ws)
    assert st == M.MOE_OK
    inp = W.make_inputs(wl)
    r = O.route(wl, inp)
    layer = M.MoELayer(cfg, weights_dev(wl, inp))
    o = layer.forward(to_dev(inp["x"]), logits_in=to_dev(r["logits"].astype(np.float32)))
    layer.check()
    ref = O.forward(wl, inp, routing=r)
    assert out_close(host_f64(o["out"]), ref["out"], "bf16")[0]


# the first expert GEMM reading its rows straight from x (gather) against the
# expert-sorted copy: every forward output bit for bit
DISPATCH_CASES = [w for w in SMALL_WORKLOADS if w.dtype == "bf16"] + \
    [W.WORKLOADS[n] for n in ("llama4moe_t4096", "longctx_zipf_t32768", "decode_t64_e64", "flat_gelu_t8192")]


@pytest.mark.parametrize("wl", DISPATCH_CASES, ids=lambda w: w.name)
def test_gather_dispatch_equals_copy(wl):
    inp = W.make_inputs(wl)
    wd = weights_dev(wl, inp)
    x = to_dev(inp["x"])
    outs = {}
    for mode in ("copy", "gather"):
        for gemm in ("one_cta", "cta_pair"):
            layer = M.MoELayer(M.MoEConfig.of(wl, gemm_kernel=gemm, dispatch=mode), wd)
            o = layer.forward(x)
            layer.check()
            outs[(mode, gemm)] = {n: v.clone() for n, v in o.items()}
    ref = outs[("copy", "one_cta")]
    R = int(ref["offsets"][-1])
    for key, o in outs.items():
        for n, v in ref.items():
            a, b = v, o[n]
            if n == "src_assign":
                a, b = a[:R], b[:R]
            assert torch.equal(a, b), f"{key}: {n} differs"


# the llama4moe layer with one shared expert and 10 % padding, at full size
SHARED_FULL = W.WORKLOADS["llama4moe_t4096"].with_(name="llama4moe_t4096_shared1_pad10", n_shared=1, pad_fraction=0.1)


@pytest.mark.parametrize("gemm", ["auto", "cta_pair"])
def test_shared_experts_and_padding_full_size(gemm):
    _check_workload(SHARED_FULL, full_size=True, gemm=gemm)
