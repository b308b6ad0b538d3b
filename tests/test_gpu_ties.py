"""GPU parity on exact ties in the router's top-k.

The tie rule (equal logits: the lower expert id is chosen first) is the
stable reading of the pages' top-k calls ("MoE: gating, experts, load
balancing, capacity factor", dpshk.com/news/6005940, §3.1 ``logits.topk``;
"Llama-MoE架构解析", coreui.cn/article/2610641, §3.1 ``torch.topk``).
Continuous random logits never tie, so these cases build ties on purpose:

  * fed logits: integer values in {-2..2} (ties everywhere, across the k-th
    place too), rows whose logits are all equal, and rows with k-1 clear
    winners followed by a run of equal values straddling the k-th place;
  * the router's own GEMM: x and W_r with entries in {-1, 0, 1}, so every
    logit is a small integer that fp32 accumulation produces exactly in any
    summation order.  The GPU's logits must then equal the oracle's bit for
    bit, and both sides decide on identical values without feeding anything.

All three routers are covered: the two warp-MMA kernels (resident weight and
slab-staged; every shape, fed or own logits) and the tcgen05 kernel (own
logits, E % 8 == 0; it refuses fed logits).  Indices, counts, offsets, slots and src_assign are compared bit for
bit with the oracle, probabilities and weights within 1e-5 relative, and the
layer output within the bf16 / fp32 output tolerance.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_37_b200 as M
import workloads as W
from oracle import moe_oracle as O
from gpu_common import host_f64, out_close, rel_close, to_dev, weights_dev

pytestmark = pytest.mark.gpu

BF16_ONE, BF16_MINUS_ONE = 0x3F80, 0xBF80


def _encode(vals: np.ndarray, dtype: str) -> np.ndarray:
    """{-1, 0, 1}-valued float array as the workload's input encoding."""
    if dtype == "f32":
        return vals.astype(np.float32)
    out = np.zeros(vals.shape, dtype=np.uint16)
    out[vals == 1] = BF16_ONE
    out[vals == -1] = BF16_MINUS_ONE
    return out


def integer_router_inputs(wl, seed: int) -> dict:
    """The workload's expert weights with x and W_r replaced by sparse
    {-1, 0, 1} patterns: logits are integers in [-3, 3]; the first rows of x
    are all zero, so their logits are all equal."""
    inp = W.make_inputs(wl)
    rng = np.random.default_rng(seed)
    x = np.zeros((wl.T, wl.d))
    for t in range(wl.T):
        nnz = 0 if t < 3 else int(rng.integers(1, 4))
        cols = rng.choice(wl.d, size=nnz, replace=False)
        x[t, cols] = rng.choice([-1.0, 1.0], size=nnz)
    wr = rng.choice([-1.0, 0.0, 1.0], size=(wl.d, wl.E), p=[0.25, 0.5, 0.25])
    inp = dict(inp)
    inp["x"] = _encode(x, wl.dtype)
    inp["w_router"] = _encode(wr, wl.dtype)
    inp["router_bias"] = None
    return inp


def tied_logits(T: int, E: int, k: int, seed: int) -> np.ndarray:
    """Integer logits in {-2..2}; rows 0-2 all equal; rows 3-9 hold k-1 clear
    winners (value 3) and then a run of equal values (value 1) that straddles
    the k-th place."""
    rng = np.random.default_rng(seed)
    L = rng.integers(-2, 3, size=(T, E)).astype(np.float32)
    L[0:3] = np.array([1.0, 0.0, -2.0], dtype=np.float32)[:, None]
    for t in range(3, min(10, T)):
        L[t] = -2.0
        perm = rng.permutation(E)
        L[t, perm[:k - 1]] = 3.0
        run = min(E - (k - 1), 2 + t % 3)
        L[t, perm[k - 1:k - 1 + run]] = 1.0
    return L


def _router_check(cfg, wl, inp, r, x, wd, logits_in=None, exact_logits=False):
    T, E, k = wl.T, wl.E, wl.k
    ws = M.Workspace(cfg)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    lo = torch.empty((T, E), dtype=torch.float32, device="cuda")
    probs = torch.empty((T, E), dtype=torch.float32, device="cuda")
    M.moe_router_topk(cfg, x, wd["w_router"], None, logits_in, idx, tw, lo, probs, ws)
    torch.cuda.synchronize()
    if exact_logits:
        assert np.array_equal(lo.cpu().numpy().astype(np.float64), r["logits64"]), "integer logits not exact"
    assert np.array_equal(idx.cpu().numpy(), r["idx"]), "top-k indices differ on tied logits"
    assert rel_close(tw.cpu().numpy(), r["w"])[0]
    assert rel_close(probs.cpu().numpy(), r["p"])[0]
    assert M.moe_check_device_status(ws)[0] == M.MOE_OK


def _forward_check(cfg, wl, inp, r, x, wd, logits_in=None):
    layer = M.MoELayer(cfg, wd)
    o = layer.forward(x, logits_in=logits_in)
    layer.check()
    R = int(r["offsets"][-1])
    for name in ("topk_idx", "counts", "offsets", "slot"):
        want = r["idx"] if name == "topk_idx" else r[name]
        assert np.array_equal(o[name].cpu().numpy(), want), f"{name} differs on tied logits"
    assert np.array_equal(o["src_assign"].cpu().numpy()[:R], r["src_assign"])
    assert rel_close(o["topk_w"].cpu().numpy(), r["w"])[0]
    assert rel_close(o["f"].cpu().numpy(), r["f"])[0]
    assert rel_close(o["p"].cpu().numpy(), r["p_mean"])[0]
    ref = O.forward(wl, inp, routing=r)
    ok, err, scale = out_close(host_f64(o["out"]), ref["out"], wl.dtype)
    assert ok, f"layer output max err {err} vs scale {scale}"


TIE_CASES = [(4, "bf16", 300), (6, "bf16", 300), (8, "bf16", 1000), (64, "bf16", 1000), (6, "f32", 200),
             (64, "f32", 200)]


@pytest.mark.parametrize("E,dtype,T", TIE_CASES, ids=[f"E{e}-{dt}-T{t}" for e, dt, t in TIE_CASES])
def test_router_ties_bit_exact(E, dtype, T):
    routers = ["warp_mma", "warp_mma_staged"] + (["tcgen05"] if dtype == "bf16" and E % 8 == 0 else [])
    for k in range(1, min(E, 8) + 1):
        wl = W.Workload(f"ties_e{E}_k{k}", T=T, d=128, ffn=64, E=E, k=k, act="swiglu" if k % 2 else "gelu_bias",
                        dtype=dtype, capacity_factor=1.0, seed=300 + 10 * E + k)
        inp = integer_router_inputs(wl, seed=wl.seed)
        wd = weights_dev(wl, inp)
        x = to_dev(inp["x"])
        # the router's own GEMM: exact integer logits, decided identically
        r_own = O.route(wl, inp)
        assert (r_own["logits64"] == np.round(r_own["logits64"])).all()
        n_tied = int((np.ptp(np.sort(r_own["logits64"], axis=1)[:, ::-1][:, k - 1:k + 1], axis=1) == 0).sum()) \
            if k < E else T
        assert n_tied > T // 10, "the case should tie at the k-th place often"
        for router in routers:
            cfg = M.MoEConfig.of(wl, router_kernel=router)
            _router_check(cfg, wl, inp, r_own, x, wd, exact_logits=True)
            _forward_check(cfg, wl, inp, r_own, x, wd)
        # fed logits (the warp routers' selection paths)
        L = tied_logits(T, E, k, seed=wl.seed + 1)
        r_fed = O.route(wl, inp, logits_feed=L)
        Ld = to_dev(L)
        for router in ("warp_mma", "warp_mma_staged"):
            cfg = M.MoEConfig.of(wl, router_kernel=router)
            _router_check(cfg, wl, inp, r_fed, x, wd, logits_in=Ld)
            _forward_check(cfg, wl, inp, r_fed, x, wd, logits_in=Ld)
        if "tcgen05" in routers:
            tc = M.MoEConfig.of(wl, router_kernel="tcgen05")
            with pytest.raises(M.MoEError) as e:
                M.MoELayer(tc, wd).forward(x, logits_in=Ld)
            assert e.value.status == M.MOE_ERR_UNSUPPORTED
