"""Helpers shared by the GPU parity tests: moving seeded inputs to the device,
oracle evaluation on token samples, and the tolerances the tests enforce.

Tolerances (stated once, used everywhere):
  * indices, counts, offsets, slots, permutation, drop mask: bit-exact;
  * fp32 router probabilities, top-k weights, f, p, L_aux: relative 1e-5;
  * bf16 layer / expert outputs: max|gpu - ref| <= 2e-2 * max|ref|;
  * fp32 layer / expert outputs (SIMT FMA path): max|gpu - ref| <= 1e-4 * max|ref|;
  * GPU-computed router logits: |gpu - ref| <= (d/16 + 16) * 2^-24 * sum_i |x_i w_i|,
    the bound of fp32 accumulation over d/16 sequential tensor-core steps.
"""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_layer_37_b200 as M
import workloads as W
from oracle import moe_oracle as O

PROB_RTOL = 1e-5
OUT_TOL = {"bf16": 2e-2, "f32": 1e-4}


def to_dev(a):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def weights_dev(wl, inp) -> dict:
    w = {"w_router": to_dev(inp["w_router"])}
    if inp.get("router_bias") is not None:
        w["router_bias"] = to_dev(np.asarray(inp["router_bias"], dtype=np.float32))
    for n in ("w_gate", "w_up", "w_down", "w1", "b1", "w2", "b2", "shared_gate", "shared_up", "shared_down",
              "shared_w1", "shared_b1", "shared_w2", "shared_b2"):
        if n in inp:
            w[n] = to_dev(inp[n])
    return w


def mask_dev(inp):
    """The padding mask of the inputs on the device, or None."""
    m = inp.get("token_mask")
    return None if m is None else torch.from_numpy(np.ascontiguousarray(m)).cuda()


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_close(gpu, ref, rtol=PROB_RTOL, atol=1e-30):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(gpu - ref)
    bad = err > rtol * np.abs(ref) + atol
    return not bad.any(), float((err / np.maximum(np.abs(ref), 1e-300)).max()) if err.size else 0.0


def out_close(gpu, ref, dtype):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    err = float(np.abs(gpu - ref).max()) if ref.size else 0.0
    return err <= OUT_TOL[dtype] * scale + 1e-30, err, scale


def sample_tokens(wl, routing, n_random=512, per_expert=64, seed=0) -> np.ndarray:
    """Token sample for full-size configs: the first and last `per_expert`
    kept tokens of every expert, some dropped tokens, and random tokens."""
    T, k = wl.T, wl.k
    rng = np.random.default_rng(seed)
    picks = set(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    src = routing["src_assign"]
    off = routing["offsets"]
    for e in range(wl.E):
        rows = src[off[e]:off[e + 1]] // k
        picks.update(rows[:per_expert].tolist())
        picks.update(rows[-per_expert:].tolist())
    dropped = np.nonzero((routing["slot"] < 0).any(axis=1))[0]
    picks.update(dropped[:64].tolist())
    picks.update([0, T - 1])
    return np.array(sorted(picks), dtype=np.int64)


def expert_rows_ref(wl, inp, routing, rows: np.ndarray) -> np.ndarray:
    """Oracle expert output for sorted rows `rows` (float64 [len(rows), d])."""
    assigns = routing["src_assign"][rows].astype(np.int64)
    y = O.expert_outputs(wl, inp, routing, assigns)
    return np.stack([y[int(a)] for a in assigns]) if len(assigns) else np.zeros((0, wl.d))


def logit_error_bound(wl, inp, tokens: np.ndarray) -> np.ndarray:
    x = O.to_f64(inp["x"][tokens], wl.dtype)
    w = O.to_f64(inp["w_router"], wl.dtype)
    absum = np.abs(x) @ np.abs(w)
    return (wl.d / 16 + 16) * 2.0 ** -24 * absum + 1e-30


SMALL_WORKLOADS = [
    W.Workload("ragged_swiglu", T=1000, d=256, ffn=384, E=6, k=2, act="swiglu", dtype="bf16",
               capacity_factor=1.0, seed=101),
    W.Workload("drops_gelu_k3", T=777, d=192, ffn=320, E=5, k=3, act="gelu_bias", dtype="bf16",
               capacity_factor=0.8, seed=102),
    W.Workload("dense_e1_k1", T=300, d=128, ffn=256, E=1, k=1, act="swiglu", dtype="bf16",
               capacity_factor=0.0, seed=103),
    W.Workload("f32_gelu", T=150, d=64, ffn=96, E=3, k=2, act="gelu_bias", dtype="f32",
               capacity_factor=1.0, seed=104),
    W.Workload("topk_eq_E", T=200, d=128, ffn=128, E=4, k=4, act="swiglu", dtype="bf16",
               capacity_factor=1.0, seed=105),
    W.Workload("single_token", T=1, d=64, ffn=64, E=8, k=2, act="swiglu", dtype="bf16",
               capacity_factor=1.25, seed=106),
    W.Workload("zipf_heavy_drops", T=513, d=128, ffn=192, E=16, k=2, act="swiglu", dtype="bf16",
               capacity_factor=0.5, zipf_router_bias=True, seed=107, w_std=0.05),
    W.Workload("e64_k8_f32", T=96, d=32, ffn=48, E=64, k=8, act="swiglu", dtype="f32",
               capacity_factor=0.0, seed=108),
    # padding mask and shared experts (readings R16, R17)
    W.Workload("shared2_swiglu_pad", T=700, d=128, ffn=192, E=8, k=2, act="swiglu", dtype="bf16",
               capacity_factor=1.0, seed=110, n_shared=2, pad_fraction=0.2),
    W.Workload("shared_gelu_pad", T=333, d=128, ffn=128, E=6, k=2, act="gelu_bias", dtype="bf16",
               capacity_factor=0.9, seed=111, n_shared=1, pad_fraction=0.3),
    W.Workload("f32_shared_pad", T=130, d=64, ffn=96, E=4, k=2, act="swiglu", dtype="f32",
               capacity_factor=1.0, seed=112, n_shared=1, pad_fraction=0.25),
]
