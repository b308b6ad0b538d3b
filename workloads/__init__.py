"""Seeded synthetic workloads for the MoE layer forward.

This module is the one piece shared by both sides of the parity check: it
describes each workload's shapes and value distributions and produces the
input bytes (x, router weight, expert weights, biases) from a counter-based
generator (``gen.c``).  It contains none of the layer's arithmetic: no
routing, capacity, activation or combine.  The same bytes are handed to the
CPU oracle and to the CUDA library.

Workload shapes follow the five benchmark configurations of the layer (tiny
fp32 check, page-1 LLaMA4-MoE layer, flattened-expert GELU layer,
long-context skewed routing, decode-sized weight streaming).  The pages'
own datasets (a private corpus, BraTS2021) are not available; these seeded
Gaussian tensors stand in for them with the stated shapes and scales.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_gen.so")
_lib = None

# stream ids of the generator, one per tensor
STREAM_X, STREAM_WR, STREAM_W1, STREAM_WUP, STREAM_W2, STREAM_B1, STREAM_B2 = 1, 2, 3, 4, 5, 6, 7
# shared experts' parameters and the padding draw
STREAM_SW1, STREAM_SWUP, STREAM_SW2, STREAM_SB1, STREAM_SB2, STREAM_PAD = 8, 9, 10, 11, 12, 13


def build_generator(force: bool = False) -> str:
    """Compile gen.c into an in-tree shared object (gcc, OpenMP)."""
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", src, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_generator())
        u64, i64, dbl, ptr = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.wl_uniform_f64.argtypes = [u64, u64, u64, i64, ptr]
        lib.wl_normal_f32.argtypes = [u64, u64, u64, i64, dbl, dbl, ptr]
        lib.wl_normal_bf16.argtypes = [u64, u64, u64, i64, dbl, dbl, ptr]
        lib.wl_normal_bf16_rows.argtypes = [u64, u64, ptr, i64, i64, dbl, dbl, ptr]
        lib.wl_stream_key.argtypes = [u64, u64]
        lib.wl_stream_key.restype = u64
        _lib = lib
    return _lib


def uniform_f64(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _load().wl_uniform_f64(seed, stream, start, n, out.ctypes.data)
    return out


def normal(seed: int, stream: int, shape, std: float, dtype: str, mean: float = 0.0) -> np.ndarray:
    """N(mean, std^2) samples; dtype 'f32' -> float32 array, 'bf16' -> uint16 bit patterns."""
    n = int(np.prod(shape)) if len(shape) else 1
    if dtype == "f32":
        out = np.empty(n, dtype=np.float32)
        _load().wl_normal_f32(seed, stream, 0, n, mean, std, out.ctypes.data)
    elif dtype == "bf16":
        out = np.empty(n, dtype=np.uint16)
        _load().wl_normal_bf16(seed, stream, 0, n, mean, std, out.ctypes.data)
    else:
        raise ValueError(dtype)
    return out.reshape(shape)


def normal_rows_bf16(seed: int, stream: int, rows: np.ndarray, row_len: int, std: float) -> np.ndarray:
    """Rows ``rows`` of a [*, row_len] bf16 stream, without generating the others."""
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((rows.size, row_len), dtype=np.uint16)
    _load().wl_normal_bf16_rows(seed, stream, rows.ctypes.data, rows.size, row_len, 0.0, std, out.ctypes.data)
    return out


@dataclass(frozen=True)
class Workload:
    """Shapes, precisions and distributions of one MoE layer forward."""
    name: str
    T: int
    d: int
    ffn: int
    E: int
    k: int
    act: str                  # "swiglu" | "gelu_bias"
    dtype: str                # "f32" | "bf16"
    capacity_factor: float    # <= 0: no capacity limit
    aux_alpha: float = 0.01
    zipf_router_bias: bool = False   # b_e = 0.5*ln(1/(e+1)), e zero-based
    x_std: float = 1.0
    w_std: float = 0.02
    b_std: float = 0.01
    seed: int = 0
    n_shared: int = 0         # always-on shared experts (same FFN form as the routed ones)
    pad_fraction: float = 0.0  # expected fraction of padding tokens (token_mask = 0)
    weights: str = "native"   # routed experts' weights: "native" (the dtype) or "int8" (quantised by the layer)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", T=64, d=128, ffn=256, E=4, k=2, act="swiglu", dtype="f32",
                         capacity_factor=1.25, seed=20260001),
    "llama4moe_t4096": Workload("llama4moe_t4096", T=4096, d=2048, ffn=4096, E=8, k=2, act="swiglu",
                                dtype="bf16", capacity_factor=1.25, seed=20260002),
    "flat_gelu_t8192": Workload("flat_gelu_t8192", T=8192, d=4096, ffn=16384, E=8, k=2, act="gelu_bias",
                                dtype="bf16", capacity_factor=1.25, seed=20260003),
    "longctx_zipf_t32768": Workload("longctx_zipf_t32768", T=32768, d=4096, ffn=4096, E=32, k=2,
                                    act="swiglu", dtype="bf16", capacity_factor=1.0,
                                    zipf_router_bias=True, seed=20260004),
    "decode_t64_e64": Workload("decode_t64_e64", T=64, d=2048, ffn=2048, E=64, k=2, act="swiglu",
                               dtype="bf16", capacity_factor=0.0, seed=20260005),
}
WORKLOAD_ORDER = ["tiny_f32", "llama4moe_t4096", "flat_gelu_t8192", "longctx_zipf_t32768", "decode_t64_e64"]


def zipf_bias(E: int) -> np.ndarray:
    """Fixed per-expert router logit bias 0.5*ln(1/(e+1)), e = 0..E-1 (a workload input)."""
    return np.array([0.5 * math.log(1.0 / (e + 1)) for e in range(E)], dtype=np.float32)


def make_inputs(wl: Workload, seed: Optional[int] = None, with_experts: bool = True) -> dict:
    """All inputs of one forward.  bf16 tensors are uint16 bit patterns."""
    s = wl.seed if seed is None else seed
    dt = wl.dtype
    out = {
        "x": normal(s, STREAM_X, (wl.T, wl.d), wl.x_std, dt),
        "w_router": normal(s, STREAM_WR, (wl.d, wl.E), wl.w_std, dt),
        "router_bias": zipf_bias(wl.E) if wl.zipf_router_bias else None,
    }
    if wl.pad_fraction > 0:
        # token t is padding when its uniform draw falls below pad_fraction
        out["token_mask"] = (uniform_f64(s, STREAM_PAD, wl.T) >= wl.pad_fraction).astype(np.uint8)
    if with_experts:
        out.update(make_expert_weights(wl, s))
        if wl.n_shared > 0:
            out.update(make_shared_weights(wl, s))
    return out


def make_shared_weights(wl: Workload, seed: Optional[int] = None) -> dict:
    """Parameters of the n_shared always-on experts, same shapes per expert as the routed ones."""
    s = wl.seed if seed is None else seed
    dt = wl.dtype
    S, d, F = wl.n_shared, wl.d, wl.ffn
    if wl.act == "swiglu":
        return {
            "shared_gate": normal(s, STREAM_SW1, (S, d, F), wl.w_std, dt),
            "shared_up": normal(s, STREAM_SWUP, (S, d, F), wl.w_std, dt),
            "shared_down": normal(s, STREAM_SW2, (S, F, d), wl.w_std, dt),
        }
    return {
        "shared_w1": normal(s, STREAM_SW1, (S, d, F), wl.w_std, dt),
        "shared_b1": normal(s, STREAM_SB1, (S, F), wl.b_std, dt),
        "shared_w2": normal(s, STREAM_SW2, (S, F, d), wl.w_std, dt),
        "shared_b2": normal(s, STREAM_SB2, (S, d), wl.b_std, dt),
    }


def make_expert_weights(wl: Workload, seed: Optional[int] = None) -> dict:
    s = wl.seed if seed is None else seed
    dt = wl.dtype
    E, d, F = wl.E, wl.d, wl.ffn
    if wl.act == "swiglu":
        return {
            "w_gate": normal(s, STREAM_W1, (E, d, F), wl.w_std, dt),
            "w_up": normal(s, STREAM_WUP, (E, d, F), wl.w_std, dt),
            "w_down": normal(s, STREAM_W2, (E, F, d), wl.w_std, dt),
        }
    if wl.act == "gelu_bias":
        return {
            "w1": normal(s, STREAM_W1, (E, d, F), wl.w_std, dt),
            "b1": normal(s, STREAM_B1, (E, F), wl.b_std, dt),
            "w2": normal(s, STREAM_W2, (E, F, d), wl.w_std, dt),
            "b2": normal(s, STREAM_B2, (E, d), wl.b_std, dt),
        }
    raise ValueError(wl.act)


def x_rows(wl: Workload, rows: np.ndarray, seed: Optional[int] = None) -> np.ndarray:
    """Rows of x for a token subset (bf16 workloads), identical to make_inputs()['x'][rows]."""
    s = wl.seed if seed is None else seed
    assert wl.dtype == "bf16"
    return normal_rows_bf16(s, STREAM_X, rows, wl.d, wl.x_std)
