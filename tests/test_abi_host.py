"""C ABI checks that need no GPU: the library loads, exports every symbol the
header declares, validates arguments on the host before any launch, and
computes the capacity exactly as the oracle does."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import mixture_experts_layer_37_b200 as M
from oracle import moe_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from mixture_experts_layer_37_b200 import build
    build.build()
    return M.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 15, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(names) == set(M.EXPORTED_SYMBOLS)


def test_config_struct_layout_matches_header():
    assert ctypes.sizeof(M.MoEConfigC) == 72
    assert M.MoEConfigC.capacity_factor.offset == 32 and M.MoEConfigC.n_shared.offset == 56
    assert M.MoEConfigC.weighting.offset == 64
    assert ctypes.sizeof(M.MoEWeightsC) == 15 * 8 and ctypes.sizeof(M.MoEOutputsC) == 12 * 8


@pytest.mark.parametrize("T,k,E,cf", [(64, 2, 4, 1.25), (4096, 2, 8, 1.25), (8192, 2, 8, 1.25), (32768, 2, 32, 1.0),
                                      (64, 2, 64, 0.0), (10, 2, 3, 1.1), (4, 1, 1, 0.5), (1000, 3, 7, 0.9),
                                      (333, 2, 5, 1.0 / 3.0), (1, 1, 1, 1e-9), (12345, 8, 64, 2.5), (7, 2, 3, -1.0)])
def test_capacity_matches_oracle(lib, T, k, E, cf):
    cfg = M.MoEConfig(T=T, d=64, ffn=64, E=E, k=k, capacity_factor=cf)
    assert M.moe_capacity(cfg) == O.capacity(T, k, E, cf)
    cap = min(O.capacity(T, k, E, cf), T)
    assert M.moe_max_rows(cfg) == min(T * k, E * cap)


def test_capacity_random_sweep(lib):
    rng = np.random.default_rng(9)
    for _ in range(2000):
        E = int(rng.integers(1, 65))
        k = int(rng.integers(1, min(E, 8) + 1))
        T = int(rng.integers(0, 200000))
        cf = float(rng.choice([rng.uniform(0.01, 4.0), round(rng.uniform(0.5, 2), 2), 1.0, 1.25, 0.0]))
        cfg = M.MoEConfig(T=T, d=64, ffn=64, E=E, k=k, capacity_factor=cf)
        assert M.moe_capacity(cfg) == O.capacity(T, k, E, cf)


def _status(fn, *args):
    return fn(*args)


def test_invalid_configs_rejected_on_host(lib):
    size = ctypes.c_size_t()
    bad = [
        (dict(E=65, k=2), M.MOE_ERR_UNSUPPORTED),
        (dict(E=4, k=5), M.MOE_ERR_INVALID_ARG),
        (dict(E=16, k=9), M.MOE_ERR_UNSUPPORTED),
        (dict(d=100), M.MOE_ERR_UNSUPPORTED),          # bf16 needs d % 64
        (dict(ffn=96), M.MOE_ERR_UNSUPPORTED),
        (dict(T=-1), M.MOE_ERR_INVALID_ARG),
        (dict(E=0), M.MOE_ERR_INVALID_ARG),
        (dict(capacity_factor=float("nan")), M.MOE_ERR_INVALID_ARG),
        (dict(T=2 ** 30, k=2), M.MOE_ERR_UNSUPPORTED),  # T*k must stay below 2^31
        (dict(router_kernel="tcgen05", E=12), M.MOE_ERR_UNSUPPORTED),  # tensor-core router: E % 8
        (dict(router_kernel="tcgen05", dtype="f32", d=96), M.MOE_ERR_UNSUPPORTED),  # and bf16 only
    ]
    for kw, want in bad:
        base = dict(T=128, d=128, ffn=128, E=8, k=2)
        base.update(kw)
        cfg = M.MoEConfig(**base).c()
        assert lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(size)) == want, kw
    f32 = M.MoEConfig(T=8, d=100, ffn=12, E=2, k=1, dtype="f32").c()
    assert lib.moe_workspace_size(ctypes.byref(f32), ctypes.byref(size)) == M.MOE_OK
    cfg = M.MoEConfig(T=8, d=128, ffn=128, E=4, k=2).c()
    cfg.dtype = 7
    assert lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(size)) == M.MOE_ERR_INVALID_ARG
    for rk in (-1, 4):
        cfg = M.MoEConfig(T=8, d=128, ffn=128, E=8, k=2).c()
        cfg.router_kernel = rk
        assert lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(size)) == M.MOE_ERR_INVALID_ARG
    for name in ("auto", "warp_mma", "tcgen05", "warp_mma_staged"):
        cfg = M.MoEConfig(T=8, d=128, ffn=128, E=8, k=2, router_kernel=name).c()
        assert lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(size)) == M.MOE_OK
    for name in ("auto", "one_cta", "cta_pair"):
        cfg = M.MoEConfig(T=8, d=128, ffn=128, E=8, k=2, gemm_kernel=name).c()
        assert lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(size)) == M.MOE_OK
    for name in ("auto", "copy", "gather"):
        cfg = M.MoEConfig(T=8, d=128, ffn=128, E=8, k=2, dispatch=name).c()
        assert lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(size)) == M.MOE_OK
    for name in ("auto", "combine", "epilogue"):
        cfg = M.MoEConfig(T=8, d=128, ffn=128, E=8, k=2, weighting=name).c()
        assert lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(size)) == M.MOE_OK
    assert lib.moe_workspace_size(ctypes.byref(M.MoEConfig(T=8, d=128, ffn=128, E=8, k=2, n_shared=8).c()),
                                  ctypes.byref(size)) == M.MOE_OK
    assert lib.moe_workspace_size(ctypes.byref(M.MoEConfig(T=8, d=128, ffn=128, E=8, k=2, n_shared=9).c()),
                                  ctypes.byref(size)) == M.MOE_ERR_UNSUPPORTED
    assert lib.moe_workspace_size(ctypes.byref(M.MoEConfig(T=8, d=128, ffn=128, E=8, k=2, weights="int8").c()),
                                  ctypes.byref(size)) == M.MOE_OK
    assert lib.moe_workspace_size(ctypes.byref(M.MoEConfig(T=8, d=128, ffn=128, E=8, k=2, dtype="f32",
                                                           weights="int8").c()), ctypes.byref(size)) == \
        M.MOE_ERR_UNSUPPORTED
    for field, v in (("gemm_kernel", 3), ("gemm_kernel", -1), ("dispatch", 3), ("dispatch", -1), ("n_shared", -1),
                     ("weight_format", 2), ("weight_format", -1), ("weighting", 3), ("weighting", -1)):
        cfg = M.MoEConfig(T=8, d=128, ffn=128, E=8, k=2).c()
        setattr(cfg, field, v)
        assert lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(size)) == M.MOE_ERR_INVALID_ARG


def test_null_and_workspace_errors_launch_nothing(lib):
    """Bad pointers and short workspaces are refused before any CUDA call, so
    these calls are safe without a GPU."""
    cfg = M.MoEConfig(T=128, d=128, ffn=128, E=8, k=2)
    c = cfg.c()
    w = M.MoEWeightsC()
    o = M.MoEOutputsC()
    assert lib.moe_forward(ctypes.byref(c), ctypes.byref(w), None, None, None, ctypes.byref(o), None, 0, None) == \
        M.MOE_ERR_INVALID_ARG
    assert lib.moe_forward(ctypes.byref(c), None, None, None, None, None, None, 0, None) == M.MOE_ERR_INVALID_ARG
    # well-formed pointers (never dereferenced) but no workspace
    fake = ctypes.c_void_p(1 << 40)
    w = M.MoEWeightsC(fake, None, fake, fake, fake, None, None, None, None, None, None, None)
    o = M.MoEOutputsC(*([fake] * 10 + [None, None]))
    assert lib.moe_forward(ctypes.byref(c), ctypes.byref(w), fake, None, None, ctypes.byref(o), None, 0, None) == \
        M.MOE_ERR_WORKSPACE
    need = M.moe_workspace_size(cfg)
    assert lib.moe_forward(ctypes.byref(c), ctypes.byref(w), fake, None, None, ctypes.byref(o), fake, need - 1,
                           None) == M.MOE_ERR_WORKSPACE
    # misaligned activation pointer
    mis = ctypes.c_void_p((1 << 40) + 8)
    assert lib.moe_forward(ctypes.byref(c), ctypes.byref(w), mis, None, None, ctypes.byref(o), fake, need, None) == \
        M.MOE_ERR_INVALID_ARG
    # shared experts without their weights
    cs = M.MoEConfig(T=128, d=128, ffn=128, E=8, k=2, n_shared=1)
    need_s = M.moe_workspace_size(cs)
    assert need_s > need
    assert lib.moe_forward(ctypes.byref(cs.c()), ctypes.byref(w), fake, None, None, ctypes.byref(o), fake, need_s,
                           None) == M.MOE_ERR_INVALID_ARG
    assert M.moe_forward_launch_count(cs) == 7
    # swiglu without w_up
    w2 = M.MoEWeightsC(fake, None, fake, None, fake, None, None, None, None, None, None, None)
    assert lib.moe_expert_ffn(ctypes.byref(c), ctypes.byref(w2), fake, fake, fake, fake, need, None) == \
        M.MOE_ERR_INVALID_ARG
    assert lib.moe_router_topk(ctypes.byref(c), fake, fake, None, None, None, None, fake, None, None, fake, need,
                               None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(ctypes.byref(c), None, fake, fake, fake, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_aux_stats(ctypes.byref(c), None, fake, fake, fake, fake, None) == M.MOE_ERR_INVALID_ARG
    # the tensor-core router has no path for fed logits: refused, not swapped for the warp router
    tc = M.MoEConfig(T=128, d=128, ffn=128, E=8, k=2, router_kernel="tcgen05")
    need_tc = M.moe_workspace_size(tc)
    assert lib.moe_router_topk(ctypes.byref(tc.c()), fake, fake, None, fake, None, fake, fake, None, None, fake,
                               need_tc, None) == M.MOE_ERR_UNSUPPORTED
    assert lib.moe_forward(ctypes.byref(tc.c()), ctypes.byref(w), fake, fake, None, ctypes.byref(o), fake, need_tc,
                           None) == M.MOE_ERR_UNSUPPORTED


def test_workspace_size_accounts_for_buffers(lib):
    cfg = M.MoEConfig(T=4096, d=2048, ffn=4096, E=8, k=2)
    rows = M.moe_max_rows(cfg)
    assert rows == 8192
    ws = M.moe_workspace_size(cfg)
    assert ws >= rows * (2048 * 2 * 2 + 4096 * 2)
    assert M.moe_forward_launch_count(cfg) == 5
    assert M.moe_forward_launch_count(M.MoEConfig(T=0, d=64, ffn=64, E=2, k=1)) == 1


def test_expert_parallel_arguments_checked_on_host(lib):
    """The expert-parallel calls validate world, rank and pointers before any
    CUDA call (no GPU needed)."""
    c = M.MoEConfig(T=64, d=128, ffn=128, E=6, k=2)
    with pytest.raises(M.MoEError) as e:
        M.moe_ep_recv_rows(c, 128, 4)          # E % world != 0
    assert e.value.status == M.MOE_ERR_INVALID_ARG
    with pytest.raises(M.MoEError) as e:
        M.moe_ep_recv_rows(M.MoEConfig(T=64, d=128, ffn=128, E=16, k=2), 128, 16)
    assert e.value.status == M.MOE_ERR_UNSUPPORTED
    with pytest.raises(M.MoEError) as e:
        M.moe_ep_recv_rows(c, 32, 2)           # T_global below the slice
    assert e.value.status == M.MOE_ERR_INVALID_ARG
    assert M.moe_ep_recv_rows(c, 128, 2) == min(128 * 2, 3 * O.capacity(128, 2, 6, 1.25))
    assert M.moe_ep_recv_rows(M.MoEConfig(T=64, d=128, ffn=128, E=6, k=2, capacity_factor=0.0), 128, 3) == 256
    assert M.moe_ep_workspace_size(c, 128, 2) < M.moe_dp_workspace_size(c, 128)
    cfg = c.c()
    fake = ctypes.c_void_p(1 << 20)
    arr2 = (ctypes.c_void_p * 2)(1 << 20, 1 << 21)
    arr_null = (ctypes.c_void_p * 2)(1 << 20, None)
    oc = M.MoEOutputsC()
    ws = ctypes.c_size_t(1 << 30)
    disp = lib.moe_ep_dispatch
    disp.argtypes = [M._CFG, ctypes.c_int64, M._P, M._P, M._P, ctypes.c_int32, ctypes.c_int32, M._P,
                     ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(M.MoEOutputsC), M._P, M._P, ctypes.c_size_t,
                     M._P]
    disp.restype = ctypes.c_int
    # rank out of range, missing counts, a null peer buffer, missing outputs: all refused before any launch
    assert disp(ctypes.byref(cfg), 128, fake, fake, None, 2, 2, fake, arr2, ctypes.byref(oc), fake, fake, ws, None) == \
        M.MOE_ERR_INVALID_ARG
    assert disp(ctypes.byref(cfg), 128, None, fake, None, 2, 0, fake, arr2, ctypes.byref(oc), fake, fake, ws, None) == \
        M.MOE_ERR_INVALID_ARG
    assert disp(ctypes.byref(cfg), 128, fake, fake, None, 2, 0, fake, arr_null, ctypes.byref(oc), fake, fake, ws,
                None) == M.MOE_ERR_INVALID_ARG
    assert disp(ctypes.byref(cfg), 128, fake, fake, None, 2, 0, fake, arr2, ctypes.byref(oc), fake, fake, ws, None) == \
        M.MOE_ERR_INVALID_ARG
    comb = lib.moe_ep_combine
    comb.argtypes = [M._CFG, ctypes.c_int64, ctypes.c_int32, ctypes.POINTER(ctypes.c_void_p),
                     ctypes.POINTER(M.MoEOutputsC), M._P, ctypes.c_size_t, M._P]
    comb.restype = ctypes.c_int
    assert comb(ctypes.byref(cfg), 128, 2, arr_null, ctypes.byref(oc), fake, ws, None) == M.MOE_ERR_INVALID_ARG
    assert comb(ctypes.byref(cfg), 128, 2, arr2, ctypes.byref(oc), None, ws, None) == M.MOE_ERR_WORKSPACE
    # a padding mask without the real-token count to exchange is refused
    route = lib.moe_dp_route
    route.argtypes = [M._CFG, ctypes.c_int64, ctypes.POINTER(M.MoEWeightsC), M._P, M._P, M._P,
                      ctypes.POINTER(M.MoEOutputsC), M._P, M._P, M._P, M._P, ctypes.c_size_t, M._P]
    route.restype = ctypes.c_int
    w = M.MoEWeightsC()
    w.w_router = 1 << 20
    oc2 = M.MoEOutputsC()
    oc2.offsets = oc2.topk_idx = oc2.topk_w = 1 << 20
    assert route(ctypes.byref(cfg), 128, ctypes.byref(w), fake, None, fake, ctypes.byref(oc2), fake, fake, None,
                 fake, ws, None) == M.MOE_ERR_INVALID_ARG
    ipc_open = lib.moe_ipc_open
    ipc_open.argtypes = [M._P, M._P]
    ipc_open.restype = ctypes.c_int
    assert ipc_open(None, None) == M.MOE_ERR_INVALID_ARG
    assert ctypes.sizeof(M.MoEIpcBufferC) == 80


def test_status_strings(lib):
    for s in range(7):
        assert M.moe_status_string(s).startswith("MOE_")
    assert "UNKNOWN" in M.moe_status_string(99)


def test_pipeline_arguments_checked_before_any_cuda_call(lib):
    """moe_pipeline_* refuse bad arguments on the host (no GPU needed)."""
    P = ctypes.c_void_p
    lib.moe_pipeline_create.argtypes = [ctypes.POINTER(M.MoEConfigC), ctypes.POINTER(M.MoEWeightsC), ctypes.c_int32,
                                        ctypes.POINTER(P)]
    lib.moe_pipeline_submit.argtypes = [P, P, P, P, P, P, ctypes.POINTER(ctypes.c_int64)]
    lib.moe_pipeline_wait.argtypes = [P, ctypes.c_int64]
    lib.moe_pipeline_check.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.moe_pipeline_destroy.argtypes = [P]
    cfg = M.MoEConfig(T=128, d=128, ffn=128, E=8, k=2).c()
    w = M.MoEWeightsC(16, None, 32, 48, 64, None, None)  # never dereferenced on the host
    h = P()
    assert lib.moe_pipeline_create(ctypes.byref(cfg), ctypes.byref(w), 2, None) == M.MOE_ERR_INVALID_ARG
    for depth in (0, 5, -1):
        assert lib.moe_pipeline_create(ctypes.byref(cfg), ctypes.byref(w), depth, ctypes.byref(h)) == \
            M.MOE_ERR_INVALID_ARG
        assert h.value is None
    bad = M.MoEConfig(T=128, d=100, ffn=128, E=8, k=2).c()
    assert lib.moe_pipeline_create(ctypes.byref(bad), ctypes.byref(w), 2, ctypes.byref(h)) == M.MOE_ERR_UNSUPPORTED
    now = M.MoEWeightsC(None, None, 32, 48, 64, None, None)
    assert lib.moe_pipeline_create(ctypes.byref(cfg), ctypes.byref(now), 2, ctypes.byref(h)) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_pipeline_submit(None, None, None, None, None, None, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_pipeline_wait(None, -1) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_pipeline_check(None, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_pipeline_destroy(None) == M.MOE_ERR_INVALID_ARG


def test_local_expert_weights_slices_the_expert_axis():
    """A rank's weights under expert parallelism: its contiguous block of E/world
    routed experts (weights, biases and INT8 scales), router and shared experts
    as they are (reading R19: rank r holds experts [r*E/world, (r+1)*E/world))."""
    import torch
    E, d, F = 8, 4, 6
    full = {"w_router": torch.randn(d, E), "w_gate": torch.randn(E, d, F), "w_up": torch.randn(E, d, F),
            "w_down": torch.randn(E, F, d), "w_gate_scale": torch.randn(E, F), "shared_gate": torch.randn(1, d, F),
            "b1": torch.randn(E, F)}
    for world in (1, 2, 4, 8):
        for r in range(world):
            loc = M.local_expert_weights(full, world, r)
            el = E // world
            for n in ("w_gate", "w_up", "w_down", "w_gate_scale", "b1"):
                assert torch.equal(loc[n], full[n][r * el:(r + 1) * el]), (n, world, r)
                assert loc[n].is_contiguous()
            assert loc["w_router"] is full["w_router"] and loc["shared_gate"] is full["shared_gate"]
