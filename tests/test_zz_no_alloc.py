"""The allocation-free dispatch entry point, moe_dispatch_noalloc.

It exists for callers that cannot allocate device memory and so cannot pass
a workspace (for example a plugin that only receives its input and output
buffers from a host framework owning every allocation).  Its scratch lives in
a fixed array inside the library.  This file checks, through the C ABI, that
two calls in a row give exactly what the workspace-based moe_dispatch gives
(index work is compared bit for bit, row copies byte for byte), with the
second call running on scratch the first one left behind, and that shapes
beyond the array's limit are refused before anything runs.  It sits in its
own file, collected last, and needs nothing from the other test files."""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_layer_37_b200 as M
import workloads as W
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def _dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _outputs(cfg):
    rows = max(M.moe_max_rows(cfg), 1)
    return {
        "counts": torch.full((cfg.E,), -1, dtype=torch.int32, device="cuda"),
        "offsets": torch.full((cfg.E + 1,), -1, dtype=torch.int32, device="cuda"),
        "slot": torch.full((cfg.T, cfg.k), -9, dtype=torch.int32, device="cuda"),
        "src_assign": torch.full((rows,), -9, dtype=torch.int32, device="cuda"),
        "x_perm": torch.zeros((rows, cfg.d), dtype=cfg.torch_dtype, device="cuda"),
    }


def _compare(wl):
    cfg = M.MoEConfig.of(wl)
    inp = W.make_inputs(wl, with_experts=False)
    idx = _dev(O.route(wl, inp)["idx"])
    x = _dev(inp["x"])
    ref = _outputs(cfg)
    ws = M.Workspace(cfg)
    M.moe_dispatch(cfg, x, idx, ref["counts"], ref["offsets"], ref["slot"], ref["src_assign"], ref["x_perm"], ws)
    got = _outputs(cfg)
    M.moe_dispatch_noalloc(cfg, x, idx, got["counts"], got["offsets"], got["slot"], got["src_assign"],
                           got["x_perm"])
    torch.cuda.synchronize()
    R = int(ref["offsets"][-1].item())
    for n in ("counts", "offsets", "slot"):
        assert torch.equal(got[n], ref[n]), n
    assert torch.equal(got["src_assign"][:R], ref["src_assign"][:R])
    as_int = torch.int16 if wl.dtype == "bf16" else torch.int32
    assert torch.equal(got["x_perm"][:R].view(as_int), ref["x_perm"][:R].view(as_int))
    return R


def test_noalloc_dispatch_matches_workspace_dispatch_twice():
    # first call: a large batch fills many scratch entries
    big = W.WORKLOADS["llama4moe_t4096"]
    assert _compare(big) > 0
    # second call, right after: a different shape (ragged T, k=3, drops) on the
    # scratch the first call left behind
    small = W.Workload("noalloc_second", T=777, d=192, ffn=320, E=5, k=3, act="gelu_bias", dtype="bf16",
                       capacity_factor=0.8, seed=202)
    assert _compare(small) > 0


def test_noalloc_dispatch_rejects_shapes_beyond_its_scratch():
    cfg = M.MoEConfig(T=64 * 1024 + 1, d=64, ffn=64, E=64, k=2).c()
    fake = ctypes.c_void_p(1 << 40)
    f = M.lib().moe_dispatch_noalloc
    f.argtypes = [ctypes.POINTER(M.MoEConfigC)] + [ctypes.c_void_p] * 8
    f.restype = ctypes.c_int
    assert f(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake, fake, None) == M.MOE_ERR_UNSUPPORTED
    ok = M.MoEConfig(T=64 * 1024, d=64, ffn=64, E=64, k=2)
    assert M.moe_workspace_size(ok) > 0  # the largest accepted shape is a valid config
