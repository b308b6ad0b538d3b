"""Python binding of libmoe, the B200 (sm_100a) MoE layer forward.

Argument marshalling only: every step of the layer runs in the CUDA kernels
of ``libmoe.so`` behind the C ABI declared in ``include/moe.h``.  PyTorch is
used for device memory and streams.  There is no CPU fallback: if the
library is missing or fails to load, the calls raise.

The functions below carry the C names (``moe_forward``, ``moe_router_topk``,
...) and take torch tensors (or None for optional pointers); ``MoELayer``
bundles weights, outputs and workspace for the common case.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

(MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT,
 MOE_ERR_RANGE) = range(7)
MOE_MAX_RANKS = 8  # ranks of one expert-parallel group
MOE_DT_F32, MOE_DT_BF16 = 0, 1
MOE_ACT_SWIGLU, MOE_ACT_GELU_BIAS = 0, 1
MOE_ROUTER_AUTO, MOE_ROUTER_WARP_MMA, MOE_ROUTER_TCGEN05, MOE_ROUTER_WARP_MMA_STAGED = 0, 1, 2, 3
ROUTER_KERNELS = {"auto": MOE_ROUTER_AUTO, "warp_mma": MOE_ROUTER_WARP_MMA, "tcgen05": MOE_ROUTER_TCGEN05,
                  "warp_mma_staged": MOE_ROUTER_WARP_MMA_STAGED}
MOE_GEMM_AUTO, MOE_GEMM_ONE_CTA, MOE_GEMM_CTA_PAIR = 0, 1, 2
GEMM_KERNELS = {"auto": MOE_GEMM_AUTO, "one_cta": MOE_GEMM_ONE_CTA, "cta_pair": MOE_GEMM_CTA_PAIR}
MOE_DISPATCH_AUTO, MOE_DISPATCH_COPY, MOE_DISPATCH_GATHER = 0, 1, 2
DISPATCH_MODES = {"auto": MOE_DISPATCH_AUTO, "copy": MOE_DISPATCH_COPY, "gather": MOE_DISPATCH_GATHER}
MOE_WEIGHTING_AUTO, MOE_WEIGHTING_COMBINE, MOE_WEIGHTING_EPILOGUE = 0, 1, 2
WEIGHTINGS = {"auto": MOE_WEIGHTING_AUTO, "combine": MOE_WEIGHTING_COMBINE, "epilogue": MOE_WEIGHTING_EPILOGUE}


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {moe_status_string(status)}")


class MoEConfigC(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("ffn", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("dtype", ctypes.c_int32), ("act", ctypes.c_int32),
                ("capacity_factor", ctypes.c_double), ("aux_alpha", ctypes.c_float), ("router_kernel", ctypes.c_int32),
                ("gemm_kernel", ctypes.c_int32), ("dispatch", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("weight_format", ctypes.c_int32), ("weighting", ctypes.c_int32)]


class MoEWeightsC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w_router", "router_logit_bias", "w_gate_or_w1", "w_up", "w_down_or_w2", "b1", "b2",
                 "shared_gate_or_w1", "shared_up", "shared_down_or_w2", "shared_b1", "shared_b2",
                 "gate_or_w1_scale", "up_scale", "down_or_w2_scale")]


class MoEOutputsC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("out", "topk_idx", "topk_w", "counts", "offsets", "slot", "src_assign", "f", "p", "l_aux",
                 "logits_out", "probs_out")]


_lib = None
_P = ctypes.c_void_p
_CFG = ctypes.POINTER(MoEConfigC)


def lib() -> ctypes.CDLL:
    """Load libmoe.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmoe.so not built ({LIB_PATH}); run `python -m mixture_experts_layer_37_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    st = ctypes.c_int
    L.moe_status_string.argtypes = [st]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_capacity.argtypes = [_CFG, ctypes.POINTER(ctypes.c_int64)]
    L.moe_max_rows.argtypes = [_CFG, ctypes.POINTER(ctypes.c_int64)]
    L.moe_workspace_size.argtypes = [_CFG, ctypes.POINTER(ctypes.c_size_t)]
    L.moe_workspace_init.argtypes = [_P, ctypes.c_size_t, _P]
    L.moe_router_topk.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
    L.moe_dispatch.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
    L.moe_expert_ffn.argtypes = [_CFG, ctypes.POINTER(MoEWeightsC), _P, _P, _P, _P, ctypes.c_size_t, _P]
    L.moe_combine.argtypes = [_CFG, _P, _P, _P, _P, _P]
    L.moe_aux_stats.argtypes = [_CFG, _P, _P, _P, _P, _P, _P]
    L.moe_forward.argtypes = [_CFG, ctypes.POINTER(MoEWeightsC), _P, _P, _P, ctypes.POINTER(MoEOutputsC), _P,
                              ctypes.c_size_t, _P]
    L.moe_forward_profiled.argtypes = [_CFG, ctypes.POINTER(MoEWeightsC), _P, _P, _P, ctypes.POINTER(MoEOutputsC),
                                       _P, ctypes.c_size_t, _P, ctypes.POINTER(ctypes.c_void_p)]
    L.moe_forward_hostio.argtypes = [_CFG, ctypes.POINTER(MoEWeightsC), _P, _P, ctypes.POINTER(MoEOutputsC), _P, _P,
                                     _P, ctypes.c_size_t, _P]
    L.moe_check_device_status.argtypes = [_P, ctypes.c_size_t, _P, ctypes.POINTER(ctypes.c_uint32)]
    L.moe_set_wait_timeout_ms.argtypes = [ctypes.c_uint32]
    L.moe_set_wait_timeout_ms.restype = None
    L.moe_selftest_bounded_wait.argtypes = [_P, ctypes.c_size_t, ctypes.c_uint32, _P]
    L.moe_forward_launch_count.argtypes = [_CFG]
    for name in ("moe_capacity", "moe_max_rows", "moe_workspace_size", "moe_workspace_init", "moe_router_topk",
                 "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_aux_stats", "moe_forward",
                 "moe_forward_hostio", "moe_check_device_status", "moe_selftest_bounded_wait",
                 "moe_forward_launch_count", "moe_forward_profiled"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


EXPORTED_SYMBOLS = ("moe_status_string", "moe_capacity", "moe_max_rows", "moe_workspace_size", "moe_workspace_init",
                    "moe_router_topk", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_aux_stats",
                    "moe_forward", "moe_forward_hostio", "moe_check_device_status", "moe_set_wait_timeout_ms",
                    "moe_selftest_bounded_wait", "moe_forward_launch_count", "moe_forward_profiled",
                    "moe_dispatch_noalloc", "moe_dp_workspace_size", "moe_dp_max_rows", "moe_dp_route",
                    "moe_dp_finish", "moe_pipeline_create", "moe_pipeline_submit", "moe_pipeline_wait",
                    "moe_pipeline_check", "moe_pipeline_destroy", "moe_quantize_int8", "moe_ep_recv_rows",
                    "moe_ep_workspace_size", "moe_ep_route", "moe_ep_dispatch", "moe_ep_expert_ffn",
                    "moe_ep_combine", "moe_ipc_export", "moe_ipc_open", "moe_ipc_close")


# ---------------------------------------------------------------- config
@dataclass(frozen=True)
class MoEConfig:
    T: int
    d: int
    ffn: int
    E: int
    k: int
    dtype: str = "bf16"        # "bf16" | "f32"
    act: str = "swiglu"        # "swiglu" | "gelu_bias"
    capacity_factor: float = 1.25
    aux_alpha: float = 0.01
    router_kernel: str = "auto"  # "auto" | "warp_mma" | "tcgen05" | "warp_mma_staged"
    gemm_kernel: str = "auto"    # "auto" | "one_cta" | "cta_pair"
    dispatch: str = "auto"       # "auto" | "copy" | "gather"
    n_shared: int = 0            # shared experts, applied to every token with weight 1
    weights: str = "native"      # routed experts' weights: "native" (the dtype) or "int8" (codes + scales)
    weighting: str = "auto"      # routing weights applied in: "auto" | "combine" | "epilogue" (second GEMM)

    def c(self) -> MoEConfigC:
        return MoEConfigC(self.T, self.d, self.ffn, self.E, self.k,
                          MOE_DT_BF16 if self.dtype == "bf16" else MOE_DT_F32,
                          MOE_ACT_SWIGLU if self.act == "swiglu" else MOE_ACT_GELU_BIAS,
                          float(self.capacity_factor), float(self.aux_alpha), ROUTER_KERNELS[self.router_kernel],
                          GEMM_KERNELS[self.gemm_kernel], DISPATCH_MODES[self.dispatch], int(self.n_shared),
                          1 if self.weights == "int8" else 0, WEIGHTINGS[self.weighting])

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @staticmethod
    def of(wl, router_kernel: str = "auto", gemm_kernel: str = "auto", dispatch: str = "auto") -> "MoEConfig":
        """From a workload description (anything with the same field names)."""
        return MoEConfig(wl.T, wl.d, wl.ffn, wl.E, wl.k, wl.dtype, wl.act, wl.capacity_factor, wl.aux_alpha,
                         router_kernel, gemm_kernel, dispatch, getattr(wl, "n_shared", 0),
                         getattr(wl, "weights", "native"))


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr() if t.numel() > 0 else None


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoEError(status, where)


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def moe_capacity(cfg: MoEConfig) -> int:
    v = ctypes.c_int64()
    _check(lib().moe_capacity(ctypes.byref(cfg.c()), ctypes.byref(v)), "moe_capacity")
    return v.value


def moe_max_rows(cfg: MoEConfig) -> int:
    v = ctypes.c_int64()
    _check(lib().moe_max_rows(ctypes.byref(cfg.c()), ctypes.byref(v)), "moe_max_rows")
    return v.value


def moe_workspace_size(cfg: MoEConfig) -> int:
    v = ctypes.c_size_t()
    _check(lib().moe_workspace_size(ctypes.byref(cfg.c()), ctypes.byref(v)), "moe_workspace_size")
    return v.value


class Workspace:
    """A 1024-byte-aligned device buffer of moe_workspace_size() bytes, status word cleared."""

    def __init__(self, cfg: MoEConfig, device="cuda", stream=None, nbytes: Optional[int] = None):
        self.nbytes = moe_workspace_size(cfg) if nbytes is None else nbytes
        self._buf = torch.empty(self.nbytes + 1024, dtype=torch.uint8, device=device)
        off = (-self._buf.data_ptr()) % 1024
        self.tensor = self._buf[off:off + self.nbytes]
        self.ptr = self.tensor.data_ptr()
        _check(lib().moe_workspace_init(self.ptr, self.nbytes, _stream(stream)), "moe_workspace_init")


def moe_workspace_init(ws: Workspace, stream=None) -> None:
    _check(lib().moe_workspace_init(ws.ptr, ws.nbytes, _stream(stream)), "moe_workspace_init")


def moe_router_topk(cfg: MoEConfig, x, w_router, logit_bias, logits_in, topk_idx, topk_w, logits_out, probs_out,
                    ws: Workspace, stream=None, token_mask=None) -> None:
    _check(lib().moe_router_topk(ctypes.byref(cfg.c()), _ptr(x), _ptr(w_router), _ptr(logit_bias), _ptr(logits_in),
                                 _ptr(token_mask), _ptr(topk_idx), _ptr(topk_w), _ptr(logits_out), _ptr(probs_out),
                                 ws.ptr, ws.nbytes, _stream(stream)), "moe_router_topk")


def moe_dispatch(cfg: MoEConfig, x, topk_idx, counts, offsets, slot, src_assign, x_perm, ws: Workspace,
                 stream=None) -> None:
    _check(lib().moe_dispatch(ctypes.byref(cfg.c()), _ptr(x), _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(slot),
                              _ptr(src_assign), _ptr(x_perm), ws.ptr, ws.nbytes, _stream(stream)), "moe_dispatch")


def _weights_c(w: dict) -> MoEWeightsC:
    """Weights by name: w_router, router_bias, w_gate/w_up/w_down (SwiGLU) or
    w1/b1/w2/b2 (GELU), and the shared experts' shared_gate/shared_up/
    shared_down or shared_w1/shared_b1/shared_w2/shared_b2."""
    g = lambda n: _ptr(w.get(n))  # noqa: E731
    return MoEWeightsC(g("w_router"), g("router_bias"), g("w_gate") if "w_gate" in w else g("w1"), g("w_up"),
                       g("w_down") if "w_down" in w else g("w2"), g("b1"), g("b2"),
                       g("shared_gate") if "shared_gate" in w else g("shared_w1"), g("shared_up"),
                       g("shared_down") if "shared_down" in w else g("shared_w2"), g("shared_b1"), g("shared_b2"),
                       g("w_gate_scale") if "w_gate_scale" in w else g("w1_scale"), g("w_up_scale"),
                       g("w_down_scale") if "w_down_scale" in w else g("w2_scale"))


def moe_expert_ffn(cfg: MoEConfig, weights: dict, x_perm, offsets, y_perm, ws: Workspace, stream=None) -> None:
    wc = _weights_c(weights)
    _check(lib().moe_expert_ffn(ctypes.byref(cfg.c()), ctypes.byref(wc), _ptr(x_perm), _ptr(offsets), _ptr(y_perm),
                                ws.ptr, ws.nbytes, _stream(stream)), "moe_expert_ffn")


def moe_combine(cfg: MoEConfig, y_perm, slot, topk_w, out, stream=None) -> None:
    _check(lib().moe_combine(ctypes.byref(cfg.c()), _ptr(y_perm), _ptr(slot), _ptr(topk_w), _ptr(out),
                             _stream(stream)), "moe_combine")


def moe_aux_stats(cfg: MoEConfig, counts, probs, f, p, l_aux, stream=None) -> None:
    _check(lib().moe_aux_stats(ctypes.byref(cfg.c()), _ptr(counts), _ptr(probs), _ptr(f), _ptr(p), _ptr(l_aux),
                               _stream(stream)), "moe_aux_stats")


_OUT_FIELDS = ("out", "topk_idx", "topk_w", "counts", "offsets", "slot", "src_assign", "f", "p", "l_aux",
               "logits_out", "probs_out")


def _outputs_c(o: dict) -> MoEOutputsC:
    return MoEOutputsC(*[_ptr(o.get(n)) for n in _OUT_FIELDS])


def allocate_outputs(cfg: MoEConfig, device="cuda", with_logits: bool = False, with_probs: bool = False) -> dict:
    T, E, k = cfg.T, cfg.E, cfg.k
    o = {
        "out": torch.empty((T, cfg.d), dtype=cfg.torch_dtype, device=device),
        "topk_idx": torch.empty((T, k), dtype=torch.int32, device=device),
        "topk_w": torch.empty((T, k), dtype=torch.float32, device=device),
        "counts": torch.empty(E, dtype=torch.int32, device=device),
        "offsets": torch.empty(E + 1, dtype=torch.int32, device=device),
        "slot": torch.empty((T, k), dtype=torch.int32, device=device),
        "src_assign": torch.empty(max(moe_max_rows(cfg), 1), dtype=torch.int32, device=device),
        "f": torch.empty(E, dtype=torch.float32, device=device),
        "p": torch.empty(E, dtype=torch.float32, device=device),
        "l_aux": torch.empty(1, dtype=torch.float32, device=device),
    }
    if with_logits:
        o["logits_out"] = torch.empty((T, E), dtype=torch.float32, device=device)
    if with_probs:
        o["probs_out"] = torch.empty((T, E), dtype=torch.float32, device=device)
    return o


def moe_forward(cfg: MoEConfig, weights: dict, x, outputs: dict, ws: Workspace, logits_in=None, stream=None,
                token_mask=None) -> None:
    wc = _weights_c(weights)
    oc = _outputs_c(outputs)
    _check(lib().moe_forward(ctypes.byref(cfg.c()), ctypes.byref(wc), _ptr(x), _ptr(logits_in), _ptr(token_mask),
                             ctypes.byref(oc), ws.ptr, ws.nbytes, _stream(stream)), "moe_forward")


def moe_forward_profiled(cfg: MoEConfig, weights: dict, x, outputs: dict, ws: Workspace, events: list,
                         logits_in=None, stream=None, token_mask=None) -> None:
    """moe_forward recording torch.cuda.Event objects `events` (n+1 of them,
    n = moe_forward_launch_count) around each kernel launch on `stream`."""
    wc = _weights_c(weights)
    oc = _outputs_c(outputs)
    arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    _check(lib().moe_forward_profiled(ctypes.byref(cfg.c()), ctypes.byref(wc), _ptr(x), _ptr(logits_in),
                                      _ptr(token_mask), ctypes.byref(oc), ws.ptr, ws.nbytes, _stream(stream), arr),
           "moe_forward_profiled")


def moe_forward_hostio(cfg: MoEConfig, weights: dict, x_host, x_dev, outputs: dict, out_host, l_aux_host,
                       ws: Workspace, stream=None) -> None:
    wc = _weights_c(weights)
    oc = _outputs_c(outputs)
    _check(lib().moe_forward_hostio(ctypes.byref(cfg.c()), ctypes.byref(wc), _ptr(x_host), _ptr(x_dev),
                                    ctypes.byref(oc), _ptr(out_host), _ptr(l_aux_host), ws.ptr, ws.nbytes,
                                    _stream(stream)), "moe_forward_hostio")


def moe_check_device_status(ws: Workspace, stream=None) -> tuple:
    """(status, site): synchronises the stream, reads and clears the status word."""
    site = ctypes.c_uint32(0)
    st = lib().moe_check_device_status(ws.ptr, ws.nbytes, _stream(stream), ctypes.byref(site))
    return st, site.value


def moe_set_wait_timeout_ms(ms: int) -> None:
    lib().moe_set_wait_timeout_ms(int(ms))


def moe_selftest_bounded_wait(ws: Workspace, timeout_ms: int, stream=None) -> None:
    _check(lib().moe_selftest_bounded_wait(ws.ptr, ws.nbytes, int(timeout_ms), _stream(stream)),
           "moe_selftest_bounded_wait")


def moe_forward_launch_count(cfg: MoEConfig) -> int:
    return lib().moe_forward_launch_count(ctypes.byref(cfg.c()))


# ---------------------------------------------------------------- layer
class MoELayer:
    """Weights + preallocated outputs and workspace for repeated forwards."""

    def __init__(self, cfg: MoEConfig, weights: dict, device="cuda", with_logits=False, with_probs=False):
        self.cfg = cfg
        self.weights = weights
        self.outputs = allocate_outputs(cfg, device, with_logits, with_probs)
        self.ws = Workspace(cfg, device)

    def forward(self, x: torch.Tensor, logits_in: Optional[torch.Tensor] = None, stream=None,
                token_mask: Optional[torch.Tensor] = None) -> dict:
        moe_forward(self.cfg, self.weights, x, self.outputs, self.ws, logits_in, stream, token_mask)
        return self.outputs

    def capture(self, x: torch.Tensor, logits_in: Optional[torch.Tensor] = None,
                token_mask: Optional[torch.Tensor] = None) -> "torch.cuda.CUDAGraph":
        """Records one forward on the fixed buffers `x` / `logits_in` into a CUDA
        graph (five kernel launches, no host work when replayed).  A replay
        reads `x` as it is at that time; results land in `self.outputs`."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.forward(x, logits_in, token_mask=token_mask)  # uncaptured first call: kernel attributes
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.forward(x, logits_in, token_mask=token_mask)
        self.graph = g
        return g

    def replay(self) -> dict:
        """Replays the graph made by `capture` on the current stream."""
        self.graph.replay()
        return self.outputs

    def check(self, stream=None) -> None:
        st, site = moe_check_device_status(self.ws, stream)
        if st != MOE_OK:
            raise MoEError(st, f"device status (site 0x{site:x})")


def moe_dispatch_noalloc(cfg: MoEConfig, x, topk_idx, counts, offsets, slot, src_assign, x_perm, stream=None) -> None:
    """moe_dispatch without a workspace, for callers that cannot allocate device
    memory: the scratch lives in a fixed array inside the library (see
    include/moe.h for the size limit and the rule that calls must not overlap)."""
    L = lib()
    f = L.moe_dispatch_noalloc
    f.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P, _P]
    f.restype = ctypes.c_int
    _check(f(ctypes.byref(cfg.c()), _ptr(x), _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(slot),
             _ptr(src_assign), _ptr(x_perm), _stream(stream)), "moe_dispatch_noalloc")


# ---------------------------------------------------------------- data-parallel shards of one batch
def moe_dp_workspace_size(cfg: MoEConfig, T_global: int) -> int:
    L = lib()
    f = L.moe_dp_workspace_size
    f.argtypes = [_CFG, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)]
    f.restype = ctypes.c_int
    v = ctypes.c_size_t()
    _check(f(ctypes.byref(cfg.c()), int(T_global), ctypes.byref(v)), "moe_dp_workspace_size")
    return v.value


def moe_dp_max_rows(cfg: MoEConfig, T_global: int) -> int:
    L = lib()
    f = L.moe_dp_max_rows
    f.argtypes = [_CFG, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]
    f.restype = ctypes.c_int
    v = ctypes.c_int64()
    _check(f(ctypes.byref(cfg.c()), int(T_global), ctypes.byref(v)), "moe_dp_max_rows")
    return v.value


def moe_dp_route(cfg: MoEConfig, T_global: int, weights: dict, x, outputs: dict, local_counts, local_psum,
                 ws: Workspace, logits_in=None, stream=None, token_mask=None, local_real=None) -> None:
    L = lib()
    f = L.moe_dp_route
    f.argtypes = [_CFG, ctypes.c_int64, ctypes.POINTER(MoEWeightsC), _P, _P, _P, ctypes.POINTER(MoEOutputsC), _P, _P,
                  _P, _P, ctypes.c_size_t, _P]
    f.restype = ctypes.c_int
    wc = _weights_c(weights)
    oc = _outputs_c(outputs)
    _check(f(ctypes.byref(cfg.c()), int(T_global), ctypes.byref(wc), _ptr(x), _ptr(logits_in), _ptr(token_mask),
             ctypes.byref(oc), _ptr(local_counts), _ptr(local_psum), _ptr(local_real), ws.ptr, ws.nbytes,
             _stream(stream)), "moe_dp_route")


def moe_dp_finish(cfg: MoEConfig, T_global: int, all_counts, all_psum, world: int, rank: int, weights: dict, x,
                  outputs: dict, ws: Workspace, stream=None, all_real=None) -> None:
    L = lib()
    f = L.moe_dp_finish
    f.argtypes = [_CFG, ctypes.c_int64, _P, _P, _P, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(MoEWeightsC), _P,
                  ctypes.POINTER(MoEOutputsC), _P, ctypes.c_size_t, _P]
    f.restype = ctypes.c_int
    wc = _weights_c(weights)
    oc = _outputs_c(outputs)
    _check(f(ctypes.byref(cfg.c()), int(T_global), _ptr(all_counts), _ptr(all_psum), _ptr(all_real), int(world),
             int(rank), ctypes.byref(wc), _ptr(x), ctypes.byref(oc), ws.ptr, ws.nbytes, _stream(stream)),
           "moe_dp_finish")


# ---------------------------------------------------------------- expert parallelism
_EXPERT_KEYS = ("w_gate", "w_up", "w_down", "w1", "b1", "w2", "b2", "w_gate_scale", "w_up_scale", "w_down_scale",
                "w1_scale", "w2_scale")


def local_expert_weights(weights: dict, world: int, rank: int) -> dict:
    """The weights rank `rank` holds under expert parallelism: its contiguous
    block of E/world routed experts (views along the expert axis), with the
    router and the shared experts as they are (replicated)."""
    out = dict(weights)
    for n in _EXPERT_KEYS:
        if n in weights and weights[n] is not None:
            E = weights[n].shape[0]
            el = E // world
            out[n] = weights[n][rank * el:(rank + 1) * el]
    return out


def _ptr_array(ptrs) -> ctypes.Array:
    vals = [p.data_ptr() if isinstance(p, torch.Tensor) else int(p) for p in ptrs]
    return (ctypes.c_void_p * len(vals))(*vals)


def _ep_fn(name: str, argtypes: list):
    f = getattr(lib(), name)
    f.argtypes = argtypes
    f.restype = ctypes.c_int
    return f


def moe_ep_recv_rows(cfg: MoEConfig, T_global: int, world: int) -> int:
    v = ctypes.c_int64()
    f = _ep_fn("moe_ep_recv_rows", [_CFG, ctypes.c_int64, ctypes.c_int32, ctypes.POINTER(ctypes.c_int64)])
    _check(f(ctypes.byref(cfg.c()), int(T_global), int(world), ctypes.byref(v)), "moe_ep_recv_rows")
    return v.value


def moe_ep_workspace_size(cfg: MoEConfig, T_global: int, world: int) -> int:
    v = ctypes.c_size_t()
    f = _ep_fn("moe_ep_workspace_size", [_CFG, ctypes.c_int64, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)])
    _check(f(ctypes.byref(cfg.c()), int(T_global), int(world), ctypes.byref(v)), "moe_ep_workspace_size")
    return v.value


def moe_ep_route(cfg: MoEConfig, T_global: int, world: int, weights: dict, x, outputs: dict, local_counts,
                 local_psum, ws: Workspace, logits_in=None, stream=None, token_mask=None, local_real=None) -> None:
    f = _ep_fn("moe_ep_route", [_CFG, ctypes.c_int64, ctypes.c_int32, ctypes.POINTER(MoEWeightsC), _P, _P, _P,
                                ctypes.POINTER(MoEOutputsC), _P, _P, _P, _P, ctypes.c_size_t, _P])
    wc = _weights_c(weights)
    oc = _outputs_c(outputs)
    _check(f(ctypes.byref(cfg.c()), int(T_global), int(world), ctypes.byref(wc), _ptr(x), _ptr(logits_in),
             _ptr(token_mask), ctypes.byref(oc), _ptr(local_counts), _ptr(local_psum), _ptr(local_real), ws.ptr,
             ws.nbytes, _stream(stream)), "moe_ep_route")


def moe_ep_dispatch(cfg: MoEConfig, T_global: int, all_counts, all_psum, world: int, rank: int, x, x_recv,
                    outputs: dict, recv_offsets, ws: Workspace, stream=None, all_real=None) -> None:
    """x_recv: every rank's receive buffer (tensors on this device, or device
    pointers this process can dereference), in rank order."""
    f = _ep_fn("moe_ep_dispatch", [_CFG, ctypes.c_int64, _P, _P, _P, ctypes.c_int32, ctypes.c_int32, _P,
                                   ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(MoEOutputsC), _P, _P,
                                   ctypes.c_size_t, _P])
    oc = _outputs_c(outputs)
    _check(f(ctypes.byref(cfg.c()), int(T_global), _ptr(all_counts), _ptr(all_psum), _ptr(all_real), int(world),
             int(rank), _ptr(x), _ptr_array(x_recv), ctypes.byref(oc), _ptr(recv_offsets), ws.ptr, ws.nbytes,
             _stream(stream)), "moe_ep_dispatch")


def moe_ep_expert_ffn(cfg: MoEConfig, T_global: int, world: int, weights: dict, x, x_recv, recv_offsets, y_recv,
                      ws: Workspace, stream=None) -> None:
    """weights: this rank's experts (local_expert_weights) and the shared experts."""
    f = _ep_fn("moe_ep_expert_ffn", [_CFG, ctypes.c_int64, ctypes.c_int32, ctypes.POINTER(MoEWeightsC), _P, _P, _P,
                                     _P, _P, ctypes.c_size_t, _P])
    wc = _weights_c(weights)
    _check(f(ctypes.byref(cfg.c()), int(T_global), int(world), ctypes.byref(wc), _ptr(x), _ptr(x_recv),
             _ptr(recv_offsets), _ptr(y_recv), ws.ptr, ws.nbytes, _stream(stream)), "moe_ep_expert_ffn")


def moe_ep_combine(cfg: MoEConfig, T_global: int, world: int, y_recv, outputs: dict, ws: Workspace,
                   stream=None) -> None:
    """y_recv: every rank's output buffer, in rank order (as x_recv of moe_ep_dispatch)."""
    f = _ep_fn("moe_ep_combine", [_CFG, ctypes.c_int64, ctypes.c_int32, ctypes.POINTER(ctypes.c_void_p),
                                  ctypes.POINTER(MoEOutputsC), _P, ctypes.c_size_t, _P])
    oc = _outputs_c(outputs)
    _check(f(ctypes.byref(cfg.c()), int(T_global), int(world), _ptr_array(y_recv), ctypes.byref(oc), ws.ptr,
             ws.nbytes, _stream(stream)), "moe_ep_combine")


class MoEIpcBufferC(ctypes.Structure):
    _fields_ = [("handle", ctypes.c_uint8 * 64), ("offset", ctypes.c_uint64), ("bytes", ctypes.c_uint64)]


def moe_ipc_export(t: torch.Tensor) -> bytes:
    """The record (bytes) naming device tensor t's memory for other processes."""
    rec = MoEIpcBufferC()
    f = _ep_fn("moe_ipc_export", [_P, ctypes.POINTER(MoEIpcBufferC)])
    _check(f(t.data_ptr(), ctypes.byref(rec)), "moe_ipc_export")
    return bytes(rec)


def moe_ipc_open(record: bytes) -> int:
    """Maps another process's exported buffer; returns its device pointer here."""
    rec = MoEIpcBufferC.from_buffer_copy(record)
    ptr = ctypes.c_void_p()
    f = _ep_fn("moe_ipc_open", [ctypes.POINTER(MoEIpcBufferC), ctypes.POINTER(ctypes.c_void_p)])
    _check(f(ctypes.byref(rec), ctypes.byref(ptr)), "moe_ipc_open")
    return int(ptr.value)


def moe_ipc_close(ptr: int, record: bytes) -> None:
    rec = MoEIpcBufferC.from_buffer_copy(record)
    f = _ep_fn("moe_ipc_close", [_P, ctypes.POINTER(MoEIpcBufferC)])
    _check(f(ptr, ctypes.byref(rec)), "moe_ipc_close")


# ---------------------------------------------------------------- pipelined forwards on host batches
class Pipeline:
    """moe_pipeline_*: forwards on host-resident batches, the copy in of the
    next batch and the copy out of the previous one overlapping the current
    forward.  Host tensors should be pinned (``pin_memory()``); they must stay
    untouched (inputs) or unread (outputs) until ``wait`` covers their step."""

    def __init__(self, cfg: MoEConfig, weights: dict, depth: int = 2):
        L = lib()
        L.moe_pipeline_create.argtypes = [_CFG, ctypes.POINTER(MoEWeightsC), ctypes.c_int32, ctypes.POINTER(_P)]
        L.moe_pipeline_submit.argtypes = [_P, _P, _P, _P, _P, _P, ctypes.POINTER(ctypes.c_int64)]
        L.moe_pipeline_wait.argtypes = [_P, ctypes.c_int64]
        L.moe_pipeline_check.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32)]
        L.moe_pipeline_destroy.argtypes = [_P]
        for n in ("moe_pipeline_create", "moe_pipeline_submit", "moe_pipeline_wait", "moe_pipeline_check",
                  "moe_pipeline_destroy"):
            getattr(L, n).restype = ctypes.c_int
        self._L = L
        self.cfg = cfg
        self.weights = weights  # kept alive: the pipeline reads them on every step
        self._wc = _weights_c(weights)
        h = _P()
        _check(L.moe_pipeline_create(ctypes.byref(cfg.c()), ctypes.byref(self._wc), int(depth), ctypes.byref(h)),
               "moe_pipeline_create")
        self._h = h

    def submit(self, x_host: torch.Tensor, out_host: torch.Tensor, l_aux_host: torch.Tensor,
               start_event=None, end_event=None) -> int:
        t = ctypes.c_int64()
        _check(self._L.moe_pipeline_submit(self._h, _ptr(x_host), _ptr(out_host), _ptr(l_aux_host),
                                           start_event.cuda_event if start_event is not None else None,
                                           end_event.cuda_event if end_event is not None else None,
                                           ctypes.byref(t)), "moe_pipeline_submit")
        return t.value

    def wait(self, ticket: int = -1) -> None:
        _check(self._L.moe_pipeline_wait(self._h, int(ticket)), "moe_pipeline_wait")

    def check(self) -> None:
        site = ctypes.c_uint32()
        st = self._L.moe_pipeline_check(self._h, ctypes.byref(site))
        if st != MOE_OK:
            raise MoEError(st, f"pipeline device status (site 0x{site.value:x})")

    def close(self) -> None:
        if getattr(self, "_h", None):
            _check(self._L.moe_pipeline_destroy(self._h), "moe_pipeline_destroy")
            self._h = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_quantize_int8(cfg: MoEConfig, w: torch.Tensor, stream=None):
    """INT8 codes and per-expert, per-output-column scales of expert weights
    w [E, K, N] (moe_quantize_int8).  Returns (codes int8 [E, K, N], scales
    float32 [E, N]), both on w's device."""
    L = lib()
    f = L.moe_quantize_int8
    f.argtypes = [_CFG, _P, ctypes.c_int64, ctypes.c_int64, _P, _P, _P]
    f.restype = ctypes.c_int
    E, K, N = w.shape
    q = torch.empty((E, K, N), dtype=torch.int8, device=w.device)
    s = torch.empty((E, N), dtype=torch.float32, device=w.device)
    _check(f(ctypes.byref(cfg.c()), _ptr(w), int(K), int(N), _ptr(q), _ptr(s), _stream(stream)), "moe_quantize_int8")
    return q, s


def quantize_expert_weights(cfg: MoEConfig, weights: dict, stream=None) -> dict:
    """A copy of `weights` whose routed experts are stored as INT8 codes plus
    scales (w_gate/w_up/w_down or w1/w2 replaced by codes, with *_scale added)."""
    out = dict(weights)
    for name in (("w_gate", "w_up", "w_down") if cfg.act == "swiglu" else ("w1", "w2")):
        q, s = moe_quantize_int8(cfg, weights[name], stream)
        out[name] = q
        out[name + "_scale"] = s
    return out
