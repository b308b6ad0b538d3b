#!/usr/bin/env python
"""Benchmark of the MoE layer forward (tokens/s) through the libmoe C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]
                    [--mode replicas|ep]

One step = one whole layer forward (router, top-k, dispatch, expert FFNs,
combine, aux statistics: five kernel launches) over one batch of the workload,
inputs resident in HBM.  Between steps, outside the timed events, a 256 MiB
buffer (twice the L2) is written and a second one read, so every step starts
with a cold L2 that holds no dirty lines.  The K timed steps (L2 clearing and
forward each) are captured into one CUDA graph and replayed once, so the host
adds no gaps between launches; the forward's own events (recorded by
moe_forward_profiled between its launches, as external records that stay in
the graph) time each step and each stage, the dominant stage giving the
roofline.  The same steps run eagerly (launches from the host each step) are
reported beside it.  Under torchrun each rank runs its own independent batch
(weak scaling, no collective on the data path); the time is the maximum over
ranks.

With no --workload, the line is the largest single-GPU workload
(longctx_zipf_t32768: T=32768, E=32, d=ffn=4096, capacity drops) and, at one
GPU, carries a ``per_config`` table with the same measurements (tokens/s,
stage times, roofline of the dominant kernel, host-buffer e2e, and the CPU
oracle on all host cores and on one core) for all five benchmark workloads.

``--impl reference`` times the CPU oracle (numpy, float64) on the host cores
on a bounded token sample of the same workload.  ``--mode ep`` shards the
experts over the GPUs instead (see run_ep).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd tokens/s; grouped-FFN TFLOP/s & HBM GB/s vs B200 peak"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "longctx_zipf_t32768"
ALL_WORKLOADS = ("tiny_f32", "llama4moe_t4096", "flat_gelu_t8192", "longctx_zipf_t32768", "decode_t64_e64")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
FLUSH_BYTES = 256 << 20
ORACLE_SAMPLE_TOKENS = 64


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None, help=f"one workload (default {DEFAULT_WORKLOAD} plus the per-config table)")
    ap.add_argument("--per-config-steps", type=int, default=10, help="timed steps of each other workload in per_config")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--mode", default="replicas", choices=["replicas", "ep"],
                    help="replicas: an independent batch per GPU (default); ep: experts sharded over the GPUs")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=10.0, help="per oracle leg, headline workload")
    ap.add_argument("--per-config-cpu-seconds", type=float, default=4.0, help="per oracle leg, other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--router-kernel", default="auto", choices=["auto", "warp_mma", "tcgen05"])
    ap.add_argument("--gemm-kernel", default="auto", choices=["auto", "one_cta", "cta_pair"])
    ap.add_argument("--dispatch", default="auto", choices=["auto", "copy", "gather"])
    ap.add_argument("--n-shared", type=int, default=None, help="shared experts (default: the workload's)")
    ap.add_argument("--pad-fraction", type=float, default=None, help="padding tokens (default: the workload's)")
    ap.add_argument("--weights", default=None, choices=["native", "int8"], help="routed experts' weight storage")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- oracle timing
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample_tokens(wl) -> int:
    """Tokens of the oracle's sub-batch per step: the largest n <= 64 (at least
    1) whose experts' weights (decoded to float64 by the oracle for every
    expert the sub-batch reaches, at most min(E, n*k) of them) stay near 4e8
    values, so that one step takes a few seconds at most."""
    per_expert = (3 if wl.act == "swiglu" else 2) * wl.d * wl.ffn
    n = 64
    while n > 1 and min(wl.E, n * wl.k) * per_expert > 4e8:
        n //= 2
    return min(n, wl.T)


def oracle_sample(wl, inp, n: int):
    """The first n tokens of the workload as a batch of their own (same weights):
    x, and the padding mask when there is one, cut to n rows."""
    sub = wl.with_(T=n)
    si = dict(inp)
    si["x"] = inp["x"][:n]
    if inp.get("token_mask") is not None:
        si["token_mask"] = inp["token_mask"][:n]
    return sub, si


def oracle_step(sub, si):
    """One whole forward of the oracle (routing, capacity dispatch, expert FFNs,
    combine, statistics) on the sub-batch."""
    from oracle import moe_oracle as O
    O.forward(sub, si)


def time_oracle(wl, inp, steps=None, seconds=None, warmup=0, threads=None):
    """The oracle as it stands, on `threads` BLAS threads (None: all of them)."""
    from threadpoolctl import threadpool_limits
    n = oracle_sample_tokens(wl)
    sub, si = oracle_sample(wl, inp, n)
    with threadpool_limits(limits=threads):
        cores = blas_threads()
        for _ in range(warmup):
            oracle_step(sub, si)
        k, t0 = 0, time.perf_counter()
        while True:
            oracle_step(sub, si)
            k += 1
            el = time.perf_counter() - t0
            if (steps is not None and k >= steps) or (seconds is not None and el >= seconds):
                break
    return {"value": k * n / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "cpu": cpu_model(), "host_cores": os.cpu_count(),
            "sample": f"{k} oracle steps; each a whole layer forward (float64, numpy/BLAS) of a batch of the "
                      f"workload's first {n} tokens with its weights (capacity of that batch); "
                      f"value = output tokens / second",
            "seconds": round(el, 3)}


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_id: str):
        self.proc = None
        self.path = tempfile.mktemp(prefix="clocks_", suffix=".csv")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", dev_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        loaded = [s for s in sm if s > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# --------------------------------------------------------------------------- native
GEMM_SOURCES = ("gemm_sm100.cu", "gemm_sm100_pair.cu", "gemm_common.cuh", "common.cuh")


def kernel_source_hash() -> str:
    """Hash of the grouped-GEMM sources; recorded ncu traffic is used only while it matches."""
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "mixture_experts_layer_37_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(f"{kernel}@{workload}")
    if not ent or ent.get("source_sha") != kernel_source_hash():
        return None
    return ent.get("bytes_per_launch")


def bench_workload(a, name: str, steps: int, warmup: int, cpu_seconds: float, world: int, rank: int, local: int):
    """Every measurement of one workload: graph-replayed and eager device
    steps, stage times and the dominant kernel's roofline, the host-buffer e2e
    paths, and (rank 0, one GPU) the CPU oracle on all cores and on one core.
    Returns the JSON line's fields (on every rank; only rank 0 prints)."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import mixture_experts_layer_37_b200 as M
    import workloads as W

    wl = W.WORKLOADS[name]
    if a.n_shared is not None:
        wl = wl.with_(n_shared=a.n_shared)
    if a.pad_fraction is not None:
        wl = wl.with_(pad_fraction=a.pad_fraction)
    if a.weights is not None:
        wl = wl.with_(weights=a.weights)
    cfg = M.MoEConfig.of(wl, a.router_kernel, a.gemm_kernel, a.dispatch)
    seed = wl.seed + 1000 * rank
    inp = W.make_inputs(wl, seed=seed)

    def dev(arr):
        if arr.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(np.ascontiguousarray(arr)).cuda()

    wnames = ("w_router", "w_gate", "w_up", "w_down", "w1", "b1", "w2", "b2", "shared_gate", "shared_up",
              "shared_down", "shared_w1", "shared_b1", "shared_w2", "shared_b2")
    weights = {n: dev(inp[n]) for n in wnames if n in inp}
    if inp.get("router_bias") is not None:
        weights["router_bias"] = dev(np.asarray(inp["router_bias"], dtype=np.float32))
    if wl.weights == "int8":
        weights = M.quantize_expert_weights(cfg, weights)  # once, before anything is timed
        torch.cuda.synchronize()
    x = dev(inp["x"])
    tmask = dev(inp["token_mask"]) if "token_mask" in inp else None
    layer = M.MoELayer(cfg, weights)
    nl = M.moe_forward_launch_count(cfg)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    evict = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")

    def clear_l2():
        # the write leaves the L2 full of dirty lines of `flush`; reading `evict`
        # writes them back here, outside the timed events, and leaves it cold
        flush.zero_()
        evict.sum()

    def make_events(n):
        evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n)]
        for e in evs:
            e.record(stream)
        return evs

    for _ in range(warmup):
        clear_l2()
        layer.forward(x, token_mask=tmask)
    torch.cuda.synchronize()
    layer.check()

    # eager steps, for comparison: every launch issued from the host
    eager = [make_events(nl + 1) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        clear_l2()
        M.moe_forward_profiled(cfg, weights, x, layer.outputs, layer.ws, eager[i], token_mask=tmask)
    torch.cuda.synchronize()
    eager_ms = float(sum(ev[0].elapsed_time(ev[nl]) for ev in eager))

    # the timed region: K steps captured into one graph
    step_ev = [make_events(nl + 1) for _ in range(steps)]
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(steps):
            clear_l2()
            M.moe_forward_profiled(cfg, weights, x, layer.outputs, layer.ws, step_ev[i], token_mask=tmask)
    graph.replay()  # upload and warm the graph
    torch.cuda.synchronize()
    layer.check()
    dev_id = str(torch.cuda.get_device_properties(local).uuid) if hasattr(torch.cuda.get_device_properties(local), "uuid") else str(local)
    if not dev_id.startswith("GPU-") and len(dev_id) > 8:
        dev_id = "GPU-" + dev_id
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev_id)
    time.sleep(0.2)
    graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    layer.check()

    stage_ms = np.array([[ev[j].elapsed_time(ev[j + 1]) for j in range(nl)] for ev in step_ev])
    step_ms = np.array([ev[0].elapsed_time(ev[nl]) for ev in step_ev])
    total_ms = float(step_ms.sum())
    if world > 1:
        t = torch.tensor([total_ms, eager_ms], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms, eager_ms = float(t[0].item()), float(t[1].item())
    value = world * wl.T * steps / (total_ms / 1e3)

    # ---------------- roofline of the dominant kernel
    R = int(layer.outputs["offsets"][-1].item())
    # router includes the fused dispatch scan; two GEMMs per shared expert before the combine
    names = ["router", "scatter", "gemm1", "gemm2"] + \
        [f"shared{i}_gemm{j}" for i in range(wl.n_shared) for j in (1, 2)] + ["combine"]
    assert len(names) == nl, (names, nl)
    mean_stage = stage_ms.mean(axis=0)
    pk, pk_src = peaks()
    bpe = 2 if wl.dtype == "bf16" else 4
    gemm1_flops = (4 if wl.act == "swiglu" else 2) * wl.d * wl.ffn * R
    gemm2_flops = 2 * wl.d * wl.ffn * R
    # each expert GEMM is bound by the tensor cores or by streaming the weights of
    # the experts that received rows, whichever its FLOP per byte puts it under
    hit = int((layer.outputs["offsets"].diff() > 0).sum().item())
    wbpe = 1 if wl.weights == "int8" else bpe
    nmat1 = 2 if wl.act == "swiglu" else 1
    gemm1_bytes = hit * nmat1 * wl.d * wl.ffn * wbpe + R * (wl.d + wl.ffn) * bpe
    gemm2_bytes = hit * wl.d * wl.ffn * wbpe + R * (wl.d + wl.ffn) * bpe
    balance = pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)

    def gemm_bound(flops, nbytes):
        return ("tensor", flops) if flops / nbytes >= balance else ("hbm", nbytes)

    algo = {
        "router": ("hbm", wl.T * wl.d * bpe + wl.d * wl.E * bpe + wl.T * wl.k * 8),
        "scatter": ("hbm", 2 * R * wl.d * bpe + wl.T * wl.k * 4 * 3),
        "gemm1": gemm_bound(gemm1_flops, gemm1_bytes),
        "gemm2": gemm_bound(gemm2_flops, gemm2_bytes),
        "combine": ("hbm", R * wl.d * bpe + (1 + wl.n_shared) * wl.T * wl.d * bpe + wl.T * wl.k * 8),
    }
    for i in range(wl.n_shared):
        algo[f"shared{i}_gemm1"] = ("tensor", (4 if wl.act == "swiglu" else 2) * wl.d * wl.ffn * wl.T)
        algo[f"shared{i}_gemm2"] = ("tensor", 2 * wl.d * wl.ffn * wl.T)
    dom = int(np.argmax(mean_stage))
    dname = names[dom]
    bound, work = algo[dname]
    dur_s = mean_stage[dom] / 1e3
    if bound == "tensor":
        achieved = work / dur_s / 1e12
        peak = pk["bf16_tflops"]
        unit = "TFLOP/s"
    else:
        achieved = work / dur_s / 1e9
        peak = pk["hbm_gbs"]
        unit = "GB/s"
    roofline = {"bound": bound, "kernel": f"grouped expert GEMM ({dname})" if "gemm" in dname else dname,
                "achieved": round(achieved, 2), "peak": peak, "peak_source": f"{pk_src} ({'bf16 dense burst' if bound == 'tensor' else 'HBM copy'})",
                "unit": unit, "frac": round(achieved / peak, 4),
                "traffic": recorded_traffic(dname, name) if "gemm" in dname and wl.weights == "native" else None}
    # the whole forward against HBM: every stage's algorithmic bytes (GEMMs: the
    # weights of the experts hit plus their activation rows) over the step time;
    # the bound that matters when the weights dominate (decode)
    shared_bytes = wl.n_shared * ((nmat1 + 1) * wl.d * wl.ffn * bpe + 2 * wl.T * (wl.d + wl.ffn) * bpe)
    fwd_bytes = algo["router"][1] + algo["scatter"][1] + gemm1_bytes + gemm2_bytes + shared_bytes + \
        algo["combine"][1]
    fwd_gbs = fwd_bytes / (total_ms / steps / 1e3) / 1e9
    forward_roofline = {"bound": "hbm", "bytes_per_step": int(fwd_bytes), "achieved": round(fwd_gbs, 1),
                        "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(fwd_gbs / pk["hbm_gbs"], 4)}
    stages = {}
    for j, n in enumerate(names):
        b, w = algo[n]
        ent = {"ms": round(float(mean_stage[j]), 4)}
        if b == "tensor":
            ent["TFLOP/s"] = round(w / (mean_stage[j] / 1e3) / 1e12, 1)
        elif w:
            ent["GB/s"] = round(w / (mean_stage[j] / 1e3) / 1e9, 1)
        stages[n] = ent

    # ---------------- end to end from host memory
    # (a) the pipelined C-ABI object: step i+1's copy in and step i-1's copy out
    #     overlap step i's forward; every step copies its own batch in and its
    #     output and L_aux out.  Steps overlap, so the L2 is not flushed between
    #     them; every step streams the expert weights, which exceed the L2.
    def pinned_x():
        if wl.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(inp["x"]).view(np.int16)).view(torch.bfloat16).pin_memory()
        return torch.from_numpy(np.ascontiguousarray(inp["x"])).pin_memory()

    depth = 2
    xs_host = [pinned_x() for _ in range(depth)]
    outs_host = [torch.empty_like(xs_host[0]).pin_memory() for _ in range(depth)]
    ls_host = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(depth)]
    pipe = M.Pipeline(cfg, weights, depth=depth)
    for i in range(max(3, warmup)):
        pipe.submit(xs_host[i % depth], outs_host[i % depth], ls_host[i % depth])
    pipe.wait()
    e_start, e_end = make_events(2)  # created and recorded once here; the pipeline re-records them
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    for i in range(steps):
        pipe.submit(xs_host[i % depth], outs_host[i % depth], ls_host[i % depth],
                    start_event=e_start if i == 0 else None, end_event=e_end if i == steps - 1 else None)
    pipe.wait()
    torch.cuda.synchronize()
    e2e_ms = e_start.elapsed_time(e_end)
    pipe.check()
    pipe.close()
    ref_out = layer.forward(x)["out"].cpu()  # the host-buffer paths take no padding mask
    assert torch.equal(outs_host[(steps - 1) % depth], ref_out), "pipelined output differs from the forward"

    # (b) one synchronous-style call per step (moe_forward_hostio: copy in,
    #     forward, copy out on one stream), L2 flushed between steps
    x_host, out_host, l_host = xs_host[0], outs_host[0], ls_host[0]
    x_dev = torch.empty_like(x)
    e2e_ev = [make_events(2) for _ in range(steps)]
    for _ in range(max(1, warmup // 2)):
        clear_l2()
        M.moe_forward_hostio(cfg, weights, x_host, x_dev, layer.outputs, out_host, l_host, layer.ws)
    torch.cuda.synchronize()
    for i in range(steps):
        clear_l2()
        e2e_ev[i][0].record(stream)
        M.moe_forward_hostio(cfg, weights, x_host, x_dev, layer.outputs, out_host, l_host, layer.ws)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    serial_ms = float(sum(ev[0].elapsed_time(ev[1]) for ev in e2e_ev))
    if world > 1:
        t = torch.tensor([e2e_ms, serial_ms], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms, serial_ms = float(t[0].item()), float(t[1].item())
    layer.check()
    bx = wl.T * wl.d * bpe
    wbytes = sum(int(v.numel() * v.element_size()) for v in weights.values())
    e2e = {"value": round(world * wl.T * steps / (e2e_ms / 1e3), 1), "unit": UNIT,
           "h2d_bytes_per_step": bx, "d2h_bytes_per_step": bx + 4,
           "api": f"moe_pipeline_submit (depth {depth}): copy in, forward, copy out per step, overlapped across steps",
           "l2": f"not flushed (steps overlap); expert weights {wbytes / 2**20:.0f} MiB > L2",
           "unpipelined": {"value": round(world * wl.T * steps / (serial_ms / 1e3), 1), "unit": UNIT,
                           "api": "moe_forward_hostio, one stream, L2 flushed between steps"}}

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = time_oracle(wl, inp, seconds=cpu_seconds)
        one = time_oracle(wl, inp, seconds=cpu_seconds, threads=1)
        cpu["one_core"] = {"value": one["value"], "unit": UNIT, "cores": one["cores"], "sample": one["sample"],
                           "seconds": one["seconds"]}

    if world > 1:
        dist.barrier()
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": round(total_ms / steps, 4),
        "eager_ms_per_step": round(eager_ms / steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic (seeded, generated on host)",
        "config": {"workload": name, "T": wl.T, "d": wl.d, "ffn": wl.ffn, "E": wl.E, "k": wl.k,
                   "act": wl.act, "capacity_factor": wl.capacity_factor, "rows_dispatched": R,
                   "parallelism": f"dp{world} (independent batches per GPU)",
                   "l2": "flushed between steps outside the timed events: 256 MiB written, then 256 MiB read",
                   "launch": "timed steps replayed from one captured CUDA graph",
                   "router_kernel": a.router_kernel, "gemm_kernel": a.gemm_kernel, "dispatch": a.dispatch},
        "roofline": roofline, "forward_roofline": forward_roofline, "stages": stages, "e2e": e2e, "gpu_launches": nl * steps,
        "clocks": clocks, "cpu_baseline": cpu,
    }
    del layer, weights, x, flush, evict, graph
    torch.cuda.empty_cache()
    return line


def per_config_entry(line: dict) -> dict:
    """The summary of one workload's line kept in the headline's per_config table."""
    keep = ("value", "unit", "ms_per_step", "steps", "dtype", "roofline", "forward_roofline", "stages", "clocks")
    ent = {k: line[k] for k in keep}
    ent["rows_dispatched"] = line["config"]["rows_dispatched"]
    ent["e2e"] = {k: line["e2e"][k] for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step")}
    ent["e2e_unpipelined"] = line["e2e"]["unpipelined"]["value"]
    cpu = line.get("cpu_baseline")
    if cpu:
        ent["cpu_oracle_all_cores"] = {"value": round(cpu["value"], 3), "cores": cpu["cores"]}
        ent["cpu_oracle_one_core"] = {"value": round(cpu["one_core"]["value"], 3), "cores": 1}
    return ent


def run_native(a):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    head = a.workload or DEFAULT_WORKLOAD
    line = bench_workload(a, head, a.steps, a.warmup, a.cpu_baseline_seconds, world, rank, local)
    if a.workload is None and world == 1:
        # the other benchmark workloads, measured the same way with fewer steps
        table = {}
        for name in ALL_WORKLOADS:
            if name == head:
                table[name] = per_config_entry(line)
                continue
            other = bench_workload(a, name, a.per_config_steps, max(3, min(a.warmup, 5)),
                                   a.per_config_cpu_seconds, world, rank, local)
            table[name] = per_config_entry(other)
        line["per_config"] = table
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_ep(a):
    """--mode ep: expert parallelism.  One batch of world x T tokens, each rank
    holding a slice of T tokens and E/world experts (ExpertParallelMoE: rows
    stored into and loaded from the other ranks' buffers over CUDA IPC
    mappings, NCCL for the count all-gathers and the two barriers).  Weak
    scaling: tokens and experts per GPU stay fixed as world grows.  Steps run
    eagerly (the collectives are host calls); the time is the maximum over
    ranks of the summed CUDA-event step times."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import mixture_experts_layer_37_b200 as M
    import workloads as W
    from mixture_experts_layer_37_b200.ep import ExpertParallelMoE

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29531")
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    name = a.workload or DEFAULT_WORKLOAD
    wl = W.WORKLOADS[name]
    if wl.E % world != 0 or world > M.MOE_MAX_RANKS:
        raise SystemExit(f"--mode ep needs E % world == 0 and world <= {M.MOE_MAX_RANKS} (E={wl.E}, world={world})")
    T, T_global = wl.T, world * wl.T
    wlg = wl.with_(T=T_global)
    inp = W.make_inputs(wlg)
    El = wl.E // world

    def dev(arr):
        if arr.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(np.ascontiguousarray(arr)).cuda()

    weights = {}
    for n in ("w_router", "shared_gate", "shared_up", "shared_down", "shared_w1", "shared_b1", "shared_w2",
              "shared_b2"):
        if n in inp:
            weights[n] = dev(inp[n])
    for n in ("w_gate", "w_up", "w_down", "w1", "b1", "w2", "b2"):
        if n in inp:
            weights[n] = dev(inp[n][rank * El:(rank + 1) * El])   # this rank's experts only
    if inp.get("router_bias") is not None:
        weights["router_bias"] = dev(np.asarray(inp["router_bias"], dtype=np.float32))
    x = dev(inp["x"][rank * T:(rank + 1) * T])
    cfg = M.MoEConfig(T=T, d=wl.d, ffn=wl.ffn, E=wl.E, k=wl.k, dtype=wl.dtype, act=wl.act,
                      capacity_factor=wl.capacity_factor, aux_alpha=wl.aux_alpha, router_kernel=a.router_kernel,
                      gemm_kernel=a.gemm_kernel, n_shared=wl.n_shared)
    ep = ExpertParallelMoE(cfg, weights, T_global=T_global)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    evict = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")

    def clear_l2():
        flush.zero_()
        evict.sum()

    def make_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record()
        return evs

    for _ in range(a.warmup):
        clear_l2()
        ep.forward(x)
    torch.cuda.synchronize()
    st = M.moe_check_device_status(ep.ws)[0]
    assert st == M.MOE_OK, M.moe_status_string(st)
    steps = [make_events(6) for _ in range(a.steps)]
    props = torch.cuda.get_device_properties(local)
    dev_id = str(props.uuid) if hasattr(props, "uuid") else str(local)
    if not dev_id.startswith("GPU-") and len(dev_id) > 8:
        dev_id = "GPU-" + dev_id
    dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev_id)
    time.sleep(0.2)
    for i in range(a.steps):
        clear_l2()
        ep.forward(x, events=steps[i])
    torch.cuda.synchronize()
    dist.barrier()
    clocks = sampler.stop()
    st = M.moe_check_device_status(ep.ws)[0]
    assert st == M.MOE_OK, M.moe_status_string(st)
    ph = np.array([[ev[j].elapsed_time(ev[j + 1]) for j in range(5)] for ev in steps])
    total_ms = float(sum(ev[0].elapsed_time(ev[5]) for ev in steps))
    recv = int(ep.recv_offsets[-1].item())
    t = torch.tensor([total_ms], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t[0].item())
    value = world * T * a.steps / (total_ms / 1e3)
    # the owner's expert FFNs (two grouped GEMMs over the received rows) against the bf16 peak
    ffn_ms = float(ph[:, 2].mean())
    flops = ((6 if wl.act == "swiglu" else 4) * wl.d * wl.ffn * recv
             + wl.n_shared * (6 if wl.act == "swiglu" else 4) * wl.d * wl.ffn * T)
    pk, pk_src = peaks()
    achieved = flops / (ffn_ms / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": "expert FFN phase of rank 0 (grouped GEMMs over the received rows)",
                "achieved": round(achieved, 2), "peak": pk["bf16_tflops"],
                "peak_source": f"{pk_src} (bf16 dense burst)",
                "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_tflops"], 4), "traffic": None}
    phase_names = ["route+all-gather+dispatch", "barrier_before_ffn", "expert FFN", "barrier_before_combine", "combine"]
    phases = {n: round(float(ph[:, j].mean()), 4) for j, n in enumerate(phase_names)}
    launches = (6 + 2 * wl.n_shared) * a.steps
    ep.close()
    dist.barrier()
    dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(total_ms / a.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic (seeded, generated on host)",
        "config": {"workload": name, "T_per_gpu": T, "T_global": T_global, "d": wl.d, "ffn": wl.ffn,
                   "E": wl.E, "experts_per_gpu": El, "k": wl.k, "act": wl.act,
                   "capacity_factor": wl.capacity_factor, "rows_received_rank0": recv,
                   "parallelism": f"ep{world} (experts sharded, one batch over all ranks)",
                   "l2": "flushed between steps outside the timed events: 256 MiB written, then 256 MiB read",
                   "launch": "eager (the count all-gathers and barriers are NCCL calls)"},
        "roofline": roofline, "phases_ms_rank0": phases,
        "e2e": None, "e2e_note": "device-resident inputs only in this mode",
        "gpu_launches": launches, "clocks": clocks,
        "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


def run_reference(a):
    import workloads as W
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = a.workload or DEFAULT_WORKLOAD
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    res = time_oracle(wl, inp, steps=a.steps, warmup=a.warmup)
    line = {"metric": METRIC, "value": round(res["value"], 3), "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": round(1e3 * res["seconds"] / a.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, generated on host)",
            "config": {"workload": name, "T": wl.T, "d": wl.d, "ffn": wl.ffn, "E": wl.E, "k": wl.k,
                       "act": wl.act, "capacity_factor": wl.capacity_factor},
            "impl": "reference",
            "cpu_baseline": {"kind": "oracle", "cores": res["cores"], "sample": res["sample"], "value": round(res["value"], 3),
                             "unit": UNIT},
            "e2e": {"value": round(res["value"], 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    elif a.mode == "ep":
        run_ep(a)
    else:
        run_native(a)


if __name__ == "__main__":
    main()
