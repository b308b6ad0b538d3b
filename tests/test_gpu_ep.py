"""Expert parallelism (experts sharded over ranks), checked on one GPU.

Emulated ranks: every rank's buffers live on the one GPU and the calls run
rank after rank on one stream (moe_ep_route for all, the stacked counts as the
all-gather, then moe_ep_dispatch, moe_ep_expert_ffn and moe_ep_combine for
all); stream order stands in for the barriers, and "peer" buffers are the
other ranks' buffers on the same device.  No kernel waits on another.  The
results must equal one moe_forward over the whole batch bit for bit, every
slot and receive offset must be the oracle's expert-parallel layout, and
every received row must be its token's row, byte for byte.

Two processes on the one GPU then run the same path through
ExpertParallelMoE with CUDA IPC mappings of each other's buffers and host
barriers (gloo), and a refusal test feeds counts and slots that do not match
the routing and checks that the kernels refuse the rows (MOE_ERR_RANGE)
instead of touching memory outside the buffers."""
import dataclasses
import os
import socket

import numpy as np
import pytest
import torch

import mixture_experts_layer_37_b200 as M
import workloads as W
from oracle import moe_oracle as O
from gpu_common import host_f64, mask_dev, out_close, sample_tokens, to_dev, weights_dev

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

ZIPF = W.Workload("ep_zipf_drops", T=1000, d=128, ffn=192, E=16, k=2, act="swiglu", dtype="bf16",
                  capacity_factor=0.6, zipf_router_bias=True, seed=301, w_std=0.05)
CASES = [
    (ZIPF, [0, 1000]),
    (ZIPF, [0, 300, 301, 777, 1000]),
    (ZIPF, [0, 100, 200, 300, 400, 500, 600, 700, 1000]),
    (W.Workload("ep_gelu_k3", T=600, d=192, ffn=256, E=6, k=3, act="gelu_bias", dtype="bf16",
                capacity_factor=0.9, seed=302), [0, 0, 333, 600]),
    (W.Workload("ep_shared", T=517, d=128, ffn=128, E=8, k=2, act="swiglu", dtype="bf16", capacity_factor=1.0,
                n_shared=1, seed=303), [0, 259, 517]),
    (W.Workload("ep_int8", T=300, d=256, ffn=128, E=8, k=2, act="swiglu", dtype="bf16", capacity_factor=1.25,
                weights="int8", seed=304), [0, 150, 300]),
    (W.WORKLOADS["tiny_f32"], [0, 40, 64]),
    (W.Workload("ep_shared_pad", T=700, d=128, ffn=192, E=8, k=2, act="swiglu", dtype="bf16", capacity_factor=0.8,
                n_shared=1, pad_fraction=0.2, seed=305), [0, 170, 171, 520, 700]),
    (W.WORKLOADS["longctx_zipf_t32768"], [i * 4096 for i in range(9)]),
]
IDS = [f"{wl.name}-{len(b) - 1}" for wl, b in CASES]


def _slice_cfg(wl, t0, t1, router="auto"):
    return M.MoEConfig(T=t1 - t0, d=wl.d, ffn=wl.ffn, E=wl.E, k=wl.k, dtype=wl.dtype, act=wl.act,
                       capacity_factor=wl.capacity_factor, aux_alpha=wl.aux_alpha, router_kernel=router,
                       n_shared=wl.n_shared, weights=wl.weights)


def run_emulated(wl, bounds, wd, x, all_counts_fn=None, fill=None, mask=None):
    """Runs the four expert-parallel calls for every emulated rank; returns the
    ranks' state.  `fill`: a value written into the receive buffers first."""
    world = len(bounds) - 1
    El = wl.E // world
    ranks = []
    for r in range(world):
        t0, t1 = bounds[r], bounds[r + 1]
        c = _slice_cfg(wl, t0, t1)
        rows = max(M.moe_ep_recv_rows(c, wl.T, world), 1)
        st = dict(cfg=c, t0=t0, t1=t1, rows=rows,
                  x_recv=torch.empty((rows, wl.d), dtype=c.torch_dtype, device="cuda"),
                  y_recv=torch.empty((rows, wl.d), dtype=c.torch_dtype, device="cuda"),
                  recv_offsets=torch.full((El + 1,), -7, dtype=torch.int32, device="cuda"),
                  out=M.allocate_outputs(c),
                  ws=M.Workspace(c, nbytes=M.moe_ep_workspace_size(c, wl.T, world)),
                  lc=torch.zeros(wl.E, dtype=torch.int32, device="cuda"),
                  lp=torch.zeros(wl.E, dtype=torch.float64, device="cuda"),
                  lr=torch.zeros(1, dtype=torch.int32, device="cuda"))
        if fill is not None:
            st["x_recv"].fill_(fill)
            st["y_recv"].fill_(fill)
        M.moe_ep_route(c, wl.T, world, wd, x[t0:t1], st["out"], st["lc"], st["lp"], st["ws"],
                       token_mask=None if mask is None else mask[t0:t1], local_real=st["lr"])
        ranks.append(st)
    all_counts = torch.stack([s["lc"] for s in ranks])
    all_psum = torch.stack([s["lp"] for s in ranks])
    all_real = torch.cat([s["lr"] for s in ranks])
    if all_counts_fn is not None:
        all_counts = all_counts_fn(all_counts)
    xr = [s["x_recv"] for s in ranks]
    yr = [s["y_recv"] for s in ranks]
    for r, s in enumerate(ranks):
        M.moe_ep_dispatch(s["cfg"], wl.T, all_counts, all_psum, world, r, x[s["t0"]:s["t1"]], xr, s["out"],
                          s["recv_offsets"], s["ws"], all_real=all_real)
    for r, s in enumerate(ranks):
        M.moe_ep_expert_ffn(s["cfg"], wl.T, world, M.local_expert_weights(wd, world, r), x[s["t0"]:s["t1"]],
                            s["x_recv"], s["recv_offsets"], s["y_recv"], s["ws"])
    for s in ranks:
        M.moe_ep_combine(s["cfg"], wl.T, world, yr, s["out"], s["ws"])
    torch.cuda.synchronize()
    return ranks


def _whole_cfg(wl):
    """The one-device forward the expert-parallel calls must equal bit for bit:
    they weight the expert rows in the combine, so this one does too."""
    return dataclasses.replace(M.MoEConfig.of(wl), weighting="combine")


def _device_weights(wl, inp):
    wd = weights_dev(wl, inp)
    if wl.weights == "int8":
        wd = M.quantize_expert_weights(M.MoEConfig.of(wl), wd)
    return wd


@pytest.mark.parametrize("wl,bounds", CASES, ids=IDS)
def test_ep_equals_whole_batch(wl, bounds):
    inp = W.make_inputs(wl)
    wd = _device_weights(wl, inp)
    x = to_dev(inp["x"])
    mask = mask_dev(inp)
    whole = M.MoELayer(_whole_cfg(wl), wd).forward(x, token_mask=mask)
    torch.cuda.synchronize()
    world = len(bounds) - 1
    El = wl.E // world
    ranks = run_emulated(wl, bounds, wd, x, mask=mask)
    for s in ranks:
        assert M.moe_check_device_status(s["ws"])[0] == M.MOE_OK
    cat = lambda n: torch.cat([s["out"][n] for s in ranks]).cpu()  # noqa: E731
    idx, slot_whole = whole["topk_idx"].cpu().numpy(), whole["slot"].cpu().numpy()
    assert torch.equal(cat("topk_idx"), whole["topk_idx"].cpu())
    lay = O.expert_parallel_layout(idx, slot_whole, wl.E, world)
    assert np.array_equal(cat("slot").numpy(), lay["row"]), "rows in the owners' buffers"
    for r, s in enumerate(ranks):
        assert s["recv_offsets"].cpu().numpy().tolist() == lay["recv_offsets"][r].tolist()
        n = int(lay["recv_offsets"][r][-1])
        src_tok = torch.from_numpy(lay["recv_src"][r] // wl.k).cuda()
        assert torch.equal(s["x_recv"][:n].view(torch.int16 if wl.dtype == "bf16" else torch.int32),
                           x[src_tok].view(torch.int16 if wl.dtype == "bf16" else torch.int32)), \
            f"rank {r}: received rows are not the tokens' rows"
        assert torch.equal(s["out"]["counts"].cpu(), whole["counts"].cpu())
        assert torch.equal(s["out"]["offsets"].cpu(), whole["offsets"].cpu())
        assert torch.equal(s["out"]["f"].cpu(), whole["f"].cpu())
        np.testing.assert_allclose(s["out"]["p"].cpu().numpy(), whole["p"].cpu().numpy(), rtol=1e-6)
        np.testing.assert_allclose(s["out"]["l_aux"].cpu().numpy(), whole["l_aux"].cpu().numpy(), rtol=1e-6)
    view = torch.int16 if wl.dtype == "bf16" else torch.int32
    assert torch.equal(cat("out").view(view), whole["out"].cpu().view(view)), "layer output differs from one device"
    if wl.capacity_factor > 0 and wl.T >= 600:
        assert (slot_whole < 0).any(), "the case must exercise drops"
    # and against the oracle where its routing agrees with the GPU's
    r_or = O.route(wl, inp)
    toks = np.arange(wl.T) if wl.T <= 2048 else sample_tokens(wl, r_or, n_random=64, per_expert=2)
    agree = (idx == r_or["idx"]).all(axis=1) & ((slot_whole >= 0) == (r_or["slot"] >= 0)).all(axis=1)
    toks = toks[agree[toks]]
    ref = O.forward(wl, inp, routing=r_or, tokens=toks)
    ok, e_, s_ = out_close(host_f64(cat("out"))[toks], ref["out"], wl.dtype)
    assert ok, f"max err {e_} vs scale {s_}"
    assert El * world == wl.E


def test_ep_refuses_inconsistent_counts_and_slots():
    """Counts that do not match the routing (a negative entry) make the prepare
    step keep nothing and report MOE_ERR_RANGE; a slot past the receive buffer
    handed to the combine is refused (term skipped, MOE_ERR_RANGE).  With the
    counts refused, no row of any receive buffer is written."""
    wl = ZIPF
    inp = W.make_inputs(wl)
    wd = weights_dev(wl, inp)
    x = to_dev(inp["x"])
    bounds = [0, 500, 1000]

    def bad_counts(ac):
        ac = ac.clone()
        ac[1, 3] = -1
        return ac

    ranks = run_emulated(wl, bounds, wd, x, all_counts_fn=bad_counts, fill=3.0)
    for s in ranks:
        assert (s["x_recv"].float() == 3.0).all() and (s["y_recv"].float() == 3.0).all()
        assert M.moe_check_device_status(s["ws"])[0] == M.MOE_ERR_RANGE
        assert (s["out"]["slot"] == -1).all()
        assert (s["recv_offsets"] == 0).all()
        assert (s["out"]["out"].float() == 0).all()
        assert M.moe_check_device_status(s["ws"])[0] == M.MOE_OK  # cleared by the read
    # a slot past the buffer, handed to the combine
    ranks = run_emulated(wl, bounds, wd, x)
    s = ranks[0]
    good = s["out"]["out"].clone()
    t = int(torch.nonzero(s["out"]["slot"][:, 0] >= 0)[0, 0])
    s["out"]["slot"][t, 0] = s["rows"] + 5
    M.moe_ep_combine(s["cfg"], wl.T, 2, [r["y_recv"] for r in ranks], s["out"], s["ws"])
    assert M.moe_check_device_status(s["ws"])[0] == M.MOE_ERR_RANGE
    changed = (s["out"]["out"] != good).any(dim=1).nonzero().flatten().tolist()
    assert changed == [t], changed


# ------------------------------------------------------------------ two processes, CUDA IPC
def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _ipc_child(rec, n, q):
    import sys
    import traceback
    sys.path.insert(0, ROOT)
    try:
        import torch as T_
        import mixture_experts_layer_37_b200 as M_
        ptr = M_.moe_ipc_open(rec)

        class _Arr:
            __cuda_array_interface__ = {"shape": (n,), "typestr": "<f4", "data": (ptr, False), "version": 3}

        t = T_.as_tensor(_Arr(), device="cuda")
        seen = t.cpu().numpy().copy()
        t.mul_(2.0)
        T_.cuda.synchronize()
        M_.moe_ipc_close(ptr, rec)
        q.put(seen)
    except Exception:
        q.put(traceback.format_exc())


def test_ipc_export_open_between_processes():
    import torch.multiprocessing as mp
    buf = torch.arange(4096, dtype=torch.float32, device="cuda")
    sub = buf[1000:2000]                                  # inside the allocation: the record carries the offset
    rec = M.moe_ipc_export(sub)
    torch.cuda.synchronize()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_ipc_child, args=(rec, 1000, q))
    p.start()
    seen = q.get(timeout=240)
    p.join(timeout=60)
    assert not isinstance(seen, str), seen
    assert p.exitcode == 0
    assert np.array_equal(seen, np.arange(1000, 2000, dtype=np.float32))
    assert torch.equal(buf[1000:2000].cpu(), torch.arange(1000, 2000, dtype=torch.float32) * 2)
    assert torch.equal(buf[:1000].cpu(), torch.arange(1000, dtype=torch.float32))


def _ep_worker(rank, world, port, bounds, q):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    import workloads as W_
    import mixture_experts_layer_37_b200 as M_
    from mixture_experts_layer_37_b200.ep import ExpertParallelMoE
    from gpu_common import to_dev as to_dev_, weights_dev as weights_dev_

    import traceback
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=120))
    try:
        wl = ZIPF
        inp = W_.make_inputs(wl)
        wd = weights_dev_(wl, inp)
        x = to_dev_(inp["x"])
        t0, t1 = bounds[rank], bounds[rank + 1]
        ep = ExpertParallelMoE(_slice_cfg(wl, t0, t1), M_.local_expert_weights(wd, world, rank), T_global=wl.T)
        res = ep.forward(x[t0:t1])
        res2 = ep.forward(x[t0:t1])                          # the buffers are reused by a second forward
        torch.cuda.synchronize()
        status = M_.moe_check_device_status(ep.ws)[0]
        q.put((rank, status, res2["out"].cpu().view(torch.int16).numpy(), res["slot"].cpu().numpy()))
        ep.close()
    except Exception:
        q.put((rank, traceback.format_exc(), None, None))
        raise
    finally:
        dist.destroy_process_group()


def test_ep_two_processes_over_ipc():
    """ExpertParallelMoE in two processes on the one GPU: each maps the other's
    receive buffers through CUDA IPC; barriers on the host (gloo)."""
    import torch.multiprocessing as mp
    wl = ZIPF
    inp = W.make_inputs(wl)
    wd = weights_dev(wl, inp)
    x = to_dev(inp["x"])
    whole = M.MoELayer(_whole_cfg(wl), wd).forward(x)
    torch.cuda.synchronize()
    bounds = [0, 420, 1000]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, 2, port, bounds, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(2):
        r, status, out, slot = q.get(timeout=300)
        assert status == M.MOE_OK, f"rank {r}: {status}"
        got[r] = (out, slot)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = np.concatenate([got[0][0], got[1][0]])
    assert np.array_equal(out, whole["out"].cpu().view(torch.int16).numpy())
    lay = O.expert_parallel_layout(whole["topk_idx"].cpu().numpy(), whole["slot"].cpu().numpy(), wl.E, 2)
    assert np.array_equal(np.concatenate([got[0][1], got[1][1]]), lay["row"])
