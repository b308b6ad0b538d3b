"""Data-parallel sharding of one batch, on CPU ranks (gloo, world sizes 2 and 3).

The orchestration of mixture_experts_layer_37_b200.dp (slice order, the two
all-gathers in rank order, the whole-batch token count) runs for real over
torch.distributed; the two device phases are replaced by stand-ins built from
the oracle, so no GPU is needed.  The stand-in finish phase applies the rule
the device phase implements: rank r may keep max(0, cap - base_e) rows of
expert e, base_e = assignments to e on lower ranks.  The test checks that the
sharded result equals the oracle's dispatch and statistics of the whole batch,
also with padding tokens masked out (the real-token counts travel with the
expert counts, and f and p divide by their sum)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _workload(T, pad_fraction=0.0):
    import workloads as W
    return W.Workload("dp", T=T, d=32, ffn=64, E=6, k=2, act="swiglu", dtype="f32", capacity_factor=0.7,
                      zipf_router_bias=True, seed=31, w_std=0.2, pad_fraction=pad_fraction)


def _worker(rank, world, port, bounds, pad, q):
    import sys
    sys.path.insert(0, ROOT)
    import workloads as W
    from oracle import moe_oracle as O
    from mixture_experts_layer_37_b200 import MoEConfig
    from mixture_experts_layer_37_b200.dp import DataParallelMoE

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = _workload(bounds[-1], pad)
        inp = W.make_inputs(wl, with_experts=False)
        t0, t1 = bounds[rank], bounds[rank + 1]
        full = O.route(wl, inp)
        logits_local = full["logits"][t0:t1]
        mask = inp.get("token_mask")
        cap = O.capacity(wl.T, wl.k, wl.E, wl.capacity_factor)
        state = {}

        def route(x, logits_in, token_mask):
            assert (token_mask is None) == (mask is None)
            real = O.real_tokens(None if token_mask is None else token_mask.numpy(), t1 - t0)
            p = O.softmax(logits_local) * real[:, None]
            idx, _ = O.mask_padding(O.select_topk(logits_local, wl.k), np.zeros((t1 - t0, wl.k)),
                                    None if token_mask is None else token_mask.numpy())
            state["idx"] = idx
            dp.local_counts.copy_(torch.from_numpy(np.bincount(idx[idx >= 0], minlength=wl.E).astype(np.int32)))
            dp.local_psum.copy_(torch.from_numpy(p.sum(axis=0)))
            dp.local_real.fill_(int(real.sum()))

        def finish(x, all_counts, all_psum, all_real):
            ac = all_counts.numpy().astype(np.int64)
            base = ac[:rank].sum(axis=0)
            cap_left = np.maximum(0, cap - base)
            d = O.dispatch(state["idx"], wl.E, 10 ** 9)
            kept = (state["idx"] >= 0) & (d["rank"] < cap_left[np.maximum(state["idx"], 0)])
            gcounts = ac.sum(axis=0)
            t_real = int(all_real.numpy().sum())
            f, pm, l = O.aux_stats(gcounts, np.zeros((0, wl.E)), t_real, wl.k, wl.aux_alpha)
            pm = all_psum.numpy().sum(axis=0) / t_real
            l = wl.aux_alpha * wl.E * float(np.sum(f * pm))
            return {"kept": kept, "counts": gcounts, "f": f, "p": pm, "l_aux": l, "all_real": all_real.numpy()}

        cfg = MoEConfig(T=t1 - t0, d=wl.d, ffn=wl.ffn, E=wl.E, k=wl.k, dtype="f32", capacity_factor=wl.capacity_factor)
        dp = DataParallelMoE(cfg, {}, device="cpu", route=route, finish=finish)
        assert dp.T_global == wl.T and dp.world == world and dp.rank == rank
        tm = None if mask is None else torch.from_numpy(mask[t0:t1].copy())
        res = dp.forward(torch.zeros((t1 - t0, wl.d)), token_mask=tm)
        q.put((rank, res["kept"], res["counts"], res["f"], res["p"], res["l_aux"], res["all_real"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bounds,pad", [([0, 120, 257], 0.0), ([0, 50, 51, 200], 0.0), ([0, 90, 257], 0.2)],
                         ids=["world2", "world3", "world2-padding"])
def test_sharded_batch_equals_whole_batch(bounds, pad):
    import workloads as W
    from oracle import moe_oracle as O

    world = len(bounds) - 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, bounds, pad, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        r, kept, counts, f, p, l, all_real = q.get(timeout=120)
        results[r] = (kept, counts, f, p, l, all_real)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = _workload(bounds[-1], pad)
    inp = W.make_inputs(wl, with_experts=False)
    full = O.route(wl, inp)
    kept_all = np.concatenate([results[r][0] for r in range(world)])
    assert np.array_equal(kept_all, full["slot"] >= 0)
    assert (full["slot"] < 0).any(), "the case must exercise drops"
    real = O.real_tokens(inp.get("token_mask"), wl.T)
    if pad:
        assert not real.all(), "the case must exercise padding"
    for r in range(world):
        _, counts, f, p, l, all_real = results[r]
        assert all_real.tolist() == [int(real[bounds[i]:bounds[i + 1]].sum()) for i in range(world)]
        assert np.array_equal(counts, full["counts"])
        np.testing.assert_allclose(f, full["f"], rtol=1e-15)
        np.testing.assert_allclose(p, full["p_mean"], rtol=1e-12)
        assert abs(l - full["l_aux"]) <= 1e-12 * abs(full["l_aux"])


@pytest.mark.parametrize("world,E", [(1, 8), (2, 6), (3, 5), (1, 64)])
def test_slice_stats_pack_and_unpack(world, E):
    """The packed per-slice statistics (fp64 sums, int32 counts, int32 real
    tokens) come back exactly from gathered rows, also for a single rank."""
    from mixture_experts_layer_37_b200.dp import SliceStats
    rows = []
    for r in range(world):
        st = SliceStats(E, "cpu")
        st.psum.copy_(torch.arange(E, dtype=torch.float64) * 0.25 + r)
        st.counts.copy_(torch.arange(E, dtype=torch.int32) * 3 + r)
        st.real.fill_(100 + r)
        assert st.buf.numel() % 8 == 0
        rows.append(st.buf.clone())
    counts, psum, real = SliceStats.unpack(torch.stack(rows), E)
    for r in range(world):
        assert torch.equal(psum[r], torch.arange(E, dtype=torch.float64) * 0.25 + r)
        assert torch.equal(counts[r], torch.arange(E, dtype=torch.int32) * 3 + r)
        assert int(real[r]) == 100 + r
    assert counts.is_contiguous() and psum.is_contiguous() and real.is_contiguous()
