"""Expert parallelism over CPU ranks (gloo, world sizes 2 and 3).

The orchestration of mixture_experts_layer_37_b200.ep runs for real over
torch.distributed: the whole-batch token count, the all-gathers in rank
order, the two barriers and the peer-buffer plumbing.  The receive buffers
are shared-memory CPU tensors that every rank holds (standing in for the
NVLink peer mappings), and the four device phases are stand-ins built from
the oracle that put every row where the library's kernels put it: a slice's
kept rows of expert e start, in the owner's buffer, after the blocks of the
owner's lower experts (each of size min(total, cap)), plus
min(rows of e on lower ranks, cap).  Ranks above 0 wait before they write
rows, so a missing barrier would let an owner read rows that have not landed.
The test checks the sharded forward against the oracle's whole-batch layer,
and every slot against the oracle's expert-parallel layout."""
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


def _workload(T, E=6):
    import workloads as W
    return W.Workload("ep", T=T, d=16, ffn=24, E=E, k=2, act="swiglu", dtype="f32", capacity_factor=0.7,
                      zipf_router_bias=True, seed=41, w_std=0.2)


def _worker(rank, world, port, bounds, E, xr, yr, q):
    import sys
    import time
    sys.path.insert(0, ROOT)
    import workloads as W
    from oracle import moe_oracle as O
    from mixture_experts_layer_37_b200 import MoEConfig
    from mixture_experts_layer_37_b200.ep import ExpertParallelMoE

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = _workload(bounds[-1], E)
        inp = W.make_inputs(wl)
        full = O.route(wl, inp)
        x = O.to_f64(inp["x"], wl.dtype)
        t0, t1 = bounds[rank], bounds[rank + 1]
        E, k, El, cap = wl.E, wl.k, wl.E // world, full["cap"]
        st = {}

        def route(x_, logits_in, token_mask):
            assert token_mask is None
            idx = full["idx"][t0:t1]
            st["idx"] = idx
            ep.local_counts.copy_(torch.from_numpy(np.bincount(idx[idx >= 0], minlength=E).astype(np.int32)))
            ep.local_psum.copy_(torch.from_numpy(full["p"][t0:t1].sum(axis=0)))
            ep.local_real.fill_(t1 - t0)

        def dispatch(x_, all_counts, all_psum, all_real):
            assert all_real.tolist() == [bounds[i + 1] - bounds[i] for i in range(world)]
            ac = all_counts.numpy().astype(np.int64)
            base, total = ac[:rank].sum(axis=0), ac.sum(axis=0)
            kept_total = np.minimum(total, cap)
            dest = np.array([kept_total[(e // El) * El:e].sum() for e in range(E)]) + np.minimum(base, cap)
            left = np.minimum(np.maximum(cap - base, 0), ac[rank])
            local_rank = O.dispatch(st["idx"], E, 10 ** 9)["rank"]
            slot = np.full(st["idx"].shape, -1, dtype=np.int64)
            time.sleep(0.3 * rank)
            for t in range(t1 - t0):
                for j in range(k):
                    e = int(st["idx"][t, j])
                    if e >= 0 and local_rank[t, j] < left[e]:
                        slot[t, j] = dest[e] + local_rank[t, j]
                        xr[e // El][slot[t, j]] = torch.from_numpy(x[t0 + t])
            st["slot"] = slot
            st["recv_off"] = [int(kept_total[rank * El:rank * El + i].sum()) for i in range(El + 1)]
            st["stats"] = (total, all_psum.numpy().sum(axis=0) / wl.T)

        def ffn(x_):
            offs = st["recv_off"]
            time.sleep(0.3 * rank)
            for el in range(El):
                rows = xr[rank][offs[el]:offs[el + 1]].numpy()
                if rows.shape[0]:
                    y = O.expert_apply(wl, O.expert_weights_f64(wl, inp, rank * El + el), rows)
                    yr[rank][offs[el]:offs[el + 1]] = torch.from_numpy(y)

        def combine():
            out = np.zeros((t1 - t0, wl.d))
            for t in range(t1 - t0):
                for j in range(k):
                    s = st["slot"][t, j]
                    if s >= 0:
                        out[t] += full["w"][t0 + t, j] * yr[int(st["idx"][t, j]) // El][s].numpy()
            return {"out": out, "slot": st["slot"], "counts": st["stats"][0], "p": st["stats"][1]}

        cfg = MoEConfig(T=t1 - t0, d=wl.d, ffn=wl.ffn, E=E, k=k, dtype="f32", capacity_factor=wl.capacity_factor)
        ep = ExpertParallelMoE(cfg, {}, device="cpu", peers=(xr, yr),
                               phases=dict(route=route, dispatch=dispatch, ffn=ffn, combine=combine))
        assert ep.T_global == wl.T and ep.world == world and ep.rank == rank and ep.E_local == El
        res = ep.forward(torch.zeros((t1 - t0, wl.d)))
        q.put((rank, res["out"], res["slot"], res["counts"], res["p"]))
    finally:
        dist.destroy_process_group()


# the first case is the pages' own multi-process check (LLaMA4-MoE page §3.1):
# two ranks holding two of four experts each, against the single-process layer
@pytest.mark.parametrize("bounds,E", [([0, 60, 130], 4), ([0, 120, 257], 6), ([0, 50, 51, 200], 6),
                                      ([0, 0, 90], 6)],
                         ids=["world2-E4", "world2", "world3-one-token", "world2-empty-slice"])
def test_expert_parallel_forward_equals_whole_batch(bounds, E):
    import workloads as W
    from oracle import moe_oracle as O

    world = len(bounds) - 1
    wl = _workload(bounds[-1], E)
    inp = W.make_inputs(wl)
    full = O.forward(wl, inp)
    El = wl.E // world
    rows = min(wl.T * wl.k, El * full["cap"])
    xr = [torch.zeros((rows, wl.d), dtype=torch.float64).share_memory_() for _ in range(world)]
    yr = [torch.zeros((rows, wl.d), dtype=torch.float64).share_memory_() for _ in range(world)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, bounds, E, xr, yr, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        r, out, slot, counts, pm = q.get(timeout=180)
        results[r] = (out, slot, counts, pm)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert (full["slot"] < 0).any(), "the case must exercise drops"
    out = np.concatenate([results[r][0] for r in range(world)])
    np.testing.assert_allclose(out, full["out"], rtol=1e-12, atol=1e-14)
    lay = O.expert_parallel_layout(full["idx"], full["slot"], wl.E, world)
    slot = np.concatenate([results[r][1] for r in range(world)])
    assert np.array_equal(slot, lay["row"])
    for r in range(world):
        assert np.array_equal(results[r][2], full["counts"])
        np.testing.assert_allclose(results[r][3], full["p_mean"], rtol=1e-12)
