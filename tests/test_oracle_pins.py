"""Pins of the CPU oracle to facts fixed by the pages and by mathematics.

Each ``check_*`` function asserts one fact about an oracle module; the tests
run them on the real oracle, and ``test_planted_mistakes`` runs them on
copies of the oracle with one plausible mistake planted (a wrong tie rule, a
dropped k in the capacity, renormalising after drops, ...) to show that some
pin fails for each.  Mistakes are only ever planted in the oracle, on the CPU.
"""
import itertools
import json
import math
import os
import types

import numpy as np
import pytest

from oracle import moe_oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _wl(**kw):
    base = dict(name="t", T=16, d=8, ffn=12, E=4, k=2, act="swiglu", dtype="f32",
                capacity_factor=0.0, aux_alpha=0.01)
    base.update(kw)
    return W.Workload(**base)


# ----------------------------------------------------------------------------
# checks (each takes the oracle module as argument)
# ----------------------------------------------------------------------------
def check_worked_example(o):
    """MoE-basics page §2.3: 4 experts, 8 tokens, 7 routed to expert 1 -> f_1 = 0.875."""
    g = _load("worked_example_f.json")
    T, E, k = g["T"], g["E"], g["k"]
    logits = np.full((T, E), -1.0)
    for t, e in enumerate(g["expert_of_token"]):
        logits[t, e] = 1.0
    idx = o.select_topk(logits, k)
    disp = o.dispatch(idx, E, o.capacity(T, k, E, 0.0))
    f, _, _ = o.aux_stats(disp["counts"], o.softmax(logits), T, k, 0.01)
    np.testing.assert_allclose(f, g["f"], rtol=0, atol=1e-15)
    assert f[1] == 0.875


def check_uniform_alpha(o):
    """f_e = p_e = 1/E -> L_aux = alpha (LLaMA4-MoE page §3.2; MoE-basics page §2.3).
    Exercised through the whole routing path: token t prefers expert t mod E by a
    tiny margin, so routing is balanced and p is uniform up to that margin."""
    for E, k in [(4, 1), (8, 2), (6, 3)]:
        T = 6 * E
        eps = 1e-9
        logits = np.zeros((T, E))
        for t in range(T):
            for j in range(k):
                logits[t, (t + j) % E] = eps * (k - j)
        idx = o.select_topk(logits, k)
        disp = o.dispatch(idx, E, o.capacity(T, k, E, 0.0))
        f, pm, laux = o.aux_stats(disp["counts"], o.softmax(logits), T, k, 0.05)
        np.testing.assert_allclose(f, 1.0 / E, rtol=0, atol=1e-15)
        np.testing.assert_allclose(pm, 1.0 / E, rtol=1e-7)
        assert abs(laux - 0.05) < 1e-8
    # directly on the statistic
    E = 5
    f, pm, laux = o.aux_stats(np.full(E, 7, dtype=np.int32), np.full((7, E), 1.0 / E), 7, E, 0.01)
    assert abs(laux - 0.01) < 1e-15


def check_sums_to_one(o):
    """Renormalised top-k weights sum to 1 (Llama-MoE page §3.1); sum f = 1 and
    sum p = 1 under the T*k normalisation (reading R4)."""
    rng = np.random.default_rng(1)
    for E, k in [(4, 2), (8, 2), (16, 4), (64, 8), (3, 3)]:
        T = 257
        l = rng.normal(size=(T, E)) * 2
        p = o.softmax(l)
        idx = o.select_topk(l, k)
        w = o.renormalise(p, idx)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-14)
        disp = o.dispatch(idx, E, o.capacity(T, k, E, 1.0))
        f, pm, _ = o.aux_stats(disp["counts"], p, T, k, 0.01)
        assert abs(f.sum() - 1.0) < 1e-14 and abs(pm.sum() - 1.0) < 1e-13


def check_topk_bruteforce(o):
    """Brute force over all k-subsets on tiny E with integer logits (many ties):
    the chosen set is the unique S with, for every s in S and u not in S,
    l_s > l_u or (l_s == l_u and s < u); idx lists S best first (ties: lower id)."""
    rng = np.random.default_rng(2)
    for E in range(1, 7):
        for k in range(1, E + 1):
            l = rng.integers(-2, 3, size=(60, E)).astype(np.float64)
            idx = o.select_topk(l, k)
            for t in range(l.shape[0]):
                ok = []
                for S in itertools.combinations(range(E), k):
                    comp = [u for u in range(E) if u not in S]
                    if all(l[t, s] > l[t, u] or (l[t, s] == l[t, u] and s < u) for s in S for u in comp):
                        ok.append(S)
                assert len(ok) == 1
                assert sorted(idx[t].tolist()) == list(ok[0])
                order = sorted(ok[0], key=lambda e: (-l[t, e], e))
                assert idx[t].tolist() == order


def check_tie_lower_id(o):
    """Equal logits: the lower expert id is chosen first (reading R5)."""
    l = np.array([[0.5, 0.5, 0.5, 0.5], [0.0, 1.0, 1.0, 0.0], [2.0, -1.0, 2.0, 2.0]])
    idx = o.select_topk(l, 2)
    assert idx.tolist() == [[0, 1], [1, 2], [0, 2]]


def check_renorm_is_selected_softmax(o):
    """p_j / sum_sel p (Llama-MoE page §3.1) equals softmax over the k selected
    logits (MoE-basics page §3.1): two page formulas, one value."""
    rng = np.random.default_rng(3)
    l = rng.normal(size=(100, 8)) * 3
    idx = o.select_topk(l, 3)
    w = o.renormalise(o.softmax(l), idx)
    sel = np.take_along_axis(l, idx.astype(np.int64), axis=1)
    z = np.exp(sel - sel.max(axis=1, keepdims=True))
    np.testing.assert_allclose(w, z / z.sum(axis=1, keepdims=True), rtol=1e-13)


def check_softmax_closed_form(o):
    """Two experts: softmax is the logistic function; shift invariance; large logits stay finite."""
    a = np.array([[0.3, -1.2], [5.0, 5.0], [800.0, 799.0]])
    p = o.softmax(a)
    expect0 = 1.0 / (1.0 + np.exp(a[:, 1] - a[:, 0]))
    np.testing.assert_allclose(p[:, 0], expect0, rtol=1e-14)
    np.testing.assert_allclose(o.softmax(a + 17.0), p, rtol=1e-14)


def check_capacity(o):
    """cap = ceil(T*k/E*cf) (MoE-basics page §2.4 scaled by k, reading R1), by hand:
    64*2/4*1.25 = 40; 4096*2/8*1.25 = 1280; 8192*2/8*1.25 = 2560; 32768*2/32*1 = 2048;
    no limit (cf <= 0) -> T; 10*2/3*1.1 = 7.33.. -> 8; T=4, k=1, E=1, cf=0.5 -> 2."""
    assert o.capacity(64, 2, 4, 1.25) == 40
    assert o.capacity(4096, 2, 8, 1.25) == 1280
    assert o.capacity(8192, 2, 8, 1.25) == 2560
    assert o.capacity(32768, 2, 32, 1.0) == 2048
    assert o.capacity(64, 2, 64, 0.0) == 64
    assert o.capacity(10, 2, 3, 1.1) == 8
    assert o.capacity(4, 1, 1, 0.5) == 2


def check_dispatch_hand_case(o):
    """T=4, E=1, k=1, cf=0.5: cap 2, tokens 2 and 3 dropped, kept rows in token order."""
    idx = np.zeros((4, 1), dtype=np.int32)
    d = o.dispatch(idx, 1, o.capacity(4, 1, 1, 0.5))
    assert d["counts"].tolist() == [4] and d["kept"].tolist() == [2]
    assert d["offsets"].tolist() == [0, 2]
    assert d["slot"][:, 0].tolist() == [0, 1, -1, -1]
    assert d["src_assign"].tolist() == [0, 1]


def check_dispatch_bruteforce(o):
    """Independent O((Tk)^2) recount of each assignment's rank on tiny inputs, and
    the layout invariants: src_assign is a bijection onto the kept assignments,
    each expert's rows are contiguous and in ascending token order, and
    sum kept = sum min(n_e, cap); cap = T drops nothing."""
    rng = np.random.default_rng(4)
    for trial in range(200):
        T = int(rng.integers(1, 9))
        E = int(rng.integers(1, 5))
        k = int(rng.integers(1, E + 1))
        l = rng.integers(-3, 4, size=(T, E)).astype(np.float64)
        idx = o.select_topk(l, k)
        cap = int(rng.integers(0, T + 2))
        d = o.dispatch(idx, E, cap)
        kept_total = 0
        for e in range(E):
            n_e = int((idx == e).sum())
            assert d["counts"][e] == n_e
            kept_total += min(n_e, cap)
        assert d["offsets"][-1] == kept_total == d["src_assign"].size
        seen = set()
        for t in range(T):
            for j in range(k):
                e = idx[t, j]
                r = sum(1 for t2 in range(T) for j2 in range(k)
                        if (t2, j2) < (t, j) and idx[t2, j2] == e)
                s = d["slot"][t, j]
                if r < cap:
                    assert s == d["offsets"][e] + r
                    assert d["src_assign"][s] == t * k + j
                    seen.add(int(s))
                else:
                    assert s == -1
        assert seen == set(range(kept_total))
        for e in range(E):
            rows = d["src_assign"][d["offsets"][e]:d["offsets"][e + 1]]
            assert all(idx.reshape(-1)[a] == e for a in rows)
            assert list(rows) == sorted(rows)
        if cap >= T:
            assert (d["slot"] >= 0).all()


def check_activation_closed_forms(o):
    """silu and exact-erf gelu at 0, +-1, 2 (values in closed_forms.json) and their
    large-|z| limits; cross-checked against torch's CPU float64 silu / gelu."""
    g = _load("closed_forms.json")
    for z, v in g["silu"]:
        assert abs(float(o.silu(np.array([z]))[0]) - v) <= 1e-15 * max(1.0, abs(v))
    for z, v in g["gelu"]:
        assert abs(float(o.gelu(np.array([z]))[0]) - v) <= 1e-15 * max(1.0, abs(v))
    big = np.array([40.0, -40.0])
    np.testing.assert_allclose(o.silu(big), [40.0, 0.0], atol=1e-15)
    np.testing.assert_allclose(o.gelu(big), [40.0, 0.0], atol=1e-15)
    import torch
    z = np.linspace(-8, 8, 1001)
    tz = torch.from_numpy(z)
    np.testing.assert_allclose(o.silu(z), torch.nn.functional.silu(tz).numpy(), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(o.gelu(z), torch.nn.functional.gelu(tz).numpy(), rtol=1e-13, atol=1e-15)


def _dense_inputs(act, T=37, d=16, F=24, seed=5):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(T, d)).astype(np.float32)
    inp = {"x": x, "w_router": rng.normal(size=(d, 1)).astype(np.float32), "router_bias": None}
    if act == "swiglu":
        inp.update(w_gate=rng.normal(size=(1, d, F)).astype(np.float32) * 0.2,
                   w_up=rng.normal(size=(1, d, F)).astype(np.float32) * 0.2,
                   w_down=rng.normal(size=(1, F, d)).astype(np.float32) * 0.2)
    else:
        inp.update(w1=rng.normal(size=(1, d, F)).astype(np.float32) * 0.2,
                   b1=rng.normal(size=(1, F)).astype(np.float32) * 0.1,
                   w2=rng.normal(size=(1, F, d)).astype(np.float32) * 0.2,
                   b2=rng.normal(size=(1, d)).astype(np.float32) * 0.1)
    return inp


def check_dense_reduction(o):
    """E=1, k=1, no capacity limit: the layer is the dense FFN (weight 1, no
    gather).  Reference: a textbook dense FFN in torch float64 on the CPU."""
    import torch
    for act in ("swiglu", "gelu_bias"):
        wl = _wl(T=37, d=16, ffn=24, E=1, k=1, act=act, capacity_factor=0.0)
        inp = _dense_inputs(act)
        res = o.forward(wl, inp)
        x = torch.from_numpy(inp["x"].astype(np.float64))
        if act == "swiglu":
            g = x @ torch.from_numpy(inp["w_gate"][0].astype(np.float64))
            u = x @ torch.from_numpy(inp["w_up"][0].astype(np.float64))
            ref = (torch.nn.functional.silu(g) * u) @ torch.from_numpy(inp["w_down"][0].astype(np.float64))
        else:
            lin1 = torch.nn.Linear(16, 24, dtype=torch.float64)
            lin2 = torch.nn.Linear(24, 16, dtype=torch.float64)
            with torch.no_grad():
                lin1.weight.copy_(torch.from_numpy(inp["w1"][0].T.astype(np.float64)))
                lin1.bias.copy_(torch.from_numpy(inp["b1"][0].astype(np.float64)))
                lin2.weight.copy_(torch.from_numpy(inp["w2"][0].T.astype(np.float64)))
                lin2.bias.copy_(torch.from_numpy(inp["b2"][0].astype(np.float64)))
                ref = lin2(torch.nn.GELU()(lin1(x)))
        np.testing.assert_allclose(res["out"], ref.detach().numpy(), rtol=1e-12, atol=1e-12)
        assert (res["w"] == 1.0).all()


def check_teaching_layer(o):
    """With no capacity cut, the oracle equals the masked-loop semantics of the
    minimal MoELayer (MoE-basics page §3.1): for each top-k slot i and expert e,
    out[ids_i == e] += w_i * expert_e(x[ids_i == e]); restated here from the
    page's description, with the expert as nn.Linear -> GELU -> nn.Linear."""
    import torch
    rng = np.random.default_rng(6)
    T, d, F, E, k = 29, 12, 20, 5, 2
    wl = _wl(T=T, d=d, ffn=F, E=E, k=k, act="gelu_bias", capacity_factor=0.0)
    inp = {"x": rng.normal(size=(T, d)).astype(np.float32),
           "w_router": rng.normal(size=(d, E)).astype(np.float32), "router_bias": None,
           "w1": (rng.normal(size=(E, d, F)) * 0.3).astype(np.float32),
           "b1": (rng.normal(size=(E, F)) * 0.1).astype(np.float32),
           "w2": (rng.normal(size=(E, F, d)) * 0.3).astype(np.float32),
           "b2": (rng.normal(size=(E, d)) * 0.1).astype(np.float32)}
    res = o.forward(wl, inp)
    x = torch.from_numpy(inp["x"].astype(np.float64))
    logits = x @ torch.from_numpy(inp["w_router"].astype(np.float64))
    logits = logits.float().double()          # reading R5: routing decided on fp32 logits
    scores, ids = logits.topk(k, dim=-1)
    probs = torch.softmax(scores, dim=-1)
    experts = []
    for e in range(E):
        l1 = torch.nn.Linear(d, F, dtype=torch.float64)
        l2 = torch.nn.Linear(F, d, dtype=torch.float64)
        with torch.no_grad():
            l1.weight.copy_(torch.from_numpy(inp["w1"][e].T.astype(np.float64)))
            l1.bias.copy_(torch.from_numpy(inp["b1"][e].astype(np.float64)))
            l2.weight.copy_(torch.from_numpy(inp["w2"][e].T.astype(np.float64)))
            l2.bias.copy_(torch.from_numpy(inp["b2"][e].astype(np.float64)))
        experts.append(torch.nn.Sequential(l1, torch.nn.GELU(), l2))
    out = torch.zeros_like(x)
    with torch.no_grad():
        for i in range(k):
            for e in range(E):
                m = ids[:, i] == e
                if m.any():
                    out[m] += probs[m, i].unsqueeze(-1) * experts[e](x[m])
    np.testing.assert_allclose(res["out"], out.numpy(), rtol=1e-10, atol=1e-12)


def check_combine_properties(o):
    """k=1 with no drops -> out = expert output; one-hot weights select; out is
    linear in the expert rows; dropped assignments add nothing and the survivors
    are not renormalised (reading R3); an all-dropped token outputs 0."""
    rng = np.random.default_rng(7)
    T, d, k = 6, 5, 2
    slot = np.array([[0, 1], [2, -1], [-1, -1], [3, 4], [5, 6], [7, 8]])
    w = rng.random((T, k))
    y = {a: rng.normal(size=d) for a in range(T * k)}
    out = o.combine(y, slot, w, T, d)
    assert np.array_equal(out[2], np.zeros(d))
    np.testing.assert_allclose(out[1], w[1, 0] * y[2], rtol=1e-15)
    y2 = {a: 3.0 * v for a, v in y.items()}
    np.testing.assert_allclose(o.combine(y2, slot, w, T, d), 3.0 * out, rtol=1e-14)
    w1h = np.zeros((T, k)); w1h[:, 1] = 1.0
    o1 = o.combine(y, slot, w1h, T, d)
    np.testing.assert_allclose(o1[0], y[1]); np.testing.assert_allclose(o1[3], y[7])
    slot1 = np.arange(T).reshape(T, 1)
    np.testing.assert_allclose(o.combine({t: y[t] for t in range(T)}, slot1, np.ones((T, 1)), T, d),
                               np.stack([y[t] for t in range(T)]))


def check_drop_path_end_to_end(o):
    """One expert, cap 2 of 4 tokens (cf 0.5), k=1: tokens 0,1 get the expert's
    output with weight 1, tokens 2,3 (dropped) get exactly 0."""
    wl = _wl(T=4, d=16, ffn=24, E=1, k=1, act="swiglu", capacity_factor=0.5)
    inp = _dense_inputs("swiglu", T=4)
    res = o.forward(wl, inp)
    assert res["slot"][:, 0].tolist() == [0, 1, -1, -1]
    assert np.array_equal(res["out"][2:], np.zeros((2, 16)))
    x = inp["x"].astype(np.float64)
    ref = o.expert_swiglu(x[:2], inp["w_gate"][0].astype(np.float64), inp["w_up"][0].astype(np.float64),
                          inp["w_down"][0].astype(np.float64))
    np.testing.assert_allclose(res["out"][:2], ref, rtol=1e-14)


def check_empty(o):
    """T = 0: nothing routed, f = p = 0, L_aux = 0 (reading R7)."""
    wl = _wl(T=0, E=3, k=2)
    inp = {"x": np.zeros((0, 8), np.float32), "w_router": np.ones((8, 3), np.float32), "router_bias": None,
           "w_gate": np.zeros((3, 8, 12), np.float32), "w_up": np.zeros((3, 8, 12), np.float32),
           "w_down": np.zeros((3, 12, 8), np.float32)}
    r = o.route(wl, inp)
    assert r["offsets"].tolist() == [0, 0, 0, 0] and r["l_aux"] == 0.0
    assert r["src_assign"].size == 0


def check_padding_mask(o):
    """Reading R16 (padding kept out of expert selection, LLaMA4-MoE page §4.1):
    an all-ones mask changes nothing; with no capacity limit, the real tokens of
    a padded batch route exactly as the batch of real tokens alone, with the
    same statistics; padding selects nothing and outputs 0; padding does not use
    capacity (hand case); an all-padding batch has zero statistics."""
    wl = _wl(T=24, d=8, ffn=12, E=4, k=2, capacity_factor=0.0)
    inp = W.make_inputs(wl.with_(seed=11))
    base = o.route(wl, inp)
    ones = o.route(wl, {**inp, "token_mask": np.ones(wl.T, dtype=np.uint8)})
    for key in ("idx", "w", "counts", "offsets", "slot", "f", "p_mean"):
        np.testing.assert_array_equal(base[key], ones[key])
    mask = np.ones(wl.T, dtype=np.uint8)
    pad = np.array([0, 3, 4, 10, 17, 23])
    mask[pad] = 0
    real = np.nonzero(mask)[0]
    masked = o.forward(wl, {**inp, "token_mask": mask})
    wl_r = wl.with_(T=real.size)
    alone = o.forward(wl_r, {**inp, "x": inp["x"][real]})
    np.testing.assert_array_equal(masked["idx"][real], alone["idx"])
    np.testing.assert_allclose(masked["w"][real], alone["w"], rtol=0, atol=0)
    np.testing.assert_array_equal(masked["counts"], alone["counts"])
    np.testing.assert_allclose(masked["f"], alone["f"], rtol=1e-15)
    np.testing.assert_allclose(masked["p_mean"], alone["p_mean"], rtol=1e-13)
    assert abs(masked["l_aux"] - alone["l_aux"]) <= 1e-15
    assert (masked["idx"][pad] == -1).all() and (masked["w"][pad] == 0).all() and (masked["slot"][pad] == -1).all()
    np.testing.assert_allclose(masked["out"][real], alone["out"], rtol=1e-13, atol=1e-15)
    assert (masked["out"][pad] == 0).all()
    # hand case: T=4, E=1, k=1, cf=0.5 -> cap 2; token 0 is padding, so tokens 1, 2 are kept, 3 dropped
    wl1 = _wl(T=4, d=8, ffn=12, E=1, k=1, capacity_factor=0.5)
    inp1 = W.make_inputs(wl1.with_(seed=3))
    r1 = o.route(wl1, {**inp1, "token_mask": np.array([0, 1, 1, 1], dtype=np.uint8)})
    assert r1["slot"][:, 0].tolist() == [-1, 0, 1, -1] and r1["counts"].tolist() == [3]
    assert abs(r1["f"][0] - 1.0) < 1e-15
    # every token padding
    r0 = o.route(wl, {**inp, "token_mask": np.zeros(wl.T, dtype=np.uint8)})
    assert (r0["counts"] == 0).all() and (r0["f"] == 0).all() and (r0["p_mean"] == 0).all() and r0["l_aux"] == 0.0
    assert r0["offsets"][-1] == 0


def check_shared_experts(o):
    """Reading R17 (shared experts in every token's computation, LLaMA4-MoE
    page §5.2): with one routed expert (E=1, k=1, no limit) and one shared
    expert the layer is the sum of two textbook dense FFNs; two identical shared
    experts add twice one; padding tokens get the shared output only."""
    import torch
    for act in ("swiglu", "gelu_bias"):
        wl = _wl(T=21, d=16, ffn=24, E=1, k=1, act=act, capacity_factor=0.0, n_shared=1)
        inp = _dense_inputs(act, T=21)
        sh = _dense_inputs(act, T=21, seed=9)
        keys = ("w_gate", "w_up", "w_down") if act == "swiglu" else ("w1", "b1", "w2", "b2")
        shared = {"shared_" + {"w_gate": "gate", "w_up": "up", "w_down": "down"}.get(k_, k_): sh[k_] for k_ in keys}
        res = o.forward(wl, {**inp, **shared})
        x = torch.from_numpy(inp["x"].astype(np.float64))

        def ffn(params):
            if act == "swiglu":
                g = x @ torch.from_numpy(params["w_gate"][0].astype(np.float64))
                u = x @ torch.from_numpy(params["w_up"][0].astype(np.float64))
                return (torch.nn.functional.silu(g) * u) @ torch.from_numpy(params["w_down"][0].astype(np.float64))
            h = torch.nn.functional.gelu(x @ torch.from_numpy(params["w1"][0].astype(np.float64))
                                         + torch.from_numpy(params["b1"][0].astype(np.float64)))
            return h @ torch.from_numpy(params["w2"][0].astype(np.float64)) + torch.from_numpy(params["b2"][0].astype(np.float64))

        ref = ffn(inp) + ffn(sh)
        np.testing.assert_allclose(res["out"], ref.numpy(), rtol=1e-12, atol=1e-12)
        two = {k_: np.concatenate([v, v]) for k_, v in shared.items()}
        res2 = o.forward(wl.with_(n_shared=2), {**inp, **two})
        np.testing.assert_allclose(res2["out"] - res["out"], ffn(sh).numpy(), rtol=1e-12, atol=1e-12)
        pad = o.forward(wl, {**inp, **shared, "token_mask": np.zeros(21, dtype=np.uint8)})
        np.testing.assert_allclose(pad["out"], ffn(sh).numpy(), rtol=1e-12, atol=1e-12)


def check_int8_quantization(o):
    """Reading R18 (INT8 weights with a per-expert, per-dimension scale, the
    long-context MoE page §3): hand codes, the half-step error bound
    |w - q*s| <= s/2, exact recovery of matrices already on the code grid,
    codes within [-127, 127] with +-127 reached in every non-zero column, an
    all-zero column, and the layer on int8 weights equal to the layer on the
    dequantised weights."""
    w = np.array([[127.0, 0.0, 1.0], [-63.5, 0.0, -0.25], [0.4, 0.0, 0.5]], dtype=np.float32)
    q, s = o.quantize_int8(w)
    assert s.tolist() == [np.float32(1.0), 0.0, np.float32(1.0) / np.float32(127.0)]
    assert q[:, 0].tolist() == [127, -64, 0]          # -63.5 rounds to the even -64
    assert q[:, 1].tolist() == [0, 0, 0]
    assert q[0, 2] == 127 and q[2, 2] == 64           # 0.5 * 127 = 63.5 -> 64 (even)
    rng = np.random.default_rng(4)
    w = (rng.normal(size=(64, 48)) * rng.uniform(0.01, 3.0, size=(1, 48))).astype(np.float32)
    q, s = o.quantize_int8(w)
    assert q.dtype == np.int8 and np.abs(q.astype(int)).max() <= 127
    assert (np.abs(q.astype(int)).max(axis=0) == 127).all()
    err = np.abs(w.astype(np.float64) - o.dequantize_int8(q, s))
    assert (err <= s.astype(np.float64)[None, :] * (0.5 + 1e-6)).all()
    grid = o.dequantize_int8(q, s).astype(np.float32)
    q2, s2 = o.quantize_int8(grid)
    np.testing.assert_array_equal(q2, q)
    np.testing.assert_allclose(o.dequantize_int8(q2, s2), grid, rtol=1e-6)
    # the layer on int8 weights is the layer on the dequantised weights
    wl = _wl(T=19, d=16, ffn=24, E=2, k=1, act="swiglu", capacity_factor=0.0, weights="int8")
    inp = W.make_inputs(wl.with_(weights="native", seed=8))
    deq = {}
    for n in ("w_gate", "w_up", "w_down"):
        deq[n] = np.stack([o.dequantize_int8(*o.quantize_int8(inp[n][e].astype(np.float32))) for e in range(2)])
    a = o.forward(wl, inp)
    # (the f32 workload's inputs are read as float32, so the dequantised weights pass through one fp32 rounding)
    b = o.forward(wl.with_(weights="native"), {**inp, **{n: v.astype(np.float32) for n, v in deq.items()}})
    assert np.abs(a["out"] - b["out"]).max() <= 1e-6 * np.abs(b["out"]).max()
    assert np.abs(a["out"] - o.forward(wl.with_(weights="native"), inp)["out"]).max() > 1e-9  # quantisation shows


def check_expert_parallel_layout(o):
    """Reading R19 (expert parallelism, LLaMA4-MoE page §2.5, MoE-basics page
    §4.1).  Hand cases (E=4 on 2 ranks: experts 0 and 1 on rank 0, 2 and 3 on
    rank 1; with and without drops); one rank reduces to the single-device
    dispatch; one expert per rank gives row = slot - offsets[e]; an independent
    simulation of the all-to-all over random contiguous token slices (each
    source rank sends every owner its kept rows expert by expert, and the owner
    stacks each expert's parts in source-rank order) gives the same rows; and
    the layer computed owner by owner equals the single-device layer."""
    idx = np.array([[3, 0], [1, 3], [0, 2]], dtype=np.int32)
    lay = o.expert_parallel_layout(idx, o.dispatch(idx, 4, 3)["slot"], 4, 2)
    assert lay["owner"].tolist() == [[1, 0], [0, 1], [0, 1]]
    assert lay["row"].tolist() == [[1, 0], [2, 2], [1, 0]]
    assert lay["recv_offsets"].tolist() == [[0, 2, 3], [0, 1, 3]]
    assert [r.tolist() for r in lay["recv_src"]] == [[1, 4, 2], [5, 0, 3]]
    lay = o.expert_parallel_layout(idx, o.dispatch(idx, 4, 1)["slot"], 4, 2)   # cap 1: assignments 3 and 4 dropped
    assert lay["owner"].tolist() == [[1, 0], [0, -1], [-1, 1]]
    assert lay["row"].tolist() == [[1, 0], [1, -1], [-1, 0]]
    assert lay["recv_offsets"].tolist() == [[0, 1, 2], [0, 1, 2]]
    rng = np.random.default_rng(19)
    for trial in range(150):
        world = int(rng.choice([1, 2, 3, 4]))
        El = int(rng.integers(1, 4))
        E = world * El
        k = int(rng.integers(1, min(E, 3) + 1))
        T = int(rng.integers(0, 12))
        idx = o.select_topk(rng.integers(-3, 4, size=(T, E)).astype(np.float64), k)
        idx[rng.random(T) < 0.15] = -1                     # padding tokens (R16)
        cap = int(rng.integers(0, T + 2))
        d = o.dispatch(idx, E, cap)
        lay = o.expert_parallel_layout(idx, d["slot"], E, world)
        keep = d["slot"] >= 0
        assert np.array_equal(lay["row"] >= 0, keep) and np.array_equal(lay["owner"] >= 0, keep)
        if world == 1:
            assert np.array_equal(lay["row"], d["slot"])
            assert lay["recv_offsets"][0].tolist() == d["offsets"].tolist()
        if El == 1:
            assert np.array_equal(lay["row"][keep], d["slot"][keep] - d["offsets"][idx[keep]])
        cuts = sorted(int(c) for c in rng.integers(0, T + 1, size=world - 1))
        bounds = [0, *cuts, T]
        part = {}
        for src in range(world):
            for own in range(world):
                for e in range(own * El, (own + 1) * El):
                    part.setdefault((own, e), []).extend(
                        t * k + j for t in range(bounds[src], bounds[src + 1]) for j in range(k)
                        if idx[t, j] == e and d["slot"][t, j] >= 0)
        for own in range(world):
            rows = [a for e in range(own * El, (own + 1) * El) for a in part[(own, e)]]
            assert lay["recv_src"][own].tolist() == rows
            sizes = [len(part[(own, e)]) for e in range(own * El, (own + 1) * El)]
            assert lay["recv_offsets"][own].tolist() == [0, *np.cumsum(sizes).tolist()]
            for r_, a in enumerate(rows):
                assert lay["owner"].reshape(-1)[a] == own and lay["row"].reshape(-1)[a] == r_
    # the layer, computed owner by owner on the received rows, equals the single-device layer
    wl = _wl(T=29, d=8, ffn=12, E=6, k=2, capacity_factor=0.8, seed=12, w_std=0.3)
    inp = W.make_inputs(wl)
    x = o.to_f64(inp["x"], wl.dtype)
    ref = o.forward(wl, inp)
    lay = o.expert_parallel_layout(ref["idx"], ref["slot"], wl.E, 3)
    y = {}
    for own in range(3):
        src = lay["recv_src"][own]
        offs = lay["recv_offsets"][own]
        for el in range(2):
            rows = src[offs[el]:offs[el + 1]]
            if rows.size:
                ye = o.expert_apply(wl, o.expert_weights_f64(wl, inp, own * 2 + el), x[rows // wl.k])
                y.update({int(a): ye[i] for i, a in enumerate(rows)})
    out = o.combine(y, ref["slot"], ref["w"], wl.T, wl.d)
    assert (ref["slot"] < 0).any(), "the case must exercise drops"
    np.testing.assert_allclose(out, ref["out"], rtol=1e-12, atol=1e-14)


CHECKS = [check_worked_example, check_uniform_alpha, check_sums_to_one, check_topk_bruteforce,
          check_tie_lower_id, check_renorm_is_selected_softmax, check_softmax_closed_form,
          check_capacity, check_dispatch_hand_case, check_dispatch_bruteforce,
          check_activation_closed_forms, check_dense_reduction, check_teaching_layer,
          check_combine_properties, check_drop_path_end_to_end, check_empty, check_padding_mask,
          check_shared_experts, check_int8_quantization, check_expert_parallel_layout]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(O)


# ----------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin
# ----------------------------------------------------------------------------
def _mutant(**overrides):
    m = types.ModuleType("oracle_mutant")
    m.__dict__.update({k: v for k, v in O.__dict__.items() if not k.startswith("__")})
    m.__dict__["__builtins__"] = O.__dict__["__builtins__"]
    # rebind the oracle's functions to the mutant's globals, so that a planted
    # function is the one its callers (route, forward, ...) reach
    for name, fn in list(m.__dict__.items()):
        if isinstance(fn, types.FunctionType) and fn.__module__ == O.__name__:
            m.__dict__[name] = types.FunctionType(fn.__code__, m.__dict__, fn.__name__, fn.__defaults__)
    m.__dict__.update(overrides)
    return m


def _topk_upper_tie(l, k):
    T, E = l.shape
    work = l.copy()
    idx = np.empty((T, k), dtype=np.int32)
    for j in range(k):
        e = E - 1 - np.argmax(work[:, ::-1], axis=1)
        idx[:, j] = e
        work[np.arange(T), e] = -np.inf
    return idx


def _cap_without_k(T, k, E, cf):
    return T if cf <= 0 else int(math.ceil(T / E * cf))


def _aux_f_over_T(counts, p, T, k, alpha):
    E = counts.shape[0]
    if T == 0:
        return np.zeros(E), np.zeros(E), 0.0
    f = counts / float(T)
    pm = p.mean(axis=0)
    return f, pm, float(alpha * E * np.sum(f * pm))


def _gelu_tanh(z):
    return 0.5 * z * (1 + np.tanh(math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)))


def _combine_renorm(y, slot, w, T, d, tokens=None):
    w = w * (slot >= 0)
    s = w.sum(axis=1, keepdims=True)
    w = np.where(s > 0, w / np.where(s > 0, s, 1), 0)
    return O.combine(y, slot, w, T, d, tokens)


def _softmax_no_shift_wrong_axis(l):
    z = np.exp(l)
    return z / z.sum(axis=0, keepdims=True)


def _dispatch_expert_major_rank(idx, E, cap):
    # ranks by slot position j first (all first choices before second choices)
    T, k = idx.shape
    order = np.array([t * k + j for j in range(k) for t in range(T)])
    flat = idx.reshape(-1).astype(np.int64)
    rank = np.empty(T * k, dtype=np.int64)
    counts = np.zeros(E, dtype=np.int64)
    for e in range(E):
        pos = order[flat[order] == e]
        rank[pos] = np.arange(pos.size)
        counts[e] = pos.size
    kept = np.minimum(counts, cap)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    keep = rank < cap
    slot = np.where(keep, offsets[flat] + rank, -1)
    src = np.empty(int(offsets[-1]), dtype=np.int64)
    src[slot[keep]] = np.nonzero(keep)[0]
    return {"counts": counts.astype(np.int32), "kept": kept.astype(np.int32), "offsets": offsets.astype(np.int32),
            "slot": slot.reshape(T, k).astype(np.int32), "src_assign": src.astype(np.int32), "rank": rank.reshape(T, k)}


def _swiglu_swapped(xr, wg, wu, wd):
    return np.matmul(O.silu(np.matmul(xr, wu)) * np.matmul(xr, wg), wd)


def _mask_ignored(idx, w, token_mask):
    return idx, w


def _stats_over_all_tokens(token_mask, T):
    return np.ones(T, dtype=bool)


def _shared_averaged(wl, inputs, xr):
    acc = np.zeros((xr.shape[0], wl.d))
    for s_ in range(wl.n_shared):
        acc = acc + O.expert_apply(wl, O.shared_weights_f64(wl, inputs, s_), xr)
    return acc / max(wl.n_shared, 1)


def _quant_global_scale(w):
    w = np.asarray(w, dtype=np.float32)
    s = np.full(w.shape[1], np.abs(w).max() / np.float32(127.0), dtype=np.float32)
    q = np.clip(np.rint(w / s[None, :]), -127, 127).astype(np.int8)
    return q, s


def _quant_truncating(w):
    w = np.asarray(w, dtype=np.float32)
    s = (np.abs(w).max(axis=0) / np.float32(127.0)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0))
    q = np.where(s[None, :] > 0, np.clip(np.trunc(w / safe[None, :]), -127, 127), 0).astype(np.int8)
    return q, s


def _ep_owner_round_robin(e, E, world):
    return np.asarray(e) % world


def _ep_layout_token_major(idx, slot, E, world):
    # an owner's rows in token order across its experts (not grouped by expert)
    T, k = idx.shape
    El = E // world
    flat = idx.reshape(-1).astype(np.int64)
    kept = slot.reshape(-1) >= 0
    owner = np.full(T * k, -1, dtype=np.int64)
    row = np.full(T * k, -1, dtype=np.int64)
    recv_offsets = np.zeros((world, El + 1), dtype=np.int64)
    recv_src = []
    for own in range(world):
        rows = [int(a) for a in np.nonzero(kept & (flat >= 0) & (flat // El == own))[0]]
        for r_, a in enumerate(rows):
            owner[a], row[a] = own, r_
        for el in range(El + 1):
            recv_offsets[own, el] = sum(1 for a in rows if flat[a] - own * El < el)
        recv_src.append(np.array(rows, dtype=np.int64))
    return {"owner": owner.reshape(T, k), "row": row.reshape(T, k), "recv_offsets": recv_offsets,
            "recv_src": recv_src}


MUTANTS = {
    "ep_owner_round_robin": dict(expert_owner=_ep_owner_round_robin),
    "ep_rows_token_major": dict(expert_parallel_layout=_ep_layout_token_major),
    "int8_global_scale": dict(quantize_int8=_quant_global_scale),
    "int8_truncating_codes": dict(quantize_int8=_quant_truncating),
    "padding_selects_experts": dict(mask_padding=_mask_ignored),
    "padding_counted_in_stats": dict(real_tokens=_stats_over_all_tokens),
    "shared_experts_averaged": dict(shared_outputs=_shared_averaged),
    "tie_upper_id": dict(select_topk=_topk_upper_tie),
    "capacity_without_k": dict(capacity=_cap_without_k),
    "f_divided_by_T": dict(aux_stats=_aux_f_over_T),
    "gelu_tanh_approx": dict(gelu=_gelu_tanh),
    "renormalise_after_drop": dict(combine=_combine_renorm),
    "softmax_wrong_axis": dict(softmax=_softmax_no_shift_wrong_axis),
    "drop_order_slot_major": dict(dispatch=_dispatch_expert_major_rank),
    "swiglu_gate_up_swapped": dict(expert_swiglu=_swiglu_swapped),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes(name):
    m = _mutant(**MUTANTS[name])
    caught = []
    for c in CHECKS:
        try:
            with np.errstate(all="ignore"):
                c(m)
        except AssertionError:
            caught.append(c.__name__)
        except Exception:  # a crash of the mutant elsewhere is not a pin catching it
            pass
    assert caught, f"planted mistake {name} slipped through every pin"


def test_real_oracle_is_self_consistent_on_workload_shapes():
    """Routing on the tiny fp32 workload: invariants hold at a real shape."""
    wl = W.WORKLOADS["tiny_f32"]
    inp = W.make_inputs(wl)
    res = O.forward(wl, inp)
    assert res["cap"] == 40
    assert res["offsets"][-1] == res["src_assign"].size
    np.testing.assert_allclose(res["w"].sum(axis=1), 1.0, atol=1e-14)
    assert np.isfinite(res["out"]).all()
