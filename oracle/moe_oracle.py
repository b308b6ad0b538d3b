"""CPU oracle of the top-k routed MoE FFN layer forward.  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or run this module.  The
library never does; it shares no code, header, table or helper with it.

Plain, slow, obviously-correct numpy in float64.  Library primitives used as
single steps: ``numpy.matmul`` (a matrix product), ``numpy.exp``,
``scipy.special.erf``.  No blocking, fusion or reordering beyond the
definitions below.

Pages cited (the web pages that define the method; titles as the pages give
them, or, where a page prints only its site's boilerplate title, its subject):
  [LLaMA4-MoE]  "Hand-building a LLaMA4-MoE" (dpshk.com/news/5809432)
  [MoE-basics]  "MoE: gating, experts, load balancing, capacity factor, and a
                minimal PyTorch MoELayer" (dpshk.com/news/6005940)
  [Loop-MoE]    "How to Loop MoE: Flatten the Experts, Untie the Attention"
                (discosf.com/news/5228035)
  [Llama-MoE]   "Llama-MoE架构解析：混合专家系统如何实现大模型高效训练与推理"
                (coreui.cn/article/2610641)

Readings taken where the pages are silent or disagree (each also listed in
the design doc):
  R1  capacity = ceil(T*k/E * cf): the buffer counts assignments, so the
      tokens-only form of [MoE-basics] §2.4 is scaled by k; cf <= 0 means
      "no limit" (cap = T).
  R2  overflow is dropped in token-major order (t ascending, then j).
  R3  a dropped assignment contributes 0; surviving weights are NOT
      renormalised; a token with every assignment dropped outputs 0.
  R4  f_e counts the router's selections before the capacity cut and divides
      by T*k (so sum f = 1 and uniform routing gives L_aux = alpha).
  R5  top-k compares logits; equal logits -> lower expert id first.  The
      decision is taken on fp32 logits (the kernel's precision): fp64 logits
      are rounded to fp32 before selection, and softmax uses those values.
  R6  GELU is the exact erf form (PyTorch nn.GELU() default).
  R7  T = 0: nothing is routed; f = p = 0 and L_aux = 0.
  R16 padding tokens ([LLaMA4-MoE] §4.1: padding is kept out of expert
      selection): a token with token_mask = 0 selects no expert (index -1,
      weight 0, no dispatch, no routed output) and is left out of f and p,
      which divide by the number of real tokens T_real; the capacity stays
      ceil(T*k/E * cf) of the whole batch T.  T_real = 0 gives zero statistics.
  R18 INT8 expert weights (the long-context MoE page, §3: INT8 weights times
      a scale computed per expert and per dimension, dequantised for use):
      per expert and output column n, scale s = max_k |W[k,n]| / 127 and code
      q = clamp(rint(W / s), -127, 127) (ties to even), both in fp32, the
      precision the library takes the decision in (an all-zero column has
      s = 0, q = 0); the layer then runs on the dequantised weights q * s.
      Shared experts keep their native weights.
  R17 shared experts ([LLaMA4-MoE] §5.2: fixed experts take part in every
      token's computation): n_shared experts of the routed experts' form, own
      weights, applied to every token (padding included) with weight 1 and
      added after the routed terms: out[t] = sum_j w[t,j] y(t,j) + sum_s y_s(t).

  R19 expert parallelism ([LLaMA4-MoE] §2.5, [MoE-basics] §4.1: each GPU
      holds some of the experts; tokens go to the GPUs of their experts by an
      all-to-all and the results come back by a second one): with E experts
      over `world` ranks, rank o holds the contiguous block
      [o*E/world, (o+1)*E/world) (the page's example puts 32 experts on 8
      GPUs, 4 on each).  An owner's receive buffer groups its experts' rows by
      expert in ascending id, each expert's rows in the batch's token order:
      the single-device grouping restricted to the owner's experts.  Capacity,
      drops and statistics are those of the whole batch, so the layer's
      result does not depend on `world`.

Parity pins: every function here is pinned by tests/test_oracle_pins.py
(worked example, closed forms, brute force, invariants, library
cross-checks); none is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np
from scipy.special import erf as _erf


# --------------------------------------------------------------------------
# input decoding (data format only)
# --------------------------------------------------------------------------
def to_f64(a: Optional[np.ndarray], dtype: str) -> Optional[np.ndarray]:
    """Decode an input tensor to float64: bf16 bit patterns (uint16) or float32."""
    if a is None:
        return None
    if dtype == "bf16":
        assert a.dtype == np.uint16
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# routing
# --------------------------------------------------------------------------
def router_logits(x: np.ndarray, w_r: np.ndarray, bias: Optional[np.ndarray] = None) -> np.ndarray:
    """score = x . W_r, a bias-free linear router ([MoE-basics] §2.1 and §3.1).

    ``bias`` is the long-context workload's fixed per-expert logit offset,
    added to the logits before the softmax (so it enters p_e as well)."""
    l = np.matmul(x, w_r)
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)[None, :]
    return l


def decision_logits(l: np.ndarray) -> np.ndarray:
    """R5: the top-k decision is taken on fp32 logits (rounded, then held in fp64)."""
    return l.astype(np.float32).astype(np.float64)


def softmax(l: np.ndarray) -> np.ndarray:
    """Softmax over all E experts ([MoE-basics] §2.1; [Llama-MoE] §3.1), max-shifted."""
    m = l.max(axis=1, keepdims=True)
    z = np.exp(l - m)
    return z / z.sum(axis=1, keepdims=True)


def select_topk(l: np.ndarray, k: int) -> np.ndarray:
    """k experts with the largest logits per token, best first ([MoE-basics] §3.1
    ``logits.topk``; [Llama-MoE] §3.1 ``torch.topk``).  Repeatedly takes the
    maximum over the not-yet-chosen experts; numpy's argmax returns the first
    (lowest) index among equal values, which is the tie rule R5."""
    T, E = l.shape
    work = l.copy()
    idx = np.empty((T, k), dtype=np.int32)
    rows = np.arange(T)
    for j in range(k):
        e = np.argmax(work, axis=1)
        idx[:, j] = e
        work[rows, e] = -np.inf
    return idx


def renormalise(p: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """w_j = p_j / sum of the k selected p ([Llama-MoE] §3.1: top-k weights divided
    by their sum).  Equal to a softmax over the k selected logits ([MoE-basics] §3.1)."""
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def capacity(T: int, k: int, E: int, capacity_factor: float) -> int:
    """Per-expert capacity ([MoE-basics] §2.4, [Llama-MoE] §3.1), reading R1:
    ceil(T*k/E * cf) evaluated in double exactly as written; cf <= 0 -> T."""
    if capacity_factor <= 0:
        return int(T)
    return int(math.ceil(T * k / E * capacity_factor))


def dispatch(idx: np.ndarray, E: int, cap: int) -> dict:
    """Capacity-bounded dispatch in token order (readings R1-R3).

    Walks the assignments (t, j) in token-major order keeping a running count
    per expert; assignment (t, j) gets rank = count so far and is kept iff
    rank < cap.  Kept rows of expert e are laid out contiguously, in token
    order, from offsets[e] = sum over e' < e of min(n_e', cap)
    ([LLaMA4-MoE] §2.4: sort the top-k indices by expert id, per-expert token
    counts, split into one contiguous group per expert).

    Returns counts[E] (before the cut), kept[E], offsets[E+1],
    slot[T,k] (row in the expert-sorted buffer, or -1 when dropped),
    src_assign[R] (= t*k + j of each row), rank[T,k].
    """
    T, k = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    rank = np.full(T * k, np.iinfo(np.int64).max, dtype=np.int64)  # index -1 (padding, R16): never kept
    counts = np.zeros(E, dtype=np.int64)
    for e in range(E):
        pos = np.nonzero(flat == e)[0]          # ascending assignment order = token-major
        rank[pos] = np.arange(pos.size)
        counts[e] = pos.size
    kept = np.minimum(counts, cap)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    keep = (flat >= 0) & (rank < cap)
    slot = np.where(keep, offsets[flat] + rank, -1)
    src_assign = np.empty(int(offsets[-1]), dtype=np.int64)
    src_assign[slot[keep]] = np.nonzero(keep)[0]
    return {
        "counts": counts.astype(np.int32),
        "kept": kept.astype(np.int32),
        "offsets": offsets.astype(np.int32),
        "slot": slot.reshape(T, k).astype(np.int32),
        "src_assign": src_assign.astype(np.int32),
        "rank": rank.reshape(T, k),
    }


# --------------------------------------------------------------------------
# experts
# --------------------------------------------------------------------------
def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z / (1 + exp(-z)), the gate of SwiGLU."""
    return z / (1.0 + np.exp(-z))


def gelu(z: np.ndarray) -> np.ndarray:
    """Exact GELU z * Phi(z) = z/2 * (1 + erf(z/sqrt 2)) (reading R6)."""
    return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))


def expert_swiglu(xr: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """SwiGLU expert W_down(silu(x W_gate) * (x W_up)) ([MoE-basics] §2.2 lists
    SwiGLU inside experts; [Llama-MoE] §2.1: Llama's SwiGLU FFN as the expert)."""
    h = silu(np.matmul(xr, w_gate)) * np.matmul(xr, w_up)
    return np.matmul(h, w_down)


def expert_gelu(xr: np.ndarray, w1: np.ndarray, b1: np.ndarray, w2: np.ndarray, b2: np.ndarray) -> np.ndarray:
    """Two-matrix expert with bias, w2(gelu(w1 x + b1)) + b2 ([MoE-basics] §3.1
    ExpertFFN; weight pool [E, d, ffn] + bias [E, ffn] of [Loop-MoE] §2.1)."""
    h = gelu(np.matmul(xr, w1) + b1[None, :])
    return np.matmul(h, w2) + b2[None, :]


def combine(y_by_assignment: dict, slot: np.ndarray, w: np.ndarray, T: int, d: int,
            tokens: Optional[np.ndarray] = None) -> np.ndarray:
    """out[t] = sum over kept j of w[t,j] * y(t,j) ([LLaMA4-MoE] §2.4 weighted
    mix; [MoE-basics] §3.1 out[mask] += w * y), j ascending; dropped j add 0.

    ``y_by_assignment`` maps t*k + j -> expert output row (float64 [d])."""
    k = slot.shape[1]
    tokens = np.arange(T) if tokens is None else tokens
    out = np.zeros((tokens.size, d), dtype=np.float64)
    for i, t in enumerate(tokens):
        for j in range(k):
            if slot[t, j] >= 0:
                out[i] += w[t, j] * y_by_assignment[int(t) * k + j]
    return out


def mask_padding(idx: np.ndarray, w: np.ndarray, token_mask: Optional[np.ndarray]) -> tuple:
    """Reading R16: a padding token (token_mask = 0) selects no expert: its
    indices become -1 and its weights 0 ([LLaMA4-MoE] §4.1)."""
    if token_mask is None:
        return idx, w
    pad = np.asarray(token_mask) == 0
    idx = idx.copy()
    w = w.copy()
    idx[pad] = -1
    w[pad] = 0.0
    return idx, w


def real_tokens(token_mask: Optional[np.ndarray], T: int) -> np.ndarray:
    """Reading R16: the tokens that count in f and p (all of them without a mask)."""
    if token_mask is None:
        return np.ones(T, dtype=bool)
    return np.asarray(token_mask) != 0


def aux_stats(counts: np.ndarray, p: np.ndarray, T: int, k: int, alpha: float) -> tuple:
    """Load-balance statistics ([MoE-basics] §2.3 and §3.1; [LLaMA4-MoE] §3.2):
    f_e = n_e / (T*k) (reading R4), p_e = mean over tokens of the full softmax,
    L_aux = alpha * E * sum_e f_e * p_e.  T = 0 gives zeros (reading R7)."""
    E = counts.shape[0]
    if T == 0:
        return np.zeros(E), np.zeros(E), 0.0
    f = counts.astype(np.float64) / float(T * k)
    pm = p.sum(axis=0) / float(T)
    return f, pm, float(alpha * E * np.sum(f * pm))


# --------------------------------------------------------------------------
# whole layer
# --------------------------------------------------------------------------
def route(wl, inputs: dict, logits_feed: Optional[np.ndarray] = None) -> dict:
    """Router, softmax, top-k, renormalisation, capacity dispatch and aux stats
    over all T tokens.  ``logits_feed`` (float32 [T,E]) replaces the router
    product when both sides must take the discrete decisions on identical
    logits; it must come from this oracle or from the input generator.
    ``inputs['token_mask']`` (uint8 [T], optional) marks padding (R16)."""
    T, E, k = wl.T, wl.E, wl.k
    if logits_feed is None:
        x = to_f64(inputs["x"], wl.dtype)
        wr = to_f64(inputs["w_router"], wl.dtype)
        l64 = router_logits(x, wr, inputs.get("router_bias"))
    else:
        l64 = np.asarray(logits_feed, dtype=np.float32).astype(np.float64)
    l = decision_logits(l64)
    p = softmax(l) if T > 0 else np.zeros((0, E))
    idx = select_topk(l, k) if T > 0 else np.zeros((0, k), dtype=np.int32)
    w = renormalise(p, idx) if T > 0 else np.zeros((0, k))
    mask = inputs.get("token_mask")
    idx, w = mask_padding(idx, w, mask)
    cap = capacity(T, k, E, wl.capacity_factor)
    disp = dispatch(idx, E, cap)
    real = real_tokens(mask, T)
    f, pm, laux = aux_stats(disp["counts"], p[real], int(real.sum()), k, wl.aux_alpha)
    return {"logits64": l64, "logits": l, "p": p, "idx": idx, "w": w, "cap": cap,
            "f": f, "p_mean": pm, "l_aux": laux, "t_real": int(real.sum()), **disp}


def quantize_int8(w: np.ndarray) -> tuple:
    """Reading R18: per-output-channel symmetric INT8 codes of one expert's
    matrix w [K, N] (float32 values): s[n] = max_k |w[k,n]| / 127 and
    q = clamp(rint(w / s), -127, 127), all in float32; s = 0 gives q = 0."""
    w = np.asarray(w, dtype=np.float32)
    amax = np.abs(w).max(axis=0).astype(np.float32)
    s = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    q = np.rint((w / safe[None, :]).astype(np.float32))
    q = np.clip(q, -127, 127)
    q = np.where(s[None, :] > 0, q, 0).astype(np.int8)
    return q, s


def dequantize_int8(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Reading R18: the weights the INT8 layer uses, q * s (float64)."""
    return q.astype(np.float64) * s.astype(np.float64)[None, :]


def expert_weights_f64(wl, inputs: dict, e: int) -> tuple:
    """Expert e's parameters decoded to float64 (dequantised INT8 weights when
    the workload stores its routed experts in INT8, reading R18)."""
    dt = wl.dtype
    if getattr(wl, "weights", "native") == "int8":
        def dq(name):
            q, s = quantize_int8(to_f64(inputs[name][e], dt).astype(np.float32))
            return dequantize_int8(q, s)
        if wl.act == "swiglu":
            return (dq("w_gate"), dq("w_up"), dq("w_down"))
        return (dq("w1"), to_f64(inputs["b1"][e], dt), dq("w2"), to_f64(inputs["b2"][e], dt))
    if wl.act == "swiglu":
        return (to_f64(inputs["w_gate"][e], dt), to_f64(inputs["w_up"][e], dt), to_f64(inputs["w_down"][e], dt))
    return (to_f64(inputs["w1"][e], dt), to_f64(inputs["b1"][e], dt),
            to_f64(inputs["w2"][e], dt), to_f64(inputs["b2"][e], dt))


def shared_weights_f64(wl, inputs: dict, s: int) -> tuple:
    """Shared expert s's parameters decoded to float64 (reading R17)."""
    dt = wl.dtype
    if wl.act == "swiglu":
        return (to_f64(inputs["shared_gate"][s], dt), to_f64(inputs["shared_up"][s], dt),
                to_f64(inputs["shared_down"][s], dt))
    return (to_f64(inputs["shared_w1"][s], dt), to_f64(inputs["shared_b1"][s], dt),
            to_f64(inputs["shared_w2"][s], dt), to_f64(inputs["shared_b2"][s], dt))


def expert_apply(wl, params: tuple, xr: np.ndarray) -> np.ndarray:
    if wl.act == "swiglu":
        return expert_swiglu(xr, *params)
    return expert_gelu(xr, *params)


def expert_outputs(wl, inputs: dict, routing: dict, assignments: np.ndarray, x_rows: Optional[dict] = None) -> dict:
    """Expert output row y(t, j) for each kept assignment a = t*k + j listed.

    ``x_rows`` optionally maps token -> float64 row (for token subsets whose x
    was generated without the rest)."""
    k = wl.k
    idx = routing["idx"]
    by_e: dict = {}
    for a in assignments:
        t, j = divmod(int(a), k)
        if routing["slot"][t, j] >= 0:
            by_e.setdefault(int(idx[t, j]), []).append(int(a))
    out = {}
    x_all = None
    for e, alist in sorted(by_e.items()):
        toks = [a // k for a in alist]
        if x_rows is not None:
            xr = np.stack([x_rows[t] for t in toks])
        else:
            if x_all is None:
                x_all = inputs["x"]
            xr = to_f64(x_all[np.asarray(toks)], wl.dtype)
        y = expert_apply(wl, expert_weights_f64(wl, inputs, e), xr)
        for a, row in zip(alist, y):
            out[a] = row
    return out


def forward(wl, inputs: dict, logits_feed: Optional[np.ndarray] = None,
            tokens: Optional[np.ndarray] = None, routing: Optional[dict] = None,
            x_rows: Optional[dict] = None) -> dict:
    """The MoE layer forward: routing over all tokens, then expert FFNs and the
    weighted combine for ``tokens`` (all tokens when None).  A token's output
    depends only on its own row and its routing, so a subset is exact."""
    r = route(wl, inputs, logits_feed) if routing is None else routing
    T, k = wl.T, wl.k
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    assigns = np.array([t * k + j for t in toks for j in range(k)], dtype=np.int64)
    y = expert_outputs(wl, inputs, r, assigns, x_rows)
    out = combine(y, r["slot"], r["w"], T, wl.d, toks)
    n_shared = getattr(wl, "n_shared", 0)
    if n_shared > 0 and toks.size > 0:
        if x_rows is not None:
            xr = np.stack([x_rows[int(t)] for t in toks])
        else:
            xr = to_f64(inputs["x"][toks], wl.dtype)
        out = out + shared_outputs(wl, inputs, xr)
    return {**r, "out": out, "tokens": toks, "y": y}


# --------------------------------------------------------------------------
# expert parallelism
# --------------------------------------------------------------------------
def expert_owner(e, E: int, world: int):
    """Reading R19: the rank holding expert e when E experts are split over
    `world` ranks in contiguous blocks of E/world ([MoE-basics] §4.1)."""
    assert world >= 1 and E % world == 0
    return np.asarray(e) // (E // world)


def expert_parallel_layout(idx: np.ndarray, slot: np.ndarray, E: int, world: int) -> dict:
    """Reading R19: the row each kept assignment takes in the receive buffer of
    the rank that holds its expert ([LLaMA4-MoE] §2.5; [MoE-basics] §4.1).
    An owner's rows are grouped by its experts in ascending id, and each
    expert's rows follow the batch's token order ([LLaMA4-MoE] §2.4 grouping).

    ``idx`` [T,k] are the selected experts (-1 = padding) and ``slot`` [T,k]
    the single-device dispatch, of which only "kept" (slot >= 0) is read.
    Returns owner [T,k] and row [T,k] (-1 where dropped), recv_offsets
    [world, E/world + 1] (each owner's per-expert row offsets) and recv_src, a
    list over owners of the assignment t*k + j held in each row."""
    T, k = idx.shape
    El = E // world
    flat = idx.reshape(-1).astype(np.int64)
    kept = slot.reshape(-1) >= 0
    owner = np.full(T * k, -1, dtype=np.int64)
    row = np.full(T * k, -1, dtype=np.int64)
    recv_offsets = np.zeros((world, El + 1), dtype=np.int64)
    recv_src = []
    for o in range(world):
        mine = [e for e in range(E) if int(expert_owner(e, E, world)) == o]
        rows_o = []
        for el, e in enumerate(mine):
            recv_offsets[o, el] = len(rows_o)
            for a in np.nonzero(kept & (flat == e))[0]:  # ascending assignment = token order
                owner[a] = o
                row[a] = len(rows_o)
                rows_o.append(int(a))
        recv_offsets[o, len(mine):] = len(rows_o)
        recv_src.append(np.array(rows_o, dtype=np.int64))
    return {"owner": owner.reshape(T, k), "row": row.reshape(T, k), "recv_offsets": recv_offsets,
            "recv_src": recv_src}


def shared_outputs(wl, inputs: dict, xr: np.ndarray) -> np.ndarray:
    """Reading R17: the sum over the shared experts (in order, weight 1 each) of
    their outputs on rows ``xr`` ([LLaMA4-MoE] §5.2)."""
    acc = np.zeros((xr.shape[0], wl.d), dtype=np.float64)
    for s_ in range(wl.n_shared):
        acc = acc + expert_apply(wl, shared_weights_f64(wl, inputs, s_), xr)
    return acc
