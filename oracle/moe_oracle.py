"""CPU oracle of the MoE layer forward path (router -> grouping -> SwiGLU experts -> combine).

TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check in ``__graft_entry__`` and the
CPU-baseline leg of ``bench.py`` may import this module. The CUDA library never calls it, and
it shares no code, table or constant with the CUDA sources.

Everything here is plain NumPy in float64 (a matmul and a stable sort are the only library
primitives used as steps). Inputs arrive as NumPy arrays whose values are exactly the values the
GPU sees (bf16 values are passed widened to float32, which is exact).

Sources, cited by page title and section:

* [P1] "MoE 模型的 FlashAttention 跟普通模型有什么不一样？" (framerc.cn)
  - section "FlashAttention 在 MoE 模型里的位置": the five-step flow (route top-k, group tokens
    by expert, per-expert FFN, merge weighted by the routing weights).
  - section "融合二：expert 计算的输出 + 合并结果": merge is ``accum += route_weight * expert_output``.
  - section "手动编译 MoE 融合算子": router weight ``[hidden_dim, num_experts]``, expert weights
    stacked with a leading expert dimension, ``activation="silu"``.
* [P4] "MoE Router" on Ascend CANN (2048ai.net)
  - section "Router 就是一个小型网络": gate = Linear(hidden, E, bias=False); softmax over all E;
    torch.topk; divide the k selected weights by their sum.
  - section "昇腾NPU的通信计算重叠": capacity C = (total tokens / E) x 1.25; assignments beyond
    C are dropped and take the residual path (contribute nothing to the MoE output).
* [P5] "大模型推理加速200%+？这套国产融合算子库把CUDA/Triton全替换了" (csdn.net)
  - section "3.1 Moe Fuse Gate & Softmax TopK": exp only over the selected k, which equals the
    renormalised full softmax in exact arithmetic; the gate selects expert groups first
    ("优先选组") and keeps each group's top-1 / top-2.
  - section "3.2 Fuse RMS RoPE & MoE Align & MoE Sum": the MoE sum also adds the shared expert's
    output with a factor, and a bias.

Readings taken where the pages are silent or disagree (each also listed in the design notes):

* "total tokens" in the capacity formula counts assignments, T*k (the preceding section of [P4]
  counts T*k expert accesses); C = ceil(cf*T*k/E), computed exactly, capped at T; cf <= 0 means
  no capacity limit (C = T).
* Drops go in token order: the earliest tokens keep their slot. Survivors are not renormalised;
  a dropped assignment contributes 0, a fully dropped token has output 0.
* Top-k ranks float32 logits (softmax is monotone); equal logits (including -0 vs +0) go to the
  lower expert index; the k indices are listed by descending logit, then ascending index.
* SwiGLU expert: y = (silu(x Wg) * (x Wu)) Wd, silu(z) = z / (1 + exp(-z)); experts have no bias.
* Group-limited routing (the pages name it, give no formula): the E experts form n_group equal
  contiguous groups; a group's score is the float32 sum of its two largest logits (its only
  logit when a group holds one expert); the topk_group groups with the highest scores are kept
  (ties to the lower group index); the k largest logits among the kept groups' experts are
  selected with the plain top-k rule; weights are renormalised over the k as before.
* FP8 expert weights ([P5] section "4.3 MOE量化方案矩阵" lists W16A16, W8A8 (INT8/FP8), W4A8
  and W4A16 expert GEMMs with offline weight repacking, without a numeric scheme; the reading
  taken is the FP8 weight format of W8A8 with the 16-bit activations of W4A16): weights only, e4m3 (OCP FP8: 1 sign, 4
  exponent bits with bias 7, 3 mantissa bits, subnormals, no infinities, 448 the largest
  finite value); one float32 scale per output channel, scale = max_k |W[k, m]| / 448 (1 when
  the column is all zero); code = e4m3(W / scale) rounded to nearest, ties to even, saturating
  at +-448; the GEMM uses decode(code) * scale. Activations stay bf16 (W8A16).
* FP8 weights and activations (W8A8, the same [P5] section): the weights as above; the
  activations entering each expert GEMM quantised per row to e4m3 the same way (one float32 scale
  per token row of x, one per slot row of h: scale = max |row| / 448, code = e4m3(v / scale)).
  The SwiGLU intermediate h is rounded to bfloat16 before its quantisation, since the GPU keeps h
  in bf16 between the two GEMMs and a quantised code is decided in the kernel's precision. Both
  scales of a product are applied to the accumulated sum: y[m] = s_act * s_w[m] * sum_k
  decode(q_act[k]) * decode(q_w[k, m]).
* Shared expert and bias in the combine: out[t] = sum_j w[t,j] y[slot] + factor * shared[t] + b,
  with shared[t] the shared expert's output row (computed by the caller) and b a per-feature
  bias; both terms apply to every token, including a fully dropped one.

Every function below is pinned by tests that do not re-run its own formula (brute force,
closed forms, hand-worked fixtures under tests/golden, special cases reducing to a dense FFN).
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

__all__ = [
    "router_logits",
    "select_topk",
    "group_scores",
    "select_topk_grouped",
    "route_weights",
    "route",
    "route_grouped",
    "capacity",
    "e4m3_decode",
    "e4m3_encode",
    "quantize_weights_fp8",
    "dequantize_weights_fp8",
    "bf16_round",
    "quantize_rows_fp8",
    "swiglu_expert_w8a8",
    "align",
    "swiglu_expert",
    "grouped_ffn_slots",
    "combine",
    "layer_forward",
]


def router_logits(x, w_router, logit_bias=None):
    """Gate logits l[t,e] = sum_h x[t,h] * Wr[h,e] (+ bias[e]), float64, rounded once to float32.

    [P4] "Router 就是一个小型网络": the gate is a bias-free Linear(hidden, E). The optional
    per-expert bias is an input of the skewed-load workload (not a learned gate bias).
    """
    x64 = np.asarray(x, dtype=np.float64)
    w64 = np.asarray(w_router, dtype=np.float64)
    logits = x64 @ w64
    if logit_bias is not None:
        logits = logits + np.asarray(logit_bias, dtype=np.float64)[None, :]
    return logits.astype(np.float32)


def select_topk(logits, k):
    """Indices of the k largest float32 logits per row, ordered by (logit desc, index asc).

    [P4] "Router 就是一个小型网络" (torch.topk over the softmax scores; softmax is monotone so
    ranking logits ranks scores). A stable sort on the negated logits keeps equal values in
    ascending expert order, which is the tie rule.
    """
    l32 = np.asarray(logits, dtype=np.float32)
    if k < 1 or k > l32.shape[1]:
        raise ValueError("need 1 <= k <= E")
    order = np.argsort(-l32, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def route_weights(logits, topk_idx):
    """Renormalised routing weights, float64.

    [P4] "Router 就是一个小型网络": p = softmax(l) over all E experts, then the k selected
    probabilities are divided by their sum so that they add to 1.
    """
    l64 = np.asarray(logits, dtype=np.float32).astype(np.float64)
    m = l64.max(axis=1, keepdims=True)
    p = np.exp(l64 - m)
    p = p / p.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(p, np.asarray(topk_idx, dtype=np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def route(x, w_router, k, logit_bias=None, logits=None):
    """Router step: returns (logits f32 [T,E], topk_idx i32 [T,k], topk_w f64 [T,k])."""
    if logits is None:
        logits = router_logits(x, w_router, logit_bias)
    idx = select_topk(logits, k)
    return np.asarray(logits, dtype=np.float32), idx, route_weights(logits, idx)


def group_scores(logits, n_group):
    """Score of each expert group per row: the float32 sum of the group's two largest float32
    logits (the single logit when a group holds one expert). Shape [T, n_group], float32.

    [P5] "3.1 Moe Fuse Gate & Softmax TopK" (select groups first, keep each group's top-1 and
    top-2). The sum is one float32 addition, the same rounding the kernel performs.
    """
    l32 = np.asarray(logits, dtype=np.float32)
    T, E = l32.shape
    if n_group < 1 or E % n_group != 0:
        raise ValueError("n_group must divide E")
    gs = E // n_group
    g = np.sort(l32.reshape(T, n_group, gs), axis=2)[:, :, ::-1]
    if gs == 1:
        return g[:, :, 0].astype(np.float32)
    return (g[:, :, 0] + g[:, :, 1]).astype(np.float32)


def select_topk_grouped(logits, k, n_group, topk_group):
    """Group-limited top-k: keep the topk_group best-scoring groups (scores from group_scores,
    ties to the lower group index), then the k largest logits among their experts, ordered and
    tie-broken exactly as select_topk.

    [P5] "3.1 Moe Fuse Gate & Softmax TopK" ("优先选组"). With topk_group == n_group (or
    n_group == 1) this is select_topk.
    """
    l32 = np.asarray(logits, dtype=np.float32)
    T, E = l32.shape
    if not (1 <= topk_group <= n_group):
        raise ValueError("need 1 <= topk_group <= n_group")
    gs = E // n_group
    if k < 1 or k > topk_group * gs:
        raise ValueError("need 1 <= k <= topk_group * (E / n_group)")
    sc = group_scores(l32, n_group)
    gorder = np.argsort(-sc, axis=1, kind="stable")[:, :topk_group]
    keep = np.zeros((T, n_group), dtype=bool)
    np.put_along_axis(keep, gorder, True, axis=1)
    order = np.argsort(-l32, axis=1, kind="stable")
    out = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        cand = [int(e) for e in order[t] if keep[t, int(e) // gs]]
        out[t] = cand[:k]
    return out


def route_grouped(x, w_router, k, n_group, topk_group, logit_bias=None, logits=None):
    """Router step with group-limited selection: (logits f32, topk_idx i32, topk_w f64)."""
    if logits is None:
        logits = router_logits(x, w_router, logit_bias)
    idx = select_topk_grouped(logits, k, n_group, topk_group)
    return np.asarray(logits, dtype=np.float32), idx, route_weights(logits, idx)


def e4m3_decode(codes):
    """Value of each FP8 e4m3 code (uint8), float64, from the format's definition:
    sign s, exponent field e (4 bits, bias 7), mantissa field m (3 bits);
    e > 0: (-1)^s * 2^(e-7) * (1 + m/8); e == 0: (-1)^s * 2^-6 * (m/8); e == 15 and m == 7: NaN.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e > 0, np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64)),
                   np.ldexp(m / 8.0, -6))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def e4m3_encode(values):
    """Nearest e4m3 code of each float32 value, ties to the even code (even mantissa field),
    saturating to +-448 (the largest finite magnitude); -0 keeps its sign. Finite inputs only.

    Chosen among the 127 finite non-negative codes by exact float64 comparison: the nearest
    magnitude wins; at an exact midpoint the code with an even mantissa field wins.
    """
    v = np.asarray(values, dtype=np.float32).astype(np.float64)
    if not np.all(np.isfinite(v)):
        raise ValueError("e4m3_encode takes finite values")
    mags = e4m3_decode(np.arange(127, dtype=np.uint8))      # codes 0..126: 0 .. 448, ascending
    a = np.minimum(np.abs(v), 448.0)
    hi = np.searchsorted(mags, a, side="left")               # first magnitude >= a
    hi = np.minimum(hi, 126)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - mags[lo]
    d_hi = mags[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(a == mags[hi], hi, np.where(pick_hi, hi, lo)).astype(np.int64)
    sign = np.signbit(v).astype(np.int64)
    return (code | (sign << 7)).astype(np.uint8)


def quantize_weights_fp8(w):
    """Per-output-channel e4m3 quantisation of expert weights w [E, K, M] (reduction dim K,
    output channels M): scale[e, m] = float32(max_k |w[e, k, m]| / 448) (1 when the column is
    all zero), code[e, k, m] = e4m3(float32(w / scale)). Returns (codes uint8, scale float32).
    Both divisions are single float32 operations, the rounding the GPU performs."""
    w32 = np.asarray(w, dtype=np.float32)
    amax = np.max(np.abs(w32), axis=1)                       # [E, M], exact
    scale = np.where(amax > 0, (amax / np.float32(448.0)).astype(np.float32), np.float32(1.0))
    scale = scale.astype(np.float32)
    q = e4m3_encode((w32 / scale[:, None, :]).astype(np.float32))
    return q, scale


def dequantize_weights_fp8(codes, scale):
    """decode(code) * scale, float64 [E, K, M]: the weights the FP8 expert GEMMs apply."""
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[:, None, :]


def bf16_round(values):
    """Nearest bfloat16 of each value, as float32: rounded to float32 first (the precision the
    GPU computes h in), then to the 8 significant bits of bfloat16, ties to the even pattern."""
    f = np.ascontiguousarray(np.asarray(values, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).reshape(f.shape)


def quantize_rows_fp8(a):
    """Per-row e4m3 quantisation of activations a [N, K]: scale[n] = float32(max_k |a[n, k]| /
    448) (1 for an all-zero row), code[n, k] = e4m3(float32(a[n, k] / scale[n])), nearest-even,
    saturating. Returns (codes uint8 [N, K], scale float32 [N]); both divisions are single
    float32 operations, as on the GPU."""
    a32 = np.asarray(a, dtype=np.float32)
    if a32.shape[0] == 0:
        return np.zeros(a32.shape, dtype=np.uint8), np.zeros(0, dtype=np.float32)
    amax = np.max(np.abs(a32), axis=1)
    scale = np.where(amax > 0, (amax / np.float32(448.0)).astype(np.float32),
                     np.float32(1.0)).astype(np.float32)
    return e4m3_encode((a32 / scale[:, None]).astype(np.float32)), scale


def swiglu_expert_w8a8(x_rows, wg, wu, wd):
    """One expert's SwiGLU FFN with e4m3 weights and e4m3 activations (W8A8), float64 sums.

    wg, wu, wd are (codes, scale) pairs of the expert's weights as quantize_weights_fp8 makes
    them ([K, M] codes, [M] scales). x rows are quantised per row; the intermediate
    h = silu(g) * u is rounded to bfloat16 and quantised per row before the down projection:
      g[m] = s_x * s_g[m] * sum_k dec(q_x[k]) dec(q_g[k, m])   (u likewise)
      y[m] = s_h * s_d[m] * sum_i dec(q_h[i]) dec(q_d[i, m])
    """
    qx, sx = quantize_rows_fp8(x_rows)
    xd = e4m3_decode(qx) * sx.astype(np.float64)[:, None]

    def deq(w):
        q, sc = w
        return e4m3_decode(q) * np.asarray(sc, dtype=np.float64)[None, :]

    g = xd @ deq(wg)
    u = xd @ deq(wu)
    with np.errstate(over="ignore"):
        h = g * u / (1.0 + np.exp(-g))
    qh, sh = quantize_rows_fp8(bf16_round(h))
    hd = e4m3_decode(qh) * sh.astype(np.float64)[:, None]
    return hd @ deq(wd)


def capacity(T, k, E, capacity_factor):
    """Per-expert capacity C = ceil(cf * T * k / E), exact rational arithmetic, capped at T.

    [P4] "昇腾NPU的通信计算重叠": C = (total_tokens / num_experts) x 1.25, with total tokens read
    as the T*k assignments. cf is taken as the float32 value the C ABI receives. cf <= 0: no limit.
    """
    cf = Fraction(float(np.float32(capacity_factor)))
    if cf <= 0:
        return int(T)
    c = math.ceil(cf * int(T) * int(k) / int(E))
    return int(min(c, int(T)))


def align(topk_idx, E, C):
    """Capacity-limited grouping of assignments by expert, token order first.

    [P1] "FlashAttention 在 MoE 模型里的位置" step 3 (pick the tokens that go to the same
    expert) and [P4] "昇腾NPU的通信计算重叠" (at most C per expert, overflow dropped).

    Assignment a = t*k + j goes to expert idx[t,j]. Its rank is the number of earlier
    assignments (smaller t) to the same expert. Kept iff rank < C.

    Returns dict with counts [E], offsets [E+1], sorted_ids [T*k] (slot -> a, -1 past the kept
    total), slot_of [T*k] (a -> slot or -1), drop_mask [T*k] (1 = dropped), raw [E], rank [T*k].
    """
    idx = np.asarray(topk_idx, dtype=np.int64)
    T, k = idx.shape
    A = T * k
    seen = [0] * E
    rank = [0] * A
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            rank[t * k + j] = seen[e]
            seen[e] += 1
    counts = [min(r, C) for r in seen]
    offsets = [0]
    for e in range(E):
        offsets.append(offsets[-1] + counts[e])
    sorted_ids = np.full(A, -1, dtype=np.int32)
    slot_of = np.full(A, -1, dtype=np.int32)
    drop_mask = np.zeros(A, dtype=np.uint8)
    for t in range(T):
        for j in range(k):
            a = t * k + j
            e = int(idx[t, j])
            if rank[a] < C:
                slot = offsets[e] + rank[a]
                sorted_ids[slot] = a
                slot_of[a] = slot
            else:
                drop_mask[a] = 1
    return {
        "counts": np.asarray(counts, dtype=np.int32),
        "offsets": np.asarray(offsets, dtype=np.int32),
        "sorted_ids": sorted_ids,
        "slot_of": slot_of,
        "drop_mask": drop_mask,
        "raw": np.asarray(seen, dtype=np.int64),
        "rank": np.asarray(rank, dtype=np.int64),
    }


def swiglu_expert(x_rows, w_gate_e, w_up_e, w_down_e):
    """One expert's FFN on a block of rows: (silu(x Wg) * (x Wu)) Wd, all in float64.

    [P1] "手动编译 MoE 融合算子" (activation="silu", weights [hidden, ffn] per expert);
    silu(z) = z * sigmoid(z) = z / (1 + exp(-z)).
    """
    xr = np.asarray(x_rows, dtype=np.float64)
    g = xr @ np.asarray(w_gate_e, dtype=np.float64)
    u = xr @ np.asarray(w_up_e, dtype=np.float64)
    with np.errstate(over="ignore"):
        h = g * u / (1.0 + np.exp(-g))
    return h @ np.asarray(w_down_e, dtype=np.float64)


def grouped_ffn_slots(x, sorted_ids, offsets, k, w_gate, w_up, w_down, slots=None,
                      expert_fn=None):
    """Expert output per kept slot: y[s] = expert_e(x[sorted_ids[s] // k]) for s in expert e's range.

    [P1] "FlashAttention 在 MoE 模型里的位置" step 4. ``w_*`` may be arrays or any object whose
    ``[e]`` returns expert e's matrix (or what ``expert_fn`` takes for it). ``slots`` restricts
    the evaluation to a subset (returned as a dict slot -> row); by default every kept slot is
    evaluated into a [A_kept, H] array. ``expert_fn`` (default swiglu_expert) evaluates one
    expert on a block of rows: swiglu_expert_w8a8 for FP8 weights and activations.
    """
    expert_fn = swiglu_expert if expert_fn is None else expert_fn
    offsets = np.asarray(offsets, dtype=np.int64)
    E = len(offsets) - 1
    sorted_ids = np.asarray(sorted_ids, dtype=np.int64)
    x = np.asarray(x)
    want = None if slots is None else set(int(s) for s in slots)
    result = {}
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        sl = [s for s in range(lo, hi) if want is None or s in want]
        if not sl:
            continue
        toks = sorted_ids[sl] // k
        y = expert_fn(x[toks], w_gate[e], w_up[e], w_down[e])
        for i, s in enumerate(sl):
            result[s] = y[i]
    if slots is not None:
        return result
    a_kept = int(offsets[-1])
    H = (len(next(iter(result.values()))) if result else 0) if a_kept else 0
    out = np.zeros((a_kept, H), dtype=np.float64)
    for s, row in result.items():
        out[s] = row
    return out


def combine(y_slots, slot_of, topk_w, tokens=None, shared=None, shared_factor=0.0,
            out_bias=None):
    """Weighted merge back to token order: out[t] = sum_{kept j} w[t,j] * y[slot_of[t*k+j]]
    (+ shared_factor * shared[t] + out_bias when given).

    [P1] "融合二：expert 计算的输出 + 合并结果" (accum += route_weight * expert_output);
    [P5] "3.2 ... MoE Sum" (shared expert factor and bias added in the sum).
    A dropped assignment (slot -1) contributes nothing; a fully dropped token gives 0 plus the
    shared and bias terms. ``y_slots`` may be an array or a dict slot -> row; ``shared`` is
    indexed by token.
    """
    w = np.asarray(topk_w, dtype=np.float64)
    T, k = w.shape
    slot_of = np.asarray(slot_of, dtype=np.int64).reshape(T, k)
    toks = range(T) if tokens is None else tokens
    H = None
    rows = {}
    for t in toks:
        acc = None
        for j in range(k):
            s = int(slot_of[t, j])
            if s < 0:
                continue
            y = np.asarray(y_slots[s], dtype=np.float64)
            acc = w[t, j] * y if acc is None else acc + w[t, j] * y
            H = y.shape[0]
        rows[t] = acc
    if H is None:
        H = np.asarray(y_slots[0]).shape[-1] if len(y_slots) else 0
    if H is None and shared is not None:
        H = np.asarray(shared).shape[-1]
    if H is None and out_bias is not None:
        H = np.asarray(out_bias).shape[-1]
    out = np.zeros((len(rows), H), dtype=np.float64)
    for i, t in enumerate(toks):
        if rows[t] is not None:
            out[i] = rows[t]
        if shared is not None:
            out[i] += float(shared_factor) * np.asarray(shared[t], dtype=np.float64)
        if out_bias is not None:
            out[i] += np.asarray(out_bias, dtype=np.float64)
    return out


def layer_forward(x, w_router, w_gate, w_up, w_down, k, capacity_factor,
                  logit_bias=None, logits=None, tokens=None, n_group=1, topk_group=1,
                  shared=None, shared_factor=0.0, out_bias=None, expert_fn=None):
    """Whole MoE layer: route -> align -> experts -> combine, float64 throughout.

    [P1] "FlashAttention 在 MoE 模型里的位置" steps 2-5. ``logits`` (float32) may be supplied
    to route from given gate logits. ``tokens`` restricts the expert FFN and the combine to a
    subset of tokens (routing and capacity still see every token, since ranks depend on all).
    ``n_group``/``topk_group`` select group-limited routing; ``shared``/``shared_factor``/
    ``out_bias`` add the shared-expert and bias terms of the combine. ``expert_fn`` replaces the
    expert FFN (swiglu_expert_w8a8 for FP8 weights and activations, with ``w_*[e]`` the
    (codes, scale) pairs).
    Returns dict with out [len(tokens) or T, H] and all routing intermediates.
    """
    x = np.asarray(x)
    T = x.shape[0]
    if n_group > 1:
        logits, idx, w = route_grouped(x, w_router, k, n_group, topk_group,
                                       logit_bias=logit_bias, logits=logits)
    else:
        logits, idx, w = route(x, w_router, k, logit_bias=logit_bias, logits=logits)
    E = logits.shape[1]
    C = capacity(T, k, E, capacity_factor)
    al = align(idx, E, C)
    tok_list = list(range(T)) if tokens is None else [int(t) for t in tokens]
    need = set()
    for t in tok_list:
        for j in range(k):
            s = int(al["slot_of"][t * k + j])
            if s >= 0:
                need.add(s)
    y = grouped_ffn_slots(x, al["sorted_ids"], al["offsets"], k, w_gate, w_up, w_down,
                          slots=sorted(need), expert_fn=expert_fn)
    out = combine(y, al["slot_of"], w, tokens=tok_list, shared=shared,
                  shared_factor=shared_factor, out_bias=out_bias)
    res = dict(al)
    res.update({"logits": logits, "topk_idx": idx, "topk_w": w, "C": C, "out": out,
                "tokens": tok_list})
    return res
