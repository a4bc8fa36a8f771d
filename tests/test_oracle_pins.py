"""Pins for the CPU oracle: each check rests on something other than the oracle's own formula
(brute force, closed forms, hand-worked fixtures, textbook special cases)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as orc
from expert_dispatch_gate_b200 import workloads as wlm


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- router logits

def test_router_logits_match_scalar_dot_products():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 7)).astype(np.float32)
    w = rng.standard_normal((7, 3)).astype(np.float32)
    b = rng.standard_normal(3).astype(np.float32)
    got = orc.router_logits(x, w, b)
    assert got.dtype == np.float32 and got.shape == (5, 3)
    for t in range(5):
        for e in range(3):
            ref = math.fsum(float(x[t, h]) * float(w[h, e]) for h in range(7)) + float(b[e])
            assert got[t, e] == np.float32(ref)


# ---------------------------------------------------------------- top-k selection

def _valid_topk_sets(l, k):
    """Every k-subset S with: for i in S, j not in S, l_i > l_j or (l_i == l_j and i < j)."""
    E = len(l)
    found = []
    for S in itertools.combinations(range(E), k):
        ok = all((l[i] > l[j]) or (l[i] == l[j] and i < j)
                 for i in S for j in range(E) if j not in S)
        if ok:
            found.append(set(S))
    return found


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    for E in range(1, 8):
        for k in range(1, E + 1):
            l = rng.integers(-2, 3, size=(6, E)).astype(np.float32) * 0.5
            # plant signed zeros
            l[rng.random(l.shape) < 0.2] = -0.0
            idx = orc.select_topk(l, k)
            for t in range(l.shape[0]):
                sets = _valid_topk_sets(list(l[t]), k)
                assert len(sets) == 1
                assert set(idx[t].tolist()) == sets[0]
                # listed by descending logit, then ascending index
                for a, b in zip(idx[t][:-1], idx[t][1:]):
                    assert l[t, a] > l[t, b] or (l[t, a] == l[t, b] and a < b)


def test_topk_is_max_sum_subset_for_distinct_logits():
    rng = np.random.default_rng(7)
    for _ in range(20):
        E = int(rng.integers(2, 9))
        k = int(rng.integers(1, E + 1))
        l = rng.permutation(E).astype(np.float32) + rng.random(E).astype(np.float32) * 0.1
        best = max(itertools.combinations(range(E), k), key=lambda S: sum(float(l[i]) for i in S))
        assert set(orc.select_topk(l[None, :], k)[0].tolist()) == set(best)


def test_routing_golden(golden_dir):
    g = _load(golden_dir, "routing_tiny.json")
    logits = np.asarray(g["logits"], dtype=np.float32)
    # the fixture's -0.0 must survive json
    assert math.copysign(1.0, float(logits[2, 1])) == -1.0
    _, idx, w = orc.route(None, None, g["k"], logits=logits)
    assert idx.tolist() == g["topk_idx"]
    np.testing.assert_allclose(w, np.asarray(g["topk_w"]), atol=g["tolerance"], rtol=0)


# ---------------------------------------------------------------- routing weights

def test_weights_sum_to_one_and_k1_is_exactly_one():
    l = wlm.random_logits(200, 16, seed=3).numpy()
    for k in (1, 2, 5, 16):
        idx = orc.select_topk(l, k)
        w = orc.route_weights(l, idx)
        assert np.all(w > 0)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-14, rtol=0)
        if k == 1:
            assert np.all(w == 1.0)


def test_weights_two_experts_logistic_closed_form():
    rng = np.random.default_rng(11)
    l = (rng.standard_normal((50, 2)) * 3).astype(np.float32)
    idx = orc.select_topk(l, 2)
    w = orc.route_weights(l, idx)
    for t in range(50):
        a, b = idx[t]
        da = float(l[t, a]) - float(l[t, b])
        assert abs(w[t, 0] - 1.0 / (1.0 + math.exp(-da))) < 1e-14
        assert abs(w[t, 1] - 1.0 / (1.0 + math.exp(da))) < 1e-14


def test_weights_ratio_and_independence_from_unselected():
    rng = np.random.default_rng(12)
    l = rng.standard_normal((40, 12)).astype(np.float32)
    idx = orc.select_topk(l, 4)
    w = orc.route_weights(l, idx)
    # w_i / w_j = exp(l_i - l_j) for selected i, j
    for t in range(40):
        for a in range(4):
            for b in range(4):
                r = w[t, a] / w[t, b]
                assert abs(r - math.exp(float(l[t, idx[t, a]]) - float(l[t, idx[t, b]]))) < 1e-12 * max(1, r)
    # lowering an unselected logit changes the full softmax but not the renormalised weights
    l2 = l.copy()
    for t in range(40):
        for e in range(12):
            if e not in idx[t]:
                l2[t, e] -= 3.0
    idx2 = orc.select_topk(l2, 4)
    assert np.array_equal(idx, idx2)
    np.testing.assert_allclose(orc.route_weights(l2, idx2), w, atol=1e-14, rtol=0)


def test_routing_shift_invariance():
    l = wlm.random_logits(100, 32, seed=5).numpy()
    idx = orc.select_topk(l, 6)
    w = orc.route_weights(l, idx)
    l2 = (l.astype(np.float64) + 0.5).astype(np.float32)  # exact: |l| < 8, step 2^-20
    assert np.array_equal(orc.select_topk(l2, 6), idx)
    np.testing.assert_allclose(orc.route_weights(l2, idx), w, atol=1e-6, rtol=0)


# ---------------------------------------------------------------- capacity

def test_capacity_golden(golden_dir):
    g = _load(golden_dir, "capacity_cases.json")
    for c in g["cases"]:
        assert orc.capacity(c["T"], c["k"], c["E"], c["cf"]) == c["C"], c


# ---------------------------------------------------------------- align

def test_align_golden(golden_dir):
    g = _load(golden_dir, "align_tiny.json")
    al = orc.align(np.asarray(g["topk_idx"]), g["E"], g["C"])
    for key in ("counts", "offsets", "sorted_ids", "slot_of", "drop_mask"):
        assert al[key].tolist() == g[key], key


def _check_align_invariants(idx, E, C, al):
    T, k = idx.shape
    A = T * k
    counts, offsets = al["counts"], al["offsets"]
    sid, slot_of, drop = al["sorted_ids"], al["slot_of"], al["drop_mask"]
    raw = np.bincount(idx.reshape(-1), minlength=E)
    assert np.array_equal(counts, np.minimum(raw, C))
    assert np.all(counts <= C)
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    kept = int(offsets[-1])
    assert kept == A - int(drop.sum())
    # bijection between slots [0, kept) and kept assignments
    assert np.all(sid[kept:] == -1)
    assert sorted(sid[:kept].tolist()) == sorted(np.nonzero(drop == 0)[0].tolist())
    for s in range(kept):
        assert slot_of[sid[s]] == s
    assert np.all((slot_of == -1) == (drop == 1))
    # each slot sits inside its expert's range
    flat = idx.reshape(-1)
    for s in range(kept):
        e = flat[sid[s]]
        assert offsets[e] <= s < offsets[e + 1]
    # token order, checked by listing each expert's tokens: the first C of them are kept,
    # in ascending token order
    for e in range(E):
        toks = [a for a in range(A) if flat[a] == e]
        keep = toks[:C]
        assert sid[offsets[e]:offsets[e + 1]].tolist() == keep
        assert all(drop[a] == 1 for a in toks[C:])


@pytest.mark.parametrize("mode", ["uniform", "zipf", "one"])
def test_align_invariants(mode):
    for (T, E, k, cf) in [(50, 8, 2, 1.25), (97, 16, 4, 1.0), (64, 4, 4, 0.0), (33, 64, 6, 1.25)]:
        idx = wlm.random_topk_idx(T, E, k, seed=T + E, mode=mode).numpy()
        C = orc.capacity(T, k, E, cf)
        al = orc.align(idx, E, C)
        _check_align_invariants(idx, E, C, al)
        if cf <= 0:
            assert al["drop_mask"].sum() == 0


def test_align_all_to_one_expert_keeps_first_C():
    T, E, k = 40, 8, 1
    idx = np.zeros((T, 1), dtype=np.int32)
    C = orc.capacity(T, k, E, 1.25)  # ceil(50/8) = 7
    assert C == 7
    al = orc.align(idx, E, C)
    assert al["counts"].tolist() == [7] + [0] * 7
    assert al["sorted_ids"][:7].tolist() == list(range(7))
    assert al["drop_mask"].tolist() == [0] * 7 + [1] * 33


# ---------------------------------------------------------------- expert FFN + combine

def test_layer_golden(golden_dir):
    g = _load(golden_dir, "layer_tiny.json")
    arr = lambda key: np.asarray(g[key], dtype=np.float64)
    res = orc.layer_forward(arr("x"), arr("w_router"), arr("w_gate"), arr("w_up"), arr("w_down"),
                            g["k"], g["capacity_factor"])
    assert res["topk_idx"].tolist() == g["topk_idx"]
    np.testing.assert_allclose(res["out"], arr("out"), atol=g["tolerance"], rtol=0)


def _dense_swiglu_torch(x, wg, wu, wd):
    x, wg, wu, wd = (torch.as_tensor(np.asarray(a, dtype=np.float64)) for a in (x, wg, wu, wd))
    return (torch.nn.functional.silu(x @ wg) * (x @ wu) @ wd).numpy()


def test_single_expert_top1_is_dense_swiglu():
    wl = wlm.Workload("t", 0, 37, 24, 1, 1, 40, "f32", 1.25)
    inp = wlm.make_inputs(wl)
    a = {k_: (v.numpy() if v is not None else None) for k_, v in inp.items()}
    res = orc.layer_forward(a["x"], a["w_router"], a["w_gate"], a["w_up"], a["w_down"], 1, 1.25)
    assert res["C"] == 37 and res["drop_mask"].sum() == 0
    assert np.all(res["topk_w"] == 1.0)
    ref = _dense_swiglu_torch(a["x"], a["w_gate"][0], a["w_up"][0], a["w_down"][0])
    np.testing.assert_allclose(res["out"], ref, rtol=1e-12, atol=1e-12)


def test_identical_experts_equal_dense_ffn_for_any_routing():
    wl = wlm.Workload("t", 0, 29, 16, 6, 3, 20, "f32", 0.0)
    inp = wlm.make_inputs(wl)
    a = {k_: (v.numpy() if v is not None else None) for k_, v in inp.items()}
    wg = np.repeat(a["w_gate"][:1], 6, axis=0)
    wu = np.repeat(a["w_up"][:1], 6, axis=0)
    wd = np.repeat(a["w_down"][:1], 6, axis=0)
    res = orc.layer_forward(a["x"], a["w_router"], wg, wu, wd, 3, 0.0)
    ref = _dense_swiglu_torch(a["x"], wg[0], wu[0], wd[0])
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-10)


def test_one_hot_routing_linearity_and_drops():
    wl = wlm.Workload("t", 0, 24, 16, 4, 1, 12, "f32", 1.0)
    inp = wlm.make_inputs(wl)
    a = {k_: (v.numpy() if v is not None else None) for k_, v in inp.items()}
    # force every token to expert 2 through the logits; C = ceil(24/4) = 6
    logits = np.zeros((24, 4), dtype=np.float32)
    logits[:, 2] = 1.0
    res = orc.layer_forward(a["x"], None, a["w_gate"], a["w_up"], a["w_down"], 1, 1.0, logits=logits)
    assert res["C"] == 6
    ref = _dense_swiglu_torch(a["x"], a["w_gate"][2], a["w_up"][2], a["w_down"][2])
    np.testing.assert_allclose(res["out"][:6], ref[:6], rtol=1e-12, atol=1e-12)
    assert np.all(res["out"][6:] == 0.0)  # dropped tokens take the residual path only
    # linear in the down projection
    res2 = orc.layer_forward(a["x"], None, a["w_gate"], a["w_up"], 2.0 * a["w_down"], 1, 1.0,
                             logits=logits)
    np.testing.assert_allclose(res2["out"], 2.0 * res["out"], rtol=1e-12, atol=1e-12)


def test_token_subset_matches_full_layer():
    wl = wlm.Workload("t", 0, 31, 16, 8, 2, 24, "f32", 1.25)
    inp = wlm.make_inputs(wl)
    a = {k_: (v.numpy() if v is not None else None) for k_, v in inp.items()}
    full = orc.layer_forward(a["x"], a["w_router"], a["w_gate"], a["w_up"], a["w_down"], 2, 1.25)
    sub = orc.layer_forward(a["x"], a["w_router"], a["w_gate"], a["w_up"], a["w_down"], 2, 1.25,
                            tokens=[30, 3, 17])
    # same values up to the BLAS blocking of the matmul (rows batched differently)
    np.testing.assert_allclose(sub["out"], full["out"][[30, 3, 17]], rtol=1e-13, atol=1e-15)


def test_silu_textbook_values():
    # silu(0) = 0 kills the gate: zero x rows give zero output for every expert
    x = np.zeros((3, 4))
    rng = np.random.default_rng(2)
    y = orc.swiglu_expert(x, rng.standard_normal((4, 5)), rng.standard_normal((4, 5)),
                          rng.standard_normal((5, 4)))
    assert np.all(y == 0.0)
    # large positive gate: silu(z) -> z; very negative: -> 0 without overflow warnings
    one = np.ones((1, 1))
    assert abs(orc.swiglu_expert(one * 40.0, one, one, one)[0, 0] - 1600.0) < 1e-9
    assert abs(orc.swiglu_expert(one * -800.0, one, one, one)[0, 0]) < 1e-300


# ---------------------------------------------------------------- sizes printed on the pages

def test_page_sizes(golden_dir):
    g = _load(golden_dir, "page_sizes.json")
    r = g["router_params"]
    assert r["H"] * r["E"] == 1048576  # "about 1M"
    d = g["dispatch_volume"]
    assert d["T"] * d["k"] == d["page_accesses"]
    assert d["H"] * d["bytes_per_elem"] == 8192  # 8 KB per access
    assert d["T"] * d["k"] * d["H"] * d["bytes_per_elem"] == 256 * 1024 * 1024  # "about 256MB"
    fine = wlm.WORKLOADS["fine"]
    assert (fine.T, fine.k, fine.H, fine.E) == (d["T"], d["k"], d["H"], r["E"])
    mix = wlm.WORKLOADS["mixtral"]
    assert (mix.E, mix.k) == (g["mixtral_active"]["E"], g["mixtral_active"]["k"])


# ---------------------------------------------------------------- group-limited routing


def test_grouped_topk_hand_worked(golden_dir):
    for c in _load(golden_dir, "grouped_routing.json")["cases"]:
        l = np.asarray([c["logits"]], dtype=np.float32)
        got = orc.select_topk_grouped(l, c["k"], c["n_group"], c["topk_group"])
        assert got[0].tolist() == c["expected"], c["note"]
        assert orc.select_topk(l, c["k"])[0].tolist() == c["plain"], c["note"]


def test_grouped_topk_reduces_to_plain():
    rng = np.random.default_rng(5)
    l = np.round(rng.standard_normal((200, 32)) * 2).astype(np.float32) / 2  # many ties
    for k in (1, 3, 8):
        plain = orc.select_topk(l, k)
        assert np.array_equal(orc.select_topk_grouped(l, k, 1, 1), plain)
        assert np.array_equal(orc.select_topk_grouped(l, k, 4, 4), plain)
        assert np.array_equal(orc.select_topk_grouped(l, k, 32, 32), plain)


def test_grouped_topk_order_invariants():
    """Kept groups beat every other group under (score desc, index asc); the selection beats
    every other candidate of the kept groups under (logit desc, index asc)."""
    rng = np.random.default_rng(6)
    E, G, g, k = 64, 8, 3, 6
    gs = E // G
    l = np.round(rng.standard_normal((300, E)) * 3).astype(np.float32) / 4
    idx = orc.select_topk_grouped(l, k, G, g)
    for t in range(l.shape[0]):
        row = l[t]
        # group scores by brute force: best pair sum over distinct members
        sc = []
        for gi in range(G):
            m = row[gi * gs:(gi + 1) * gs]
            sc.append(max(np.float32(m[a]) + np.float32(m[b])
                          for a in range(gs) for b in range(gs) if a != b))
        sel = [int(e) for e in idx[t]]
        kept = {e // gs for e in sel}
        assert len(kept) <= g
        # the kept set is exactly the g best groups
        best = sorted(range(G), key=lambda gi: (-sc[gi], gi))[:g]
        assert kept <= set(best)
        cand = [e for e in range(E) if e // gs in best]
        for s in sel:
            for c in cand:
                if c not in sel:
                    assert row[s] > row[c] or (row[s] == row[c] and s < c)
        # listed by (logit desc, index asc)
        for a, b in zip(sel, sel[1:]):
            assert row[a] > row[b] or (row[a] == row[b] and a < b)


def test_group_scores_single_member_groups_are_the_logits():
    l = np.asarray([[0.5, -1.0, 2.0, 0.0]], dtype=np.float32)
    assert np.array_equal(orc.group_scores(l, 4), l)


# ---------------------------------------------------------------- shared expert + bias in the combine


def test_combine_shared_and_bias_hand_worked():
    # T=2, k=2, H=2; token 0 keeps both slots, token 1 is fully dropped
    y = np.asarray([[1.0, 2.0], [3.0, -1.0]])
    slot_of = np.asarray([0, 1, -1, -1])
    w = np.asarray([[0.75, 0.25], [0.5, 0.5]])
    shared = np.asarray([[4.0, 8.0], [-2.0, 6.0]])
    bias = np.asarray([0.5, -0.5])
    out = orc.combine(y, slot_of, w, shared=shared, shared_factor=0.5, out_bias=bias)
    # token 0: 0.75*[1,2] + 0.25*[3,-1] = [1.5, 1.25]; + 0.5*[4,8] = [3.5, 5.25]; + bias
    # token 1: dropped -> 0.5*[-2,6] + bias = [-0.5, 2.5]
    assert np.array_equal(out, np.asarray([[4.0, 4.75], [-0.5, 2.5]]))


def test_combine_shared_terms_are_additive():
    rng = np.random.default_rng(7)
    T, k, H = 9, 3, 16
    y = rng.standard_normal((T * k, H))
    slot_of = rng.permutation(T * k)
    slot_of[::4] = -1
    w = rng.random((T, k))
    shared = rng.standard_normal((T, H))
    bias = rng.standard_normal(H)
    base = orc.combine(y, slot_of, w)
    assert np.array_equal(orc.combine(y, slot_of, w, shared=shared, shared_factor=0.0), base)
    with_terms = orc.combine(y, slot_of, w, shared=shared, shared_factor=1.5, out_bias=bias)
    assert np.allclose(with_terms - base, 1.5 * shared + bias, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- FP8 (e4m3) weights


def test_e4m3_decode_landmarks():
    d = orc.e4m3_decode(np.arange(256, dtype=np.uint8))
    # format landmarks: zero, smallest subnormal 2^-9, largest subnormal 7*2^-9, smallest
    # normal 2^-6, one, largest finite 448; NaN only at S.1111.111
    assert d[0x00] == 0.0 and d[0x01] == 2.0 ** -9 and d[0x07] == 7 * 2.0 ** -9
    assert d[0x08] == 2.0 ** -6 and d[0x38] == 1.0 and d[0x7E] == 448.0
    assert np.isnan(d[0x7F]) and np.isnan(d[0xFF]) and np.sum(np.isnan(d)) == 2
    assert np.array_equal(d[0x80:0xFF], -d[0x00:0x7F])
    # the 127 non-negative finite codes are strictly increasing
    assert np.all(np.diff(d[:0x7F]) > 0)
    # within a binade the step is 2^(e-7)/8
    for e in range(1, 16):
        codes = [(e << 3) | m for m in range(8) if (e << 3) | m < 0x7F]
        steps = np.diff(d[codes])
        assert np.all(steps == 2.0 ** (e - 7) / 8)


def test_e4m3_roundtrip_and_ties():
    codes = np.asarray([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = orc.e4m3_decode(codes)
    assert np.array_equal(orc.e4m3_encode(vals.astype(np.float32)), codes)
    mags = orc.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = (mags[:-1] + mags[1:]) / 2          # exact in float32 (4 significant bits)
    assert np.array_equal(mids.astype(np.float32).astype(np.float64), mids)
    got = orc.e4m3_encode(mids.astype(np.float32)).astype(np.int64)
    lo = np.arange(126)
    assert np.array_equal(got, np.where(lo % 2 == 0, lo, lo + 1))  # ties to the even code
    assert np.array_equal(orc.e4m3_encode((mids * (1 - 2.0 ** -12)).astype(np.float32)), lo)
    assert np.array_equal(orc.e4m3_encode((mids * (1 + 2.0 ** -12)).astype(np.float32)), lo + 1)
    # saturation
    assert orc.e4m3_encode(np.float32([1e6, -1e6, 480.0, 449.0]))[:4].tolist() == [0x7E, 0xFE, 0x7E, 0x7E]


def test_e4m3_encode_matches_torch_conversion_in_range():
    rng = np.random.default_rng(8)
    v = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.1, 1.0, 30.0)])
    v = np.clip(v, -463.0, 463.0).astype(np.float32)   # torch does not saturate above that
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(orc.e4m3_encode(v), ref)


def test_quantize_weights_fp8_per_channel():
    rng = np.random.default_rng(9)
    E, K, M = 3, 64, 48
    w = (rng.standard_normal((E, K, M)) * rng.uniform(1e-3, 5, size=(1, 1, M))).astype(np.float32)
    w[1, :, 7] = 0.0                                     # an all-zero column
    q, scale = orc.quantize_weights_fp8(w)
    assert q.dtype == np.uint8 and scale.dtype == np.float32 and scale.shape == (E, M)
    assert scale[1, 7] == 1.0 and np.all(q[1, :, 7] == 0)
    deq = orc.dequantize_weights_fp8(q, scale)
    amax = np.abs(w).max(axis=1)
    # each column's largest element lands on +-448 (code 0x7E) and stays within rounding of itself
    for e in range(E):
        for m in range(M):
            if amax[e, m] > 0:
                assert np.abs(orc.e4m3_decode(q[e, :, m])).max() == 448.0
    # error bound: half an e4m3 step at the element's magnitude (relative 2^-4 for normals,
    # 2^-10 * scale below the normal range), plus the float32 division's rounding
    a = np.abs(w.astype(np.float64))
    bound = np.maximum(a * 2.0 ** -4, 2.0 ** -10 * scale[:, None, :]) * (1 + 1e-6)
    assert np.all(np.abs(deq - w) <= bound)


# ---------------------------------------------------------------- grouped routing through the whole layer


def _grouped_fixture(golden_dir):
    g = _load(golden_dir, "layer_grouped.json")
    arr = {k_: np.asarray(g[k_], dtype=np.float64)
           for k_ in ("x", "w_router", "w_gate", "w_up", "w_down", "shared", "out_bias")}
    return g, arr


def _grouped_layer(g, arr, n_group=None, topk_group=None):
    return orc.layer_forward(arr["x"], arr["w_router"], arr["w_gate"], arr["w_up"], arr["w_down"],
                             g["k"], g["capacity_factor"],
                             n_group=g["n_group"] if n_group is None else n_group,
                             topk_group=g["topk_group"] if topk_group is None else topk_group,
                             shared=arr["shared"], shared_factor=g["shared_factor"],
                             out_bias=arr["out_bias"])


def _matches(res, g):
    return (res["topk_idx"].tolist() == g["topk_idx"]
            and np.allclose(res["topk_w"], np.asarray(g["topk_w"]), rtol=0, atol=g["tolerance"])
            and np.allclose(res["out"], np.asarray(g["out"]), rtol=0, atol=g["tolerance"]))


def test_route_grouped_hand_worked(golden_dir):
    g, arr = _grouped_fixture(golden_dir)
    logits, idx, w = orc.route_grouped(arr["x"], arr["w_router"], g["k"], g["n_group"],
                                       g["topk_group"])
    assert np.array_equal(logits, arr["x"].astype(np.float32))
    assert idx.tolist() == g["topk_idx"]
    np.testing.assert_allclose(w, np.asarray(g["topk_w"]), rtol=0, atol=g["tolerance"])
    # the fixture's tokens all select differently without the group step
    _, plain, _ = orc.route(arr["x"], arr["w_router"], g["k"])
    assert plain.tolist() == g["plain_topk_idx"]
    assert all(a != b for a, b in zip(plain.tolist(), g["topk_idx"]))


def test_layer_grouped_hand_worked(golden_dir):
    g, arr = _grouped_fixture(golden_dir)
    res = _grouped_layer(g, arr)
    assert res["C"] == g["C"]
    assert res["topk_idx"].tolist() == g["topk_idx"]
    np.testing.assert_allclose(res["topk_w"], np.asarray(g["topk_w"]), rtol=0, atol=g["tolerance"])
    assert res["counts"].tolist() == g["counts"]
    assert res["slot_of"].tolist() == g["slot_of"]
    np.testing.assert_allclose(res["out"], np.asarray(g["out"]), rtol=0, atol=g["tolerance"])


def test_layer_grouped_fixture_rejects_planted_mistakes(golden_dir, monkeypatch):
    """The fixture fails for the plausible mistakes in the grouped layer path."""
    g, arr = _grouped_fixture(golden_dir)
    assert _matches(_grouped_layer(g, arr), g)
    # n_group and topk_group swapped: one group means plain routing
    assert not _matches(_grouped_layer(g, arr, n_group=g["topk_group"], topk_group=g["n_group"]), g)
    with pytest.raises(ValueError):
        orc.select_topk_grouped(arr["x"], g["k"], g["topk_group"], g["n_group"])

    real = orc.route_grouped

    def weights_from_plain_selection(x, w_router, k, n_group, topk_group, logit_bias=None,
                                     logits=None):
        lg, idx, _ = real(x, w_router, k, n_group, topk_group, logit_bias=logit_bias,
                          logits=logits)
        return lg, idx, orc.route_weights(lg, orc.select_topk(lg, k))

    monkeypatch.setattr(orc, "route_grouped", weights_from_plain_selection)
    assert not _matches(_grouped_layer(g, arr), g)

    def groups_scored_by_top1(x, w_router, k, n_group, topk_group, logit_bias=None, logits=None):
        lg = orc.router_logits(x, w_router, logit_bias) if logits is None else logits
        l32 = np.asarray(lg, dtype=np.float32)
        T, E = l32.shape
        gs = E // n_group
        sc = l32.reshape(T, n_group, gs).max(axis=2)
        keep = np.argsort(-sc, axis=1, kind="stable")[:, :topk_group]
        masked = np.full_like(l32, -np.inf)
        for t in range(T):
            for grp in keep[t]:
                masked[t, grp * gs:(grp + 1) * gs] = l32[t, grp * gs:(grp + 1) * gs]
        idx = orc.select_topk(masked, k)
        return l32, idx, orc.route_weights(l32, idx)

    monkeypatch.setattr(orc, "route_grouped", groups_scored_by_top1)
    assert not _matches(_grouped_layer(g, arr), g)


# ---------------------------------------------------------------- FP8 weights and activations (W8A8)


def test_bf16_round_matches_torch_including_ties():
    rng = np.random.default_rng(21)
    v = np.concatenate([rng.standard_normal(50000) * s for s in (1e-30, 1e-3, 1.0, 1e20)])
    v = v.astype(np.float32)
    # exact ties: float32 patterns whose low 16 bits are 0x8000, both parities of bit 16
    ties = (rng.integers(0x00800000, 0x7f000000, size=4000, dtype=np.uint32) & ~np.uint32(0xffff)) \
        | np.uint32(0x8000)
    v = np.concatenate([v, ties.view(np.float32), -ties.view(np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy()
    assert np.array_equal(orc.bf16_round(v), ref)
    # float64 input: rounded to float32 first, then to bfloat16
    d = rng.standard_normal(20000) * 3.0
    assert np.array_equal(orc.bf16_round(d),
                          torch.from_numpy(d.astype(np.float32)).to(torch.bfloat16).float().numpy())


def test_quantize_rows_fp8_matches_torch_and_landmarks():
    rng = np.random.default_rng(22)
    a = (rng.standard_normal((40, 96)) * rng.uniform(1e-3, 50, size=(40, 1))).astype(np.float32)
    a[5] = 0.0
    q, sc = orc.quantize_rows_fp8(a)
    assert q.shape == a.shape and q.dtype == np.uint8 and sc.shape == (40,)
    t = torch.from_numpy(a)
    sc_t = t.abs().amax(dim=1) / 448.0
    sc_t = torch.where(sc_t > 0, sc_t, torch.ones_like(sc_t))
    q_t = (t / sc_t[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(sc, sc_t.numpy()) and np.array_equal(q, q_t)
    assert sc[5] == 1.0 and np.all(q[5] == 0)
    dec = orc.e4m3_decode(q)
    assert np.all(np.abs(np.delete(dec, 5, axis=0)).max(axis=1) == 448.0)
    # a row already on the e4m3 grid with max 448 * 2^-8 is reproduced exactly
    grid = orc.e4m3_decode(np.arange(0, 127, 3, dtype=np.uint8)) * 2.0 ** -8
    row = np.concatenate([grid, -grid[::-1], [448.0 * 2.0 ** -8]]).astype(np.float32)[None]
    q2, s2 = orc.quantize_rows_fp8(row)
    assert s2[0] == 2.0 ** -8 and np.array_equal(orc.e4m3_decode(q2) * s2[0], row.astype(np.float64))
    # no rows
    q0, s0 = orc.quantize_rows_fp8(np.zeros((0, 8), dtype=np.float32))
    assert q0.shape == (0, 8) and s0.shape == (0,)


def _w8a8_expert_torch(x, wg, wu, wd):
    """The W8A8 expert written independently with torch ops: per-row e4m3 of the activations by
    torch's float8 conversion, float64 matmuls, torch's silu, torch's bfloat16 rounding of h."""
    def q_rows(a):
        a = torch.as_tensor(a, dtype=torch.float32)
        sc = a.abs().amax(dim=1) / 448.0
        sc = torch.where(sc > 0, sc, torch.ones_like(sc))
        return (a / sc[:, None]).to(torch.float8_e4m3fn).to(torch.float64) * sc.double()[:, None]

    def deq(w):
        q, sc = w
        return (torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64)
                * torch.from_numpy(sc).double()[None, :])

    xd = q_rows(x)
    g, u = xd @ deq(wg), xd @ deq(wu)
    h = (torch.nn.functional.silu(g) * u).float().to(torch.bfloat16).float()
    return (q_rows(h) @ deq(wd)).numpy()


def test_swiglu_expert_w8a8_matches_an_independent_torch_composition(monkeypatch):
    rng = np.random.default_rng(23)
    H, I, n = 64, 48, 9
    x = rng.standard_normal((n, H)).astype(np.float32)
    ws = [orc.quantize_weights_fp8((rng.standard_normal((1, H, I)) / 8).astype(np.float32)),
          orc.quantize_weights_fp8((rng.standard_normal((1, H, I)) / 8).astype(np.float32)),
          orc.quantize_weights_fp8((rng.standard_normal((1, I, H)) / 7).astype(np.float32))]
    wg, wu, wd = [(q[0], s[0]) for q, s in ws]
    got = orc.swiglu_expert_w8a8(x, wg, wu, wd)
    ref = _w8a8_expert_torch(x, wg, wu, wd)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # planted mistakes fail: h not rounded to bf16 before its quantisation, or the activation
    # scale of x dropped
    real_round, real_rows = orc.bf16_round, orc.quantize_rows_fp8
    monkeypatch.setattr(orc, "bf16_round", lambda v: np.asarray(v, dtype=np.float64))
    bad = orc.swiglu_expert_w8a8(x, wg, wu, wd)
    assert not np.allclose(bad, ref, rtol=1e-9, atol=1e-9 * np.abs(ref).max())
    monkeypatch.setattr(orc, "bf16_round", real_round)

    def rows_without_scale(a):
        q, sc = real_rows(a)
        return q, np.ones_like(sc)
    monkeypatch.setattr(orc, "quantize_rows_fp8", rows_without_scale)
    bad = orc.swiglu_expert_w8a8(x, wg, wu, wd)
    assert not np.allclose(bad, ref, rtol=1e-3, atol=1e-3 * np.abs(ref).max())


def test_layer_w8a8_close_to_the_exact_layer():
    """The quantised layer stays within the e4m3 error scale of the exact float64 layer on the
    same routing (each quantised operand is within 2^-4 relative; the output error is a few
    percent of the output's scale)."""
    wl = wlm.Workload("q", 0, 24, 64, 4, 2, 32, "f32", 0.0)
    a = {k_: (v.numpy() if v is not None else None) for k_, v in wlm.make_inputs(wl).items()}
    qs = [orc.quantize_weights_fp8(a[n]) for n in ("w_gate", "w_up", "w_down")]
    pairs = [[(q[e], s[e]) for e in range(wl.E)] for q, s in qs]
    exact = orc.layer_forward(a["x"], a["w_router"], a["w_gate"], a["w_up"], a["w_down"], wl.k, 0.0)
    quant = orc.layer_forward(a["x"], a["w_router"], pairs[0], pairs[1], pairs[2], wl.k, 0.0,
                              expert_fn=orc.swiglu_expert_w8a8)
    assert np.array_equal(quant["topk_idx"], exact["topk_idx"])
    err = np.abs(quant["out"] - exact["out"]).max() / np.abs(exact["out"]).max()
    assert 1e-4 < err < 0.1


def _torch_swiglu(xr, wg, wu, wd):
    """Independent float64 composition with torch's own SiLU: (silu(x Wg) * (x Wu)) Wd."""
    xt = torch.as_tensor(xr, dtype=torch.float64)
    g = xt @ torch.as_tensor(wg, dtype=torch.float64)
    u = xt @ torch.as_tensor(wu, dtype=torch.float64)
    return (torch.nn.functional.silu(g) * u) @ torch.as_tensor(wd, dtype=torch.float64)


def test_grouped_ffn_slots_pinned_per_slot():
    """grouped_ffn_slots: slot s of expert e holds expert e's SwiGLU FFN of token
    sorted_ids[s] // k ([P1] step 4), checked slot by slot against a torch composition, on a
    grouping with drops (so slots and assignments are not the identity). Planted mistakes fail:
    gate and up exchanged, the expert of the neighbouring range, the assignment index taken as
    the token."""
    g = np.random.default_rng(7)
    T, H, E, k, I = 11, 6, 4, 2, 5
    x = g.standard_normal((T, H))
    wg, wu, wd = (g.standard_normal((E, H, I)), g.standard_normal((E, H, I)),
                  g.standard_normal((E, I, H)))
    idx = np.stack([g.choice(E, k, replace=False) for _ in range(T)])
    al = orc.align(idx, E, 4)  # capacity 4 of 5.5 mean: drops
    assert al["drop_mask"].sum() > 0
    y = orc.grouped_ffn_slots(x, al["sorted_ids"], al["offsets"], k, wg, wu, wd)
    offs = al["offsets"]

    def expected(s, e, tok_of=lambda a: a // k, gate=wg, up=wu):
        a = int(al["sorted_ids"][s])
        return _torch_swiglu(x[tok_of(a)][None], gate[e], up[e], wd[e])[0].numpy()

    for e in range(E):
        for s in range(int(offs[e]), int(offs[e + 1])):
            np.testing.assert_allclose(y[s], expected(s, e), rtol=1e-12, atol=1e-12)
    # planted mistakes, each caught on at least one slot
    def differs(fn):
        return any(not np.allclose(y[s], fn(s, e), rtol=1e-9, atol=1e-9)
                   for e in range(E) for s in range(int(offs[e]), int(offs[e + 1])))
    assert differs(lambda s, e: expected(s, e, gate=wu, up=wg))
    assert differs(lambda s, e: expected(s, (e + 1) % E))
    assert differs(lambda s, e: expected(s, e, tok_of=lambda a: a % T))
