"""CUDA path vs the CPU oracle, through the C ABI (libmoe.so), on one B200.

Every stage is tested on oracle-produced inputs (bit-exact for integer outputs, tolerance for
floating point), then the whole layer is compared, at small sizes in full and at the workload
sizes on sampled tokens/slots.
"""
import numpy as np
import pytest
import torch

from expert_dispatch_gate_b200 import _lib as L
from expert_dispatch_gate_b200 import layer as M
from expert_dispatch_gate_b200 import workloads as W
from oracle import moe_oracle as orc
from tests.parity import (TOL_LOGITS, TOL_OUT, TOL_W, ExpertWeights, assert_close_rel,
                          decided_tokens_grouped,
                          check_topk_valid, decided_tokens, inputs_np, np32, npi, to_dev)

pytestmark = pytest.mark.gpu

# Parity sizes: several tiles and ragged tails, oracle-friendly.
SMALL = {
    "tiny": W.WORKLOADS["tiny"],
    "e8_two_token_blocks": W.Workload("e8", 10, 1500, 128, 8, 2, 256, "bf16", 1.25),
    "e32_ragged": W.Workload("e32", 11, 517, 256, 32, 4, 384, "bf16", 1.25),
    "e64_zipf": W.Workload("e64z", 12, 300, 256, 64, 6, 256, "bf16", 1.25, zipf_s=1.2),
    "e256_k8": W.Workload("e256", 13, 200, 128, 256, 8, 128, "bf16", 1.25),
    "e16_nocap": W.Workload("e16n", 14, 97, 256, 16, 4, 256, "bf16", 0.0),
    "dense_e1": W.Workload("e1", 15, 130, 128, 1, 1, 128, "bf16", 1.25),
    "e64_k16_f32": W.Workload("e64f", 16, 77, 64, 64, 16, 96, "f32", 1.0),
    # E = 96: the router's second 64-expert chunk is half zero-filled (N = 96, two
    # accumulators); I = 640 leaves the last GEMM1 pair tile half outside the weight; H = 384
    # runs GEMM2 with one feature block per tile
    "e96_partial_tiles": W.Workload("e96", 19, 333, 384, 96, 4, 640, "bf16", 1.25),
    # T = 50, H = 1024: one token tile, the router's K split into 4 ranges
    "e128_router_t50": W.Workload("e128", 20, 50, 1024, 128, 6, 256, "bf16", 1.25),
    # T = 90: one token tile of the tensor-core router, its K split into 4 ranges
    "e128_router_ksplit": W.Workload("e128k", 21, 90, 1024, 128, 6, 256, "bf16", 1.25),
    # H = 192 and I = 320, multiples of 64 only: partial last feature blocks in both GEMMs (and
    # a partial last K stage of the e4m3 operands)
    "h192_i320": W.Workload("h192", 22, 300, 192, 16, 4, 320, "bf16", 1.25),
}


@pytest.fixture(scope="session", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    L.lib()  # fails loudly when libmoe.so is missing


_cache = {}


def small_inputs(name):
    if name not in _cache:
        wl = SMALL[name]
        cpu = W.make_inputs(wl, "cpu")
        dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
        _cache[name] = (wl, cpu, dev)
    return _cache[name]


def oracle_routing(wl, cpu):
    host = inputs_np(cpu)
    logits = orc.router_logits(host["x"], host["w_router"], host["logit_bias"])
    idx = orc.select_topk(logits, wl.k)
    w = orc.route_weights(logits, idx)
    C = orc.capacity(wl.T, wl.k, wl.E, wl.capacity_factor)
    return logits, idx, w, C, orc.align(idx, wl.E, C)


# ----------------------------------------------------------------- route (selection only)

@pytest.mark.parametrize("T,E,k,ties", [
    (1, 8, 2, False), (300, 8, 1, True), (300, 64, 6, True), (1000, 256, 8, True),
    (257, 256, 16, False), (33, 16, 16, True), (4096, 256, 8, False), (129, 128, 4, True),
    # experts not a multiple of the per-lane run (scalar loads, lanes past E)
    (50, 37, 3, True), (64, 5, 2, True), (100, 200, 8, True), (77, 104, 7, True),
    # large batches: 2 lanes per token at E = 256, one thread per token at E = 64
    (40000, 256, 8, True), (100000, 64, 6, True),
])
def test_route_from_logits_bitexact(T, E, k, ties):
    logits = W.random_logits(T, E, seed=T * 7 + E + k, ties=ties)
    idx_g, w_g = M.route_from_logits(logits.cuda(), k)
    torch.cuda.synchronize()
    l32 = logits.numpy()
    idx_o = orc.select_topk(l32, k)
    w_o = orc.route_weights(l32, idx_o)
    assert np.array_equal(npi(idx_g), idx_o)
    np.testing.assert_allclose(npi(w_g), w_o, atol=TOL_W, rtol=0)
    np.testing.assert_allclose(npi(w_g).astype(np.float64).sum(1), 1.0, atol=k * 2.0 ** -23 * 2)


@pytest.mark.parametrize("T,E,k", [
    (3000, 64, 6), (1000, 64, 8), (513, 32, 2), (700, 16, 16), (300, 60, 5), (257, 64, 1),
    (100000, 64, 6),                    # one lane per token
    (4096, 256, 8), (40000, 256, 8),   # 16 and 2 lanes per token
    (77, 256, 16), (129, 200, 7), (3, 62, 4),
])
def test_lane_and_warp_selection_agree_bitwise(T, E, k):
    """Plain top-k runs G lanes per token (topk_lanes_kernel, G from 1 to 16 by T and E); the
    group-limited form with every group kept (no expert excluded) runs the warp-per-token
    kernel on the same rule. Indices and weights (the renormalising sum is taken in the same
    pairwise order) agree bit for bit."""
    logits = W.random_logits(T, E, seed=5 * T + E + k, ties=True).cuda()
    idx_t, w_t = M.route_from_logits(logits, k)
    idx_w, w_w = M.route_from_logits(logits, k, n_group=2, topk_group=2)
    torch.cuda.synchronize()
    assert torch.equal(idx_t, idx_w)
    assert torch.equal(w_t.view(torch.int32), w_w.view(torch.int32))


# ----------------------------------------------------------------- route (gate GEMM + selection)

# Router-only shapes for the tensor-core gate GEMM: CTA pairs (E % 128 == 0) over several
# 256-token tiles with a ragged tail, a pair whose second CTA has one token, the longest K split
# (T = 2, H = 4096), and a single-CTA shape with E = 192.
ROUTER = {
    "pairs_ragged": W.Workload("r1", 21, 1000, 512, 256, 8, 128, "bf16", 1.25),
    "pairs_e128_k6": W.Workload("r2", 22, 257, 2048, 128, 6, 128, "bf16", 1.25),
    "pairs_short_peer": W.Workload("r3", 23, 129, 256, 256, 8, 128, "bf16", 1.25),
    "pairs_t2_ksplit16": W.Workload("r4", 24, 2, 4096, 256, 8, 128, "bf16", 1.25),
    "single_e192": W.Workload("r5", 25, 513, 4096, 192, 8, 128, "bf16", 1.25),
    # the K split at 4 and 16 ranges with one or two token tiles
    "tc_t100_ksplit4": W.Workload("r6", 26, 100, 1024, 128, 6, 128, "bf16", 1.25),
    "tc_t65_ksplit16": W.Workload("r7", 27, 65, 4096, 256, 8, 128, "bf16", 1.25),
    # decode-sized batches: one token, a few, and E not a multiple of 128 (single CTAs)
    "tc_t1": W.Workload("r8", 28, 1, 4096, 256, 8, 128, "bf16", 0.0),
    "tc_t3_e128": W.Workload("r9", 29, 3, 2048, 128, 4, 128, "bf16", 0.0),
    "tc_t16_e96": W.Workload("r10", 30, 16, 1024, 96, 6, 128, "bf16", 1.25),
    "tc_t64_e64_zipf": W.Workload("r11", 31, 64, 2048, 64, 6, 128, "bf16", 1.25, zipf_s=1.2),
    # the CUDA-core router (E < 64 or f32) over several 256-row slabs of Wr, the last one
    # partial, in bf16 and f32, and a single token
    "simt_e8_slabs": W.Workload("r12", 32, 300, 1088, 8, 2, 128, "bf16", 1.25),
    "simt_e64_f32_slabs": W.Workload("r13", 33, 129, 520, 64, 6, 128, "f32", 1.25),
    "simt_e16_t1": W.Workload("r14", 34, 1, 4096, 16, 4, 128, "bf16", 0.0),
    # E = 64 with one K range: the persistent gate GEMM with the top-k in its epilogue, over
    # about three tiles per CTA (both TMEM buffers reused) with a ragged last tile
    "fused_e64_t60000": W.Workload("r15", 35, 60000, 256, 64, 6, 128, "bf16", 1.25),
    "fused_e64_h2048_k8": W.Workload("r16", 36, 20000, 2048, 64, 8, 128, "bf16", 1.25),
    # short batches: every K range's partials summed in one batch of loads
    "short_t5_e64": W.Workload("r19", 40, 5, 2048, 64, 6, 128, "bf16", 0.0),
    "short_t16_e256_pairs": W.Workload("r20", 41, 16, 4096, 256, 8, 128, "bf16", 1.25),
    # the same on CTA pairs: E = 256 over about three 256-token tiles per pair, E = 128
    "fused_pairs_e256_t60000": W.Workload("r17", 38, 60000, 256, 256, 8, 128, "bf16", 1.25),
    "fused_pairs_e128": W.Workload("r18", 39, 40000, 512, 128, 6, 128, "bf16", 1.25),
}


@pytest.mark.parametrize("name", list(SMALL) + list(ROUTER))
def test_router(name):
    if name in ROUTER:
        wl = ROUTER[name]
        cpu = W.make_inputs(wl, "cpu", weights=False)
        dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    else:
        wl, cpu, dev = small_inputs(name)
    idx_g, w_g, logits_g = M.route(dev["x"], dev["w_router"], wl.k, dev["logit_bias"])
    torch.cuda.synchronize()
    L_o, idx_o, w_o, _, _ = oracle_routing(wl, cpu)
    L_g = np32(logits_g)
    tol = TOL_LOGITS[wl.dtype] * max(1.0, float(np.abs(L_o).max()))
    delta = float(np.abs(L_g - L_o).max())
    assert delta <= tol, (delta, tol)
    dec = decided_tokens(L_o, wl.k, delta)
    idx_g = npi(idx_g)
    assert np.array_equal(idx_g[dec], idx_o[dec])
    check_topk_valid(L_o, idx_g, wl.k, delta, np.nonzero(~dec)[0])
    np.testing.assert_allclose(npi(w_g)[dec], w_o[dec], atol=TOL_W + wl.k * delta, rtol=0)
    # the selection the kernel made is exactly the rule applied to the logits it exported
    # (checked by the selection-only kernel on the same values, bit for bit, weights included)
    idx_s, w_s = M.route_from_logits(logits_g, wl.k)
    assert torch.equal(idx_s.cpu(), torch.as_tensor(idx_g))
    assert torch.equal(w_s.view(torch.int32), w_g.view(torch.int32))


# ----------------------------------------------------------------- align

@pytest.mark.parametrize("T,E,k,cf,mode", [
    (1, 256, 8, 1.25, "uniform"), (64, 8, 2, 0.0, "uniform"), (5000, 8, 2, 1.25, "zipf"),
    (4096, 256, 8, 1.25, "uniform"), (4096, 256, 8, 1.25, "zipf"), (3000, 64, 6, 1.25, "zipf"),
    (2500, 16, 4, 1.0, "one"), (777, 32, 3, 0.5, "uniform"), (2049, 1, 1, 1.25, "one"),
    (20000, 64, 6, 1.25, "zipf"),
    # the grouping's launch forms and their edges: one 256-thread block up to 2048
    # assignments, one cluster of 8 CTAs up to 65536, one cooperative grid beyond (86 CTAs
    # just above 65536, one per SM from about 300000)
    (256, 16, 8, 1.25, "zipf"), (1024, 128, 2, 1.0, "uniform"), (1025, 128, 2, 1.0, "uniform"),
    (4097, 256, 8, 1.25, "zipf"), (8192, 256, 8, 1.25, "zipf"), (5462, 96, 6, 0.75, "uniform"),
    (8193, 256, 8, 1.25, "uniform"), (10923, 64, 6, 1.25, "zipf"),
    (32768, 256, 8, 1.25, "zipf"), (40000, 64, 8, 1.25, "zipf"), (43691, 64, 6, 0.0, "uniform"),
    (49152, 256, 8, 1.25, "zipf"), (131072, 64, 6, 1.25, "zipf"),
])
def test_align_bitexact(T, E, k, cf, mode):
    idx = W.random_topk_idx(T, E, k, seed=T + 31 * E + k, mode=mode)
    res = M.align(idx.cuda(), E, cf)
    torch.cuda.synchronize()
    C = orc.capacity(T, k, E, cf)
    assert res["C"] == C
    al = orc.align(idx.numpy(), E, C)
    for key in ("counts", "offsets", "sorted_ids", "slot_of", "drop_mask"):
        assert np.array_equal(npi(res[key]), al[key]), key
    assert res["ws"].check() == L.MOE_OK


def test_align_chunked_form_beyond_the_grid_properties():
    """10 M assignments: more than the cooperative grid holds (148 SMs x 1024 threads x 64
    rounds), so the three chunked kernels run. Checked by the grouping's defining properties
    (numpy, any size): counts = min(histogram, C), offsets their prefix, each expert's slots the
    first C of its assignments in assignment order, everything else dropped."""
    T, E, k, cf = 1250000, 256, 8, 1.25
    idx = W.random_topk_idx(T, E, k, seed=77, mode="zipf")
    res = M.align(idx.cuda(), E, cf)
    torch.cuda.synchronize()
    C = orc.capacity(T, k, E, cf)
    flat = idx.numpy().reshape(-1).astype(np.int64)
    A = flat.size
    counts = np.minimum(np.bincount(flat, minlength=E), C)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    order = np.argsort(flat, kind="stable")          # expert-major, assignment order inside
    start = np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))])[flat[order]]
    keep = (np.arange(A) - start) < C
    sorted_ids = np.full(A, -1, np.int64)
    sorted_ids[:offsets[-1]] = order[keep]
    slot_of = np.full(A, -1, np.int64)
    slot_of[order[keep]] = np.arange(offsets[-1])
    assert np.array_equal(npi(res["counts"]), counts)
    assert np.array_equal(npi(res["offsets"]), offsets)
    assert np.array_equal(npi(res["sorted_ids"]), sorted_ids)
    assert np.array_equal(npi(res["slot_of"]), slot_of)
    assert np.array_equal(npi(res["drop_mask"]), (slot_of < 0).astype(np.uint8))
    assert res["ws"].check() == L.MOE_OK


def test_align_every_expert_exactly_at_capacity():
    # T = 64, E = 8, k = 1, cf = 1: C = 8 and each expert gets exactly 8 tokens: no drops
    idx = torch.arange(64, dtype=torch.int32).remainder(8).reshape(64, 1)
    res = M.align(idx.cuda(), 8, 1.0)
    al = orc.align(idx.numpy(), 8, 8)
    assert npi(res["drop_mask"]).sum() == 0
    for key in ("counts", "offsets", "sorted_ids", "slot_of", "drop_mask"):
        assert np.array_equal(npi(res[key]), al[key]), key


@pytest.mark.parametrize("T", [100, 3000, 140000])  # each launch form of the grouping
def test_align_flags_out_of_range_expert_ids(T):
    idx = W.random_topk_idx(T, 16, 2, seed=3)
    idx[7, 1] = 16
    idx[50, 0] = -3
    idx[T - 1, 1] = 1 << 20
    res = M.align(idx.cuda(), 16, 0.0)
    with pytest.raises(L.MoeError) as ei:
        res["ws"].check()
    assert ei.value.status == L.MOE_ERR_DEVICE
    drop = npi(res["drop_mask"])
    assert drop[7 * 2 + 1] == 1 and drop[50 * 2] == 1 and drop[2 * T - 1] == 1
    slot_of = npi(res["slot_of"])
    assert slot_of[7 * 2 + 1] == -1 and slot_of[50 * 2] == -1 and slot_of[2 * T - 1] == -1
    # every valid assignment is kept (no capacity limit) and grouped by the oracle's rule
    valid = idx.numpy().copy()
    bad = (valid < 0) | (valid >= 16)
    assert int(npi(res["counts"]).sum()) == int((~bad).sum())
    assert res["ws"].check() == L.MOE_OK  # the error word was cleared


# ----------------------------------------------------------------- grouped FFN

def _ffn_check(wl, x_dev, weights_dev, al, slots, x_host=None):
    y = M.grouped_ffn(x_dev, to_dev(al["sorted_ids"]), to_dev(al["offsets"]), weights_dev[0],
                      weights_dev[1], weights_dev[2], wl.k, wl.capacity_factor)
    torch.cuda.synchronize()
    xh = np32(x_dev) if x_host is None else x_host
    ref = orc.grouped_ffn_slots(xh, al["sorted_ids"], al["offsets"], wl.k,
                                ExpertWeights(weights_dev[0]), ExpertWeights(weights_dev[1]),
                                ExpertWeights(weights_dev[2]), slots=slots)
    got = np32(y[torch.as_tensor(sorted(ref), dtype=torch.long, device=y.device)])
    want = np.stack([ref[s] for s in sorted(ref)])
    return assert_close_rel(got, want, TOL_OUT[wl.dtype], "expert outputs")


@pytest.mark.parametrize("name", list(SMALL))
def test_grouped_ffn(name):
    wl, cpu, dev = small_inputs(name)
    _, _, _, _, al = oracle_routing(wl, cpu)
    kept = int(al["offsets"][-1])
    _ffn_check(wl, dev["x"], (dev["w_gate"], dev["w_up"], dev["w_down"]), al, list(range(kept)))


# ----------------------------------------------------------------- combine

@pytest.mark.parametrize("name", list(SMALL))
def test_combine(name):
    wl, cpu, dev = small_inputs(name)
    _, _, w_o, _, al = oracle_routing(wl, cpu)
    y = W.make_y_slots(wl, "cpu")
    w32 = w_o.astype(np.float32)
    out = M.combine(y.cuda(), to_dev(al["slot_of"]), to_dev(w32, torch.float32), wl.E)
    torch.cuda.synchronize()
    ref = orc.combine(np32(y), al["slot_of"], w32)
    got = np32(out)
    assert_close_rel(got, ref, TOL_OUT[wl.dtype], "combine")
    # arithmetic bound: fp32 accumulation, one final rounding to the output type
    ulp = 2.0 ** -8 if wl.dtype == "bf16" else 2.0 ** -22
    assert np.all(np.abs(got - ref) <= ulp * np.abs(ref) + 1e-6 * np.abs(ref).max())
    dropped_all = np.all(al["slot_of"].reshape(wl.T, wl.k) < 0, axis=1)
    assert np.all(got[dropped_all] == 0.0)


# ----------------------------------------------------------------- whole layer

def compare_layer(wl, cpu_or_dev, dev, res, sample=None, seed=0, n_group=1, topk_group=1,
                  shared=None, shared_factor=0.0, out_bias=None, weights=None, expert_fn=None):
    """Compare moe_layer_forward's outputs with the oracle (see module docstring of parity).
    With n_group > 1 the routing is group-limited; shared / out_bias (host numpy) add the
    combine's shared-expert and bias terms."""
    host = inputs_np(cpu_or_dev)
    T, E, k = wl.T, wl.E, wl.k
    L_o = orc.router_logits(host["x"], host["w_router"], host["logit_bias"])
    L_g = np32(res["logits"])
    tol = TOL_LOGITS[wl.dtype] * max(1.0, float(np.abs(L_o).max()))
    delta = float(np.abs(L_g - L_o).max())
    assert delta <= tol, (delta, tol)
    if n_group > 1:
        idx_o = orc.select_topk_grouped(L_o, k, n_group, topk_group)
        dec = decided_tokens_grouped(L_o, k, n_group, topk_group, delta)
    else:
        idx_o = orc.select_topk(L_o, k)
        dec = decided_tokens(L_o, k, delta)
    w_o = orc.route_weights(L_o, idx_o)
    idx_g, w_g = npi(res["topk_idx"]), npi(res["topk_w"])
    assert np.array_equal(idx_g[dec], idx_o[dec])
    if n_group == 1:
        check_topk_valid(L_o, idx_g, k, delta, np.nonzero(~dec)[0])
    np.testing.assert_allclose(w_g[dec], w_o[dec], atol=TOL_W + k * delta, rtol=0)
    C = orc.capacity(T, k, E, wl.capacity_factor)
    assert res["C"] == C
    al = orc.align(idx_o, E, C)
    counts_g, drop_g = npi(res["counts"]), npi(res["drop_mask"])
    # the GPU's grouping is valid for the GPU's own routing (invariants, no oracle call)
    raw_g = np.bincount(idx_g.reshape(-1), minlength=E)
    assert np.array_equal(counts_g, np.minimum(raw_g, C))
    flat_g = idx_g.reshape(-1)
    order = np.argsort(flat_g, kind="stable")
    pos = 0
    for e in range(E):
        mine = order[pos:pos + raw_g[e]]
        pos += raw_g[e]
        assert np.all(drop_g[mine[:C]] == 0) and np.all(drop_g[mine[C:]] == 1)
    # A fragile token u can change the ranks (hence drops) only of later assignments to the
    # experts it picks on either side. first_taint[e] = earliest such u for expert e.
    frag = np.nonzero(~dec)[0]
    first_taint = np.full(E, T, dtype=np.int64)
    for u in frag:
        for e in set(idx_o[u].tolist()) | set(idx_g[u].tolist()):
            first_taint[e] = min(first_taint[e], u)
    clean = first_taint == T
    assert np.array_equal(counts_g[clean], al["counts"][clean])
    tok_of = np.repeat(np.arange(T), k)
    flat_o = idx_o.reshape(-1)
    same_rank = tok_of < first_taint[flat_o]
    assert np.array_equal(drop_g[same_rank], al["drop_mask"][same_rank])
    # outputs on decided tokens all of whose experts rank them identically on both sides
    ok_tok = dec & np.all(np.arange(T)[:, None] < first_taint[idx_o], axis=1)
    comparable = np.nonzero(ok_tok)[0].tolist()
    assert len(comparable) >= min(T, 1)
    if sample is not None and len(comparable) > sample:
        rng = np.random.default_rng(seed)
        comparable = sorted(rng.choice(comparable, size=sample, replace=False).tolist())
    if weights is None:
        weights = (ExpertWeights(dev["w_gate"]), ExpertWeights(dev["w_up"]),
                   ExpertWeights(dev["w_down"]))
    ref = orc.layer_forward(host["x"], host["w_router"], weights[0], weights[1], weights[2], k,
                            wl.capacity_factor, logit_bias=host["logit_bias"], tokens=comparable,
                            n_group=n_group, topk_group=topk_group, shared=shared,
                            shared_factor=shared_factor, out_bias=out_bias, expert_fn=expert_fn)
    got = np32(res["out"])[comparable]
    r = assert_close_rel(got, ref["out"], TOL_OUT[wl.dtype], "layer output")
    return {"delta_logits": delta, "fragile": int((~dec).sum()), "compared": len(comparable),
            "rel_err": r}


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_small(name):
    wl, cpu, dev = small_inputs(name)
    res = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                          wl.k, wl.capacity_factor, logit_bias=dev["logit_bias"])
    torch.cuda.synchronize()
    assert res["ws"].check() == L.MOE_OK
    compare_layer(wl, cpu, dev, res)
    # determinism: a second run gives the same bits
    res2 = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                           wl.k, wl.capacity_factor, logit_bias=dev["logit_bias"], ws=res["ws"])
    torch.cuda.synchronize()
    for key in ("out", "topk_idx", "topk_w", "counts", "drop_mask", "logits"):
        assert torch.equal(res[key], res2[key]), key


def test_layer_empty_batch():
    wl = SMALL["e8_two_token_blocks"].with_tokens(0)
    dev = {k: (None if v is None else v.cuda()) for k, v in W.make_inputs(wl, "cpu").items()}
    res = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                          wl.k, wl.capacity_factor)
    torch.cuda.synchronize()
    assert res["out"].shape == (0, wl.H)
    assert int(res["counts"].sum()) == 0


def test_layer_heavy_drops_give_zero_rows():
    # cf = float32(0.05) = 0.0500000007...: C = ceil(5.0000000745) = 6 in exact arithmetic;
    # most assignments are dropped, many tokens fully
    wl = W.Workload("drops", 17, 400, 128, 8, 2, 128, "bf16", 0.05)
    cpu = W.make_inputs(wl, "cpu")
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    res = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                          wl.k, wl.capacity_factor)
    torch.cuda.synchronize()
    assert res["C"] == 6 == orc.capacity(wl.T, wl.k, wl.E, wl.capacity_factor)
    drop = npi(res["drop_mask"]).reshape(wl.T, wl.k)
    assert int(npi(res["counts"]).sum()) <= 6 * wl.E
    out = np32(res["out"])
    assert np.all(out[np.all(drop == 1, axis=1)] == 0.0)
    compare_layer(wl, cpu, dev, res)


# ----------------------------------------------------------------- workload sizes (sampled)

FULL = [("mixtral", None), ("fine", None), ("skewed", None), ("decode", 1), ("decode", 16),
        ("decode", 64), ("decode", 256)]


def _full_inputs(name, T):
    wl = W.WORKLOADS[name] if T is None else W.WORKLOADS[name].with_tokens(T)
    dev = W.make_inputs(wl, "cuda")
    return wl, dev


@pytest.mark.parametrize("name,T", FULL)
def test_layer_workload_sizes(name, T):
    wl, dev = _full_inputs(name, T)
    res = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                          wl.k, wl.capacity_factor, logit_bias=dev["logit_bias"])
    torch.cuda.synchronize()
    assert res["ws"].check() == L.MOE_OK
    info = compare_layer(wl, dev, dev, res, sample=64)
    print(name, T, info)
    # per-stage checks on oracle-made inputs at this size
    host = inputs_np(dev)
    L_o = orc.router_logits(host["x"], host["w_router"], host["logit_bias"])
    idx_s, w_s = M.route_from_logits(torch.as_tensor(L_o).cuda(), wl.k)
    idx_o = orc.select_topk(L_o, wl.k)
    assert np.array_equal(npi(idx_s), idx_o)
    np.testing.assert_allclose(npi(w_s), orc.route_weights(L_o, idx_o), atol=TOL_W, rtol=0)
    C = orc.capacity(wl.T, wl.k, wl.E, wl.capacity_factor)
    al_o = orc.align(idx_o, wl.E, C)
    al_g = M.align(to_dev(idx_o), wl.E, wl.capacity_factor, H=wl.H, I=wl.I)
    for key in ("counts", "offsets", "sorted_ids", "slot_of", "drop_mask"):
        assert np.array_equal(npi(al_g[key]), al_o[key]), key
    # expert outputs for every slot of a few experts: the fullest, a ragged one, the last
    counts = al_o["counts"]
    nz = np.nonzero(counts)[0]
    pick = sorted({int(nz[np.argmax(counts[nz])]), int(nz[len(nz) // 2]), int(nz[-1])})
    slots = [s for e in pick for s in range(al_o["offsets"][e], al_o["offsets"][e + 1])]
    _ffn_check(wl, dev["x"], (dev["w_gate"], dev["w_up"], dev["w_down"]), al_o, slots,
               x_host=host["x"])


# ----------------------------------------------------------------- the bench's schedule, in full

def test_layer_fine_e32_every_token_and_slot():
    """The fine-grained layer's per-expert shapes and load (H = 4096, I = 2048, k = 8, C = 160,
    about 128 tokens per expert) with 32 experts: the expert GEMMs run the same persistent CTA-pair
    schedule over all SMs as the bench (several tiles per CTA pair), and every token's output and
    every kept slot's expert output is compared with the oracle."""
    wl = W.PROFILE_WORKLOADS["fine_e32"]
    dev = W.make_inputs(wl, "cuda")
    res = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                          wl.k, wl.capacity_factor, logit_bias=dev["logit_bias"])
    torch.cuda.synchronize()
    assert res["ws"].check() == L.MOE_OK
    info = compare_layer(wl, dev, dev, res)
    print("fine_e32 layer", info)
    assert info["compared"] >= wl.T // 2
    host = inputs_np(dev)
    L_o = orc.router_logits(host["x"], host["w_router"], host["logit_bias"])
    idx_o = orc.select_topk(L_o, wl.k)
    C = orc.capacity(wl.T, wl.k, wl.E, wl.capacity_factor)
    al_o = orc.align(idx_o, wl.E, C)
    kept = int(al_o["offsets"][-1])
    r = _ffn_check(wl, dev["x"], (dev["w_gate"], dev["w_up"], dev["w_down"]), al_o,
                   list(range(kept)), x_host=host["x"])
    print("fine_e32 expert outputs: %d slots, max rel err %.3e" % (kept, r))


def test_combine_fine_every_token():
    """moe_combine at the fine-grained size (T = 4096, k = 8, H = 4096, C = 160) over every token,
    on the oracle's grouping of seeded logits and seeded expert outputs."""
    wl = W.WORKLOADS["fine"]
    logits = W.random_logits(wl.T, wl.E, seed=99)
    l32 = logits.numpy()
    idx_o = orc.select_topk(l32, wl.k)
    w32 = orc.route_weights(l32, idx_o).astype(np.float32)
    C = orc.capacity(wl.T, wl.k, wl.E, wl.capacity_factor)
    al = orc.align(idx_o, wl.E, C)
    y = W.make_y_slots(wl, "cpu")
    out = M.combine(y.cuda(), to_dev(al["slot_of"]), to_dev(w32, torch.float32), wl.E)
    torch.cuda.synchronize()
    ref = orc.combine(np32(y), al["slot_of"], w32)
    got = np32(out)
    r = assert_close_rel(got, ref, TOL_OUT[wl.dtype], "combine")
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * np.abs(ref).max())
    dropped_all = np.all(al["slot_of"].reshape(wl.T, wl.k) < 0, axis=1)
    assert np.all(got[dropped_all] == 0.0)
    print("combine fine: %d tokens, %d dropped assignments, max rel err %.3e"
          % (wl.T, int(al["drop_mask"].sum()), r))


GRAPH_SHAPES = {
    "e256_k8": None,
    # E = 64 with one K range and 72000 assignments: the fused gate GEMM + top-k and the
    # cooperative one-launch grouping inside the graph
    "fused_router_grid_align": W.Workload("g1", 37, 12000, 256, 64, 6, 128, "bf16", 1.25),
}


@pytest.mark.parametrize("name", list(GRAPH_SHAPES))
def test_layer_call_captured_in_a_cuda_graph_replays_identically(name):
    """The layer call makes no host synchronisation and launches only on its stream, so a serving
    loop can capture it in a CUDA graph: replays give the eager call's results bit for bit, for
    new inputs copied into the captured buffers too."""
    if GRAPH_SHAPES[name] is None:
        wl, cpu, dev = small_inputs(name)
    else:
        wl = GRAPH_SHAPES[name]
        cpu = W.make_inputs(wl, "cpu")
        dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    shape = M.shape_of(wl.T, wl.H, wl.E, wl.k, wl.I, wl.capacity_factor, wl.dtype)
    ws = M.Workspace(shape, "cuda")
    x = dev["x"].clone()
    ref = M.layer_forward(x, dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"], wl.k,
                          wl.capacity_factor, ws=ws)
    torch.cuda.synchronize()
    outs = {key: torch.empty_like(ref[key]) for key in ("out", "topk_idx", "topk_w", "counts",
                                                         "drop_mask", "logits")}
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())

    def call():
        L.moe_layer_forward(shape, x, dev["w_router"], None, dev["w_gate"], dev["w_up"],
                            dev["w_down"], outs["out"], outs["logits"], outs["topk_idx"],
                            outs["topk_w"], outs["counts"], outs["drop_mask"], ws.buf, ws.nbytes,
                            stream)

    with torch.cuda.stream(stream):
        call()  # first call on this stream before capture (tensor-map and attribute setup)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        call()
    for key in outs:
        outs[key].zero_()
    graph.replay()
    torch.cuda.synchronize()
    for key in outs:
        assert torch.equal(outs[key], ref[key]), key
    # new activations through the captured buffer
    x.copy_(torch.flip(dev["x"], dims=[0]))
    ref2 = M.layer_forward(x, dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"], wl.k,
                           wl.capacity_factor)
    graph.replay()
    torch.cuda.synchronize()
    assert ws.check() == L.MOE_OK
    for key in outs:
        assert torch.equal(outs[key], ref2[key]), key
    del graph
