"""Helpers for the GPU-vs-oracle parity tests: input marshalling and comparison rules.

Inputs always flow from the seeded generators (or from the oracle) into the CUDA library,
never from the CUDA library into the oracle. Where floating point decides an integer (the top-k
choice from gate logits that both sides compute in their own summation order), tokens whose
decision is fragile are identified from the oracle's logits and compared for validity only.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as orc

# Layer-output tolerances: max-abs error relative to max |reference|.
TOL_OUT = {"f32": 1e-4, "bf16": 2e-2}
# Gate-logit tolerances (relative to max |reference logit|).
TOL_LOGITS = {"f32": 1e-5, "bf16": 1e-3}
# Routing weights from identical float32 logits: a few float32 ulp of values <= 1.
TOL_W = 1e-6


def np32(t):
    """Tensor -> float32 numpy (exact for bf16 and f32)."""
    return t.detach().float().cpu().numpy()


def npi(t):
    return t.detach().cpu().numpy()


class ExpertWeights:
    """Expert e's matrix as float64 numpy, copied from a (device) [E, a, b] tensor on demand
    (not cached: the oracle visits each expert once, and the workload weights are large)."""

    def __init__(self, w):
        self.w = w

    def __getitem__(self, e):
        return self.w[int(e)].detach().cpu().double().numpy()

    def __len__(self):
        return self.w.shape[0]


class DequantExpertWeights:
    """Expert e's matrix after the oracle's FP8 quantisation (decode(code) * scale, float64),
    computed on demand from the seeded bf16 weights of a (device) [E, K, M] tensor."""

    def __init__(self, w):
        self.w = w

    def __getitem__(self, e):
        w = self.w[int(e)].detach().float().cpu().numpy()[None]
        q, sc = orc.quantize_weights_fp8(w)
        return orc.dequantize_weights_fp8(q, sc)[0]

    def __len__(self):
        return self.w.shape[0]


class W8A8ExpertWeights:
    """Expert e's weights as the oracle's (codes, scale) pair of the FP8 quantisation, computed
    on demand from the seeded bf16 weights of a (device) [E, K, M] tensor; the argument form that
    orc.swiglu_expert_w8a8 takes."""

    def __init__(self, w):
        self.w = w

    def __getitem__(self, e):
        w = self.w[int(e)].detach().float().cpu().numpy()[None]
        q, sc = orc.quantize_weights_fp8(w)
        return q[0], sc[0]

    def __len__(self):
        return self.w.shape[0]


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    return err / scale if scale > 0 else err, err, scale


def assert_close_rel(got, ref, tol, what=""):
    r, err, scale = rel_err(got, ref)
    assert r <= tol, f"{what}: max|err| = {err:.3e}, max|ref| = {scale:.3e}, ratio {r:.3e} > {tol}"
    return r


def decided_tokens(logits_ref, k, delta):
    """Tokens whose top-k list (set and order) cannot change under a perturbation of every logit
    by at most delta: every gap among the k+1 largest logits exceeds 2*delta (ties decided by
    index need exactly equal values, which a perturbation can break, so they count as fragile
    unless delta == 0)."""
    l = np.asarray(logits_ref, dtype=np.float64)
    T, E = l.shape
    kk = min(k + 1, E)
    top = -np.sort(-l, axis=1)[:, :kk]
    if kk < 2:
        return np.ones(T, dtype=bool)
    gaps = top[:, :-1] - top[:, 1:]
    if delta == 0:
        return np.ones(T, dtype=bool)
    return np.all(gaps > 2.0 * delta, axis=1)


def decided_tokens_grouped(logits_ref, k, n_group, topk_group, delta):
    """Tokens whose group-limited selection cannot change under a perturbation of every logit
    by at most delta: the topk_group+1 best group scores (each a sum of two logits, so it moves
    by at most 2*delta) are more than 4*delta apart, and the k+1 best logits among the kept
    groups' experts are more than 2*delta apart."""
    l32 = np.asarray(logits_ref, dtype=np.float32)
    T, E = l32.shape
    gs = E // n_group
    sc = orc.group_scores(l32, n_group).astype(np.float64)
    margin = 1e-6 * max(1.0, float(np.abs(sc).max()))
    dec = np.ones(T, dtype=bool)
    order = np.argsort(-sc, axis=1, kind="stable")
    if topk_group < n_group:
        top = np.take_along_axis(sc, order[:, :topk_group + 1], axis=1)
        dec &= np.all(top[:, :-1] - top[:, 1:] > 4.0 * delta + margin, axis=1)
    l64 = l32.astype(np.float64)
    for t in range(T):
        if not dec[t]:
            continue
        kept = order[t, :topk_group]
        cand = np.concatenate([l64[t, g * gs:(g + 1) * gs] for g in kept])
        top = -np.sort(-cand)[:min(k + 1, cand.size)]
        if top.size >= 2 and not np.all(top[:-1] - top[1:] > 2.0 * delta):
            dec[t] = False
    return dec


def check_topk_valid(logits_ref, idx_gpu, k, delta, rows):
    """Fragile tokens: the GPU's set must be a top-k of some perturbation within delta."""
    l = np.asarray(logits_ref, dtype=np.float64)
    for t in rows:
        sel = set(int(e) for e in idx_gpu[t])
        assert len(sel) == k
        kth = -np.sort(-l[t])[k - 1]
        for e in range(l.shape[1]):
            if e in sel:
                assert l[t, e] >= kth - 2 * delta - 1e-30
            else:
                assert l[t, e] <= kth + 2 * delta + 1e-30


def check_align_valid(idx, E, C, counts, offsets, sorted_ids, slot_of, drop):
    """Align invariants on any routing (no oracle call): counts = min(raw, C); offsets scan;
    slots are a bijection onto kept assignments; the kept ones of each expert are its first C
    assignments in token order and occupy its slot range in that order."""
    idx = np.asarray(idx).reshape(-1)
    A = idx.size
    raw = np.bincount(idx, minlength=E)
    assert np.array_equal(counts, np.minimum(raw, C))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    kept = int(offsets[-1])
    assert np.all(sorted_ids[kept:] == -1)
    order = np.argsort(idx, kind="stable")  # assignments grouped by expert, token order inside
    pos = 0
    for e in range(E):
        mine = order[pos:pos + raw[e]]
        pos += raw[e]
        keep = mine[:C]
        assert np.array_equal(sorted_ids[offsets[e]:offsets[e + 1]], keep)
        assert np.all(slot_of[keep] == np.arange(offsets[e], offsets[e + 1]))
        assert np.all(drop[keep] == 0)
        assert np.all(slot_of[mine[C:]] == -1) and np.all(drop[mine[C:]] == 1)


def inputs_np(inp):
    """Host copies of the activations/router inputs (weights stay lazy)."""
    return {
        "x": np32(inp["x"]),
        "w_router": np32(inp["w_router"]),
        "logit_bias": None if inp.get("logit_bias") is None else np32(inp["logit_bias"]),
    }


def to_dev(a, dtype=torch.int32, device="cuda"):
    return torch.as_tensor(np.ascontiguousarray(a)).to(device=device, dtype=dtype)
