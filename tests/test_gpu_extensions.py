"""GPU parity of the routing / combine extensions (moe_layer_opts): group-limited top-k and the
shared-expert + bias terms of the combine, against the oracle.

Inputs come from the seeded generators; the oracle never sees a value computed by the CUDA
library (GPU-exported logits are only compared with the oracle's, or fed back to the GPU).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from expert_dispatch_gate_b200 import _lib as L
from expert_dispatch_gate_b200 import layer as M
from expert_dispatch_gate_b200 import workloads as W
from oracle import moe_oracle as orc
from tests.parity import (TOL_LOGITS, TOL_OUT, TOL_W, assert_close_rel, decided_tokens_grouped,
                          np32, npi, to_dev)
from tests.test_gpu_parity import SMALL, compare_layer, oracle_routing, small_inputs

pytestmark = pytest.mark.gpu

# (T, E, k, n_group, topk_group, ties)
GROUPED = [
    (300, 64, 6, 8, 3, True),      # 8 experts per group
    (1000, 256, 8, 8, 4, True),    # the fine-grained router's shape, many ties
    (257, 256, 8, 8, 4, False),
    (129, 32, 4, 4, 2, True),
    (64, 128, 16, 4, 2, False),    # k = 16 from 64 candidates
    (50, 16, 2, 16, 2, True),      # one expert per group: the plain top-2
    (100, 256, 8, 32, 4, True),    # 32 groups of 8
    (7, 8, 2, 2, 1, True),
]


def _shared_and_bias(T, H, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    shared = torch.randn((T, H), generator=g).to(dtype)
    bias = torch.randn(H, generator=g, dtype=torch.float32)
    return shared, bias


@pytest.mark.parametrize("T,E,k,G,g,ties", GROUPED)
def test_route_grouped_from_logits_bitexact(T, E, k, G, g, ties):
    logits = W.random_logits(T, E, seed=T * 11 + E + k + G, ties=ties)
    idx_g, w_g = M.route_from_logits(logits.cuda(), k, n_group=G, topk_group=g)
    torch.cuda.synchronize()
    l32 = logits.numpy()
    idx_o = orc.select_topk_grouped(l32, k, G, g)
    assert np.array_equal(npi(idx_g), idx_o)
    w_o = orc.route_weights(l32, idx_o)
    np.testing.assert_allclose(npi(w_g), w_o, atol=TOL_W, rtol=0)


@pytest.mark.parametrize("name,G,g", [("e64_zipf", 8, 3), ("e256_k8", 8, 4),
                                      ("e32_ragged", 4, 2), ("e128_router_ksplit", 4, 2),
                                      ("e64_k16_f32", 4, 2)])
def test_router_grouped(name, G, g):
    wl, cpu, dev = small_inputs(name)
    idx_g, w_g, logits_g = M.route(dev["x"], dev["w_router"], wl.k, dev["logit_bias"],
                                   n_group=G, topk_group=g)
    torch.cuda.synchronize()
    L_o, _, _, _, _ = oracle_routing(wl, cpu)
    L_g = np32(logits_g)
    tol = TOL_LOGITS[wl.dtype] * max(1.0, float(np.abs(L_o).max()))
    delta = float(np.abs(L_g - L_o).max())
    assert delta <= tol, (delta, tol)
    idx_o = orc.select_topk_grouped(L_o, wl.k, G, g)
    dec = decided_tokens_grouped(L_o, wl.k, G, g, delta)
    assert dec.sum() >= wl.T // 2
    assert np.array_equal(npi(idx_g)[dec], idx_o[dec])
    w_o = orc.route_weights(L_o, idx_o)
    np.testing.assert_allclose(npi(w_g)[dec], w_o[dec], atol=TOL_W + wl.k * delta, rtol=0)
    # the router's selection is the group-limited rule applied to the logits it exported
    idx_s, _ = M.route_from_logits(logits_g, wl.k, n_group=G, topk_group=g)
    assert torch.equal(idx_s.cpu(), idx_g.cpu())


@pytest.mark.parametrize("name", ["e8_two_token_blocks", "e64_zipf", "e256_k8",
                                  "e64_k16_f32", "e96_partial_tiles"])
def test_combine_shared_and_bias(name):
    wl, cpu, dev = small_inputs(name)
    _, _, w_o, _, al = oracle_routing(wl, cpu)
    y = W.make_y_slots(wl, "cpu")
    w32 = w_o.astype(np.float32)
    shared, bias = _shared_and_bias(wl.T, wl.H, y.dtype, 1234 + wl.index)
    out = M.combine(y.cuda(), to_dev(al["slot_of"]), to_dev(w32, torch.float32), wl.E,
                    shared=shared.cuda(), shared_factor=0.75, out_bias=bias.cuda())
    torch.cuda.synchronize()
    ref = orc.combine(np32(y), al["slot_of"], w32, shared=np32(shared), shared_factor=0.75,
                      out_bias=bias.numpy())
    got = np32(out)
    assert_close_rel(got, ref, TOL_OUT[wl.dtype], "combine + shared + bias")
    ulp = 2.0 ** -8 if wl.dtype == "bf16" else 2.0 ** -22
    assert np.all(np.abs(got - ref) <= ulp * np.abs(ref) + 1e-6 * np.abs(ref).max())


@pytest.mark.parametrize("name,G,g", [("e64_zipf", 8, 3), ("e256_k8", 8, 4),
                                      ("e32_ragged", 4, 2), ("e96_partial_tiles", 4, 2),
                                      ("e64_k16_f32", 4, 2)])
def test_layer_grouped_with_shared_expert(name, G, g):
    wl, cpu, dev = small_inputs(name)
    shared, bias = _shared_and_bias(wl.T, wl.H, dev["x"].dtype, 99 + wl.index)
    res = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                          wl.k, wl.capacity_factor, logit_bias=dev["logit_bias"], n_group=G,
                          topk_group=g, shared=shared.cuda(), shared_factor=0.5,
                          out_bias=bias.cuda())
    torch.cuda.synchronize()
    assert res["ws"].check() == L.MOE_OK
    compare_layer(wl, cpu, dev, res, n_group=G, topk_group=g, shared=np32(shared),
                  shared_factor=0.5, out_bias=bias.numpy())


def test_layer_opts_defaults_match_plain_call():
    wl, cpu, dev = small_inputs("e64_zipf")
    plain = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                            wl.k, wl.capacity_factor, logit_bias=dev["logit_bias"])
    shape = M.shape_of(wl.T, wl.H, wl.E, wl.k, wl.I, wl.capacity_factor, wl.dtype)
    out = torch.empty_like(plain["out"])
    idx = torch.empty_like(plain["topk_idx"])
    w = torch.empty_like(plain["topk_w"])
    counts = torch.empty_like(plain["counts"])
    drop = torch.empty_like(plain["drop_mask"])
    L.moe_layer_forward_ex(shape, L.make_opts(), dev["x"], dev["w_router"], dev["logit_bias"],
                           dev["w_gate"], dev["w_up"], dev["w_down"], out, None, idx, w, counts,
                           drop, plain["ws"].buf, plain["ws"].nbytes)
    torch.cuda.synchronize()
    assert torch.equal(out, plain["out"]) and torch.equal(idx, plain["topk_idx"])
    assert torch.equal(w, plain["topk_w"]) and torch.equal(drop, plain["drop_mask"])
