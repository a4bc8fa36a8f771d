"""GPU parity of the FP8 (e4m3, weight-only) expert path against the oracle: the quantiser bit
for bit, the expert GEMMs and the whole layer within the bf16 tolerance of the oracle run on
the oracle's own dequantised weights (decode(code) * scale)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from expert_dispatch_gate_b200 import _lib as L
from expert_dispatch_gate_b200 import layer as M
from expert_dispatch_gate_b200 import workloads as W
from oracle import moe_oracle as orc
from tests.parity import (TOL_OUT, DequantExpertWeights, assert_close_rel, np32, npi, to_dev)
from tests.test_gpu_parity import SMALL, compare_layer, oracle_routing, small_inputs

pytestmark = pytest.mark.gpu

BF16_SMALL = [n for n, wl in SMALL.items() if wl.dtype == "bf16"]


@pytest.mark.parametrize("E,K,N", [(3, 64, 256), (2, 200, 128), (4, 128, 4096)])
def test_quantize_fp8_bitexact(E, K, N):
    g = torch.Generator().manual_seed(E * 1000 + K + N)
    w = torch.randn((E, K, N), generator=g) * torch.exp(3 * torch.randn((1, 1, N), generator=g))
    w[0, :, 5] = 0.0                       # all-zero column: scale 1, codes 0
    w[1, :, 3] *= 1e-30                    # tiny column
    w[-1, 7, :] = 1e4                      # a row of large values: each is its column's max
    w = w.to(torch.bfloat16)
    codes, scale = M.quantize_fp8(w.cuda())
    torch.cuda.synchronize()
    q_o, s_o = orc.quantize_weights_fp8(w.float().numpy())
    assert np.array_equal(npi(scale).view(np.uint32), s_o.view(np.uint32))
    assert np.array_equal(npi(codes), q_o)


@pytest.mark.parametrize("name", BF16_SMALL)
def test_grouped_ffn_fp8(name):
    wl, cpu, dev = small_inputs(name)
    _, _, _, _, al = oracle_routing(wl, cpu)
    fp8 = M.Fp8Weights(dev["w_gate"], dev["w_up"], dev["w_down"])
    y = M.grouped_ffn_w8(dev["x"], to_dev(al["sorted_ids"]), to_dev(al["offsets"]), fp8, wl.k,
                         wl.capacity_factor)
    torch.cuda.synchronize()
    kept = int(al["offsets"][-1])
    slots = list(range(kept))
    ref = orc.grouped_ffn_slots(np32(dev["x"]), al["sorted_ids"], al["offsets"], wl.k,
                                DequantExpertWeights(dev["w_gate"]),
                                DequantExpertWeights(dev["w_up"]),
                                DequantExpertWeights(dev["w_down"]), slots=slots)
    got = np32(y[:kept])
    want = np.stack([ref[s] for s in slots])
    assert_close_rel(got, want, TOL_OUT["bf16"], "expert outputs, e4m3 weights")


@pytest.mark.parametrize("name", BF16_SMALL)
def test_layer_fp8(name):
    wl, cpu, dev = small_inputs(name)
    fp8 = M.Fp8Weights(dev["w_gate"], dev["w_up"], dev["w_down"])
    res = M.layer_forward_w8(dev["x"], dev["w_router"], fp8, wl.k, wl.capacity_factor,
                             logit_bias=dev["logit_bias"])
    torch.cuda.synchronize()
    assert res["ws"].check() == L.MOE_OK
    compare_layer(wl, cpu, dev, res,
                  weights=(DequantExpertWeights(dev["w_gate"]), DequantExpertWeights(dev["w_up"]),
                           DequantExpertWeights(dev["w_down"])))


# full sizes: the oracle quantises each sampled token's experts on the host, so few tokens
@pytest.mark.parametrize("name,T", [("fine", None), ("decode", 16)])
def test_layer_fp8_workload_sizes(name, T):
    wl = W.WORKLOADS[name] if T is None else W.WORKLOADS[name].with_tokens(T)
    dev = W.make_inputs(wl, "cuda")
    fp8 = M.Fp8Weights(dev["w_gate"], dev["w_up"], dev["w_down"])
    res = M.layer_forward_w8(dev["x"], dev["w_router"], fp8, wl.k, wl.capacity_factor,
                             logit_bias=dev["logit_bias"])
    torch.cuda.synchronize()
    assert res["ws"].check() == L.MOE_OK
    info = compare_layer(wl, dev, dev, res, sample=4,
                         weights=(DequantExpertWeights(dev["w_gate"]),
                                  DequantExpertWeights(dev["w_up"]),
                                  DequantExpertWeights(dev["w_down"])))
    print(name, T, info)
    # the same routing as the bf16 layer (the router does not use the expert weights)
    ref = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                          wl.k, wl.capacity_factor, logit_bias=dev["logit_bias"])
    torch.cuda.synchronize()
    assert torch.equal(res["topk_idx"], ref["topk_idx"])
    assert torch.equal(res["drop_mask"], ref["drop_mask"])
    del dev, fp8, res, ref
    torch.cuda.empty_cache()
