"""GPU parity of the W8A8 expert path (e4m3 weights and e4m3 activations on the tensor cores)
against the oracle's W8A8 expert (orc.swiglu_expert_w8a8): the weight repacking and the row
quantiser bit for bit, the expert GEMMs and the whole layer within the bf16 tolerance."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from expert_dispatch_gate_b200 import _lib as L
from expert_dispatch_gate_b200 import layer as M
from expert_dispatch_gate_b200 import workloads as W
from oracle import moe_oracle as orc
from tests.parity import TOL_OUT, W8A8ExpertWeights, assert_close_rel, np32, npi, to_dev
from tests.test_gpu_parity import SMALL, compare_layer, oracle_routing, small_inputs

pytestmark = pytest.mark.gpu

BF16_SMALL = [n for n, wl in SMALL.items() if wl.dtype == "bf16"]


@pytest.mark.parametrize("E,K,N", [(3, 64, 256), (2, 192, 128), (2, 128, 4096), (1, 4096, 64)])
def test_pack_w8a8_bitexact(E, K, N):
    g = torch.Generator().manual_seed(E * 1000 + K + N + 7)
    w = torch.randn((E, K, N), generator=g) * torch.exp(3 * torch.randn((1, 1, N), generator=g))
    w[0, :, 5] = 0.0                       # all-zero column: scale 1, codes 0
    w[-1, 7, :] = 1e4                      # a row of large values: each is its column's max
    w = w.to(torch.bfloat16)
    codes, scale = M.pack_w8a8(w.cuda())
    torch.cuda.synchronize()
    q_o, s_o = orc.quantize_weights_fp8(w.float().numpy())
    assert np.array_equal(npi(scale).view(np.uint32), s_o.view(np.uint32))
    assert np.array_equal(npi(codes), np.ascontiguousarray(q_o.transpose(0, 2, 1)))


@pytest.mark.parametrize("N,K", [(1, 8), (37, 4096), (300, 2048), (5, 14336), (9, 1000), (3, 4104),
                                 (7, 8192)])
def test_quantize_rows_fp8_bitexact(N, K):
    g = torch.Generator().manual_seed(N * 31 + K)
    a = torch.randn((N, K), generator=g) * torch.exp(4 * torch.randn((N, 1), generator=g))
    a[0, :] = 0.0 if N > 1 else a[0, :]    # an all-zero row: scale 1, codes 0
    a = a.to(torch.bfloat16)
    codes, scale = M.quantize_rows_fp8(a.cuda())
    torch.cuda.synchronize()
    q_o, s_o = orc.quantize_rows_fp8(a.float().numpy())
    assert np.array_equal(npi(scale).view(np.uint32), s_o.view(np.uint32))
    assert np.array_equal(npi(codes), q_o)


def _oracle_weights(dev):
    return (W8A8ExpertWeights(dev["w_gate"]), W8A8ExpertWeights(dev["w_up"]),
            W8A8ExpertWeights(dev["w_down"]))


@pytest.mark.parametrize("name", BF16_SMALL)
def test_grouped_ffn_w8a8(name):
    wl, cpu, dev = small_inputs(name)
    _, _, _, _, al = oracle_routing(wl, cpu)
    wq = M.W8A8Weights(dev["w_gate"], dev["w_up"], dev["w_down"])
    y = M.grouped_ffn_w8a8(dev["x"], to_dev(al["sorted_ids"]), to_dev(al["offsets"]), wq, wl.k,
                           wl.capacity_factor)
    torch.cuda.synchronize()
    kept = int(al["offsets"][-1])
    slots = list(range(kept))
    og, ou, od = _oracle_weights(dev)
    ref = orc.grouped_ffn_slots(np32(dev["x"]), al["sorted_ids"], al["offsets"], wl.k, og, ou, od,
                                slots=slots, expert_fn=orc.swiglu_expert_w8a8)
    got = np32(y[:kept])
    want = np.stack([ref[s] for s in slots])
    r = assert_close_rel(got, want, TOL_OUT["bf16"], "expert outputs, W8A8")
    print(name, "W8A8 expert outputs: max rel err %.3e" % r)


@pytest.mark.parametrize("name", BF16_SMALL)
def test_layer_w8a8(name):
    wl, cpu, dev = small_inputs(name)
    wq = M.W8A8Weights(dev["w_gate"], dev["w_up"], dev["w_down"])
    res = M.layer_forward_w8a8(dev["x"], dev["w_router"], wq, wl.k, wl.capacity_factor,
                               logit_bias=dev["logit_bias"])
    torch.cuda.synchronize()
    assert res["ws"].check() == L.MOE_OK
    info = compare_layer(wl, cpu, dev, res, weights=_oracle_weights(dev),
                         expert_fn=orc.swiglu_expert_w8a8)
    print(name, info)
    # determinism
    res2 = M.layer_forward_w8a8(dev["x"], dev["w_router"], wq, wl.k, wl.capacity_factor,
                                logit_bias=dev["logit_bias"], ws=res["ws"])
    torch.cuda.synchronize()
    assert torch.equal(res["out"], res2["out"])


# full sizes: the oracle quantises each sampled token's experts on the host, so few tokens
@pytest.mark.parametrize("name,T", [("fine", None), ("decode", 16)])
def test_layer_w8a8_workload_sizes(name, T):
    wl = W.WORKLOADS[name] if T is None else W.WORKLOADS[name].with_tokens(T)
    dev = W.make_inputs(wl, "cuda")
    wq = M.W8A8Weights(dev["w_gate"], dev["w_up"], dev["w_down"])
    res = M.layer_forward_w8a8(dev["x"], dev["w_router"], wq, wl.k, wl.capacity_factor,
                               logit_bias=dev["logit_bias"])
    torch.cuda.synchronize()
    assert res["ws"].check() == L.MOE_OK
    info = compare_layer(wl, dev, dev, res, sample=4, weights=_oracle_weights(dev),
                         expert_fn=orc.swiglu_expert_w8a8)
    print(name, T, info)
    ref = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                          wl.k, wl.capacity_factor, logit_bias=dev["logit_bias"])
    torch.cuda.synchronize()
    assert torch.equal(res["topk_idx"], ref["topk_idx"])
    assert torch.equal(res["drop_mask"], ref["drop_mask"])
    # the quantised layer stays near the bf16 layer (e4m3 carries 3 mantissa bits)
    kept = ~np.all(npi(res["drop_mask"]).reshape(wl.T, wl.k) == 1, axis=1)
    d = np.abs(np32(res["out"])[kept] - np32(ref["out"])[kept]).max()
    assert d <= 0.15 * np.abs(np32(ref["out"])[kept]).max()
    del dev, wq, res, ref
    torch.cuda.empty_cache()
