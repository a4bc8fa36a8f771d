"""Out-of-bounds writes. Every output of the layer and of the grouping, and the workspace, sits
inside a byte buffer with 256-byte guard regions on both sides filled with 0xA5. After the call
the guards must be intact, the results must equal those of an ordinary call, and they must match
the oracle (grouping bit for bit; the layer by the parity rules of the layer tests), so that a
write that lands inside the outputs but in the wrong place fails too."""
import numpy as np
import pytest
import torch

from expert_dispatch_gate_b200 import _lib as L
from expert_dispatch_gate_b200 import layer as M
from expert_dispatch_gate_b200 import workloads as W
from oracle import moe_oracle as orc
from tests.test_gpu_parity import compare_layer, small_inputs

pytestmark = pytest.mark.gpu

G = 256  # guard bytes on each side (keeps the 16-byte alignment the ABI asks for)


def guarded(shape, dtype):
    """(buffer with guards, typed view of the middle)."""
    n = 1
    for d in shape:
        n *= d
    es = torch.empty((), dtype=dtype).element_size()
    buf = torch.full((G + n * es + G,), 0xA5, dtype=torch.uint8, device="cuda")
    return buf, buf[G:G + n * es].view(dtype).view(shape)


def intact(buf):
    return bool((buf[:G] == 0xA5).all()) and bool((buf[-G:] == 0xA5).all())


def guarded_ws(shape):
    nbytes = int(L.moe_workspace_bytes(shape))
    buf = torch.full((G + nbytes + G,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = buf[G:G + nbytes]
    ws.zero_()
    return buf, ws, nbytes


@pytest.mark.parametrize("name", ["e96_partial_tiles", "e32_ragged", "e256_k8", "e64_k16_f32",
                                  "e8_two_token_blocks", "e64_zipf", "e128_router_ksplit"])
def test_layer_writes_stay_inside_their_buffers(name):
    wl, cpu, dev = small_inputs(name)
    shape = M.shape_of(wl.T, wl.H, wl.E, wl.k, wl.I, wl.capacity_factor, wl.dtype)
    b = {
        "out": guarded((wl.T, wl.H), dev["x"].dtype),
        "logits": guarded((wl.T, wl.E), torch.float32),
        "topk_idx": guarded((wl.T, wl.k), torch.int32),
        "topk_w": guarded((wl.T, wl.k), torch.float32),
        "counts": guarded((wl.E,), torch.int32),
        "drop_mask": guarded((wl.T * wl.k,), torch.uint8),
    }
    ws_buf, ws, nbytes = guarded_ws(shape)
    L.moe_layer_forward(shape, dev["x"], dev["w_router"], dev["logit_bias"], dev["w_gate"],
                        dev["w_up"], dev["w_down"], b["out"][1], b["logits"][1],
                        b["topk_idx"][1], b["topk_w"][1], b["counts"][1], b["drop_mask"][1], ws,
                        nbytes)
    torch.cuda.synchronize()
    assert L.moe_check_error(ws) == L.MOE_OK
    for key, (buf, _) in b.items():
        assert intact(buf), key
    assert intact(ws_buf), "workspace"
    ref = M.layer_forward(dev["x"], dev["w_router"], dev["w_gate"], dev["w_up"], dev["w_down"],
                          wl.k, wl.capacity_factor, logit_bias=dev["logit_bias"])
    torch.cuda.synchronize()
    for key in b:
        assert torch.equal(b[key][1], ref[key]), key
    got = {key: view for key, (_, view) in b.items()}
    got["C"] = L.moe_capacity(shape)
    compare_layer(wl, cpu, dev, got)


# one 256-thread block (2048 assignments), the 8-CTA cluster (32768), chunked kernels (65544)
@pytest.mark.parametrize("T,E,k", [(256, 16, 8), (4096, 256, 8), (8193, 256, 8)])
def test_grouping_writes_stay_inside_their_buffers(T, E, k):
    idx = W.random_topk_idx(T, E, k, seed=T + E, mode="zipf").cuda()
    shape = M.shape_of(T, 128, E, k, 128, 1.25, L.MOE_BF16)
    A = T * k
    b = {
        "counts": guarded((E,), torch.int32),
        "offsets": guarded((E + 1,), torch.int32),
        "sorted_ids": guarded((A,), torch.int32),
        "slot_of": guarded((A,), torch.int32),
        "drop_mask": guarded((A,), torch.uint8),
    }
    ws_buf, ws, nbytes = guarded_ws(shape)
    L.moe_align(shape, idx, b["counts"][1], b["offsets"][1], b["sorted_ids"][1], b["slot_of"][1],
                b["drop_mask"][1], ws, nbytes)
    torch.cuda.synchronize()
    assert L.moe_check_error(ws) == L.MOE_OK
    for key, (buf, _) in b.items():
        assert intact(buf), key
    assert intact(ws_buf), "workspace"
    ref = M.align(idx, E, 1.25)
    torch.cuda.synchronize()
    for key in b:
        assert torch.equal(b[key][1], ref[key]), key
    al = orc.align(idx.cpu().numpy(), E, orc.capacity(T, k, E, 1.25))
    for key in b:
        assert np.array_equal(b[key][1].cpu().numpy(), al[key]), key
