"""Tensor-level wrappers over the C ABI: allocate outputs and workspace with PyTorch (device
memory is PyTorch's job), then make one library call. No arithmetic happens here."""
from __future__ import annotations

import torch

from . import _lib as L


def _dtype_code(t):
    if t.dtype == torch.float32:
        return L.MOE_F32
    if t.dtype == torch.bfloat16:
        return L.MOE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: the layer takes float32 or bfloat16")


def shape_of(T, H, E, k, I, capacity_factor, dtype):
    return L.make_shape(T, H, E, k, I, capacity_factor, dtype)


class Workspace:
    """A device byte buffer sized by moe_workspace_bytes, reused across calls of one shape."""

    def __init__(self, shape, device):
        self.nbytes = max(int(L.moe_workspace_bytes(shape)), 256)
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device)

    def check(self, stream=None):
        return L.moe_check_error(self.buf, stream)


def route(x, w_router, k, logit_bias=None, logits_out=True, ws=None, stream=None, n_group=1,
          topk_group=1):
    T, H = x.shape
    E = w_router.shape[1]
    shape = shape_of(T, H, E, k, 128, 0.0, _dtype_code(x))
    ws = ws or Workspace(shape, x.device)
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    logits = torch.empty((T, E), dtype=torch.float32, device=x.device) if logits_out else None
    if n_group > 1:
        L.moe_route_ex(shape, L.make_opts(n_group, topk_group), x, w_router, logit_bias, logits,
                       idx, w, ws.buf, ws.nbytes, stream)
    else:
        L.moe_route(shape, x, w_router, logit_bias, logits, idx, w, ws.buf, ws.nbytes, stream)
    return idx, w, logits


def route_from_logits(logits, k, stream=None, n_group=1, topk_group=1):
    """Top-k selection and weights from given float32 logits; n_group > 1 makes the selection
    group-limited (keep the topk_group best of n_group expert groups first)."""
    T, E = logits.shape
    shape = shape_of(T, 128, E, k, 128, 0.0, L.MOE_BF16 if E <= 64 or E % 8 == 0 else L.MOE_F32)
    idx = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    if n_group > 1:
        L.moe_route_from_logits_ex(shape, L.make_opts(n_group, topk_group), logits, idx, w,
                                   stream)
    else:
        L.moe_route_from_logits(shape, logits, idx, w, stream)
    return idx, w


def align(topk_idx, E, capacity_factor, H=128, I=128, dtype=L.MOE_BF16, ws=None, stream=None):
    T, k = topk_idx.shape
    shape = shape_of(T, H, E, k, I, capacity_factor, dtype)
    dev = topk_idx.device
    ws = ws or Workspace(shape, dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sorted_ids = torch.empty(T * k, dtype=torch.int32, device=dev)
    slot_of = torch.empty(T * k, dtype=torch.int32, device=dev)
    drop = torch.empty(T * k, dtype=torch.uint8, device=dev)
    L.moe_align(shape, topk_idx, counts, offsets, sorted_ids, slot_of, drop, ws.buf, ws.nbytes,
                stream)
    return {"counts": counts, "offsets": offsets, "sorted_ids": sorted_ids, "slot_of": slot_of,
            "drop_mask": drop, "C": L.moe_capacity(shape), "ws": ws}


def grouped_ffn(x, sorted_ids, offsets, w_gate, w_up, w_down, k, capacity_factor, ws=None,
                stream=None):
    T, H = x.shape
    E, _, I = w_gate.shape
    shape = shape_of(T, H, E, k, I, capacity_factor, _dtype_code(x))
    ws = ws or Workspace(shape, x.device)
    y = torch.empty((T * k, H), dtype=x.dtype, device=x.device)
    L.moe_grouped_ffn(shape, x, sorted_ids, offsets, w_gate, w_up, w_down, y, ws.buf, ws.nbytes,
                      stream)
    return y


def combine(y_slots, slot_of, topk_w, E, stream=None, shared=None, shared_factor=0.0,
            out_bias=None):
    """Weighted merge to token order; optionally + shared_factor * shared + out_bias."""
    T, k = topk_w.shape
    H = y_slots.shape[1]
    shape = shape_of(T, H, E, k, 128, 0.0, _dtype_code(y_slots))
    out = torch.empty((T, H), dtype=y_slots.dtype, device=y_slots.device)
    if shared is not None or out_bias is not None:
        opts = L.make_opts(shared_out=shared, shared_factor=shared_factor, out_bias=out_bias)
        L.moe_combine_ex(shape, opts, y_slots, slot_of, topk_w, out, stream)
    else:
        L.moe_combine(shape, y_slots, slot_of, topk_w, out, stream)
    return out


class MoELayerOutputs(dict):
    pass


def layer_forward(x, w_router, w_gate, w_up, w_down, k, capacity_factor, logit_bias=None,
                  logits_out=True, ws=None, out=None, stream=None, n_group=1, topk_group=1,
                  shared=None, shared_factor=0.0, out_bias=None):
    """Whole layer through moe_layer_forward (moe_layer_forward_ex when group-limited routing
    or a shared-expert / bias term is asked for). Returns out, topk_idx, topk_w, counts,
    drop_mask (and logits when requested)."""
    T, H = x.shape
    E, _, I = w_gate.shape
    dev = x.device
    shape = shape_of(T, H, E, k, I, capacity_factor, _dtype_code(x))
    ws = ws or Workspace(shape, dev)
    res = MoELayerOutputs()
    res["out"] = out if out is not None else torch.empty((T, H), dtype=x.dtype, device=dev)
    res["topk_idx"] = torch.empty((T, k), dtype=torch.int32, device=dev)
    res["topk_w"] = torch.empty((T, k), dtype=torch.float32, device=dev)
    res["counts"] = torch.empty(E, dtype=torch.int32, device=dev)
    res["drop_mask"] = torch.empty(T * k, dtype=torch.uint8, device=dev)
    res["logits"] = torch.empty((T, E), dtype=torch.float32, device=dev) if logits_out else None
    if n_group > 1 or shared is not None or out_bias is not None:
        opts = L.make_opts(n_group, topk_group, shared, shared_factor, out_bias)
        L.moe_layer_forward_ex(shape, opts, x, w_router, logit_bias, w_gate, w_up, w_down,
                               res["out"], res["logits"], res["topk_idx"], res["topk_w"],
                               res["counts"], res["drop_mask"], ws.buf, ws.nbytes, stream)
    else:
        L.moe_layer_forward(shape, x, w_router, logit_bias, w_gate, w_up, w_down, res["out"],
                            res["logits"], res["topk_idx"], res["topk_w"], res["counts"],
                            res["drop_mask"], ws.buf, ws.nbytes, stream)
    res["ws"] = ws
    res["C"] = L.moe_capacity(shape)
    return res


def quantize_fp8(w, stream=None):
    """e4m3 codes [E,K,M] (uint8) and per-channel float32 scales [E,M] of bf16 weights [E,K,M]."""
    E, K, M = w.shape
    codes = torch.empty((E, K, M), dtype=torch.uint8, device=w.device)
    scale = torch.empty((E, M), dtype=torch.float32, device=w.device)
    L.moe_quantize_weights_fp8(w, E, K, M, codes, scale, stream)
    return codes, scale


class Fp8Weights:
    """The three expert weights as e4m3 codes + scales (quantised on the device)."""

    def __init__(self, w_gate, w_up, w_down, stream=None):
        self.q_gate, self.s_gate = quantize_fp8(w_gate, stream)
        self.q_up, self.s_up = quantize_fp8(w_up, stream)
        self.q_down, self.s_down = quantize_fp8(w_down, stream)
        self.E, self.H, self.I = w_gate.shape

    def args(self):
        return (self.q_gate, self.q_up, self.q_down, self.s_gate, self.s_up, self.s_down)


def grouped_ffn_w8(x, sorted_ids, offsets, fp8, k, capacity_factor, ws=None, stream=None):
    T, H = x.shape
    shape = shape_of(T, H, fp8.E, k, fp8.I, capacity_factor, L.MOE_BF16)
    ws = ws or Workspace(shape, x.device)
    y = torch.empty((T * k, H), dtype=x.dtype, device=x.device)
    L.moe_grouped_ffn_w8(shape, x, sorted_ids, offsets, *fp8.args(), y, ws.buf, ws.nbytes, stream)
    return y


def layer_forward_w8(x, w_router, fp8, k, capacity_factor, logit_bias=None, logits_out=True,
                     ws=None, out=None, stream=None, opts=None):
    """Whole layer with e4m3 expert weights (moe_layer_forward_w8)."""
    T, H = x.shape
    E = w_router.shape[1]
    dev = x.device
    shape = shape_of(T, H, E, k, fp8.I, capacity_factor, _dtype_code(x))
    ws = ws or Workspace(shape, dev)
    res = MoELayerOutputs()
    res["out"] = out if out is not None else torch.empty((T, H), dtype=x.dtype, device=dev)
    res["topk_idx"] = torch.empty((T, k), dtype=torch.int32, device=dev)
    res["topk_w"] = torch.empty((T, k), dtype=torch.float32, device=dev)
    res["counts"] = torch.empty(E, dtype=torch.int32, device=dev)
    res["drop_mask"] = torch.empty(T * k, dtype=torch.uint8, device=dev)
    res["logits"] = torch.empty((T, E), dtype=torch.float32, device=dev) if logits_out else None
    L.moe_layer_forward_w8(shape, opts, x, w_router, logit_bias, *fp8.args(), res["out"],
                           res["logits"], res["topk_idx"], res["topk_w"], res["counts"],
                           res["drop_mask"], ws.buf, ws.nbytes, stream)
    res["ws"] = ws
    res["C"] = L.moe_capacity(shape)
    return res


# ---- FP8 weights and activations (W8A8)

def pack_w8a8(w, stream=None):
    """K-major e4m3 codes [E,M,K] (uint8) and per-channel float32 scales [E,M] of bf16 weights
    [E,K,M] (moe_pack_weights_w8a8)."""
    E, K, M = w.shape
    codes = torch.empty((E, M, K), dtype=torch.uint8, device=w.device)
    scale = torch.empty((E, M), dtype=torch.float32, device=w.device)
    L.moe_pack_weights_w8a8(w, E, K, M, codes, scale, stream)
    return codes, scale


def quantize_rows_fp8(a, stream=None):
    """Per-row e4m3 codes [N,K] (uint8) and float32 scales [N] of bf16 rows a [N,K]."""
    N, K = a.shape
    codes = torch.empty((N, K), dtype=torch.uint8, device=a.device)
    scale = torch.empty(N, dtype=torch.float32, device=a.device)
    L.moe_quantize_rows_fp8(a, N, K, codes, scale, stream)
    return codes, scale


class W8A8Weights:
    """The three expert weights repacked as K-major e4m3 codes + scales (on the device)."""

    def __init__(self, w_gate, w_up, w_down, stream=None):
        self.q_gate, self.s_gate = pack_w8a8(w_gate, stream)
        self.q_up, self.s_up = pack_w8a8(w_up, stream)
        self.q_down, self.s_down = pack_w8a8(w_down, stream)
        self.E, self.H, self.I = w_gate.shape

    def args(self):
        return (self.q_gate, self.q_up, self.q_down, self.s_gate, self.s_up, self.s_down)


def grouped_ffn_w8a8(x, sorted_ids, offsets, wq, k, capacity_factor, ws=None, stream=None):
    T, H = x.shape
    shape = shape_of(T, H, wq.E, k, wq.I, capacity_factor, L.MOE_BF16)
    ws = ws or Workspace(shape, x.device)
    y = torch.empty((T * k, H), dtype=x.dtype, device=x.device)
    L.moe_grouped_ffn_w8a8(shape, x, sorted_ids, offsets, *wq.args(), y, ws.buf, ws.nbytes, stream)
    return y


def layer_forward_w8a8(x, w_router, wq, k, capacity_factor, logit_bias=None, logits_out=True,
                       ws=None, out=None, stream=None, opts=None):
    """Whole layer with W8A8 expert GEMMs (moe_layer_forward_w8a8)."""
    T, H = x.shape
    E = w_router.shape[1]
    dev = x.device
    shape = shape_of(T, H, E, k, wq.I, capacity_factor, _dtype_code(x))
    ws = ws or Workspace(shape, dev)
    res = MoELayerOutputs()
    res["out"] = out if out is not None else torch.empty((T, H), dtype=x.dtype, device=dev)
    res["topk_idx"] = torch.empty((T, k), dtype=torch.int32, device=dev)
    res["topk_w"] = torch.empty((T, k), dtype=torch.float32, device=dev)
    res["counts"] = torch.empty(E, dtype=torch.int32, device=dev)
    res["drop_mask"] = torch.empty(T * k, dtype=torch.uint8, device=dev)
    res["logits"] = torch.empty((T, E), dtype=torch.float32, device=dev) if logits_out else None
    L.moe_layer_forward_w8a8(shape, opts, x, w_router, logit_bias, *wq.args(), res["out"],
                             res["logits"], res["topk_idx"], res["topk_w"], res["counts"],
                             res["drop_mask"], ws.buf, ws.nbytes, stream)
    res["ws"] = ws
    res["C"] = L.moe_capacity(shape)
    return res
