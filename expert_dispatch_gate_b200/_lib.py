"""ctypes binding of libmoe.so (the C ABI in include/moe.h).

Argument marshalling only: every function passes raw device pointers, sizes and the CUDA stream
straight to the library, which runs every step of the path in its own kernels. Tensors come
from PyTorch (device memory and streams); a missing library is an error, never a fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_DEBUG_LIB=1 selects the debug build (device-side bounds checks, see moe_debug_checks).
LIB_PATH = os.path.join(HERE, "libmoe_debug.so" if os.environ.get("MOE_DEBUG_LIB") == "1"
                        else "libmoe.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "moe.h")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE = range(6)
MOE_F32, MOE_BF16 = 0, 1
N_STAGE_EVENTS = 5  # route, align, GEMM1, GEMM2, combine


class MoeError(RuntimeError):
    def __init__(self, status, detail):
        super().__init__(f"{status_string(status)} -- {detail}")
        self.status = status
        self.detail = detail


class MoeShape(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64),
        ("H", ctypes.c_int32),
        ("E", ctypes.c_int32),
        ("k", ctypes.c_int32),
        ("I", ctypes.c_int32),
        ("capacity_factor", ctypes.c_float),
        ("dtype", ctypes.c_int32),
    ]


class MoeLayerOpts(ctypes.Structure):
    """moe_layer_opts: group-limited routing and the combine's shared-expert / bias terms."""
    _fields_ = [
        ("n_group", ctypes.c_int32),
        ("topk_group", ctypes.c_int32),
        ("shared_out", ctypes.c_void_p),
        ("shared_factor", ctypes.c_float),
        ("out_bias", ctypes.c_void_p),
    ]


_lib = None
_P = ctypes.c_void_p


def _signatures(lib):
    S = ctypes.POINTER(MoeShape)
    O = ctypes.POINTER(MoeLayerOpts)
    i64 = ctypes.c_int64
    st = ctypes.c_int
    sz = ctypes.c_size_t
    table = {
        "moe_workspace_bytes": (sz, [S]),
        "moe_capacity": (ctypes.c_int32, [S]),
        "moe_route": (st, [S, _P, _P, _P, _P, _P, _P, _P, sz, _P]),
        "moe_route_from_logits": (st, [S, _P, _P, _P, _P]),
        "moe_align": (st, [S, _P, _P, _P, _P, _P, _P, _P, sz, _P]),
        "moe_align_noalloc": (st, [S, _P, _P, _P, _P, _P, _P, _P]),
        "moe_grouped_ffn": (st, [S, _P, _P, _P, _P, _P, _P, _P, _P, sz, _P]),
        "moe_combine": (st, [S, _P, _P, _P, _P, _P]),
        "moe_layer_forward": (st, [S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, sz, _P]),
        "moe_check_error": (st, [_P, _P]),
        "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_last_error_detail": (ctypes.c_char_p, []),
        "moe_set_stage_events": (st, [ctypes.POINTER(_P), ctypes.c_int32]),
        "moe_route_ex": (st, [S, O, _P, _P, _P, _P, _P, _P, _P, sz, _P]),
        "moe_route_from_logits_ex": (st, [S, O, _P, _P, _P, _P]),
        "moe_combine_ex": (st, [S, O, _P, _P, _P, _P, _P]),
        "moe_layer_forward_ex": (st, [S, O, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, sz,
                                      _P]),
        "moe_quantize_weights_fp8": (st, [_P, i64, i64, i64, _P, _P, _P]),
        "moe_grouped_ffn_w8": (st, [S] + [_P] * 11 + [sz, _P]),
        "moe_layer_forward_w8": (st, [S, O] + [_P] * 16 + [sz, _P]),
        "moe_probe_stalled_wait": (st, [_P, sz, _P]),
        "moe_pack_weights_w8a8": (st, [_P, i64, i64, i64, _P, _P, _P]),
        "moe_debug_checks": (ctypes.c_int32, []),
        "moe_quantize_rows_fp8": (st, [_P, i64, i64, _P, _P, _P]),
        "moe_grouped_ffn_w8a8": (st, [S] + [_P] * 11 + [sz, _P]),
        "moe_layer_forward_w8a8": (st, [S, O] + [_P] * 16 + [sz, _P]),
        "moe_ep_plan": (st, [S, ctypes.c_int32, ctypes.c_int32, i64] + [_P] * 7 + [_P, sz, _P]),
        "moe_ep_dispatch": (st, [S, ctypes.c_int32, _P, _P, _P, _P, _P]),
        "moe_ep_combine": (st, [S, ctypes.c_int32, _P, _P, _P, _P, _P, _P]),
        "moe_ep_signal": (st, [ctypes.c_int32, ctypes.c_int32, ctypes.c_uint32, _P, _P]),
        "moe_ep_wait": (st, [ctypes.c_int32, ctypes.c_uint32, _P, _P, sz, _P]),
    }
    for name, (res, args) in table.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


def lib():
    """The loaded libmoe.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m expert_dispatch_gate_b200.build` "
                "(the MoE path has no fallback without its CUDA library)")
        _lib = _signatures(ctypes.CDLL(LIB_PATH))
    return _lib


def header_functions():
    """Names of the functions include/moe.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def status_string(status):
    return lib().moe_status_string(int(status)).decode()


def last_error_detail():
    return lib().moe_last_error_detail().decode()


def _check(status):
    if status != MOE_OK:
        raise MoeError(status, last_error_detail())
    return status


def ptr(t):
    """Raw pointer of a tensor (or an int address, or None for NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_shape(T, H, E, k, I, capacity_factor, dtype):
    if isinstance(dtype, str):
        dtype = MOE_F32 if dtype in ("f32", "float32") else MOE_BF16
    return MoeShape(int(T), int(H), int(E), int(k), int(I), float(capacity_factor), int(dtype))


def moe_workspace_bytes(shape):
    return lib().moe_workspace_bytes(ctypes.byref(shape))


def moe_capacity(shape):
    return lib().moe_capacity(ctypes.byref(shape))


def moe_route(shape, x, w_router, logit_bias, logits_out, topk_idx, topk_w, ws, ws_bytes,
              stream=None, check=True):
    s = lib().moe_route(ctypes.byref(shape), ptr(x), ptr(w_router), ptr(logit_bias),
                        ptr(logits_out), ptr(topk_idx), ptr(topk_w), ptr(ws), int(ws_bytes),
                        _stream(stream))
    return _check(s) if check else s


def moe_route_from_logits(shape, logits, topk_idx, topk_w, stream=None, check=True):
    s = lib().moe_route_from_logits(ctypes.byref(shape), ptr(logits), ptr(topk_idx), ptr(topk_w),
                                    _stream(stream))
    return _check(s) if check else s


def moe_align(shape, topk_idx, counts, offsets, sorted_ids, slot_of, drop_mask, ws, ws_bytes,
              stream=None, check=True):
    s = lib().moe_align(ctypes.byref(shape), ptr(topk_idx), ptr(counts), ptr(offsets),
                        ptr(sorted_ids), ptr(slot_of), ptr(drop_mask), ptr(ws), int(ws_bytes),
                        _stream(stream))
    return _check(s) if check else s


def moe_align_noalloc(shape, topk_idx, counts, offsets, sorted_ids, slot_of, drop_mask,
                      stream=None, check=True):
    s = lib().moe_align_noalloc(ctypes.byref(shape), ptr(topk_idx), ptr(counts), ptr(offsets),
                                ptr(sorted_ids), ptr(slot_of), ptr(drop_mask), _stream(stream))
    return _check(s) if check else s


def moe_grouped_ffn(shape, x, sorted_ids, offsets, w_gate, w_up, w_down, y_slots, ws, ws_bytes,
                    stream=None, check=True):
    s = lib().moe_grouped_ffn(ctypes.byref(shape), ptr(x), ptr(sorted_ids), ptr(offsets),
                              ptr(w_gate), ptr(w_up), ptr(w_down), ptr(y_slots), ptr(ws),
                              int(ws_bytes), _stream(stream))
    return _check(s) if check else s


def moe_combine(shape, y_slots, slot_of, topk_w, out, stream=None, check=True):
    s = lib().moe_combine(ctypes.byref(shape), ptr(y_slots), ptr(slot_of), ptr(topk_w), ptr(out),
                          _stream(stream))
    return _check(s) if check else s


def moe_ep_plan(shape, R, rank, T_total, topk_idx, slot_of_local, offsets_local, counts_all,
                owner, slot, own_offsets, ws, ws_bytes, stream=None, check=True):
    s = lib().moe_ep_plan(ctypes.byref(shape), int(R), int(rank), int(T_total), ptr(topk_idx),
                          ptr(slot_of_local), ptr(offsets_local), ptr(counts_all), ptr(owner),
                          ptr(slot), ptr(own_offsets), ptr(ws), int(ws_bytes), _stream(stream))
    return _check(s) if check else s


def moe_ep_dispatch(shape, R, x, owner, slot, peer_xs, stream=None, check=True):
    s = lib().moe_ep_dispatch(ctypes.byref(shape), int(R), ptr(x), ptr(owner), ptr(slot),
                              ptr(peer_xs), _stream(stream))
    return _check(s) if check else s


def moe_ep_signal(R, rank, epoch, peer_flags, stream=None, check=True):
    s = lib().moe_ep_signal(int(R), int(rank), int(epoch) & 0xffffffff, ptr(peer_flags),
                            _stream(stream))
    return _check(s) if check else s


def moe_ep_wait(R, epoch, flags, ws, ws_bytes, stream=None, check=True):
    s = lib().moe_ep_wait(int(R), int(epoch) & 0xffffffff, ptr(flags), ptr(ws), int(ws_bytes),
                          _stream(stream))
    return _check(s) if check else s


def moe_ep_combine(shape, R, peer_y, owner, slot, topk_w, out, stream=None, check=True):
    s = lib().moe_ep_combine(ctypes.byref(shape), int(R), ptr(peer_y), ptr(owner), ptr(slot),
                             ptr(topk_w), ptr(out), _stream(stream))
    return _check(s) if check else s


def moe_layer_forward(shape, x, w_router, logit_bias, w_gate, w_up, w_down, out, logits_out,
                      topk_idx, topk_w, counts, drop_mask, ws, ws_bytes, stream=None, check=True):
    s = lib().moe_layer_forward(ctypes.byref(shape), ptr(x), ptr(w_router), ptr(logit_bias),
                                ptr(w_gate), ptr(w_up), ptr(w_down), ptr(out), ptr(logits_out),
                                ptr(topk_idx), ptr(topk_w), ptr(counts), ptr(drop_mask), ptr(ws),
                                int(ws_bytes), _stream(stream))
    return _check(s) if check else s


def make_opts(n_group=1, topk_group=1, shared_out=None, shared_factor=0.0, out_bias=None):
    """A moe_layer_opts; the tensors must stay alive while the call is in flight."""
    return MoeLayerOpts(int(n_group), int(topk_group), ptr(shared_out), float(shared_factor),
                        ptr(out_bias))


def _opts(opts):
    return None if opts is None else ctypes.byref(opts)


def moe_route_ex(shape, opts, x, w_router, logit_bias, logits_out, topk_idx, topk_w, ws,
                 ws_bytes, stream=None, check=True):
    s = lib().moe_route_ex(ctypes.byref(shape), _opts(opts), ptr(x), ptr(w_router),
                           ptr(logit_bias), ptr(logits_out), ptr(topk_idx), ptr(topk_w), ptr(ws),
                           int(ws_bytes), _stream(stream))
    return _check(s) if check else s


def moe_route_from_logits_ex(shape, opts, logits, topk_idx, topk_w, stream=None, check=True):
    s = lib().moe_route_from_logits_ex(ctypes.byref(shape), _opts(opts), ptr(logits),
                                       ptr(topk_idx), ptr(topk_w), _stream(stream))
    return _check(s) if check else s


def moe_combine_ex(shape, opts, y_slots, slot_of, topk_w, out, stream=None, check=True):
    s = lib().moe_combine_ex(ctypes.byref(shape), _opts(opts), ptr(y_slots), ptr(slot_of),
                             ptr(topk_w), ptr(out), _stream(stream))
    return _check(s) if check else s


def moe_layer_forward_ex(shape, opts, x, w_router, logit_bias, w_gate, w_up, w_down, out,
                         logits_out, topk_idx, topk_w, counts, drop_mask, ws, ws_bytes,
                         stream=None, check=True):
    s = lib().moe_layer_forward_ex(ctypes.byref(shape), _opts(opts), ptr(x), ptr(w_router),
                                   ptr(logit_bias), ptr(w_gate), ptr(w_up), ptr(w_down), ptr(out),
                                   ptr(logits_out), ptr(topk_idx), ptr(topk_w), ptr(counts),
                                   ptr(drop_mask), ptr(ws), int(ws_bytes), _stream(stream))
    return _check(s) if check else s


def moe_quantize_weights_fp8(w, E, K, M, codes, scale, stream=None, check=True):
    s = lib().moe_quantize_weights_fp8(ptr(w), int(E), int(K), int(M), ptr(codes), ptr(scale),
                                       _stream(stream))
    return _check(s) if check else s


def moe_pack_weights_w8a8(w, E, K, M, codes, scale, stream=None, check=True):
    s = lib().moe_pack_weights_w8a8(ptr(w), int(E), int(K), int(M), ptr(codes), ptr(scale),
                                    _stream(stream))
    return _check(s) if check else s


def moe_quantize_rows_fp8(a, N, K, codes, scale, stream=None, check=True):
    s = lib().moe_quantize_rows_fp8(ptr(a), int(N), int(K), ptr(codes), ptr(scale),
                                    _stream(stream))
    return _check(s) if check else s


def moe_grouped_ffn_w8a8(shape, x, sorted_ids, offsets, qk_gate, qk_up, qk_down, s_gate, s_up,
                         s_down, y_slots, ws, ws_bytes, stream=None, check=True):
    s = lib().moe_grouped_ffn_w8a8(ctypes.byref(shape), ptr(x), ptr(sorted_ids), ptr(offsets),
                                   ptr(qk_gate), ptr(qk_up), ptr(qk_down), ptr(s_gate), ptr(s_up),
                                   ptr(s_down), ptr(y_slots), ptr(ws), int(ws_bytes),
                                   _stream(stream))
    return _check(s) if check else s


def moe_layer_forward_w8a8(shape, opts, x, w_router, logit_bias, qk_gate, qk_up, qk_down, s_gate,
                           s_up, s_down, out, logits_out, topk_idx, topk_w, counts, drop_mask, ws,
                           ws_bytes, stream=None, check=True):
    s = lib().moe_layer_forward_w8a8(ctypes.byref(shape), _opts(opts), ptr(x), ptr(w_router),
                                     ptr(logit_bias), ptr(qk_gate), ptr(qk_up), ptr(qk_down),
                                     ptr(s_gate), ptr(s_up), ptr(s_down), ptr(out),
                                     ptr(logits_out), ptr(topk_idx), ptr(topk_w), ptr(counts),
                                     ptr(drop_mask), ptr(ws), int(ws_bytes), _stream(stream))
    return _check(s) if check else s


def moe_grouped_ffn_w8(shape, x, sorted_ids, offsets, q_gate, q_up, q_down, s_gate, s_up, s_down,
                       y_slots, ws, ws_bytes, stream=None, check=True):
    s = lib().moe_grouped_ffn_w8(ctypes.byref(shape), ptr(x), ptr(sorted_ids), ptr(offsets),
                                 ptr(q_gate), ptr(q_up), ptr(q_down), ptr(s_gate), ptr(s_up),
                                 ptr(s_down), ptr(y_slots), ptr(ws), int(ws_bytes),
                                 _stream(stream))
    return _check(s) if check else s


def moe_layer_forward_w8(shape, opts, x, w_router, logit_bias, q_gate, q_up, q_down, s_gate,
                         s_up, s_down, out, logits_out, topk_idx, topk_w, counts, drop_mask, ws,
                         ws_bytes, stream=None, check=True):
    s = lib().moe_layer_forward_w8(ctypes.byref(shape), _opts(opts), ptr(x), ptr(w_router),
                                   ptr(logit_bias), ptr(q_gate), ptr(q_up), ptr(q_down),
                                   ptr(s_gate), ptr(s_up), ptr(s_down), ptr(out), ptr(logits_out),
                                   ptr(topk_idx), ptr(topk_w), ptr(counts), ptr(drop_mask),
                                   ptr(ws), int(ws_bytes), _stream(stream))
    return _check(s) if check else s


def moe_check_error(ws, stream=None, check=True):
    s = lib().moe_check_error(ptr(ws), _stream(stream))
    return _check(s) if check else s


def moe_set_stage_events(events):
    """events: list of N_STAGE_EVENTS torch.cuda.Event (recorded by moe_layer_forward) or None."""
    if events is None:
        return _check(lib().moe_set_stage_events(None, 0))
    for e in events:  # torch creates the CUDA event lazily, on its first record
        if not e.cuda_event:
            e.record()
    arr = (_P * len(events))(*[e.cuda_event for e in events])
    return _check(lib().moe_set_stage_events(arr, len(events)))


def moe_probe_stalled_wait(ws, ws_bytes, stream=None, check=True):
    s = lib().moe_probe_stalled_wait(ptr(ws), int(ws_bytes), _stream(stream))
    return _check(s) if check else s
