"""Host-side checks of the C ABI that need no GPU: the library loads, exports what the header
declares, computes capacities/workspace sizes, and rejects invalid calls before any launch."""
import ctypes
import json
import os

import pytest

from expert_dispatch_gate_b200 import _lib as L
from expert_dispatch_gate_b200 import build as B
from expert_dispatch_gate_b200 import workloads as W


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.lib()


def test_library_exports_every_header_function(lib):
    names = L.header_functions()
    assert len(names) >= 20
    assert "moe_layer_forward_w8" in names  # names with digits are parsed too
    for n in names:
        assert hasattr(lib, n), n
        # the binding declares every header function's argument types
        assert getattr(lib, n).argtypes is not None, n


def test_shape_struct_layout():
    assert ctypes.sizeof(L.MoeShape) == 32
    assert L.MoeShape.capacity_factor.offset == 24 and L.MoeShape.dtype.offset == 28


def test_capacity_through_abi_matches_golden(lib, golden_dir):
    with open(os.path.join(golden_dir, "capacity_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        E = c["E"]
        shape = L.make_shape(c["T"], 128, E, c["k"], 128, c["cf"], "bf16" if E <= 64 or E % 8 == 0 else "f32")
        assert L.moe_capacity(shape) == c["C"], c


def test_capacity_of_workloads(lib):
    exp = {"tiny": 64, "mixtral": 1280, "fine": 160, "decode": 16, "skewed": 3840}
    for name, wl in W.WORKLOADS.items():
        s = L.make_shape(wl.T, wl.H, wl.E, wl.k, wl.I, wl.capacity_factor, wl.dtype)
        assert L.moe_capacity(s) == exp[name], name
        assert L.moe_workspace_bytes(s) > 0


def test_workspace_bytes_cover_intermediates(lib):
    wl = W.WORKLOADS["fine"]
    s = L.make_shape(wl.T, wl.H, wl.E, wl.k, wl.I, wl.capacity_factor, wl.dtype)
    ws = L.moe_workspace_bytes(s)
    a_cap = min(wl.T * wl.k, wl.E * 160)
    # the SwiGLU intermediate and the per-slot expert outputs live in the workspace
    assert ws >= a_cap * (wl.I + wl.H) * 2 + wl.T * wl.E * 4
    assert L.moe_workspace_bytes(L.make_shape(0, 4096, 256, 8, 2048, 1.25, "bf16")) > 0


BAD = 0x1000  # fake, 16-byte aligned address: never dereferenced, validation fails first
ODD = 0x1001  # misaligned


@pytest.mark.parametrize("T,H,E,k,I,cf,dt,status", [
    (16, 128, 8, 0, 128, 1.25, "bf16", L.MOE_ERR_INVALID_ARG),   # k = 0
    (16, 128, 8, 9, 128, 1.25, "bf16", L.MOE_ERR_INVALID_ARG),   # k > E
    (16, 128, 300, 8, 128, 1.25, "bf16", L.MOE_ERR_UNSUPPORTED),  # E > 256
    (16, 128, 32, 17, 128, 1.25, "bf16", L.MOE_ERR_UNSUPPORTED),  # k > 16
    (16, 100, 8, 2, 128, 1.25, "bf16", L.MOE_ERR_UNSUPPORTED),   # H % 8
    (16, 136, 8, 2, 128, 1.25, "bf16", L.MOE_ERR_UNSUPPORTED),   # bf16 H % 64
    (16, 128, 8, 2, 200, 1.25, "bf16", L.MOE_ERR_UNSUPPORTED),   # bf16 I % 64
    (16, 128, 100, 2, 128, 1.25, "bf16", L.MOE_ERR_UNSUPPORTED),  # bf16 E > 64, E % 8
    (16, 128, 72, 2, 128, 1.25, "f32", L.MOE_ERR_UNSUPPORTED),   # f32 E > 64
    (-1, 128, 8, 2, 128, 1.25, "bf16", L.MOE_ERR_INVALID_ARG),   # T < 0
    (16, 128, 8, 2, 128, float("nan"), "bf16", L.MOE_ERR_INVALID_ARG),
])
def test_invalid_shapes_rejected(lib, T, H, E, k, I, cf, dt, status):
    s = L.make_shape(T, H, E, k, I, cf, dt)
    got = L.moe_layer_forward(s, BAD, BAD, None, BAD, BAD, BAD, BAD, None, BAD, BAD, BAD, BAD,
                              BAD, 1 << 40, stream=0, check=False)
    assert got == status, L.last_error_detail()
    assert L.moe_workspace_bytes(s) == 0 and L.moe_capacity(s) == -1


def test_invalid_dtype_rejected(lib):
    s = L.make_shape(16, 128, 8, 2, 128, 1.25, "bf16")
    s.dtype = 7
    assert L.moe_combine(s, BAD, BAD, BAD, BAD, stream=0, check=False) == L.MOE_ERR_INVALID_ARG


def _good():
    return L.make_shape(64, 128, 8, 2, 128, 1.25, "bf16")


@pytest.mark.parametrize("which", range(13))
def test_null_or_misaligned_pointers_rejected(lib, which):
    s = _good()
    ws = L.moe_workspace_bytes(s)
    args = [BAD] * 13  # x wr bias wg wu wd out logits idx w counts drop ws
    optional = {2, 7}  # logit_bias, logits_out may be NULL
    for bad in ([None, ODD] if which not in optional else [ODD]):
        a = list(args)
        a[which] = bad
        got = L.moe_layer_forward(s, a[0], a[1], a[2], a[3], a[4], a[5], a[6], a[7], a[8], a[9],
                                  a[10], a[11], a[12], ws, stream=0, check=False)
        expect = L.MOE_ERR_WORKSPACE if (which == 12 and bad is None) else L.MOE_ERR_INVALID_ARG
        assert got == expect, (which, bad, L.last_error_detail())
        assert L.last_error_detail()


def test_workspace_too_small(lib):
    s = _good()
    need = L.moe_workspace_bytes(s)
    got = L.moe_layer_forward(s, *([BAD] * 12), BAD, need - 1, stream=0, check=False)
    assert got == L.MOE_ERR_WORKSPACE
    assert "too small" in L.last_error_detail()
    got = L.moe_align(s, BAD, BAD, BAD, BAD, BAD, BAD, BAD, 16, stream=0, check=False)
    assert got == L.MOE_ERR_WORKSPACE


def test_stage_events_validation(lib):
    assert lib.moe_set_stage_events(None, 3) == L.MOE_ERR_INVALID_ARG
    arr = (ctypes.c_void_p * 2)(None, None)
    assert lib.moe_set_stage_events(arr, 2) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_set_stage_events(None, 0) == L.MOE_OK


def test_status_strings(lib):
    for s in range(6):
        assert L.status_string(s).startswith("MOE_")
    with pytest.raises(L.MoeError):
        L.moe_combine(L.make_shape(4, 128, 8, 9, 128, 0, "bf16"), BAD, BAD, BAD, BAD, stream=0)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        L.lib()


def test_layer_opts_struct_layout():
    assert ctypes.sizeof(L.MoeLayerOpts) == 32
    o = L.MoeLayerOpts
    assert (o.n_group.offset, o.topk_group.offset, o.shared_out.offset, o.shared_factor.offset,
            o.out_bias.offset) == (0, 4, 8, 16, 24)


@pytest.mark.parametrize("opts,why", [
    (dict(n_group=7, topk_group=1), "n_group must divide E"),
    (dict(n_group=8, topk_group=9), "topk_group above n_group"),
    (dict(n_group=8, topk_group=0), "topk_group below 1"),
    (dict(n_group=64, topk_group=2), "more than 32 groups"),
    (dict(n_group=16, topk_group=1), "k = 6 exceeds the 4 experts of one group"),
    (dict(shared_factor=float("inf")), "non-finite factor"),
    (dict(shared_out=ODD), "misaligned shared output"),
    (dict(out_bias=ODD), "misaligned bias"),
])
def test_invalid_layer_opts_rejected_before_launch(lib, opts, why):
    s = L.make_shape(64, 128, 64, 6, 128, 1.25, "bf16")
    o = L.make_opts(**opts)
    ws = L.moe_workspace_bytes(s)
    got = L.moe_layer_forward_ex(s, o, *([BAD] * 12), BAD, ws, stream=0, check=False)
    assert got == L.MOE_ERR_INVALID_ARG, why
    assert L.moe_route_from_logits_ex(s, o, BAD, BAD, BAD, stream=0, check=False) == \
        L.MOE_ERR_INVALID_ARG, why
    assert L.moe_combine_ex(s, o, BAD, BAD, BAD, BAD, stream=0, check=False) == \
        L.MOE_ERR_INVALID_ARG, why
    assert L.last_error_detail()


def test_stalled_wait_probe_refuses_a_missing_or_small_workspace(lib):
    # validation happens on the host: nothing is launched, so no GPU is needed
    assert L.moe_probe_stalled_wait(None, 0, check=False) == L.MOE_ERR_WORKSPACE
    buf = ctypes.create_string_buffer(512)
    addr = (ctypes.addressof(buf) + 15) & ~15
    assert L.moe_probe_stalled_wait(addr, 128, check=False) == L.MOE_ERR_WORKSPACE


def test_expert_parallel_calls_reject_bad_arguments_before_any_launch(lib):
    shape = L.make_shape(64, 128, 8, 2, 128, 1.25, "bf16")
    bogus = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    # R must divide E
    assert lib.moe_ep_dispatch(ctypes.byref(shape), 3, bogus, bogus, bogus, bogus, None) == \
        L.MOE_ERR_INVALID_ARG
    # rank outside [0, R)
    assert lib.moe_ep_signal(2, 2, 1, bogus, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_signal(2, 0, 1, None, None) == L.MOE_ERR_INVALID_ARG
    # the wait needs a workspace for its error word
    assert lib.moe_ep_wait(2, 1, bogus, None, 0, None) == L.MOE_ERR_WORKSPACE
    assert lib.moe_ep_wait(0, 1, bogus, bogus, 256, None) == L.MOE_ERR_INVALID_ARG


def test_bf16_accepts_multiples_of_64(lib):
    s = L.make_shape(300, 192, 16, 4, 320, 1.25, "bf16")
    assert L.moe_workspace_bytes(s) > 0 and L.moe_capacity(s) == 94  # ceil(1.25 * 300 * 4 / 16)
