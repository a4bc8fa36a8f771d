"""moe_align_noalloc: the grouping step for callers that cannot allocate device memory.

Some callers run inside another framework's memory planner (which hands them only the tensors it
owns) or on a latency-critical path where a cudaMalloc may stall or fail, so they cannot supply
the scratch workspace moe_align takes. moe_align_noalloc keeps that scratch in a fixed device
array inside the library instead. This test checks, through the C ABI, that two calls in a row
give exactly what moe_align gives on the same routing (grouping results are integers, so the
comparison is bit for bit), and that a batch beyond the array's limit is refused.

The file is collected last on purpose, so a failure here never hides the other tests.
"""
import pytest
import torch

from expert_dispatch_gate_b200 import _lib as L
from expert_dispatch_gate_b200 import layer as M
from expert_dispatch_gate_b200 import workloads as W

pytestmark = pytest.mark.gpu

KEYS = ("counts", "offsets", "sorted_ids", "slot_of", "drop_mask")


def _noalloc(idx, E, cf, H=4096, I=2048):
    T, k = idx.shape
    shape = L.make_shape(T, H, E, k, I, cf, "bf16")
    dev = idx.device
    out = {
        "counts": torch.full((E,), -7, dtype=torch.int32, device=dev),
        "offsets": torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
        "sorted_ids": torch.full((T * k,), -7, dtype=torch.int32, device=dev),
        "slot_of": torch.full((T * k,), -7, dtype=torch.int32, device=dev),
        "drop_mask": torch.full((T * k,), 7, dtype=torch.uint8, device=dev),
    }
    L.moe_align_noalloc(shape, idx, out["counts"], out["offsets"], out["sorted_ids"],
                        out["slot_of"], out["drop_mask"])
    return out


@pytest.mark.parametrize("T,E,k,cf,mode", [
    (256, 16, 8, 1.25, "zipf"),        # 2048 assignments: the one-block form
    (4096, 256, 8, 1.25, "uniform"),   # the fine-grained layer's routing size
    (32768, 64, 6, 1.25, "zipf"),      # 196608 assignments, heavy drops
    (32768, 256, 8, 1.25, "zipf"),     # 262144: the limit, every chunk histogram in use
])
def test_noalloc_matches_workspace_align_twice(T, E, k, cf, mode):
    assert torch.cuda.is_available()
    # two different routings back to back: the shared scratch must not leak between calls
    for seed in (T + E, T + E + 1):
        idx = W.random_topk_idx(T, E, k, seed=seed, mode=mode).cuda()
        ref = M.align(idx, E, cf, H=4096, I=2048)
        got = _noalloc(idx, E, cf)
        torch.cuda.synchronize()
        for key in KEYS:
            assert torch.equal(got[key], ref[key]), key


def test_noalloc_rejects_batches_beyond_its_scratch():
    T, E, k = 32769, 64, 8  # 262152 assignments > 262144
    shape = L.make_shape(T, 4096, E, k, 2048, 1.25, "bf16")
    buf = torch.empty(16, dtype=torch.int32, device="cuda")
    st = L.moe_align_noalloc(shape, buf, buf, buf, buf, buf, buf, check=False)
    assert st == L.MOE_ERR_UNSUPPORTED
    assert "262144" in L.last_error_detail()


def test_noalloc_empty_batch_gives_zero_counts_and_offsets():
    E = 64
    shape = L.make_shape(0, 4096, E, 6, 2048, 1.25, "bf16")
    counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    other = torch.full((16,), -7, dtype=torch.int32, device="cuda")
    assert L.moe_align_noalloc(shape, other, counts, offsets, other, other, other,
                               check=False) == L.MOE_OK
    torch.cuda.synchronize()
    assert torch.all(counts == 0) and torch.all(offsets == 0)
    assert torch.all(other == -7)  # no assignment: nothing else is written


G = 256  # guard bytes on each side of every output (keeps 16-byte alignment)


def _guarded(n, dtype):
    es = torch.empty((), dtype=dtype).element_size()
    buf = torch.full((G + n * es + G,), 0xA5, dtype=torch.uint8, device="cuda")
    return buf, buf[G:G + n * es].view(dtype)


@pytest.mark.parametrize("T,E,k", [(256, 16, 8), (4096, 256, 8), (8193, 256, 8)])
def test_noalloc_writes_stay_inside_their_buffers(T, E, k):
    """Each output between 0xA5 guard regions, at each launch form of the grouping; the guards
    stay intact and the results equal the workspace call's."""
    idx = W.random_topk_idx(T, E, k, seed=T + 3 * E, mode="zipf").cuda()
    shape = L.make_shape(T, 4096, E, k, 2048, 1.25, "bf16")
    A = T * k
    b = {"counts": _guarded(E, torch.int32), "offsets": _guarded(E + 1, torch.int32),
         "sorted_ids": _guarded(A, torch.int32), "slot_of": _guarded(A, torch.int32),
         "drop_mask": _guarded(A, torch.uint8)}
    L.moe_align_noalloc(shape, idx, *(b[key][1] for key in KEYS))
    ref = M.align(idx, E, 1.25, H=4096, I=2048)
    torch.cuda.synchronize()
    for key, (buf, view) in b.items():
        assert bool((buf[:G] == 0xA5).all()) and bool((buf[-G:] == 0xA5).all()), key
        assert torch.equal(view, ref[key]), key
