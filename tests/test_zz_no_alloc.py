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
    (4096, 256, 8, 1.25, "uniform"),   # the fine-grained layer's routing size
    (32768, 64, 6, 1.25, "zipf"),      # 196608 assignments, heavy drops
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
