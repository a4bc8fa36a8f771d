"""Failure detection on the GPU without a fault: a kernel's bounded wait that nothing satisfies
runs out, the kernel records device error 2 in the workspace error word and returns, the host
reads it through moe_check_error, and the context stays usable for the next call."""
import time

import numpy as np
import pytest
import torch

from expert_dispatch_gate_b200 import _lib as L
from expert_dispatch_gate_b200 import layer as M
from expert_dispatch_gate_b200 import workloads as W
from oracle import moe_oracle as orc

pytestmark = pytest.mark.gpu


def test_stalled_wait_ends_with_a_device_error_and_the_context_stays_usable():
    shape = L.make_shape(64, 128, 8, 2, 128, 1.25, "bf16")
    ws = M.Workspace(shape, "cuda")
    assert ws.check() == L.MOE_OK
    t0 = time.perf_counter()
    L.moe_probe_stalled_wait(ws.buf, ws.nbytes)
    with pytest.raises(L.MoeError) as ei:
        ws.check()
    elapsed = time.perf_counter() - t0
    assert ei.value.status == L.MOE_ERR_DEVICE
    assert "device error 2" in str(ei.value)
    assert 1.5 < elapsed < 60  # the wait ran to its limit (2 s), then the kernel returned
    assert ws.check() == L.MOE_OK  # the word was cleared
    # the next call on the same context and workspace works and matches the oracle
    idx = W.random_topk_idx(64, 8, 2, seed=5).cuda()
    res = M.align(idx, 8, 1.25, ws=ws)
    torch.cuda.synchronize()
    assert ws.check() == L.MOE_OK
    al = orc.align(idx.cpu().numpy(), 8, orc.capacity(64, 2, 8, 1.25))
    assert np.array_equal(res["slot_of"].cpu().numpy(), al["slot_of"])


def test_check_error_clears_the_whole_control_block():
    """A device error may leave the one-launch grouping's grid-barrier counters (control-block
    words 32 and 33) off zero; moe_check_error clears all 256 bytes with the error word. Planted
    on the host: an error code and stale counters written into the block, no kernel faulted.
    After the check, a grouping that uses the grid barrier (98304 assignments) matches the
    oracle and leaves the block at zero."""
    T, E, k = 16384, 64, 6
    shape = L.make_shape(T, 128, E, k, 128, 1.25, "bf16")
    ws = M.Workspace(shape, "cuda")
    block = ws.buf[:256].view(torch.int32)
    block[0] = 2
    block[32] = 77
    block[33] = 5
    with pytest.raises(L.MoeError) as ei:
        ws.check()
    assert ei.value.status == L.MOE_ERR_DEVICE
    assert torch.count_nonzero(ws.buf[:256]).item() == 0
    idx = W.random_topk_idx(T, E, k, seed=11, mode="zipf").cuda()
    res = M.align(idx, E, 1.25, ws=ws)
    torch.cuda.synchronize()
    assert ws.check() == L.MOE_OK
    al = orc.align(idx.cpu().numpy(), E, orc.capacity(T, k, E, 1.25))
    for key in ("counts", "offsets", "sorted_ids", "slot_of", "drop_mask"):
        assert np.array_equal(res[key].cpu().numpy(), al[key]), key
    assert torch.count_nonzero(ws.buf[:256]).item() == 0
