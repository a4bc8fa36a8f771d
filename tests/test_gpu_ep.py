"""Expert parallelism emulated on one GPU (moe_ep_plan / moe_ep_dispatch / moe_ep_combine).

R ranks' buffers live on one device and each rank's "peer" pointers point at the other ranks'
buffers. The kernels are launched rank after rank on one stream. Every rank's step signal
(moe_ep_signal) is launched before any rank's wait (moe_ep_wait), so each wait finds its flags
already set and no kernel waits on a later one. The routing is
computed once for the concatenated batch and sliced per rank, so the emulated ranks and the
one-device layer group exactly the same assignments. Then:

- owner and slot equal the protocol oracle's plan (``oracle/moe_ep_oracle.py``) bit for bit;
- each owner's expert outputs equal the one-device grouped FFN's rows for its experts bit for
  bit (same rows, same order, same weights);
- the combined output rows equal the one-device combine bit for bit.
"""
import numpy as np
import pytest
import torch

from expert_dispatch_gate_b200 import _lib as L
from expert_dispatch_gate_b200 import layer as M
from expert_dispatch_gate_b200 import workloads as W
from oracle import moe_ep_oracle as ep
from oracle import moe_oracle as orc

pytestmark = pytest.mark.gpu

# (R, tokens per rank, H, E, k, I, capacity factor, dtype, Zipf bias)
CASES = [
    (2, [300, 217], 256, 16, 4, 256, 1.0, "bf16", 1.2),
    (4, [128, 0, 200, 77], 256, 64, 6, 256, 1.25, "bf16", 1.2),  # a rank with no tokens
    (2, [150, 150], 128, 8, 2, 128, 0.5, "f32", 0.0),             # heavy drops, CUDA-core FFN
    (8, [64] * 8, 512, 256, 8, 512, 1.25, "bf16", 0.0),            # 32 experts per rank
]


def _ptr_table(tensors):
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device="cuda")


@pytest.mark.parametrize("R,T_list,H,E,k,I,cf,dtype,zipf", CASES)
def test_ep_emulated_matches_one_device(R, T_list, H, E, k, I, cf, dtype, zipf):
    T = sum(T_list)
    wl = W.Workload("ep_gpu", 40 + R, T, H, E, k, I, dtype, cf, zipf_s=zipf)
    cpu = W.make_inputs(wl, "cpu")
    dev = {n: (None if v is None else v.cuda()) for n, v in cpu.items()}
    code = L.MOE_F32 if dtype == "f32" else L.MOE_BF16
    El = E // R

    # routing once for the whole batch; the one-device grouping, expert FFN and combine
    idx_all, w_all, _ = M.route(dev["x"], dev["w_router"], k, dev["logit_bias"])
    al = M.align(idx_all, E, cf, H=H, I=I, dtype=code)
    y1 = M.grouped_ffn(dev["x"], al["sorted_ids"], al["offsets"], dev["w_gate"], dev["w_up"],
                       dev["w_down"], k, cf)
    out1 = M.combine(y1, al["slot_of"], w_all, E)
    C = orc.capacity(T, k, E, cf)
    assert al["C"] == C

    cuts = np.cumsum([0] + T_list)
    shapes = [M.shape_of(T_list[r], H, E, k, I, cf, code) for r in range(R)]
    local = [M.align(idx_all[cuts[r]:cuts[r + 1]], E, 0.0, H=H, I=I, dtype=code)
             for r in range(R)]
    counts_all = torch.stack([a["counts"] for a in local]).contiguous()
    plans = []
    for r in range(R):
        A_r = T_list[r] * k
        owner = torch.empty(max(A_r, 1), dtype=torch.int32, device="cuda")
        slot = torch.empty(max(A_r, 1), dtype=torch.int32, device="cuda")
        own_off = torch.empty(El + 1, dtype=torch.int32, device="cuda")
        ws = M.Workspace(shapes[r], "cuda")
        L.moe_ep_plan(shapes[r], R, r, T, idx_all[cuts[r]:cuts[r + 1]], local[r]["slot_of"],
                      local[r]["offsets"], counts_all, owner, slot, own_off, ws.buf, ws.nbytes)
        plans.append((owner[:A_r], slot[:A_r], own_off, ws))
    rows_cap = El * C
    xs = [torch.zeros((rows_cap, H), dtype=dev["x"].dtype, device="cuda") for _ in range(R)]
    peer_xs = _ptr_table(xs)
    # one flag array of R words per rank and per kind of signal (rows sent, outputs ready)
    flags = torch.zeros((2, R, R), dtype=torch.int32, device="cuda")
    sent = _ptr_table([flags[0, q] for q in range(R)])
    ready = _ptr_table([flags[1, q] for q in range(R)])
    epoch = 7
    for r in range(R):
        L.moe_ep_dispatch(shapes[r], R, dev["x"][cuts[r]:cuts[r + 1]], plans[r][0], plans[r][1],
                          peer_xs)
        L.moe_ep_signal(R, r, epoch, sent)
    for r in range(R):
        L.moe_ep_wait(R, epoch, flags[0, r], plans[r][3].buf, plans[r][3].nbytes)
    ys = []
    ident = torch.arange(rows_cap, dtype=torch.int32, device="cuda")
    for r in range(R):
        sl = slice(r * El, (r + 1) * El)
        ys.append(M.grouped_ffn(xs[r], ident, plans[r][2], dev["w_gate"][sl].contiguous(),
                                dev["w_up"][sl].contiguous(), dev["w_down"][sl].contiguous(), 1,
                                0.0))
    for r in range(R):
        L.moe_ep_signal(R, r, epoch, ready)
    for r in range(R):
        L.moe_ep_wait(R, epoch, flags[1, r], plans[r][3].buf, plans[r][3].nbytes)
    peer_y = _ptr_table(ys)
    outs = []
    for r in range(R):
        o = torch.empty((T_list[r], H), dtype=dev["x"].dtype, device="cuda")
        L.moe_ep_combine(shapes[r], R, peer_y, plans[r][0], plans[r][1],
                         w_all[cuts[r]:cuts[r + 1]], o)
        outs.append(o)
    torch.cuda.synchronize()
    for r in range(R):
        assert plans[r][3].check() == L.MOE_OK
    assert torch.all(flags == epoch)

    # plan: the protocol oracle's owners and slots for the same routing
    idx_np = idx_all.cpu().numpy()
    for r in range(R):
        ref = ep._plan(idx_np[cuts[r]:cuts[r + 1]], counts_all.cpu().numpy(), r, R, E, C)
        assert np.array_equal(plans[r][0].cpu().numpy(), ref["owner"])
        assert np.array_equal(plans[r][1].cpu().numpy(), ref["slot"])
        off = plans[r][2].cpu().numpy()
        assert np.array_equal(off, np.append(ref["offsets_owner"][r * El:(r + 1) * El],
                                             ref["counts"][r * El:(r + 1) * El].sum()))
    # expert outputs: each owner's rows are the one-device rows of its experts
    offsets1 = al["offsets"].cpu().numpy()
    for r in range(R):
        lo, hi = int(offsets1[r * El]), int(offsets1[(r + 1) * El])
        assert torch.equal(ys[r][:hi - lo], y1[lo:hi])
    assert torch.equal(torch.cat(outs), out1)


def test_ep_wait_for_a_rank_that_never_signals_ends_with_a_device_error():
    """Rank 1 of 2 never signals: rank 0's wait runs to its 2 s limit, records device error 2 and
    returns; the next step's wait, after both ranks signal a new epoch, succeeds."""
    import time
    R = 2
    shape = L.make_shape(64, 128, 8, 2, 128, 1.25, "bf16")
    ws = M.Workspace(shape, "cuda")
    flags = torch.zeros((R, R), dtype=torch.int32, device="cuda")
    table = _ptr_table([flags[q] for q in range(R)])
    L.moe_ep_signal(R, 0, 1, table)          # rank 0 announces epoch 1; rank 1 does not
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    L.moe_ep_wait(R, 1, flags[0], ws.buf, ws.nbytes)
    with pytest.raises(L.MoeError) as ei:
        ws.check()
    elapsed = time.perf_counter() - t0
    assert ei.value.status == L.MOE_ERR_DEVICE and "device error 2" in str(ei.value)
    assert 1.5 < elapsed < 60
    assert flags[0].tolist() == [1, 0] and flags[1].tolist() == [1, 0]
    for r in range(R):
        L.moe_ep_signal(R, r, 2, table)
    L.moe_ep_wait(R, 2, flags[0], ws.buf, ws.nbytes)
    assert ws.check() == L.MOE_OK
    assert torch.all(flags == 2)
