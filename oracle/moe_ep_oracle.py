"""Expert-parallel form of the MoE layer across R ranks: route -> dispatch -> experts -> return
-> combine. It is the oracle for the exchange protocol of an expert-parallel layer.

TEST INFRASTRUCTURE ONLY, under the same rule as ``moe_oracle``: only the test suite may import
this module, and the CUDA library shares nothing with it. The arithmetic steps (router, capacity,
expert FFN, weights) are those of ``moe_oracle``; this module adds only the partition of the work
over ranks and the messages between them.

Sources, cited by page title and section:

* [P4] "MoE Router" on Ascend CANN (2048ai.net)
  - section "Token 分发的通信瓶颈": with experts spread over devices, each device sends every
    token row to the devices that own its experts (an all-to-all with per-destination counts,
    AlltoAllV) and gets the expert outputs back the same way.
  - section "昇腾NPU的通信计算重叠": at most C assignments per expert; the overflow is dropped.

The pages give the exchange, not the bookkeeping. The reading taken here is that an
expert-parallel layer must compute exactly what one device computes on the concatenated batch
(rank 0's tokens first, then rank 1's, ...). Capacity and drop order are properties of the whole
batch, so ranks must agree on them. Protocol, for rank r of R, which holds the tokens x_r and
the experts [r*E/R, (r+1)*E/R):

1. route the local tokens;
2. count the local assignments per expert and all-gather the R x E table of these counts;
3. the global rank of a local assignment (t, j) to expert e is the count of e on ranks below
   r plus its rank among the local assignments to e (token order). It is kept iff that is
   below C = capacity(T_total, k, E, cf), T_total being the sum of the ranks' token counts;
4. the owner of e is rank e // (E/R). The owner's slot for the row is offsets_owner[e] + the
   global rank, where offsets_owner is the exclusive prefix sum of min(total count, C) over
   the owner's experts;
5. each rank sends every kept row x[t] with its slot to the owner (one all-to-all-v). The owner
   places the rows at their slots, which is expert-major order, runs its experts, and sends
   each y row back in the order it came (a second all-to-all-v);
6. each rank combines the returned rows with its routing weights.
"""
from __future__ import annotations

import numpy as np

from oracle import moe_oracle as orc


def _plan(idx_r, raw_all, rank, R, E, C):
    """Steps 3-4 for rank ``rank``: per local assignment a = t*k + j, whether it is kept, its
    owner rank and its slot in the owner's slot-major buffer. Also the owner-side offsets of
    this rank's experts and the number of rows it receives from each rank."""
    idx = np.asarray(idx_r, dtype=np.int64)
    T, k = idx.shape
    El = E // R
    raw_all = np.asarray(raw_all, dtype=np.int64)  # [R, E]
    before = raw_all[:rank].sum(axis=0)             # counts of each expert on lower ranks
    total = raw_all.sum(axis=0)
    counts = np.minimum(total, C)                   # kept per expert over the whole batch
    # owner-side offsets: exclusive prefix over each owner's own experts
    offsets_owner = np.zeros(E, dtype=np.int64)
    for d in range(R):
        run = 0
        for e in range(d * El, (d + 1) * El):
            offsets_owner[e] = run
            run += counts[e]
    seen = np.zeros(E, dtype=np.int64)
    kept = np.zeros(T * k, dtype=bool)
    owner = np.full(T * k, -1, dtype=np.int64)
    slot = np.full(T * k, -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            a = t * k + j
            e = int(idx[t, j])
            g = int(before[e] + seen[e])   # global rank of this assignment within expert e
            seen[e] += 1
            if g < C:
                kept[a] = True
                owner[a] = e // El
                slot[a] = offsets_owner[e] + g
    # rows rank d receives from each source: the kept assignments of d's experts on that source
    recv_from = np.zeros(R, dtype=np.int64)
    mine = range(rank * El, (rank + 1) * El)
    for src in range(R):
        b = raw_all[:src].sum(axis=0)
        recv_from[src] = sum(int(np.clip(C - b[e], 0, raw_all[src, e])) for e in mine)
    return {"kept": kept, "owner": owner, "slot": slot, "counts": counts,
            "offsets_owner": offsets_owner, "recv_from": recv_from}


def ep_layer_forward(comm, rank, x_r, w_router, w_gate_local, w_up_local, w_down_local, k,
                     capacity_factor, E, logit_bias=None):
    """The expert-parallel layer on rank ``rank``. ``comm`` has ``R`` (the number of ranks),
    ``all_gather(array)`` -> list of the ranks' arrays, and ``all_to_all(list of arrays, one per
    destination)`` -> list of arrays, one per source. ``w_*_local`` hold this rank's E/R
    experts. Returns the rank's output rows [T_r, H] (float64) with its routing (topk_idx,
    kept mask, owner, slot)."""
    R = comm.R
    if E % R != 0:
        raise ValueError("the experts must divide evenly over the ranks")
    El = E // R
    x_r = np.asarray(x_r)
    T, H = x_r.shape
    # 1. route
    _, idx, w = orc.route(x_r, w_router, k, logit_bias=logit_bias)
    # 2. per-expert counts of the local assignments, all-gathered
    raw = np.bincount(np.asarray(idx, dtype=np.int64).reshape(-1), minlength=E).astype(np.int64)
    raw_all = np.stack(comm.all_gather(raw))
    T_total = int(raw_all.sum()) // k
    C = orc.capacity(T_total, k, E, capacity_factor)
    # 3-4. keep decisions, owners and slots
    plan = _plan(idx, raw_all, rank, R, E, C)
    # 5. dispatch: per owner, the kept rows in local assignment order, with their slots
    send_rows, send_slots, send_order = [], [], []
    for d in range(R):
        sel = np.nonzero(plan["kept"] & (plan["owner"] == d))[0]
        send_order.append(sel)
        send_rows.append(x_r[sel // k].astype(np.float64))
        send_slots.append(plan["slot"][sel])
    recv_rows = comm.all_to_all(send_rows)
    recv_slots = comm.all_to_all(send_slots)
    n_local = int(plan["counts"][rank * El:(rank + 1) * El].sum())
    xs = np.zeros((n_local, H), dtype=np.float64)
    filled = np.zeros(n_local, dtype=bool)
    for rows, slots in zip(recv_rows, recv_slots):
        xs[slots] = rows
        filled[slots] = True
    if not filled.all():
        raise AssertionError("the dispatched rows do not cover the owner's slots")
    # the owner's experts on its slot-major rows
    y = np.zeros((n_local, w_down_local[0].shape[1] if El else 0), dtype=np.float64)
    for le in range(El):
        e = rank * El + le
        lo = int(plan["offsets_owner"][e])
        hi = lo + int(plan["counts"][e])
        if hi > lo:
            y[lo:hi] = orc.swiglu_expert(xs[lo:hi], w_gate_local[le], w_up_local[le],
                                         w_down_local[le])
    # return each y row to its sender, in the order the rows came
    back = comm.all_to_all([y[slots] for slots in recv_slots])
    # 6. combine
    y_of = {}
    for d in range(R):
        for a, row in zip(send_order[d], back[d]):
            y_of[int(a)] = row
    slot_of = np.full(T * k, -1, dtype=np.int64)
    rows = []
    for i, a in enumerate(sorted(y_of)):
        slot_of[a] = i
        rows.append(y_of[a])
    y_local = np.asarray(rows, dtype=np.float64).reshape(len(rows), H)
    # A rank without tokens still took part in every exchange above. One whose assignments
    # were all dropped gets zero rows, as on one device.
    out = orc.combine(y_local, slot_of, w) if rows else np.zeros((T, H), dtype=np.float64)
    return {"out": out, "topk_idx": idx, "topk_w": w, "kept": plan["kept"],
            "owner": plan["owner"], "slot": plan["slot"], "C": C,
            "recv_from": plan["recv_from"], "received": np.array([len(s) for s in recv_slots])}
