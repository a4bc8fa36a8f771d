"""Expert-parallel exchange protocol (``oracle/moe_ep_oracle.py``) on CPU ranks.

The property pinned: R ranks, each routing its own tokens and owning E/R experts, compute
exactly what one device computes on the concatenated batch. That covers the routing, the
capacity drops (decided by global ranks from the all-gathered count table), the owner-side slots
(the one-device slots minus the owner's first offset), and the output rows. The same protocol
code runs with all ranks as threads of one process and as two gloo processes; in both, the
collectives are the only way data moves between ranks.
"""
import datetime
import time
import os
import socket
import threading

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from expert_dispatch_gate_b200 import workloads as W
from oracle import moe_ep_oracle as ep
from oracle import moe_oracle as orc


class ThreadComm:
    """Collectives between R threads: each rank posts its part, all wait, each reads."""

    def __init__(self, R, shared, rank):
        self.R, self.s, self.rank = R, shared, rank

    def _exchange(self, part):
        self.s["slots"][self.rank] = part
        self.s["bar"].wait()
        got = list(self.s["slots"])
        self.s["bar"].wait()
        return got

    def all_gather(self, arr):
        return [np.array(a) for a in self._exchange(np.array(arr))]

    def all_to_all(self, parts):
        got = self._exchange([np.array(p) for p in parts])
        return [got[src][self.rank] for src in range(self.R)]


def run_threads(R, fn):
    shared = {"slots": [None] * R, "bar": threading.Barrier(R, timeout=60)}
    results, errors = [None] * R, []

    def body(r):
        try:
            results[r] = fn(ThreadComm(R, shared, r), r)
        except Exception as e:  # reported below; the barrier's timeout frees the others
            errors.append(e)
            shared["bar"].abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(R)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(120)
    if errors:
        raise errors[0]
    return results


def _problem(T_list, H, E, k, I, zipf, seed):
    wl = W.Workload("ep", 30 + seed, sum(T_list), H, E, k, I, "f32", 1.25, zipf_s=zipf)
    inp = W.make_inputs(wl, "cpu")
    host = {n: (None if v is None else v.numpy()) for n, v in inp.items()}
    cuts = np.cumsum([0] + list(T_list))
    return host, [host["x"][cuts[r]:cuts[r + 1]] for r in range(len(T_list))]


def _rank_fn(host, xs, E, k, cf):
    def fn(comm, r):
        El = E // comm.R
        sl = slice(r * El, (r + 1) * El)
        return ep.ep_layer_forward(comm, r, xs[r], host["w_router"], host["w_gate"][sl],
                                   host["w_up"][sl], host["w_down"][sl], k, cf, E,
                                   logit_bias=host["logit_bias"])
    return fn


def _check_against_one_device(host, res, E, k, cf):
    R = len(res)
    one = orc.layer_forward(host["x"], host["w_router"], host["w_gate"], host["w_up"],
                            host["w_down"], k, cf, logit_bias=host["logit_bias"])
    idx = np.concatenate([r["topk_idx"].reshape(-1, k) for r in res])
    assert np.array_equal(idx, one["topk_idx"])
    kept = np.concatenate([r["kept"] for r in res])
    assert np.array_equal(kept, one["drop_mask"] == 0)
    assert res[0]["C"] == orc.capacity(host["x"].shape[0], k, E, cf)
    # owner-side slots are the one-device slots minus the owner's first offset
    El = E // R
    owner = np.concatenate([r["owner"] for r in res])
    slot = np.concatenate([r["slot"] for r in res])
    base = one["offsets"][np.arange(R) * El]
    assert np.array_equal(owner[kept], one["topk_idx"].reshape(-1)[kept] // El)
    assert np.array_equal(slot[kept] + base[owner[kept]], one["slot_of"][kept])
    # every owner received exactly the rows its plan expected, from every source
    for r in res:
        assert np.array_equal(r["received"], r["recv_from"])
    out = np.concatenate([r["out"] for r in res])
    scale = max(1.0, float(np.abs(one["out"]).max()))
    np.testing.assert_allclose(out, one["out"], rtol=0, atol=1e-12 * scale)


# (R, tokens per rank, H, E, k, I, capacity factor, Zipf bias)
CASES = [
    (2, [40, 60], 32, 8, 2, 16, 1.0, 0.0),
    (3, [0, 50, 17], 32, 12, 3, 16, 0.75, 1.2),   # a rank with no tokens, heavy skew
    (4, [30, 30, 30, 30], 16, 16, 4, 8, 0.5, 1.2),  # most assignments dropped
    (2, [64, 1], 16, 4, 4, 8, 0.0, 0.0),           # k = E, no capacity limit
    (4, [9, 0, 0, 23], 16, 8, 2, 8, 1.25, 0.0),
]


@pytest.mark.parametrize("R,T_list,H,E,k,I,cf,zipf", CASES)
def test_expert_parallel_equals_one_device(R, T_list, H, E, k, I, cf, zipf):
    host, xs = _problem(T_list, H, E, k, I, zipf, seed=R + len(T_list) + E)
    res = run_threads(R, _rank_fn(host, xs, E, k, cf))
    _check_against_one_device(host, res, E, k, cf)


def test_drops_follow_global_token_order():
    # every token picks expert 0 first: with C slots, exactly the first C tokens of the
    # concatenated batch keep it, whichever rank holds them
    R, T_list, H, E, k, I = 2, [5, 7], 16, 4, 1, 8
    host, xs = _problem(T_list, H, E, k, I, 0.0, seed=3)
    host["logit_bias"] = np.array([50.0, 0.0, 0.0, 0.0], dtype=np.float32)
    cf = 0.5  # C = ceil(0.5 * 12 * 1 / 4) = 2
    res = run_threads(R, _rank_fn(host, xs, E, k, cf))
    kept = np.concatenate([r["kept"] for r in res])
    assert res[0]["C"] == 2
    assert kept.tolist() == [True, True] + [False] * 10
    _check_against_one_device(host, res, E, k, cf)


class DistComm:
    """The same collectives over torch.distributed (gloo on CPU): per-destination row counts are
    exchanged first, then the rows, each by one all_to_all_single."""

    def __init__(self):
        self.R = dist.get_world_size()

    def all_gather(self, arr):
        t = torch.as_tensor(np.ascontiguousarray(arr))
        out = [torch.empty_like(t) for _ in range(self.R)]
        dist.all_gather(out, t)
        return [o.numpy() for o in out]

    def all_to_all(self, parts):
        parts = [np.ascontiguousarray(p) for p in parts]
        tail = parts[0].shape[1:]
        width = int(np.prod(tail)) if tail else 1
        send_n = torch.tensor([p.shape[0] for p in parts], dtype=torch.int64)
        recv_n = torch.empty(self.R, dtype=torch.int64)
        dist.all_to_all_single(recv_n, send_n)
        send = torch.as_tensor(np.concatenate([p.reshape(-1) for p in parts]))
        recv = torch.empty(int(recv_n.sum()) * width, dtype=send.dtype)
        dist.all_to_all_single(recv, send, [int(n) * width for n in recv_n],
                               [int(n) * width for n in send_n])
        out, o = [], 0
        for n in recv_n.tolist():
            out.append(recv[o:o + n * width].numpy().reshape((n,) + tail))
            o += n * width
        return out


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _gloo_worker(rank, world, port, case, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        R, T_list, H, E, k, I, cf, zipf = case
        host, xs = _problem(T_list, H, E, k, I, zipf, seed=R + len(T_list) + E)
        res = _rank_fn(host, xs, E, k, cf)(DistComm(), rank)
        q.put((rank, res))
    except Exception as e:  # reported to the test instead of a silent exit
        q.put((rank, RuntimeError(f"rank {rank}: {type(e).__name__}: {e}")))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_two_gloo_ranks():
    case = (2, [33, 48], 32, 8, 3, 16, 1.0, 1.2)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_worker, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(60)
    for r in range(2):
        if isinstance(got[r], Exception):
            raise got[r]
    assert all(p.exitcode == 0 for p in procs)
    R, T_list, H, E, k, I, cf, zipf = case
    host, _ = _problem(T_list, H, E, k, I, zipf, seed=R + len(T_list) + E)
    _check_against_one_device(host, [got[0], got[1]], E, k, cf)


def _leaving_worker(rank, world, port, store_port, case, q):
    """Two gloo ranks run one expert-parallel step; rank 1 then leaves between steps. Rank 0
    learns of it on the host before launching step 2."""
    from expert_dispatch_gate_b200.ep_host import RankLost, StepHeartbeat
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    store = dist.TCPStore("127.0.0.1", store_port, world, rank == 0,
                          timeout=datetime.timedelta(seconds=30))
    hb = StepHeartbeat(store, rank, world, timeout_s=10.0)
    try:
        R, T_list, H, E, k, I, cf, zipf = case
        host, xs = _problem(T_list, H, E, k, I, zipf, seed=R + len(T_list) + E)
        hb.begin_step(1)
        res = _rank_fn(host, xs, E, k, cf)(DistComm(), rank)
        dist.barrier()  # step 1 done on both ranks: nothing of it is in flight
        if rank == 1:
            hb.leave()
            q.put((rank, "left", res))
            # keep the store's host alive until rank 0 has seen the mark
            return
        t0 = time.monotonic()
        try:
            hb.begin_step(2)
            q.put((rank, "step 2 started", None))
        except RankLost as e:
            q.put((rank, f"lost {e.rank} at step {e.step} after {time.monotonic() - t0:.2f} s",
                   res))
    except Exception as e:  # reported to the test instead of a silent exit
        q.put((rank, f"error {type(e).__name__}: {e}", None))
    finally:
        dist.destroy_process_group()


def test_rank_leaving_between_steps_is_seen_on_the_host_before_the_next_step():
    case = (2, [20, 17], 32, 8, 2, 16, 1.0, 0.0)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port, store_port = _free_port(), _free_port()
    procs = [ctx.Process(target=_leaving_worker, args=(r, 2, port, store_port, case, q))
             for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(2):
        r, msg, res = q.get(timeout=180)
        got[r] = (msg, res)
    for p in procs:
        p.join(60)
    assert got[1][0] == "left", got[1][0]
    assert got[0][0].startswith("lost 1 at step 2"), got[0][0]
    assert float(got[0][0].split(" after ")[1].split(" s")[0]) < 5.0  # seen at once, no deadline
    # step 1 itself was complete and correct on both ranks
    R, T_list, H, E, k, I, cf, zipf = case
    host, _ = _problem(T_list, H, E, k, I, zipf, seed=R + len(T_list) + E)
    _check_against_one_device(host, [got[0][1], got[1][1]], E, k, cf)
    assert all(p.exitcode == 0 for p in procs)


def test_step_heartbeat_deadline_for_a_rank_that_never_arrives():
    from expert_dispatch_gate_b200.ep_host import RankLost, StepHeartbeat
    store = dist.HashStore()
    hb0 = StepHeartbeat(store, 0, 3, timeout_s=0.2)
    hb1 = StepHeartbeat(store, 1, 3, timeout_s=0.2)
    store.set("moe_ep/rank2", "4")          # rank 2 is still at step 4
    hb1.store.set("moe_ep/rank1", "5")      # rank 1 has published step 5
    t0 = time.monotonic()
    with pytest.raises(RankLost) as ei:
        hb0.begin_step(5)
    assert ei.value.rank == 2 and ei.value.step == 5
    assert 0.2 <= time.monotonic() - t0 < 2.0
    store.set("moe_ep/rank2", "5")
    hb0.begin_step(5)                        # everyone at step 5 now
