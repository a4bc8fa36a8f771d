"""Host-side step check for expert parallelism over R ranks (one process per GPU).

[P4] "MoE Router" (2048ai.net), section "Token 分发的通信瓶颈": with experts spread over devices,
every step exchanges token rows between all ranks. On the device the exchange is ordered by flag
words (moe_ep_signal / moe_ep_wait), whose waits are bounded: a rank that has left makes the
others' waits run out after 2 s and report a device error. This module lets the ranks find out on
the host first, between steps, before any of them launches the step's kernels: each rank
publishes the step it is about to run in a key-value store shared by the group (a
torch.distributed Store), and waits, with a deadline, until every other rank has published the
same step. A rank that leaves marks its key, so the others stop at once instead of at the
deadline.
"""
from __future__ import annotations

import time


class RankLost(RuntimeError):
    """A rank of the expert-parallel group left or did not reach the step in time."""

    def __init__(self, rank, step, why):
        super().__init__(f"rank {rank} {why} before step {step}")
        self.rank, self.step = rank, step


class StepHeartbeat:
    """Per-step presence check through a torch.distributed Store (TCPStore, FileStore, ...)."""

    LEFT = "left"

    def __init__(self, store, rank, world, timeout_s=5.0, poll_s=0.005, prefix="moe_ep"):
        self.store, self.rank, self.world = store, int(rank), int(world)
        self.timeout_s, self.poll_s, self.prefix = float(timeout_s), float(poll_s), prefix

    def _key(self, q):
        return f"{self.prefix}/rank{q}"

    def _read(self, q):
        if not self.store.check([self._key(q)]):
            return None
        return self.store.get(self._key(q)).decode()

    def begin_step(self, step):
        """Publish `step` for this rank, then return once every rank has published it (or a later
        step). Raises RankLost for a rank that left or that missed the deadline."""
        step = int(step)
        self.store.set(self._key(self.rank), str(step))
        deadline = time.monotonic() + self.timeout_s
        pending = [q for q in range(self.world) if q != self.rank]
        while pending:
            still = []
            for q in pending:
                v = self._read(q)
                if v == self.LEFT:
                    raise RankLost(q, step, "left the group")
                if v is None or int(v) < step:
                    still.append(q)
            pending = still
            if pending:
                if time.monotonic() > deadline:
                    raise RankLost(pending[0], step, f"did not arrive within {self.timeout_s} s")
                time.sleep(self.poll_s)

    def leave(self):
        """Mark this rank as gone (call between steps, with none of its kernels in flight)."""
        self.store.set(self._key(self.rank), self.LEFT)
