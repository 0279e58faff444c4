"""Zigzag context parallelism across ranks: the forward ring of one rank.

"Online Draft Co-Training" (core-innovation and method-detail sections): C
context-parallel ranks each hold one zigzag shard of the packed batch (shard
q: chunks q and 2C-1-q of every sequence and the branches anchored in them).
The main-sequence K/V shards go round the ring, each rank sending its current
shard to rank q+1 and receiving the next one from rank q-1 while it attends
its queries to the shard it holds; every step's partial is merged into a
running (O, l) by the LSE rule, and the rank-local branch keys are merged
last.  The exposed cost of a step is max(t_comm, t_attn).

RingSchedule is the communication and ordering (device-agnostic: any
torch.distributed backend, any step callback); ZigzagRingAttention runs the
library's ring kernels on it.  Every computation step runs in the library's
CUDA kernels.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import numpy as np


class RingSchedule:
    """Double-buffered K/V rotation of one rank over C steps.

    step_fn(step, shard, k, v) is called for step = 0 .. C-1 with the main K/V
    of shard (rank - step) mod C.  While step t runs, the shard it holds is
    already on its way to rank + 1 and shard (rank - t - 1) mod C is arriving
    from rank - 1 into the spare buffer (batch_isend_irecv of
    torch.distributed), so the exchange overlaps the step.  The spare buffer
    is only received into once the step that read it has been issued before
    the exchange on the same stream, which orders the two on the device.
    rows[j] is the number of main rows of shard j (receive sizes)."""

    def __init__(self, C: int, rank: int, rows: Sequence[int], group=None):
        if not 0 <= rank < C:
            raise ValueError(f"rank {rank} outside a ring of {C}")
        if len(rows) != C:
            raise ValueError("need one row count per shard")
        self.C, self.rank, self.rows, self.group = C, rank, list(rows), group

    def shard_at(self, step: int) -> int:
        return (self.rank - step) % self.C

    def run(self, k, v, step_fn: Callable, alloc: Callable) -> List[int]:
        """Runs the C steps; alloc(n_rows) returns an empty (k, v) pair with
        n_rows main rows.  Returns the shard order the steps saw."""
        import torch.distributed as dist
        C, r = self.C, self.rank
        order = []
        cur = (k, v)
        spare = None
        for step in range(C):
            work = None
            if step + 1 < C:
                nxt_shard = self.shard_at(step + 1)
                nxt = alloc(self.rows[nxt_shard]) if spare is None or \
                    spare[0].shape[0] != self.rows[nxt_shard] else spare
                ops = [dist.P2POp(dist.isend, cur[0], (r + 1) % C, self.group),
                       dist.P2POp(dist.isend, cur[1], (r + 1) % C, self.group),
                       dist.P2POp(dist.irecv, nxt[0], (r - 1) % C, self.group),
                       dist.P2POp(dist.irecv, nxt[1], (r - 1) % C, self.group)]
                work = dist.batch_isend_irecv(ops)
            order.append(self.shard_at(step))
            step_fn(step, self.shard_at(step), cur[0], cur[1])
            if work is not None:
                for w in work:
                    w.wait()
                spare, cur = cur, nxt
        return order


class ZigzagRingAttention:
    """One rank's zigzag ring forward on the library's kernels.

    cu_seqlens, branch_anchor, branch_depth: host arrays of the whole batch
    (every sequence at least 2C tokens); the rank's tensors are its shard's
    rows in local order (ba_zigzag_shard's main_rows / branch_rows).  The
    index arrays of every shard are derived on the host (cheap), so each rank
    can plan every ring step without a collective."""

    def __init__(self, cu_seqlens, branch_anchor, branch_depth, hq: int, hkv: int,
                 head_dim: int, mask: int, C: int, rank: int, scale: Optional[float] = None,
                 device="cuda"):
        import torch

        from . import Problem, ba_ring_workspace_size, ba_zigzag_shard
        self.C, self.rank = C, rank
        self.device = torch.device(device)
        self.shards = [ba_zigzag_shard(cu_seqlens, branch_anchor, branch_depth, C, j)
                       for j in range(C)]
        me = self.shards[rank]
        dev = self.device
        self.local = Problem(torch.as_tensor(me["cu_local"], device=dev),
                             torch.as_tensor(me["anchor_local"], device=dev),
                             torch.as_tensor(me["depth_local"], device=dev),
                             int(me["branch_rows"].shape[0]), hq, hkv, head_dim, mask, scale, 1)
        self.cu_global = torch.as_tensor(np.asarray(cu_seqlens, dtype=np.int32), device=dev)
        self.cu_visit = [torch.as_tensor(s["cu_local"], device=dev) for s in self.shards]
        plan_b, acc_b = ba_ring_workspace_size(self.local, C)
        self.plan_ws = [torch.empty(plan_b, dtype=torch.uint8, device=dev) for _ in range(C)]
        self.acc_ws = torch.empty(acc_b, dtype=torch.uint8, device=dev)

    @property
    def main_rows(self) -> np.ndarray:
        return self.shards[self.rank]["main_rows"]

    @property
    def branch_rows(self) -> np.ndarray:
        return self.shards[self.rank]["branch_rows"]

    def rows(self) -> List[int]:
        return [int(s["main_rows"].shape[0]) for s in self.shards]

    def plan(self, stream=None) -> None:
        from . import ba_ring_plan
        for step in range(self.C):
            j = (self.rank - step) % self.C
            ba_ring_plan(self.local, self.C, self.rank, step, self.cu_global, self.cu_visit[j],
                         self.plan_ws[step], stream)

    def plan_status(self) -> List[int]:
        from . import ba_plan_status
        return [ba_plan_status(ws) for ws in self.plan_ws]

    def step(self, step: int, q_m, q_b, k_visit, v_visit, stream=None) -> None:
        from . import branch_attn_ring_step
        branch_attn_ring_step(self.local, self.C, step, self.plan_ws[step], self.acc_ws, q_m,
                              k_visit, v_visit, q_b, stream)

    def finish(self, q_m, q_b, k_b, v_b, out=None, stream=None) -> dict:
        import torch

        from . import branch_attn_ring_finish
        if out is None:
            sh = self.local.shapes()
            out = {"o_m": torch.empty(sh["q_m"], dtype=torch.bfloat16, device=self.device),
                   "o_b": torch.empty(sh["q_b"], dtype=torch.bfloat16, device=self.device),
                   "lse_m": torch.empty(sh["lse_m"], dtype=torch.float32, device=self.device),
                   "lse_b": torch.empty(sh["lse_b"], dtype=torch.float32, device=self.device)}
        branch_attn_ring_finish(self.local, self.C, self.plan_ws[0], self.acc_ws, q_m, q_b, k_b,
                                v_b, out["o_m"], out["o_b"], out["lse_m"], out["lse_b"], stream)
        return out

    def forward(self, q_m, k_m, v_m, q_b, k_b, v_b, group=None, out=None) -> dict:
        """The whole ring on this rank: C steps with the K/V rotation of
        RingSchedule over `group` (a torch.distributed process group whose
        ranks 0..C-1 hold shards 0..C-1), then the branch-local merge."""
        import torch
        sched = RingSchedule(self.C, self.rank, self.rows(), group)
        hkv, d = k_m.shape[1], k_m.shape[2]

        def alloc(n):
            return (torch.empty((n, hkv, d), dtype=k_m.dtype, device=k_m.device),
                    torch.empty((n, hkv, d), dtype=v_m.dtype, device=v_m.device))

        sched.run(k_m, v_m, lambda step, j, k, v: self.step(step, q_m, q_b, k, v), alloc)
        return self.finish(q_m, q_b, k_b, v_b, out)
