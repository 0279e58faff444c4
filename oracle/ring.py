"""Shards and ring steps of zigzag context parallelism across ranks.

TEST INFRASTRUCTURE ONLY (like the rest of oracle/): brute-force statements
of which rows a shard holds and which keys its queries see at each ring step,
used to check the library's shard helper and ring plans; never called by the
product.

"Online Draft Co-Training" (core-innovation and method-detail sections): the
packed batch is split over C ranks in zigzag order, shard q holding chunks q
and 2C-1-q of every sequence and the branches anchored in them; main K/V go
round the ring, at step t shard q's queries meet shard (q - t) mod C's main
keys under the global mask, and the branch partial stays on its rank.
"""
from typing import Dict

import numpy as np

from .branch_attention import derive, visible_keys, zigzag_chunks


def shard(st, C: int, q: int) -> Dict[str, np.ndarray]:
    """Rows of shard q in its local order: for every sequence, chunk q then
    chunk 2C-1-q (position order); the branches anchored in those rows, in
    anchor order.  Returns main_rows (batch main row of each local row),
    branches (batch branch index of each local branch), branch_rows (batch
    branch row of each local branch row), cu_local, anchor_local (anchors as
    local rows) and depth_local."""
    dv = derive(st)
    chunks = zigzag_chunks(dv.cu, C)
    main_rows, cu_local = [], [0]
    for s_chunks in chunks:
        for k in (q, 2 * C - 1 - q):
            lo, hi = s_chunks[k]
            main_rows.extend(range(lo, hi))
        cu_local.append(len(main_rows))
    main_rows = np.asarray(main_rows, dtype=np.int64)
    local_of = {int(r): i for i, r in enumerate(main_rows)}
    anchors = np.asarray(st.anchors, dtype=np.int64)
    branches = [b for b in range(anchors.shape[0]) if int(anchors[b]) in local_of]
    branches.sort(key=lambda b: (local_of[int(anchors[b])], b))
    branch_rows = [r for b in branches for r in range(int(dv.cu_branch[b]), int(dv.cu_branch[b + 1]))]
    return {"main_rows": main_rows, "branches": np.asarray(branches, dtype=np.int64),
            "branch_rows": np.asarray(branch_rows, dtype=np.int64),
            "cu_local": np.asarray(cu_local, dtype=np.int64),
            "anchor_local": np.asarray([local_of[int(anchors[b])] for b in branches], dtype=np.int64),
            "depth_local": np.asarray([int(dv.cu_branch[b + 1] - dv.cu_branch[b]) for b in branches],
                                      dtype=np.int64)}


def step_intervals(st, C: int, q: int, step: int) -> np.ndarray:
    """[lo, hi] (inclusive, local rows of the visiting shard j = (q - step) mod
    C) of the main keys each local query row of shard q sees at this ring step:
    the global mask's visible main keys of the row, kept where shard j holds
    them, mapped to j's local order.  Rows in local order, main rows then
    branch rows; hi < lo (lo, hi = 0, -1) when the row sees none.  Raises if
    the visible keys are not one contiguous run of j's local rows."""
    dv = derive(st)
    j = (q - step) % C
    sq, sj = shard(st, C, q), shard(st, C, j)
    local_j = {int(r): i for i, r in enumerate(sj["main_rows"])}
    rows = [("main", int(r)) for r in sq["main_rows"]] + \
           [("branch", int(r)) for r in sq["branch_rows"]]
    out = np.zeros((len(rows), 2), dtype=np.int64)
    for i, (kind, r) in enumerate(rows):
        mk, _ = visible_keys(st, dv, kind, r)
        seen = sorted(local_j[int(k)] for k in mk if int(k) in local_j)
        if not seen:
            out[i] = (0, -1)
            continue
        if seen[-1] - seen[0] + 1 != len(seen):
            raise AssertionError(f"row {kind} {r}: visible keys of shard {j} not contiguous")
        out[i] = (seen[0], seen[-1])
    return out
