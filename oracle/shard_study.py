"""Per-shard work of a ring over C shards: zigzag order versus sequential.

TEST INFRASTRUCTURE ONLY (like the rest of oracle/): an exact count, used to
study the tile order the zigzag path emulates, never called by the product.

"Online Draft Co-Training" (core-innovation section) contrasts a sequential
ring, where each shard holds one contiguous chunk of every sequence, with the
packed, load-balanced zigzag ring, where shard i holds chunks i and 2C-1-i of
every sequence and the branches anchored in them.  Under causal attention a
sequential shard's queries see more keys the later its chunk, so the shards
do unequal work; zigzag pairs an early chunk with a late one.

pair_matrix counts, exactly, the useful (query head, key) pairs of shard i's
queries against the main keys held by shard j; the branch-local pairs of a
branch query, computed on its anchor's shard, are added to W[i, i].  At ring
step s shard i computes W[i, (i - s) mod C].
"""
from typing import Dict

import numpy as np

from .branch_attention import derive
from .plan import row_intervals

ORDERS = ("zigzag", "sequential")


def _pieces(cu: np.ndarray, C: int, order: str):
    """Key ranges [start, end) of every piece of every sequence and the shard
    each piece belongs to: 2C zigzag chunks (chunk k -> shard k or 2C-1-k) or
    C sequential chunks (chunk k -> shard k), in position order."""
    if order not in ORDERS:
        raise ValueError(order)
    n_pieces = 2 * C if order == "zigzag" else C
    k = np.arange(n_pieces + 1, dtype=np.int64)
    start = cu[:-1, None].astype(np.int64)
    length = (cu[1:] - cu[:-1])[:, None].astype(np.int64)
    edges = start + (k[None, :] * length) // n_pieces          # [S, n_pieces + 1]
    kk = np.arange(n_pieces)
    shard = np.where(kk < C, kk, 2 * C - 1 - kk) if order == "zigzag" else kk
    return edges[:, :-1], edges[:, 1:], shard


def pair_matrix(st, C: int, order: str = "zigzag", block: int = 1 << 17) -> np.ndarray:
    """W[i, j] (int64): useful pairs, over all q heads, of shard i's queries
    against shard j's main keys, with shard i's branch-local pairs on W[i, i]."""
    dv = derive(st)
    iv = row_intervals(st)
    n = dv.n_main
    cu = np.asarray(dv.cu, dtype=np.int64)
    p_lo, p_hi, p_shard = _pieces(cu, C, order)
    seq = np.concatenate([dv.main_seq, dv.branch_seq[dv.row_branch]]).astype(np.int64)
    anchors = np.asarray(st.anchors, dtype=np.int64)
    pos = np.concatenate([np.arange(n, dtype=np.int64), anchors[dv.row_branch]])
    W = np.zeros((C, C), dtype=np.int64)
    for r0 in range(0, iv.shape[0], block):
        r1 = min(r0 + block, iv.shape[0])
        s = seq[r0:r1]
        lo, hi = iv[r0:r1, 0:1], iv[r0:r1, 1:2] + 1
        plo, phi = p_lo[s], p_hi[s]                              # [R, n_pieces]
        overlap = np.clip(np.minimum(hi, phi) - np.maximum(lo, plo), 0, None)
        q_piece = (plo <= pos[r0:r1, None]).sum(axis=1) - 1
        q_shard = p_shard[q_piece]
        for j in range(C):
            cols = np.nonzero(p_shard == j)[0]
            np.add.at(W[:, j], q_shard, overlap[:, cols].sum(axis=1))
        local = np.maximum(iv[r0:r1, 3] - iv[r0:r1, 2] + 1, 0)
        np.add.at(W, (q_shard, q_shard), local)
    return W * st.hq


def imbalance(W: np.ndarray) -> Dict[str, float]:
    """max / mean of the shards' total work, and the worst ring step's max /
    mean (the ring waits for its slowest shard at every step)."""
    C = W.shape[0]
    totals = W.sum(axis=1).astype(np.float64)
    steps = [np.array([W[i, (i - s) % C] for i in range(C)], dtype=np.float64)
             for s in range(C)]
    step_ratio = [x.max() / x.mean() for x in steps if x.mean() > 0]
    return {"total_max_over_mean": float(totals.max() / totals.mean()),
            "worst_step_max_over_mean": float(max(step_ratio)),
            "ring_time_over_ideal": float(sum(x.max() for x in steps) / (totals.sum() / C))}


if __name__ == "__main__":  # prints the imbalance table of the three batches
    import workloads as wl
    for name in ("ttt_20k", "dflash_32k", "ttt_256k"):
        st = wl.structure(name)
        for C in (2, 4, 8):
            row = []
            for order in ORDERS:
                m = imbalance(pair_matrix(st, C, order))
                row.append(f"{order}: totals {m['total_max_over_mean']:.3f}, "
                           f"worst step {m['worst_step_max_over_mean']:.3f}, "
                           f"ring / ideal {m['ring_time_over_ideal']:.3f}")
            print(f"{name} C={C}: " + " | ".join(row))
