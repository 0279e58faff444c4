"""Oracle for the tile metadata ("plan") that drives tile skipping.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages fix which keys each query sees (method-detail section: causal main
prefix up to the anchor, plus the own branch); the tile bookkeeping below is
this library's contract, written in the plain per-tile form:

  * query tiles of BM rows, main tiles first (rows [t BM, (t+1) BM) of the
    main tokens), then branch tiles (the same over branch rows);
  * for a tile whose first/last rows belong to branches b_lo <= b_hi with
    anchors a_lo <= a_hi (a main tile uses its own first/last positions):
      kv_begin = floor(cu[s(b_lo)] / BN),  kv_end = floor(a_hi / BN) + 1,
      key tile k is full iff s(b_lo) = s(b_hi), k BN >= cu[s(b_lo)] and
      (k+1) BN - 1 <= a_lo; the full tiles form [full_begin, full_end), or
      full_begin = full_end = kv_begin when there are none;
      branch-local key rows [cu_branch[b_lo], cu_branch[b_hi + 1]) (main
      tiles: [0, 0));
  * per query row: the closed interval of visible main keys and of visible
    branch-local key rows (empty = [0, -1]), read off the mask definition;
  * per key row: the main query rows and the branch query rows that see it,
    each a half-open row range (empty = [0, 0));
  * per main key tile k: the main and the branch query tiles t with
    kv_begin(t) <= k < kv_end(t), as index ranges (empty = [0, 0));
  * per branch key tile k' (rows [k' BN, (k'+1) BN)): the branch query tiles
    whose branch-local range meets it;
  * forward / backward work orders: tiles sorted by decreasing cost, ties by
    index (cost = key tiles visited, query tiles visited); the backward's
    whole walk is the sum of the backward costs;
  * zigzag (C > 1): per ring step s and query tile, the key tiles spanned by
    the rows' keys inside chunk j and inside chunk 2C-1-j of their sequence,
    j = (shard(row) - s) mod C, as two ranges (empty = [0, 0)).
"""
from __future__ import annotations

import numpy as np

from .branch_attention import MASK_BLOCK_BIDIR, derive, zigzag_chunks

PLAN_BM = 128
PLAN_BN = 128


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


def row_intervals(st) -> np.ndarray:
    """[(N + Nb), 4] int64: main_lo, main_hi, loc_lo, loc_hi per query row.

    Read off the visibility rule: a main row r of sequence s sees main keys
    [cu[s], r]; a branch row of branch b (anchor a, sequence s) sees main keys
    [cu[s], a] and branch rows [cu_branch[b], own row] (causal kinds) or
    [cu_branch[b], cu_branch[b+1] - 1] (block-bidirectional).
    """
    dv = derive(st)
    n, nb = dv.n_main, dv.n_branch_tokens
    out = np.zeros((n + nb, 4), dtype=np.int64)
    out[:n, 0] = dv.cu[dv.main_seq]
    out[:n, 1] = np.arange(n)
    out[:n, 3] = -1
    if nb:
        b = dv.row_branch
        anchors = np.asarray(st.anchors, dtype=np.int64)
        out[n:, 0] = dv.cu[dv.branch_seq[b]]
        out[n:, 1] = anchors[b]
        out[n:, 2] = dv.cu_branch[b]
        if st.mask_kind == MASK_BLOCK_BIDIR:
            out[n:, 3] = dv.cu_branch[b + 1] - 1
        else:
            out[n:, 3] = np.arange(nb)
    return out


def _interval_of_rows(lo: np.ndarray, hi: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """For each key k: the query rows r with lo[r] <= k <= hi[r], as
    [begin, end) (empty = (0, 0)); returns [len(keys), 2].

    lo and hi are non-decreasing over the rows (asserted by the caller), so
    {r : hi[r] >= k} is a suffix and {r : lo[r] <= k} a prefix, and their
    intersection is the interval between the two boundaries.
    """
    b = np.searchsorted(hi, keys, side="left")
    e = np.searchsorted(lo, keys, side="right")
    empty = b >= e
    return np.stack([np.where(empty, 0, b), np.where(empty, 0, e)], axis=1).astype(np.int64)


def key_intervals(st) -> np.ndarray:
    """[(N + Nb), 4] int64 per key row: the main query rows that see it as
    [begin, end), then the branch query rows (indexed from 0 over the branch
    rows) as [begin, end); empty = (0, 0).  Main keys first, then branch keys,
    which only branch rows see (through their branch-local interval).

    Follows from the per-row intervals (row_intervals): main rows and branch
    rows each have non-decreasing lower and upper bounds (rows in packed order,
    anchors non-decreasing), so the rows seeing one key are contiguous.
    """
    iv = row_intervals(st)
    n, nb = st.n_main, st.n_branch_tokens
    m, b = iv[:n], iv[n:]
    for part in (m[:, 0], m[:, 1], b[:, 0], b[:, 1], b[:, 2], b[:, 3]):
        assert np.all(np.diff(part) >= 0), "row bounds must be non-decreasing"
    out = np.zeros((n + nb, 4), dtype=np.int64)
    main_keys, branch_keys = np.arange(n), np.arange(nb)
    out[:n, :2] = _interval_of_rows(m[:, 0], m[:, 1], main_keys)
    out[:n, 2:] = _interval_of_rows(b[:, 0], b[:, 1], main_keys)
    out[n:, 2:] = _interval_of_rows(b[:, 2], b[:, 3], branch_keys)
    return out


def _tile_entry(cu, s_lo, s_hi, a_lo, a_hi, bl, BN):
    kv_begin = int(cu[s_lo]) // BN
    kv_end = int(a_hi) // BN + 1
    # full key tiles: k BN >= cu[s] and (k+1) BN - 1 <= a_lo, same sequence
    fb = -(-int(cu[s_lo]) // BN)
    fe = (int(a_lo) + 1) // BN
    if s_lo != s_hi or fb >= fe:
        fb = fe = kv_begin
    return [kv_begin, fb, fe, kv_end, int(bl[0]), int(bl[1])]


def plan(st, BM: int = PLAN_BM, BN: int = PLAN_BN) -> dict:
    dv = derive(st)
    cu = dv.cu
    anchors = np.asarray(st.anchors, dtype=np.int64)
    n, nb = dv.n_main, dv.n_branch_tokens
    n_mt, n_bt = _cdiv(n, BM), _cdiv(nb, BM)
    qt = []
    for t in range(n_mt):
        r0, r1 = t * BM, min((t + 1) * BM, n) - 1
        qt.append(_tile_entry(cu, dv.main_seq[r0], dv.main_seq[r1], r0, r1, (0, 0), BN))
    for t in range(n_bt):
        r0, r1 = t * BM, min((t + 1) * BM, nb) - 1
        b_lo, b_hi = dv.row_branch[r0], dv.row_branch[r1]
        qt.append(_tile_entry(cu, dv.branch_seq[b_lo], dv.branch_seq[b_hi], anchors[b_lo],
                              anchors[b_hi], (dv.cu_branch[b_lo], dv.cu_branch[b_hi + 1]), BN))
    qt = np.array(qt, dtype=np.int64).reshape(-1, 6)

    def tile_range(sel):
        ts = np.nonzero(sel)[0]
        return (int(ts.min()), int(ts.max()) + 1) if ts.size else (0, 0)

    n_kt, n_bkt = _cdiv(n, BN), _cdiv(nb, BN)
    qm, qb = qt[:n_mt], qt[n_mt:]
    kv_main = np.zeros((n_kt, 4), dtype=np.int64)
    for k in range(n_kt):
        kv_main[k, :2] = tile_range((qm[:, 0] <= k) & (k < qm[:, 3]))
        kv_main[k, 2:] = tile_range((qb[:, 0] <= k) & (k < qb[:, 3]))
    kv_branch = np.zeros((n_bkt, 2), dtype=np.int64)
    for k in range(n_bkt):
        lo, hi = k * BN, min((k + 1) * BN, nb)
        kv_branch[k] = tile_range((qb[:, 4] < hi) & (qb[:, 5] > lo))

    fwd_cost = (qt[:, 3] - qt[:, 0]) + (qt[:, 5] - qt[:, 4] + BN - 1) // BN
    bwd_cost = np.concatenate([(kv_main[:, 1] - kv_main[:, 0]) + (kv_main[:, 3] - kv_main[:, 2]),
                               kv_branch[:, 1] - kv_branch[:, 0]])
    fwd_order = np.argsort(-fwd_cost, kind="stable")
    bwd_order = np.argsort(-bwd_cost, kind="stable")
    out = {
        "cu_branch": dv.cu_branch.copy(),
        "branch_seq": dv.branch_seq.copy(),
        "row_iv": row_intervals(st),
        "key_iv": key_intervals(st),
        "qtile": qt,
        "kv_main": kv_main,
        "kv_branch": kv_branch,
        "fwd_order": fwd_order.astype(np.int64),
        "bwd_order": bwd_order.astype(np.int64),
        # the backward's whole walk: query tiles over all key tiles
        "walk": int(bwd_cost.sum()),
        # walk ahead of each position of the backward order
        "bwd_prefix": (np.cumsum(bwd_cost[bwd_order]) - bwd_cost[bwd_order]).astype(np.int64),
    }
    C = int(getattr(st, "zigzag_C", 1))
    if C > 1:
        out["zz_tiles"] = zz_tiles(st, C, BM, BN)
    return out


def zz_tiles(st, C: int, BM: int = PLAN_BM, BN: int = PLAN_BN) -> np.ndarray:
    """[C, n_qtiles, 4] key-tile ranges of each ring step (two windows).

    A row's shard is that of the chunk holding its own position (main rows)
    or its anchor (branch rows); at step s it reads chunks j and 2C-1-j of its
    sequence, j = (shard - s) mod C, intersected with its visible main keys.
    """
    dv = derive(st)
    n, nb = dv.n_main, dv.n_branch_tokens
    iv = row_intervals(st)
    chunks = zigzag_chunks(dv.cu, C)
    bounds = np.array([[lo for lo, _ in c] + [c[-1][1]] for c in chunks], dtype=np.int64)
    own = iv[:, 1]                     # own position (main) / anchor (branch)
    seq = dv.main_seq[own]
    # chunk k of a position: the k with bounds[s, k] <= pos < bounds[s, k+1]
    # (empty chunks share a boundary; searchsorted(right) picks the last one)
    k = np.zeros(own.shape[0], dtype=np.int64)
    for s_ in np.unique(seq):
        sel = seq == s_
        k[sel] = np.searchsorted(bounds[s_], own[sel], side="right") - 1
    shard = np.where(k < C, k, 2 * C - 1 - k)
    n_mt, n_bt = _cdiv(n, BM), _cdiv(nb, BM)
    # rows are stored tile by tile: main tiles, then branch tiles
    starts = np.concatenate([np.arange(n_mt) * BM, n + np.arange(n_bt) * BM])
    out = np.zeros((C, n_mt + n_bt, 4), dtype=np.int64)
    big = np.iinfo(np.int64).max
    for step in range(C):
        j = (shard - step) % C
        for w, ch in enumerate((j, 2 * C - 1 - j)):
            lo = np.maximum(bounds[seq, ch], iv[:, 0])
            hi = np.minimum(bounds[seq, ch + 1] - 1, iv[:, 1])
            ok = hi >= lo
            lo_t = np.minimum.reduceat(np.where(ok, lo, big), starts)
            hi_t = np.maximum.reduceat(np.where(ok, hi, -1), starts)
            has = hi_t >= 0
            out[step, :, 2 * w] = np.where(has, lo_t // BN, 0)
            out[step, :, 2 * w + 1] = np.where(has, hi_t // BN + 1, 0)
    return out
