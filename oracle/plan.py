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
  * per main key tile k: the main and the branch query tiles t with
    kv_begin(t) <= k < kv_end(t), as index ranges (empty = [0, 0));
  * per branch key tile k' (rows [k' BN, (k'+1) BN)): the branch query tiles
    whose branch-local range meets it;
  * forward / backward work orders: tiles sorted by decreasing cost, ties by
    index (cost = key tiles visited, query tiles visited).
"""
from __future__ import annotations

import numpy as np

from .branch_attention import derive, visible_keys

PLAN_BM = 128
PLAN_BN = 128


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


def row_intervals(st) -> np.ndarray:
    """[(N + Nb), 4] int64: main_lo, main_hi, loc_lo, loc_hi per query row."""
    dv = derive(st)
    n, nb = dv.n_main, dv.n_branch_tokens
    out = np.zeros((n + nb, 4), dtype=np.int64)
    for r in range(n):
        mk, _ = visible_keys(st, dv, "main", r)
        out[r] = (mk.min(), mk.max(), 0, -1)
    for r in range(nb):
        mk, lk = visible_keys(st, dv, "branch", r)
        out[n + r] = (mk.min(), mk.max(), lk.min(), lk.max())
    return out


def _tile_entry(cu, s_lo, s_hi, a_lo, a_hi, bl, BN):
    kv_begin = int(cu[s_lo]) // BN
    kv_end = int(a_hi) // BN + 1
    full = [k for k in range(kv_begin, kv_end)
            if s_lo == s_hi and k * BN >= cu[s_lo] and (k + 1) * BN - 1 <= a_lo]
    if full:
        assert full == list(range(full[0], full[-1] + 1))
        fb, fe = full[0], full[-1] + 1
    else:
        fb = fe = kv_begin
    return [kv_begin, fb, fe, kv_end, bl[0], bl[1]]


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

    def tile_range(ts):
        return (min(ts), max(ts) + 1) if ts else (0, 0)

    n_kt, n_bkt = _cdiv(n, BN), _cdiv(nb, BN)
    kv_main = np.zeros((n_kt, 4), dtype=np.int64)
    for k in range(n_kt):
        mt = [t for t in range(n_mt) if qt[t, 0] <= k < qt[t, 3]]
        bt = [t for t in range(n_bt) if qt[n_mt + t, 0] <= k < qt[n_mt + t, 3]]
        kv_main[k] = (*tile_range(mt), *tile_range(bt))
    kv_branch = np.zeros((n_bkt, 2), dtype=np.int64)
    for k in range(n_bkt):
        lo, hi = k * BN, min((k + 1) * BN, nb)
        bt = [t for t in range(n_bt) if qt[n_mt + t, 4] < hi and qt[n_mt + t, 5] > lo]
        kv_branch[k] = tile_range(bt)

    fwd_cost = (qt[:, 3] - qt[:, 0]) + (qt[:, 5] - qt[:, 4] + BN - 1) // BN
    bwd_cost = np.concatenate([(kv_main[:, 1] - kv_main[:, 0]) + (kv_main[:, 3] - kv_main[:, 2]),
                               kv_branch[:, 1] - kv_branch[:, 0]])
    fwd_order = np.argsort(-fwd_cost, kind="stable")
    bwd_order = np.argsort(-bwd_cost, kind="stable")
    return {
        "cu_branch": dv.cu_branch.copy(),
        "branch_seq": dv.branch_seq.copy(),
        "row_iv": row_intervals(st),
        "qtile": qt,
        "kv_main": kv_main,
        "kv_branch": kv_branch,
        "fwd_order": fwd_order.astype(np.int64),
        "bwd_order": bwd_order.astype(np.int64),
    }
