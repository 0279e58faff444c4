"""Pins of the per-shard work count (oracle/shard_study.py) against brute
force over the explicit mask, the total pair count, and closed forms."""
import numpy as np
import pytest

import oracle
import workloads as wl
from oracle import shard_study as ss


def _brute(st, C, order):
    """Loop over the explicit mask: query row -> its shard, main key column ->
    its shard; branch-key columns count on the query's own shard."""
    dv = oracle.derive(st)
    mask = oracle.dense_mask(st, dv)
    n = dv.n_main
    cu = np.asarray(dv.cu)
    pieces = 2 * C if order == "zigzag" else C

    def shard_of(pos, s):
        start, L = int(cu[s]), int(cu[s + 1] - cu[s])
        for k in range(pieces):
            if start + (k * L) // pieces <= pos < start + ((k + 1) * L) // pieces:
                return (k if k < C else 2 * C - 1 - k) if order == "zigzag" else k
        raise AssertionError("position outside its sequence")

    W = np.zeros((C, C), dtype=np.int64)
    anchors = np.asarray(st.anchors)
    for r in range(mask.shape[0]):
        if r < n:
            s, pos = int(dv.main_seq[r]), r
        else:
            b = int(dv.row_branch[r - n])
            s, pos = int(dv.branch_seq[b]), int(anchors[b])
        i = shard_of(pos, s)
        for k in np.nonzero(mask[r, :n])[0]:
            W[i, shard_of(int(k), int(dv.main_seq[k]))] += 1
        W[i, i] += int(mask[r, n:].sum())
    return W * st.hq


@pytest.mark.parametrize("seed,kind", [(1, 0), (2, 1), (3, 2), (4, 0)])
@pytest.mark.parametrize("C", [1, 2, 3])
@pytest.mark.parametrize("order", ss.ORDERS)
def test_matches_brute_force(seed, kind, C, order):
    st = wl.random_structure(seed, n_seqs=3, max_len=30, mask_kind=kind)
    np.testing.assert_array_equal(ss.pair_matrix(st, C, order, block=7), _brute(st, C, order))


@pytest.mark.parametrize("order", ss.ORDERS)
def test_total_is_the_useful_pair_count(order):
    st = wl.structure("tiny_ttt")
    for C in (1, 2, 4, 8):
        assert ss.pair_matrix(st, C, order).sum() == oracle.useful_pairs(st)


def _single_causal(L):
    return wl.Structure("causal", np.array([0, L]), np.zeros(0, dtype=np.int64),
                        np.zeros(0, dtype=np.int64), 1, 1, 8, 0)


@pytest.mark.parametrize("C", [2, 4, 8])
def test_single_causal_sequence_closed_forms(C):
    L = 2 * C * 37
    st = _single_causal(L)
    zz = ss.pair_matrix(st, C, "zigzag")
    seq = ss.pair_matrix(st, C, "sequential")
    # zigzag: every shard does exactly L (L + 1) / (2C) pairs
    assert np.all(zz.sum(axis=1) == L * (L + 1) // (2 * C))
    # sequential: shard i's rows [a, b) see r + 1 keys each; no key of a later shard
    m = L // C
    totals = []
    for i in range(C):
        a, b = i * m, (i + 1) * m
        totals.append((b * (b + 1) - a * (a + 1)) // 2)
        assert seq[i].sum() == totals[-1]
        assert np.all(seq[i, i + 1:] == 0)
    assert ss.imbalance(zz)["total_max_over_mean"] == 1.0
    assert ss.imbalance(seq)["total_max_over_mean"] == pytest.approx(
        max(totals) / (sum(totals) / C), rel=1e-12)


@pytest.mark.parametrize("C", [2, 4])
def test_prefix_differences_give_the_shard_totals(C):
    """bench.py's shard timing turns totals over the 2C prefixes of one sequence
    into per-shard sums; fed each prefix's useful-pair count it must give the
    pair matrix's shard totals, for both orders (the decomposition behind the
    measured per-shard times)."""
    import dataclasses
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    L = 2 * C * 48
    base = dataclasses.replace(wl.truncate(wl.structure("ttt_256k"), L), zigzag_C=1)
    prefix = [0] + [oracle.useful_pairs(wl.truncate(base, k * L // (2 * C)))
                    for k in range(1, 2 * C + 1)]
    split = bench.shard_split(prefix, C)
    for order in ss.ORDERS:
        np.testing.assert_array_equal(split[order], ss.pair_matrix(base, C, order).sum(axis=1))
    with pytest.raises(ValueError):
        bench.shard_split(prefix[:-1], C)


@pytest.mark.parametrize("name", ["ttt_20k", "dflash_32k"])
def test_packed_prefix_differences_give_the_shard_totals(name):
    """The packed-batch form of the same decomposition: every sequence cut to
    its first k of 2C chunks (workloads.truncate_each); the differences of the
    prefixes' pair counts, split by bench.shard_split, equal the pair matrix's
    shard totals for both orders, for C = 8 and for C = 4, 2 from every second
    or fourth prefix (the subsampling bench.py's shard timing uses)."""
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    st = wl.structure(name)
    C = 8
    prefix = [0] + [oracle.useful_pairs(wl.truncate_each(st, k, 2 * C)[0])
                    for k in range(1, 2 * C + 1)]
    assert prefix[-1] == oracle.useful_pairs(st)
    for c in (8, 4, 2):
        split = bench.shard_split(prefix[::C // c], c)
        for order in ss.ORDERS:
            np.testing.assert_array_equal(split[order], ss.pair_matrix(st, c, order).sum(axis=1))


def test_truncate_each_keeps_rows_and_branches():
    st = wl.random_structure(5, n_seqs=4, max_len=50, max_depth=4, branch_prob=0.5)
    sub, mr, br = wl.truncate_each(st, 3, 8)
    lens = np.diff(st.cu_seqlens)
    kept = (3 * lens) // 8
    assert sub.n_main == kept.sum() == len(mr)
    assert sub.n_branch_tokens == len(br)
    # the kept branches are exactly those anchored in kept rows, in order, with
    # their anchors re-indexed into the kept rows and their own rows gathered
    sel = np.nonzero(np.isin(st.anchors, mr))[0]
    np.testing.assert_array_equal(mr[sub.anchors], st.anchors[sel])
    np.testing.assert_array_equal(sub.depths, st.depths[sel])
    dv = oracle.derive(st)
    rows = [np.arange(dv.cu_branch[b], dv.cu_branch[b + 1]) for b in sel]
    np.testing.assert_array_equal(br, np.concatenate(rows) if rows else np.zeros(0, int))
    assert np.all(np.diff(sub.cu_seqlens) > 0)
