"""Zigzag ring across ranks, host side (no GPU).

- The library's shard helper (ba_zigzag_shard, host C code) against the
  oracle's brute-force shard; its argument checks.
- The oracle's ring-step intervals partition every row's visible main keys.
- RingSchedule (the K/V rotation of one rank) with 2 and 4 gloo ranks: every
  rank meets the shards in the order (rank - t) mod C, with their data; and
  the whole decomposition (per-step partials over the received shard, merged
  by the LSE rule, branch-local partial last) equals the dense forward.
"""
import os
import socket

import numpy as np
import pytest

import oracle
import speculative_draft_branch_b200 as ba
import workloads as wl
from oracle import ring as oring

KINDS = (wl.MASK_TTT_CAUSAL, wl.MASK_BLOCK_BIDIR, wl.MASK_BLOCK_CAUSAL)


def _long_enough(seed, C, kind, n_seqs=3, max_len=40, hq=2, hkv=1, d=8, p=0.5):
    """Random batch whose sequences all hold at least 2C tokens."""
    st = wl.random_structure(seed, n_seqs=n_seqs, max_len=max_len, max_depth=4, hq=hq, hkv=hkv,
                             head_dim=d, mask_kind=kind, branch_prob=p)
    lens = np.maximum(np.diff(st.cu_seqlens), 2 * C)
    cu = np.concatenate([[0], np.cumsum(lens)])
    rng = np.random.default_rng(seed)
    anchors = np.sort(np.nonzero(rng.random(int(cu[-1])) < p)[0])
    depths = rng.integers(1, 5, size=anchors.shape[0])
    return wl.Structure(f"ring{seed}", cu, anchors, depths, hq, hkv, d, kind)


@pytest.mark.parametrize("C", [1, 2, 3, 4])
@pytest.mark.parametrize("kind", KINDS)
def test_shard_helper_matches_oracle(C, kind):
    st = _long_enough(3 + C, C, kind)
    for q in range(C):
        got = ba.ba_zigzag_shard(st.cu_seqlens, st.anchors, st.depths, C, q)
        ref = oring.shard(st, C, q)
        for key in ("main_rows", "branch_rows", "cu_local", "anchor_local", "depth_local"):
            np.testing.assert_array_equal(got[key], ref[key], err_msg=f"C={C} q={q} {key}")
    # the shards partition the batch's rows
    rows = np.concatenate([ba.ba_zigzag_shard(st.cu_seqlens, st.anchors, st.depths, C, q)
                           ["main_rows"] for q in range(C)])
    np.testing.assert_array_equal(np.sort(rows), np.arange(st.n_main))


def test_shard_helper_rejects_bad_input():
    cu = np.array([0, 10, 13])
    an, de = np.array([2]), np.array([3])
    with pytest.raises(ba.BranchAttnError) as e:        # 3 tokens < 2C = 4
        ba.ba_zigzag_shard(cu, an, de, 2, 0)
    assert e.value.status == -2
    for C, q in ((0, 0), (2, 2), (65, 0), (2, -1)):
        with pytest.raises(ba.BranchAttnError) as e:
            ba.ba_zigzag_shard(np.array([0, 10, 20]), an, de, C, q)
        assert e.value.status == -1


@pytest.mark.parametrize("C", [2, 3, 4])
@pytest.mark.parametrize("kind", KINDS)
def test_step_intervals_partition_the_visible_keys(C, kind):
    """Over the C steps a row's intervals (in the visiting shards' local rows,
    mapped back to batch rows) are disjoint and cover exactly its visible main
    keys."""
    st = _long_enough(11 + C, C, kind, max_len=30)
    dv = oracle.derive(st)
    for q in range(C):
        sq = oring.shard(st, C, q)
        rows = [("main", int(r)) for r in sq["main_rows"]] + \
               [("branch", int(r)) for r in sq["branch_rows"]]
        seen = [[] for _ in rows]
        for step in range(C):
            j = (q - step) % C
            back = oring.shard(st, C, j)["main_rows"]
            for i, (lo, hi) in enumerate(oring.step_intervals(st, C, q, step)):
                seen[i].extend(int(x) for x in back[lo:hi + 1])
        for i, (kind_r, r) in enumerate(rows):
            mk, _ = oracle.visible_keys(st, dv, kind_r, r)
            assert sorted(seen[i]) == sorted(int(k) for k in mk), (q, kind_r, r)


# ---------------------------------------------------------------- gloo ranks
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _attend(q, k, v, iv, scale):
    """Partial softmax attention of rows q [R, d] over keys k/v [T, d] rows
    lo..hi of each row (empty: O = 0, l = -inf)."""
    R, d = q.shape
    o, lse = np.zeros((R, d)), np.full(R, -np.inf)
    for i in range(R):
        lo, hi = int(iv[i, 0]), int(iv[i, 1])
        if hi < lo:
            continue
        s = scale * (k[lo:hi + 1] @ q[i])
        m = s.max()
        p = np.exp(s - m)
        o[i] = p @ v[lo:hi + 1] / p.sum()
        lse[i] = m + np.log(p.sum())
    return o, lse


def _rank_main(rank, world, port, case, results):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        C = world
        st = _long_enough(40 + C, C, case["kind"], n_seqs=2, max_len=24, hq=2, hkv=1, d=8)
        rng = np.random.default_rng(7)
        t = {key: rng.standard_normal(shape) for key, shape in wl.tensor_shapes(st).items()}
        me = oring.shard(st, C, rank)
        rows = [len(oring.shard(st, C, j)["main_rows"]) for j in range(C)]
        # this rank's shard of K / V, tagged so the receiver can tell whose it is
        k_loc = torch.tensor(t["k_m"][me["main_rows"], 0], dtype=torch.float64)
        v_loc = torch.tensor(t["v_m"][me["main_rows"], 0], dtype=torch.float64)
        q_rows = np.concatenate([t["q_m"][me["main_rows"]], t["q_b"][me["branch_rows"]]])
        nloc = q_rows.shape[0]
        acc_o = np.zeros((st.hq, nloc, st.head_dim))
        acc_l = np.full((st.hq, nloc), -np.inf)
        seen = []

        def step_fn(step, j, k, v):
            nonlocal acc_o, acc_l
            ref = oring.shard(st, C, j)["main_rows"]
            # the received shard is shard j's data, rows in j's local order
            assert np.array_equal(k.numpy(), t["k_m"][ref, 0])
            seen.append(j)
            iv = oring.step_intervals(st, C, rank, step)
            for h in range(st.hq):
                o, l = _attend(q_rows[:, h], k.numpy(), v.numpy(), iv, st.scale)
                a_o, a_l = oracle.lse_merge(acc_o[h:h + 1], acc_l[h:h + 1], o[None], l[None])
                acc_o[h], acc_l[h] = a_o[0], a_l[0]

        def alloc(n):
            return (torch.empty((n, st.head_dim), dtype=torch.float64),
                    torch.empty((n, st.head_dim), dtype=torch.float64))

        order = ba.ring.RingSchedule(C, rank, rows).run(k_loc, v_loc, step_fn, alloc)
        # branch-local partial last (own branch keys of each branch row)
        dv = oracle.derive(st)
        n_m = len(me["main_rows"])
        kb = t["k_b"][:, 0]
        vb = t["v_b"][:, 0]
        for h in range(st.hq):
            for i, r in enumerate(me["branch_rows"]):
                _, lk = oracle.visible_keys(st, dv, "branch", int(r))
                o, l = _attend(q_rows[n_m + i:n_m + i + 1, h], kb[lk], vb[lk],
                               np.array([[0, len(lk) - 1]]), st.scale)
                a_o, a_l = oracle.lse_merge(acc_o[h:h + 1, n_m + i:n_m + i + 1],
                                            acc_l[h:h + 1, n_m + i:n_m + i + 1], o[None], l[None])
                acc_o[h, n_m + i], acc_l[h, n_m + i] = a_o[0, 0], a_l[0, 0]
        o_m, o_b, l_m, l_b = oracle.forward_dense(st, t)
        ref_o = np.concatenate([o_m[me["main_rows"]], o_b[me["branch_rows"]]]).transpose(1, 0, 2)
        ref_l = np.concatenate([l_m[:, me["main_rows"]], l_b[:, me["branch_rows"]]], axis=1)
        err = max(np.abs(acc_o - ref_o).max(), np.abs(acc_l - ref_l).max())
        results.put((rank, order, seen, float(err)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("kind", KINDS)
def test_ring_schedule_over_gloo_ranks(world, kind):
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, {"kind": kind}, results))
             for r in range(world)]
    for p in procs:
        p.start()
    import queue
    import time
    out, deadline = [], time.time() + 240
    while len(out) < world:
        try:
            out.append(results.get(timeout=2))
        except queue.Empty:
            dead = [p.exitcode for p in procs if p.exitcode not in (None, 0)]
            assert not dead and time.time() < deadline, f"rank processes failed: {dead}"
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, order, seen, err in out:
        expect = [(rank - t) % world for t in range(world)]
        assert order == expect and seen == expect
        assert err < 1e-12, (rank, err)
