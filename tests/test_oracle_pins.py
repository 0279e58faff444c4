"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute itself: a
hand-worked fixture, a library routine on a special case (causal SDPA), a
closed form, finite differences, or brute-force enumeration.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
KINDS = (wl.MASK_TTT_CAUSAL, wl.MASK_BLOCK_BIDIR, wl.MASK_BLOCK_CAUSAL)


def _f64_tensors(st, seed):
    rng = np.random.default_rng(seed)
    return {k: rng.standard_normal(shape) for k, shape in wl.tensor_shapes(st).items()}


def _rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    den = max(np.abs(b).max(), 1e-300)
    return np.abs(a - b).max() / den


# ---------------------------------------------------------------- merge rule
def test_lse_merge_golden():
    """Hand-worked merges (technical-contribution section of the paper pages)."""
    rows = []
    with open(os.path.join(GOLDEN, "lse_merge_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    assert len(rows) == 6
    for r in rows:
        la, lb, oa, ob, l_ref, o_ref = r[0], r[1], r[2:4], r[4:6], r[6], r[7:9]
        o, l = oracle.lse_merge(np.array([oa]), np.array([la]), np.array([ob]), np.array([lb]))
        if math.isinf(l_ref):
            assert np.isneginf(l[0])
        else:
            assert abs(l[0] - l_ref) <= 1e-12 * max(1.0, abs(l_ref))
        np.testing.assert_allclose(o[0], o_ref, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_union_softmax_equals_split_merge(kind, seed):
    """(a) softmax over the union of keys == LSE merge of the two split partials."""
    st = wl.random_structure(seed, n_seqs=3, max_len=20, max_depth=5, hq=4, hkv=2,
                             head_dim=8, mask_kind=kind)
    t = _f64_tensors(st, seed)
    ref = oracle.forward_dense(st, t)
    merged, pm, pb = oracle.split_forward(st, t)
    for a, b in zip(merged, ref):
        assert _rel(a, b) <= 1e-12
    # the split really is a split: main rows have an empty branch partial
    assert np.all(np.isneginf(pb[2]))
    assert np.all(np.isfinite(pm[2])) and np.all(np.isfinite(pm[3]))


# ------------------------------------------------------- library special cases
def _sdpa(q, k, v, scale, causal):
    """torch SDPA in fp64; q [R, d], k/v [T, d]."""
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None], is_causal=causal, scale=scale)
    return out[0, 0].numpy()


@pytest.mark.parametrize("seed", [0, 1])
def test_branch_free_is_causal_sdpa(seed):
    """(b) with no branches the path is plain causal attention per sequence."""
    st = wl.random_structure(seed, n_seqs=4, max_len=30, hq=4, hkv=2, head_dim=16,
                             branch_prob=0.0)
    assert st.n_branches == 0
    t = _f64_tensors(st, seed)
    o_m, o_b, lse_m, _ = oracle.forward_dense(st, t)
    assert o_b.shape[0] == 0
    cu = st.cu_seqlens
    for s in range(st.n_seqs):
        lo, hi = cu[s], cu[s + 1]
        for h in range(st.hq):
            g = h // (st.hq // st.hkv)
            ref = _sdpa(t["q_m"][lo:hi, h], t["k_m"][lo:hi, g], t["v_m"][lo:hi, g],
                        st.scale, True)
            np.testing.assert_allclose(o_m[lo:hi, h], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", KINDS)
def test_branch_rows_are_sdpa_over_concatenated_keys(kind):
    """A branch query equals unmasked SDPA of that one query over
    main[seq start .. anchor] ++ own branch keys (depth <= own for the causal
    kinds, the whole block for block-bidirectional)."""
    st = wl.random_structure(7, n_seqs=3, max_len=25, max_depth=6, hq=2, hkv=1,
                             head_dim=8, mask_kind=kind, branch_prob=0.7)
    t = _f64_tensors(st, 7)
    _, o_b, _, _ = oracle.forward_dense(st, t)
    cu = st.cu_seqlens
    row = 0
    for b in range(st.n_branches):
        a = int(st.anchors[b])
        s = int(np.searchsorted(cu, a, side="right") - 1)
        for j in range(int(st.depths[b])):
            upto = int(st.depths[b]) if kind == wl.MASK_BLOCK_BIDIR else j + 1
            rows = slice(row - j, row - j + upto)
            for h in range(st.hq):
                k = np.concatenate([t["k_m"][cu[s]:a + 1, 0], t["k_b"][rows, 0]])
                v = np.concatenate([t["v_m"][cu[s]:a + 1, 0], t["v_b"][rows, 0]])
                ref = _sdpa(t["q_b"][row:row + 1, h], k, v, st.scale, False)
                np.testing.assert_allclose(o_b[row, h], ref[0], rtol=1e-12, atol=1e-12)
            row += 1


# ------------------------------------------------------------ zigzag sharding
@pytest.mark.parametrize("kind", KINDS)
def test_zigzag_invariant_to_shard_count(kind):
    """(c) the C-shard zigzag ring merged by LSE equals the monolithic result."""
    st = wl.random_structure(3, n_seqs=2, max_len=40, max_depth=4, hq=2, hkv=1,
                             head_dim=8, mask_kind=kind)
    t = _f64_tensors(st, 3)
    ref = oracle.forward_dense(st, t)
    for C in (1, 2, 4, 8):
        out = oracle.zigzag_forward(st, t, C)
        for a, b in zip(out, ref):
            assert _rel(a, b) <= 1e-12, C


def test_zigzag_chunks_shape():
    """Chunk boundaries floor(kL/2C): 16 equal chunks of 16384 at 262,144 tokens."""
    ch = oracle.zigzag_chunks(np.array([0, 262144]), 8)[0]
    assert len(ch) == 16
    assert all(hi - lo == 16384 for lo, hi in ch)
    ch = oracle.zigzag_chunks(np.array([0, 10]), 2)[0]
    assert ch == [(0, 2), (2, 5), (5, 7), (7, 10)]


# -------------------------------------------------------------- gradients
@pytest.mark.parametrize("kind", KINDS)
def test_gradients_central_differences(kind):
    """(d) analytic dQ/dK/dV == central finite differences of sum(O * dO)."""
    st = wl.Structure("fd", np.array([0, 5, 12]), np.array([1, 4, 6, 9]),
                      np.array([2, 1, 3, 2]), 2, 1, 4, kind)
    t = _f64_tensors(st, 11)
    grads = oracle.backward_dense(st, t)
    names = ("q_m", "k_m", "v_m", "q_b", "k_b", "v_b")

    def loss(tt):
        o_m, o_b, _, _ = oracle.forward_dense(st, tt)
        return float((o_m * tt["do_m"]).sum() + (o_b * tt["do_b"]).sum())

    h = 1e-6
    for name, g in zip(names, grads):
        fd = np.zeros_like(t[name])
        for idx in np.ndindex(*t[name].shape):
            tp = dict(t)
            tp[name] = t[name].copy()
            tp[name][idx] += h
            lp = loss(tp)
            tp[name][idx] -= 2 * h
            lm = loss(tp)
            fd[idx] = (lp - lm) / (2 * h)
        assert _rel(g, fd) <= 1e-6, name


@pytest.mark.parametrize("kind", KINDS)
def test_gradients_match_autograd(kind):
    """Analytic gradients == torch autograd through a dense fp64 masked softmax
    whose mask is built here from the per-row rule, not by the oracle."""
    st = wl.random_structure(5, n_seqs=2, max_len=15, max_depth=4, hq=4, hkv=2,
                             head_dim=8, mask_kind=kind)
    t = _f64_tensors(st, 5)
    n, nb = st.n_main, st.n_branch_tokens
    cu = st.cu_seqlens
    seq_of = np.searchsorted(cu, np.arange(n), side="right") - 1
    mask = np.zeros((n + nb, n + nb), dtype=bool)
    pos = np.arange(n)
    for r in range(n):
        mask[r, :n] = (seq_of == seq_of[r]) & (pos <= r)
    row = 0
    for b in range(st.n_branches):
        a, D = int(st.anchors[b]), int(st.depths[b])
        for j in range(D):
            mask[n + row, :n] = (seq_of == seq_of[a]) & (pos <= a)
            hi = D if kind == wl.MASK_BLOCK_BIDIR else j + 1
            mask[n + row, n + row - j:n + row - j + hi] = True
            row += 1
    tt = {k: torch.tensor(v, requires_grad=True) for k, v in t.items()}
    q = torch.cat([tt["q_m"], tt["q_b"]])
    k = torch.cat([tt["k_m"], tt["k_b"]]).repeat_interleave(st.hq // st.hkv, dim=1)
    v = torch.cat([tt["v_m"], tt["v_b"]]).repeat_interleave(st.hq // st.hkv, dim=1)
    s = torch.einsum("qhd,khd->hqk", q, k) * st.scale
    s = s.masked_fill(~torch.from_numpy(mask)[None], float("-inf"))
    o = torch.einsum("hqk,khd->qhd", torch.softmax(s, dim=-1), v)
    loss = (o * torch.cat([tt["do_m"], tt["do_b"]])).sum()
    loss.backward()
    grads = oracle.backward_dense(st, t)
    for name, g in zip(("q_m", "k_m", "v_m", "q_b", "k_b", "v_b"), grads):
        assert _rel(g, tt[name].grad.numpy()) <= 1e-12, name


# ---------------------------------------------------------- closed forms
def test_q_zero_gives_log_of_visible_count():
    """With Q = 0 every visible key has score 0, so l_i = ln(n_i) exactly;
    n_i in closed form for the tiny TTT batch: main position p sees p+1 keys,
    depth-j branch token at anchor p sees p+1 main keys and j+1 branch keys."""
    st = wl.structure("tiny_ttt")
    t = _f64_tensors(st, 0)
    t["q_m"][:] = 0.0
    t["q_b"][:] = 0.0
    _, _, lse_m, lse_b = oracle.forward_dense(st, t)
    exp_m, exp_b = [], []
    for L in (96, 160):
        for p in range(L):
            exp_m.append(p + 1)
            exp_b.extend([p + 2, p + 3, p + 4])
    np.testing.assert_allclose(lse_m, np.log(exp_m)[None].repeat(st.hq, 0), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse_b, np.log(exp_b)[None].repeat(st.hq, 0), rtol=0, atol=1e-13)


@pytest.mark.parametrize("kind", KINDS)
def test_constant_keys_average_visible_values(kind):
    """With every key equal, O_i is the plain mean of the V rows query i sees
    (DSpark-like block layout: anchors every 4th position, depth-3 blocks)."""
    cu = np.array([0, 12, 20])
    anchors = np.array([3, 7, 11, 15, 19])
    st = wl.Structure("constk", cu, anchors, np.full(5, 3), 2, 2, 8, kind)
    t = _f64_tensors(st, 2)
    t["k_m"][:] = 0.5
    t["k_b"][:] = 0.5
    o_m, o_b, _, _ = oracle.forward_dense(st, t)
    for r in range(20):
        lo = 0 if r < 12 else 12
        np.testing.assert_allclose(o_m[r], t["v_m"][lo:r + 1].mean(axis=0), rtol=1e-12, atol=1e-13)
    for b, a in enumerate(anchors):
        lo = 0 if a < 12 else 12
        for j in range(3):
            hi = 3 if kind == wl.MASK_BLOCK_BIDIR else j + 1
            vals = np.concatenate([t["v_m"][lo:a + 1], t["v_b"][3 * b:3 * b + hi]])
            np.testing.assert_allclose(o_b[3 * b + j], vals.mean(axis=0), rtol=1e-12, atol=1e-13)


def test_useful_pair_counts_closed_form():
    """Pair counts (x all q heads) against closed forms of each layout."""
    # tiny TTT: main sum L(L+1)/2, branches 3 L(L+1)/2 + 6 L per sequence, x 4 heads
    per = sum(4 * L * (L + 1) // 2 + 6 * L for L in (96, 160))
    assert per * 4 == 286720
    assert oracle.useful_pairs(wl.structure("tiny_ttt")) == 286720
    # DSpark 64K: main L(L+1)/2; branch at p=32k+31 depth 8 block-causal:
    # sum_k 8 (p+1) + 36, x 32 heads
    L = 65536
    per = L * (L + 1) // 2 + sum(8 * (32 * k + 32) + 36 for k in range(2048))
    assert per * 32 == 85911142400
    assert oracle.useful_pairs(wl.structure("dspark_64k")) == 85911142400
    # TTT 256K: one sequence, depth-3 TTT-causal branch at every position:
    # main L(L+1)/2; branch at p sees p+1 main keys at each of its 3 depths
    # (3 L(L+1)/2) plus 1+2+3 = 6 branch keys, x 32 heads
    L = 262144
    per = L * (L + 1) // 2 + 3 * L * (L + 1) // 2 + 6 * L
    assert per * 32 == 4398113619968
    assert oracle.useful_pairs(wl.structure("ttt_256k")) == 4398113619968


def test_useful_pairs_match_dense_mask():
    for kind in KINDS:
        st = wl.random_structure(9, mask_kind=kind, hq=3, hkv=1)
        assert oracle.useful_pairs(st) == int(oracle.dense_mask(st).sum()) * st.hq


# ---------------------------------------------------------- row-wise path
@pytest.mark.parametrize("kind", KINDS)
def test_rows_forward_matches_dense(kind):
    st = wl.random_structure(4, n_seqs=3, max_len=30, max_depth=5, hq=4, hkv=2,
                             head_dim=8, mask_kind=kind)
    t = _f64_tensors(st, 4)
    o_m, o_b, lse_m, lse_b = oracle.forward_dense(st, t)
    dq_m, dk_m, dv_m, dq_b, dk_b, dv_b = oracle.backward_dense(st, t)
    mr = list(range(0, st.n_main, 3))
    br = list(range(1, st.n_branch_tokens, 2))
    out = oracle.rows_backward_dq(st, t, mr, br)
    R = len(mr)
    np.testing.assert_allclose(out["o"][:R], o_m[mr], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["o"][R:], o_b[br], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["lse"][:, :R], lse_m[:, mr], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["lse"][:, R:], lse_b[:, br], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["dq"][:R], dq_m[mr], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out["dq"][R:], dq_b[br], rtol=1e-10, atol=1e-12)
    mk = [st.n_main - 1, st.n_main - 2, 5]
    bk = [0, st.n_branch_tokens - 1]
    kb = oracle.keys_backward(st, t, mk, bk)
    np.testing.assert_allclose(kb["dk_m"], dk_m[mk], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(kb["dv_m"], dv_m[mk], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(kb["dk_b"], dk_b[bk], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(kb["dv_b"], dv_b[bk], rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------- plan
@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("tile", [4, 8])
def test_plan_matches_bruteforce(kind, seed, tile):
    """Tile metadata == brute-force enumeration over the explicit mask."""
    st = wl.random_structure(seed, n_seqs=4, max_len=30, max_depth=6, mask_kind=kind,
                             branch_prob=0.6)
    BM = BN = tile
    p = oracle.plan(st, BM, BN)
    mask = oracle.dense_mask(st)
    n, nb = st.n_main, st.n_branch_tokens
    # per-row intervals: contiguous and equal to the mask rows
    iv = p["row_iv"]
    for r in range(n + nb):
        mk = np.nonzero(mask[r, :n])[0]
        lk = np.nonzero(mask[r, n:])[0]
        assert (mk.min(), mk.max()) == tuple(iv[r, :2]) and mk.size == mk.max() - mk.min() + 1
        if lk.size:
            assert (lk.min(), lk.max()) == tuple(iv[r, 2:])
            assert lk.size == lk.max() - lk.min() + 1
        else:
            assert tuple(iv[r, 2:]) == (0, -1)
    # per-key intervals: the mask column's main rows and branch rows, each
    # exactly the listed half-open range
    ki = p["key_iv"]
    for k in range(n + nb):
        col = mask[:, k]
        for part, (lo_r, hi_r) in ((slice(0, 2), (0, n)), (slice(2, 4), (n, n + nb))):
            rows = np.nonzero(col[lo_r:hi_r])[0]
            want = (int(rows.min()), int(rows.max()) + 1) if rows.size else (0, 0)
            assert tuple(ki[k, part]) == want, (k, part)
            assert rows.size == want[1] - want[0]
    n_mt = -(-n // BM)
    qt = p["qtile"]
    tiles = [(0, t * BM, min((t + 1) * BM, n)) for t in range(n_mt)]
    tiles += [(n, t * BM, min((t + 1) * BM, nb)) for t in range(-(-nb // BM))]
    for ti, (off, r0, r1) in enumerate(tiles):
        rows = mask[off + r0:off + r1]
        kv_b, f_b, f_e, kv_e, bl_b, bl_e = qt[ti]
        seen = np.nonzero(rows[:, :n].any(axis=0))[0]
        assert kv_b == seen.min() // BN and kv_e == seen.max() // BN + 1
        for k in range(-(-n // BN)):
            block = rows[:, k * BN:min((k + 1) * BN, n)]
            full = bool(block.all()) and (k + 1) * BN <= n
            assert full == (f_b <= k < f_e), (ti, k)
        if off == 0:
            assert (bl_b, bl_e) == (0, 0)
        else:
            own = set()
            for r in range(r0, r1):
                b = np.searchsorted(np.cumsum(st.depths), r, side="right")
                lo = int(np.concatenate([[0], np.cumsum(st.depths)])[b])
                own.update(range(lo, lo + int(st.depths[b])))
            assert (bl_b, bl_e) == (min(own), max(own) + 1)
    # backward ranges: exactly the query tiles whose kv range covers key tile k
    n_mt, n_bt = len([x for x in tiles if x[0] == 0]), len([x for x in tiles if x[0] == n])
    for k in range(-(-n // BN)):
        mt = [t for t in range(n_mt) if qt[t, 0] <= k < qt[t, 3]]
        bt = [t for t in range(n_bt) if qt[n_mt + t, 0] <= k < qt[n_mt + t, 3]]
        assert mt and mt == list(range(mt[0], mt[-1] + 1))
        assert tuple(p["kv_main"][k, :2]) == (mt[0], mt[-1] + 1)
        if bt:
            assert bt == list(range(bt[0], bt[-1] + 1))
            assert tuple(p["kv_main"][k, 2:]) == (bt[0], bt[-1] + 1)
        else:
            assert tuple(p["kv_main"][k, 2:]) == (0, 0)
        # every visible (row, key) pair in this key tile belongs to a listed tile
        cols = slice(k * BN, min((k + 1) * BN, n))
        rows_seen = np.nonzero(mask[:, cols].any(axis=1))[0]
        for r in rows_seen:
            t = r // BM if r < n else n_mt + (r - n) // BM
            if t < n_mt:
                assert p["kv_main"][k, 0] <= t < p["kv_main"][k, 1]
            else:
                assert p["kv_main"][k, 2] <= t - n_mt < p["kv_main"][k, 3]
    for k in range(-(-nb // BN)):
        cols = slice(n + k * BN, n + min((k + 1) * BN, nb))
        rows_seen = np.nonzero(mask[:, cols].any(axis=1))[0]
        ts = sorted({(r - n) // BM for r in rows_seen})
        assert all(r >= n for r in rows_seen)
        lo, hi = p["kv_branch"][k]
        assert lo <= ts[0] and ts[-1] < hi
    # work orders: permutations sorted by decreasing cost, ties by index
    for key, cost in (("fwd_order", (qt[:, 3] - qt[:, 0]) + (qt[:, 5] - qt[:, 4] + BN - 1) // BN),
                      ("bwd_order", np.concatenate([
                          p["kv_main"][:, 1] - p["kv_main"][:, 0] + p["kv_main"][:, 3]
                          - p["kv_main"][:, 2], p["kv_branch"][:, 1] - p["kv_branch"][:, 0]]))):
        order = p[key]
        if key == "bwd_order":
            assert p["walk"] == int(cost.sum())
            # walk ahead of each position, summed one entry at a time
            ahead = 0
            for i, k in enumerate(order):
                assert p["bwd_prefix"][i] == ahead
                ahead += int(cost[k])
            assert ahead == p["walk"]
        assert sorted(order.tolist()) == list(range(cost.shape[0]))
        for i in range(len(order) - 1):
            a, b = order[i], order[i + 1]
            assert cost[a] > cost[b] or (cost[a] == cost[b] and a < b)


def test_zz_tiles_cover_every_ring_step_pair():
    """Each (row, key) pair the zigzag ring computes at step s lies inside the
    listed key tiles of the row's tile at step s, and every pair is computed at
    exactly one step."""
    st = wl.random_structure(6, n_seqs=3, max_len=45, max_depth=3, zigzag_C=3,
                             branch_prob=0.5)
    C, BM = 3, 8
    zz = oracle.plan(st, BM, BM)["zz_tiles"]
    dv = oracle.derive(st)
    n = dv.n_main
    chunks = oracle.zigzag_chunks(dv.cu, C)
    mask = oracle.dense_mask(st)
    n_mt = -(-n // BM)
    for r in range(n + dv.n_branch_tokens):
        own = r if r < n else int(st.anchors[dv.row_branch[r - n]])
        s = int(dv.main_seq[own])
        kc = next(k for k, (lo, hi) in enumerate(chunks[s]) if lo <= own < hi)
        shard = kc if kc < C else 2 * C - 1 - kc
        t = r // BM if r < n else n_mt + (r - n) // BM
        seen = np.zeros(n, dtype=int)
        for step in range(C):
            j = (shard - step) % C
            for w, ch in enumerate((j, 2 * C - 1 - j)):
                lo, hi = chunks[s][ch]
                keys = [k for k in range(lo, hi) if mask[r, k]]
                seen[keys] += 1
                for k in keys:
                    assert zz[step, t, 2 * w] <= k // BM < zz[step, t, 2 * w + 1]
        np.testing.assert_array_equal(seen, mask[r, :n].astype(int))


# ---------------------------------------------------------- zero queries (closed form)
@pytest.mark.parametrize("kind", KINDS)
def test_visible_counts_match_dense_mask(kind):
    st = wl.random_structure(17, n_seqs=3, max_len=40, max_depth=6, mask_kind=kind)
    n_m, n_b = oracle.visible_counts(st)
    rows = oracle.dense_mask(st).sum(axis=1)
    np.testing.assert_array_equal(np.concatenate([n_m, n_b]), rows)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("seed", [0, 1])
def test_zero_query_dv_matches_dense_backward(kind, seed):
    """With Q = 0 the dense backward (explicit mask, analytic gradients) gives
    dV = the suffix-sum closed form and dK = 0, for every main and branch key."""
    st = wl.random_structure(30 + seed, n_seqs=3, max_len=25, max_depth=5, hq=4, hkv=2,
                             head_dim=8, mask_kind=kind, branch_prob=0.6)
    t = _f64_tensors(st, 40 + seed)
    t["q_m"][:] = 0.0
    t["q_b"][:] = 0.0
    dq_m, dk_m, dv_m, dq_b, dk_b, dv_b = oracle.backward_dense(st, t)
    got_m, got_b = oracle.zero_query_dv(st, t)
    np.testing.assert_allclose(got_m, dv_m, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got_b, dv_b, rtol=1e-12, atol=1e-12)
    assert np.abs(dk_m).max() == 0.0 and np.abs(dk_b).max() == 0.0
    # a subset of groups fills only those groups
    part_m, part_b = oracle.zero_query_dv(st, t, groups=[1])
    np.testing.assert_allclose(part_m[:, 1], dv_m[:, 1], rtol=1e-12, atol=1e-12)
    assert np.abs(part_m[:, 0]).max() == 0.0 and np.abs(part_b[:, 0]).max() == 0.0


# ---------------------------------------------------------- bf16 operand model
def test_round_bf16_is_round_to_nearest_even():
    # values on the bf16 grid stay; midpoints go to the even neighbour
    assert oracle.round_bf16(np.array([1.0, 1.0 + 2 ** -7]))[1] == 1.0 + 2 ** -7
    assert oracle.round_bf16(np.array([1.0 + 2 ** -8]))[0] == 1.0          # tie -> even
    assert oracle.round_bf16(np.array([1.0 + 3 * 2 ** -8]))[0] == 1.0 + 2 ** -6
    x = np.random.default_rng(0).standard_normal(1000)
    r = oracle.round_bf16(x)
    assert np.all(np.abs(r - x) <= np.abs(x) * 2 ** -8)


@pytest.mark.parametrize("kind", KINDS)
def test_keys_backward_with_bf16_operands_matches_dense(kind):
    """operand_bf16=True equals the dense definition with P and dS rounded to
    bf16 and D taken from the bf16-rounded O (explicit mask, union softmax,
    dense products)."""
    st = wl.random_structure(23, n_seqs=2, max_len=20, max_depth=4, hq=4, hkv=2, head_dim=8,
                             mask_kind=kind, branch_prob=0.6)
    t = _f64_tensors(st, 5)
    dvr = oracle.derive(st)
    mask = oracle.dense_mask(st, dvr)
    n = dvr.n_main
    q = np.concatenate([t["q_m"], t["q_b"]])
    k = np.concatenate([t["k_m"], t["k_b"]])
    v = np.concatenate([t["v_m"], t["v_b"]])
    do = np.concatenate([t["do_m"], t["do_b"]])
    grp = st.hq // st.hkv
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for h in range(st.hq):
        g = h // grp
        s = st.scale * q[:, h] @ k[:, g].T
        s = np.where(mask, s, -np.inf)
        lse = np.log(np.exp(s - s.max(1, keepdims=True)).sum(1)) + s.max(1)
        p = np.where(mask, np.exp(s - lse[:, None]), 0.0)
        o = oracle.round_bf16(p @ v[:, g])          # the forward's bf16 output
        ds = p * (do[:, h] @ v[:, g].T - (do[:, h] * o).sum(1)[:, None])
        dv[:, g] += oracle.round_bf16(p).T @ do[:, h]
        dk[:, g] += st.scale * oracle.round_bf16(ds).T @ q[:, h]
    mk = list(range(n))
    bk = list(range(dvr.n_branch_tokens))
    got = oracle.keys_backward(st, t, mk, bk, operand_bf16=True)
    np.testing.assert_allclose(got["dv_m"], dv[:n], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dk_m"], dk[:n], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dv_b"], dv[n:], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dk_b"], dk[n:], rtol=1e-12, atol=1e-12)
