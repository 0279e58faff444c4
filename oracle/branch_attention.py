"""fp64 CPU oracle: branch attention forward / backward written from its definition.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Source: "Online Draft Co-Training" paper pages (arXiv 2609.07108):
  - technical-contribution and method-detail sections: each branch query is the
    causal attention over the main sequence up to its anchor plus the
    attention over its own (rank-local) branch keys; the two partials
    (O_m, l_m) and (O_b, l_b) combine as l = log(e^{l_m} + e^{l_b}),
    O = e^{l_m - l} O_m + e^{l_b - l} O_b;
  - core-innovation section: zigzag sharding of the packed main sequence,
    branch K/V kept with the anchor's shard, main K/V visiting every shard.
Shapes of the three draft-branch kinds (TTT-causal, block-bidirectional,
block-causal) follow the EAGLE-3 / DFlash / DSpark description in the
research-background section.

Conventions (readings of the pages where they leave a point open):
  * main tokens t = 0..N-1 packed by cu_seqlens; branch b has anchor a_b and
    depth D_b, its tokens are branch rows cu_branch[b] .. cu_branch[b+1]-1
    (anchor-major, depth-minor);
  * main query r sees main keys of its own sequence at positions <= r;
  * branch query (b, j) sees main keys of the anchor's sequence at positions
    <= a_b (anchor inclusive) and branch keys (b, j') with j' <= j (TTT-causal,
    block-causal) or all j' (block-bidirectional);
  * scores S = scale * q . k, LSE in natural log with the scale included;
  * q head h reads kv head h // (Hq / Hkv).
Everything is computed in float64 from the exact bf16 input values.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Sequence, Tuple

import numpy as np

MASK_TTT_CAUSAL = 0
MASK_BLOCK_BIDIR = 1
MASK_BLOCK_CAUSAL = 2


def to64(x) -> np.ndarray:
    """bf16/fp32 torch tensor or numpy array -> float64 numpy (exact)."""
    if isinstance(x, np.ndarray):
        return x.astype(np.float64, copy=False)
    import torch
    return x.detach().to("cpu", torch.float64).numpy()


@dataclasses.dataclass
class Derived:
    cu: np.ndarray          # [S+1] cu_seqlens
    cu_branch: np.ndarray   # [n_br+1] exclusive scan of depths
    branch_seq: np.ndarray  # [n_br] sequence of each branch's anchor
    main_seq: np.ndarray    # [N] sequence of each main token
    row_branch: np.ndarray  # [Nb] branch of each branch row
    n_main: int
    n_branch_tokens: int


def derive(st) -> Derived:
    cu = np.asarray(st.cu_seqlens, dtype=np.int64)
    anchors = np.asarray(st.anchors, dtype=np.int64)
    depths = np.asarray(st.depths, dtype=np.int64)
    n = int(cu[-1])
    cu_branch = np.zeros(anchors.shape[0] + 1, dtype=np.int64)
    for b in range(anchors.shape[0]):
        cu_branch[b + 1] = cu_branch[b] + depths[b]
    main_seq = np.zeros(n, dtype=np.int64)
    for s in range(cu.shape[0] - 1):
        main_seq[cu[s]:cu[s + 1]] = s
    branch_seq = main_seq[anchors] if anchors.shape[0] else np.zeros(0, dtype=np.int64)
    nb = int(cu_branch[-1])
    row_branch = np.zeros(nb, dtype=np.int64)
    for b in range(anchors.shape[0]):
        row_branch[cu_branch[b]:cu_branch[b + 1]] = b
    return Derived(cu, cu_branch, branch_seq, main_seq, row_branch, n, nb)


def visible_keys(st, dv: Derived, kind: str, row: int) -> Tuple[np.ndarray, np.ndarray]:
    """Visible (main key indices, branch key rows) of one query row."""
    if kind == "main":
        s = dv.main_seq[row]
        return np.arange(dv.cu[s], row + 1), np.zeros(0, dtype=np.int64)
    b = dv.row_branch[row]
    a = int(st.anchors[b])
    s = dv.branch_seq[b]
    main = np.arange(dv.cu[s], a + 1)
    if st.mask_kind == MASK_BLOCK_BIDIR:
        loc = np.arange(dv.cu_branch[b], dv.cu_branch[b + 1])
    else:
        loc = np.arange(dv.cu_branch[b], row + 1)
    return main, loc


def dense_mask(st, dv: Derived = None) -> np.ndarray:
    """Explicit boolean mask over main+branch tokens: rows = queries, cols = keys.

    Index order on both axes: main tokens 0..N-1, then branch rows N..N+Nb-1.
    """
    dv = dv or derive(st)
    n, nb = dv.n_main, dv.n_branch_tokens
    m = np.zeros((n + nb, n + nb), dtype=bool)
    for r in range(n):
        mk, _ = visible_keys(st, dv, "main", r)
        m[r, mk] = True
    for r in range(nb):
        mk, lk = visible_keys(st, dv, "branch", r)
        m[n + r, mk] = True
        m[n + r, n + lk] = True
    return m


def _softmax_attend(s: np.ndarray, mask: np.ndarray, v: np.ndarray):
    """Masked softmax attention of score rows s [R, T] over values v [T, d].

    Rows with no visible key return O = 0 and lse = -inf (empty partial).
    """
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    empty = ~np.isfinite(m[:, 0])
    m = np.where(np.isfinite(m), m, 0.0)
    p = np.exp(s - m)
    z = p.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore"):
        lse = (m + np.log(z))[:, 0]
    lse[empty] = -np.inf
    zs = np.where(z > 0, z, 1.0)
    o = (p / zs) @ v
    o[empty] = 0.0
    return o, lse


def _all_tokens(t, keys: Sequence[str]):
    return [np.concatenate([to64(t[k + "_m"]), to64(t[k + "_b"])], axis=0) for k in keys]


def forward_dense(st, t, mask: np.ndarray = None):
    """Union-softmax forward over the explicit mask (small problems)."""
    dv = derive(st)
    mask = dense_mask(st, dv) if mask is None else mask
    q, k, v = _all_tokens(t, ["q", "k", "v"])
    hq, hkv = st.hq, st.hkv
    grp = hq // hkv
    n = dv.n_main
    o = np.zeros_like(q)
    lse = np.zeros((hq, q.shape[0]))
    for h in range(hq):
        g = h // grp
        s = st.scale * (q[:, h, :] @ k[:, g, :].T)
        o[:, h, :], lse[h] = _softmax_attend(s, mask, v[:, g, :])
    return o[:n], o[n:], lse[:, :n], lse[:, n:]


def backward_dense(st, t, mask: np.ndarray = None):
    """Analytic gradients of sum(O * dO) over the explicit mask (small problems).

    D_i = dO_i . O_i; dV = P^T dO; dP = dO V^T; dS = P (dP - D);
    dQ = scale dS K; dK = scale dS^T Q; dK/dV summed over each GQA group.
    """
    dv = derive(st)
    mask = dense_mask(st, dv) if mask is None else mask
    q, k, v, do = _all_tokens(t, ["q", "k", "v", "do"])
    hq, hkv = st.hq, st.hkv
    grp = hq // hkv
    n = dv.n_main
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    for h in range(hq):
        g = h // grp
        s = st.scale * (q[:, h, :] @ k[:, g, :].T)
        o, lse = _softmax_attend(s, mask, v[:, g, :])
        p = np.where(mask, np.exp(np.where(mask, s, 0.0) - lse[:, None]), 0.0)
        dd = (do[:, h, :] * o).sum(axis=1)
        dvv[:, g, :] += p.T @ do[:, h, :]
        dp = do[:, h, :] @ v[:, g, :].T
        ds = p * (dp - dd[:, None])
        dq[:, h, :] = st.scale * (ds @ k[:, g, :])
        dk[:, g, :] += st.scale * (ds.T @ q[:, h, :])
    return dq[:n], dk[:n], dvv[:n], dq[n:], dk[n:], dvv[n:]


def lse_merge(o_a, l_a, o_b, l_b):
    """Online-softmax merge of two partials (paper: technical contribution).

    l = log(e^{l_a} + e^{l_b}),  O = e^{l_a - l} O_a + e^{l_b - l} O_b,
    evaluated stably as l = m + log(e^{l_a - m} + e^{l_b - m}), m = max(l_a, l_b).
    An empty partial has l = -inf, O = 0; two empty partials give (0, -inf).
    Shapes: o_* [..., d], l_* [...].
    """
    o_a = np.asarray(o_a, dtype=np.float64)
    o_b = np.asarray(o_b, dtype=np.float64)
    l_a = np.asarray(l_a, dtype=np.float64)
    l_b = np.asarray(l_b, dtype=np.float64)
    m = np.maximum(l_a, l_b)
    both_empty = ~np.isfinite(m)
    ms = np.where(both_empty, 0.0, m)
    with np.errstate(divide="ignore"):
        l = ms + np.log(np.exp(l_a - ms) + np.exp(l_b - ms))
    l = np.where(both_empty, -np.inf, l)
    ls = np.where(both_empty, 0.0, l)
    wa = np.where(both_empty, 0.0, np.exp(l_a - ls))
    wb = np.where(both_empty, 0.0, np.exp(l_b - ls))
    o = wa[..., None] * o_a + wb[..., None] * o_b
    return o, l


def _partial_dense(st, t, mask, cols):
    """Partial attention of every query over the key columns selected by `cols`."""
    sub = mask & cols[None, :]
    return forward_dense(st, t, mask=sub)


def split_forward(st, t):
    """Main-prefix partial and branch-local partial, merged by the LSE rule.

    Returns (o_m, o_b, lse_m, lse_b) of the merged result plus the two partials.
    """
    dv = derive(st)
    mask = dense_mask(st, dv)
    n = dv.n_main
    total = mask.shape[1]
    is_main = np.arange(total) < n
    pm = _partial_dense(st, t, mask, is_main)
    pb = _partial_dense(st, t, mask, ~is_main)
    # merge per token group: o [rows, H, d], lse [H, rows]
    out = []
    for part in range(2):  # 0 = main rows, 1 = branch rows
        o_a, l_a = pm[part], pm[2 + part]
        o_b, l_b = pb[part], pb[2 + part]
        o, l = lse_merge(o_a.transpose(1, 0, 2), l_a, o_b.transpose(1, 0, 2), l_b)
        out.append((o.transpose(1, 0, 2), l))
    return (out[0][0], out[1][0], out[0][1], out[1][1]), pm, pb


def zigzag_chunks(cu: np.ndarray, C: int) -> List[List[Tuple[int, int]]]:
    """Chunk k of sequence s is [cu[s] + floor(k L / 2C), cu[s] + floor((k+1) L / 2C))."""
    out = []
    for s in range(cu.shape[0] - 1):
        start, L = int(cu[s]), int(cu[s + 1] - cu[s])
        out.append([(start + (k * L) // (2 * C), start + ((k + 1) * L) // (2 * C))
                    for k in range(2 * C)])
    return out


def _shard_of_chunk(k: int, C: int) -> int:
    return k if k < C else 2 * C - 1 - k


def zigzag_forward(st, t, C: int):
    """Virtual zigzag ring over C shards, merged by the LSE rule.

    Shard i holds chunks i and 2C-1-i of every sequence (core-innovation
    section: packed, load-balanced zigzag) and the branches anchored in them.
    At ring step s shard i attends its queries to the main keys held by shard
    (i - s) mod C under the global mask; the partials are merged in step order
    into a running (O, l), and the rank-local branch partial is merged last.
    """
    dv = derive(st)
    mask = dense_mask(st, dv)
    n, nb = dv.n_main, dv.n_branch_tokens
    chunks = zigzag_chunks(dv.cu, C)
    key_shard = np.full(n + nb, -1, dtype=np.int64)
    for s_chunks in chunks:
        for k, (lo, hi) in enumerate(s_chunks):
            key_shard[lo:hi] = _shard_of_chunk(k, C)
    q_shard = key_shard.copy()
    anchors = np.asarray(st.anchors, dtype=np.int64)
    for r in range(nb):
        q_shard[n + r] = key_shard[anchors[dv.row_branch[r]]]
    hq, d = st.hq, st.head_dim
    acc_o = np.zeros((hq, n + nb, d))
    acc_l = np.full((hq, n + nb), -np.inf)
    for step in range(C):
        for i in range(C):
            j = (i - step) % C
            rows = q_shard == i
            cols = key_shard == j  # branch columns are -1: never main keys of a shard
            sub = mask & rows[:, None] & cols[None, :]
            o_m, o_b, l_m, l_b = forward_dense(st, t, mask=sub)
            o = np.concatenate([o_m, o_b], axis=0).transpose(1, 0, 2)
            l = np.concatenate([l_m, l_b], axis=1)
            acc_o, acc_l = lse_merge(acc_o, acc_l, o, l)
    is_branch = np.arange(n + nb) >= n
    sub = mask & is_branch[None, :]
    o_m, o_b, l_m, l_b = forward_dense(st, t, mask=sub)
    o = np.concatenate([o_m, o_b], axis=0).transpose(1, 0, 2)
    l = np.concatenate([l_m, l_b], axis=1)
    acc_o, acc_l = lse_merge(acc_o, acc_l, o, l)
    acc_o = acc_o.transpose(1, 0, 2)
    return acc_o[:n], acc_o[n:], acc_l[:, :n], acc_l[:, n:]


# ---------------------------------------------------------------------------
# Row-wise evaluation for large problems (same definition, one query at a time
# or a batch of queries from one sequence, keys gathered per row).
# ---------------------------------------------------------------------------

def _row_sets(st, dv, main_rows, branch_rows):
    items = []
    for r in main_rows:
        mk, lk = visible_keys(st, dv, "main", int(r))
        items.append(("main", int(r), mk, lk))
    for r in branch_rows:
        mk, lk = visible_keys(st, dv, "branch", int(r))
        items.append(("branch", int(r), mk, lk))
    return items


# Rows of one sequence are scored together in batches of at most this many
# score-matrix entries (rows x main keys), so that full-size sequences fit in
# host memory; batching changes which rows share a matmul, not any value.
ROW_BATCH_ENTRIES = 1 << 24


def _row_batches(items, idx):
    """Split the row indices `idx` of one sequence into batches of rows with
    similar main-key counts, each batch's score matrix within ROW_BATCH_ENTRIES."""
    order = sorted(idx, key=lambda i: items[i][2].size)
    batches, cur, width = [], [], 0
    for i in order:
        w = max(width, items[i][2].size)
        if cur and w * (len(cur) + 1) > ROW_BATCH_ENTRIES:
            batches.append(cur)
            cur, w = [], items[i][2].size
        cur.append(i)
        width = w
    if cur:
        batches.append(cur)
    return batches


def rows_forward(st, t, main_rows=(), branch_rows=(), with_dq=False, heads=None):
    """Forward (and optionally dQ) of selected query rows, each over its own key set.

    Returns dict with o [R, Hq, d], lse [Hq, R] and, if with_dq, dq [R, Hq, d],
    in the order main_rows then branch_rows.  Only q heads in `heads` (default:
    all) are computed; the others stay zero.

    Rows reading the same sequence share one score matrix S = K_prefix q^T
    (a plain matmul, taken over batches of rows); each row then masks the keys
    it does not see (main keys past its own position / anchor) and appends its
    branch-local scores.
    """
    dv = derive(st)
    items = _row_sets(st, dv, main_rows, branch_rows)
    hq, hkv, d = st.hq, st.hkv, st.head_dim
    grp = hq // hkv
    heads = list(range(hq)) if heads is None else [int(h) for h in heads]
    R = len(items)
    o = np.zeros((R, hq, d))
    lse = np.zeros((hq, R))
    dq = np.zeros((R, hq, d)) if with_dq else None
    by_seq: Dict[int, List[int]] = {}
    for i, (kind, r, mk, lk) in enumerate(items):
        by_seq.setdefault(int(dv.main_seq[mk[0]]), []).append(i)
    groups = sorted({h // grp for h in heads})
    batches = [(s, b) for s, idx in by_seq.items() for b in _row_batches(items, idx)]
    for s, idx in batches:
        lo = int(dv.cu[s])
        hi = max(int(items[i][2][-1]) for i in idx) + 1
        nm = np.array([items[i][2].size for i in idx])            # main keys per row
        assert all(items[i][2][0] == lo for i in idx)
        visible = np.arange(hi - lo)[:, None] < nm[None, :]        # [L, R]
        qs = np.stack([to64(t["q_" + ("m" if items[i][0] == "main" else "b")][items[i][1]])
                       for i in idx])                              # [R, Hq, d]
        dos = np.stack([to64(t["do_" + ("m" if items[i][0] == "main" else "b")][items[i][1]])
                        for i in idx]) if with_dq else None
        for g in groups:
            km = to64(t["k_m"][lo:hi, g])                          # [L, d]
            vm = to64(t["v_m"][lo:hi, g])
            kl = [to64(t["k_b"][items[i][3], g]) for i in idx]     # per-row local keys
            vl = [to64(t["v_b"][items[i][3], g]) for i in idx]
            for h in heads:
                if h // grp != g:
                    continue
                sm = st.scale * (km @ qs[:, h, :].T)               # [L, R]
                sm = np.where(visible, sm, -np.inf)
                sl = [st.scale * (kl[c] @ qs[c, h]) for c in range(len(idx))]
                m = np.maximum(sm.max(axis=0),
                               np.array([x.max() if x.size else -np.inf for x in sl]))
                pm = np.exp(sm - m[None, :])
                pl = [np.exp(x - m[c]) for c, x in enumerate(sl)]
                z = pm.sum(axis=0) + np.array([x.sum() for x in pl])
                pm = pm / z[None, :]
                pl = [x / z[c] for c, x in enumerate(pl)]
                oo = pm.T @ vm + np.stack([pl[c] @ vl[c] for c in range(len(idx))])
                for c, i in enumerate(idx):
                    lse[h, i] = m[c] + np.log(z[c])
                    o[i, h] = oo[c]
                if with_dq:
                    dpm = vm @ dos[:, h, :].T                      # [L, R]
                    dd = (dos[:, h, :] * oo).sum(axis=1)
                    dsm = pm * (dpm - dd[None, :])
                    dqm = st.scale * (dsm.T @ km)
                    for c, i in enumerate(idx):
                        dsl = pl[c] * (vl[c] @ dos[c, h] - dd[c])
                        dq[i, h] = dqm[c] + st.scale * (dsl @ kl[c])
    out = {"o": o, "lse": lse}
    if with_dq:
        out["dq"] = dq
    return out


def rows_backward_dq(st, t, main_rows=(), branch_rows=(), heads=None):
    return rows_forward(st, t, main_rows, branch_rows, with_dq=True, heads=heads)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """x rounded to the nearest bf16 value (ties to even), back in fp64."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(
        torch.bfloat16).to(torch.float64).numpy()


def keys_backward(st, t, main_keys=(), branch_keys=(), groups=None, operand_bf16=False):
    """dK and dV of selected key rows, summed over every query that sees them.

    P_ik = exp(S_ik - l_i) needs only q_i, k and the query's LSE l_i, which
    rows_forward gives (with O_i for D_i = dO_i . O_i); so each query scores
    just the selected keys it sees: dV_k += P_ik dO_i, dK_k += scale dS_ik q_i,
    dS_ik = P_ik (dO_i . v_k - D_i).
    Returns dict with dk_m/dv_m [len(main_keys), Hkv, d] and dk_b/dv_b
    [len(branch_keys), Hkv, d]; only kv heads in `groups` (default: all) are
    computed, each summed over all q heads of its group.

    operand_bf16=True rounds P and dS to bf16 before they multiply dO and q,
    and takes D = dO . O from the bf16-rounded O (everything else stays fp64):
    the precision in which a bf16 tensor-core backward receives them (its O is
    the forward's bf16 output), so that a kernel's error can be separated from
    what the rounding of those operands alone causes.
    """
    return _keys_backward(st, t, main_keys, branch_keys, groups, (bool(operand_bf16),))[0]


def keys_backward_both(st, t, main_keys=(), branch_keys=(), groups=None):
    """keys_backward in fp64 and with bf16 operands, sharing the row forward:
    returns (exact, bf16_operands)."""
    return tuple(_keys_backward(st, t, main_keys, branch_keys, groups, (False, True)))


def _keys_backward(st, t, main_keys, branch_keys, groups, modes):
    dv = derive(st)
    hq, hkv, d = st.hq, st.hkv, st.head_dim
    grp = hq // hkv
    groups = list(range(hkv)) if groups is None else [int(g) for g in groups]
    heads = [h for h in range(hq) if h // grp in groups]
    main_keys = np.asarray([int(k) for k in main_keys], dtype=np.int64)
    branch_keys = np.asarray([int(k) for k in branch_keys], dtype=np.int64)
    anchors = np.asarray(st.anchors, dtype=np.int64)
    q_main, q_branch = set(), set()
    for k in main_keys:
        s = dv.main_seq[k]
        q_main.update(range(int(k), int(dv.cu[s + 1])))
        for b in np.nonzero((anchors >= k) & (dv.branch_seq == s))[0]:
            q_branch.update(range(int(dv.cu_branch[b]), int(dv.cu_branch[b + 1])))
    for k in branch_keys:
        b = dv.row_branch[k]
        q_branch.update(range(int(dv.cu_branch[b]), int(dv.cu_branch[b + 1])))
    q_main = sorted(q_main)
    q_branch = sorted(q_branch)
    fw = rows_forward(st, t, q_main, q_branch, heads=heads)
    items = _row_sets(st, dv, q_main, q_branch)
    R = len(items)
    # visibility of every selected key from every visiting row: main keys in
    # the row's main interval, branch keys in its branch-local interval
    m_lo = np.array([it[2][0] for it in items], dtype=np.int64)
    m_hi = np.array([it[2][-1] for it in items], dtype=np.int64)
    b_lo = np.array([it[3][0] if it[3].size else 0 for it in items], dtype=np.int64)
    b_hi = np.array([it[3][-1] if it[3].size else -1 for it in items], dtype=np.int64)
    vis_m = (main_keys[None, :] >= m_lo[:, None]) & (main_keys[None, :] <= m_hi[:, None])
    vis_b = (branch_keys[None, :] >= b_lo[:, None]) & (branch_keys[None, :] <= b_hi[:, None])
    qx = np.zeros((R, hq, d))
    dox = np.zeros((R, hq, d))
    for i, (kind, r, _, _) in enumerate(items):
        sfx = "m" if kind == "main" else "b"
        qx[i] = to64(t["q_" + sfx][r])
        dox[i] = to64(t["do_" + sfx][r])
    km_sel = to64(t["k_m"][main_keys]) if main_keys.size else np.zeros((0, hkv, d))
    vm_sel = to64(t["v_m"][main_keys]) if main_keys.size else np.zeros((0, hkv, d))
    kb_sel = to64(t["k_b"][branch_keys]) if branch_keys.size else np.zeros((0, hkv, d))
    vb_sel = to64(t["v_b"][branch_keys]) if branch_keys.size else np.zeros((0, hkv, d))
    res = [{"dk_m": np.zeros((main_keys.size, hkv, d)), "dv_m": np.zeros((main_keys.size, hkv, d)),
            "dk_b": np.zeros((branch_keys.size, hkv, d)), "dv_b": np.zeros((branch_keys.size, hkv, d))}
           for _ in modes]
    for h in heads:
        g = h // grp
        # D_i = dO_i . O_i; with bf16 operands O is the forward's bf16 output
        dd = {False: (dox[:, h] * fw["o"][:, h]).sum(axis=1)}
        if True in modes:
            dd[True] = (dox[:, h] * round_bf16(fw["o"][:, h])).sum(axis=1)
        for vis, ksel, vsel, kind in ((vis_m, km_sel, vm_sel, "m"), (vis_b, kb_sel, vb_sel, "b")):
            if ksel.shape[0] == 0:
                continue
            s_ik = st.scale * (qx[:, h] @ ksel[:, g].T)             # [R, keys]
            p = np.where(vis, np.exp(np.where(vis, s_ik, 0.0) - fw["lse"][h][:, None]), 0.0)
            dp = dox[:, h] @ vsel[:, g].T
            for out, rounded in zip(res, modes):
                ds = p * (dp - dd[rounded][:, None])
                pp, dss = (round_bf16(p), round_bf16(ds)) if rounded else (p, ds)
                out["dv_" + kind][:, g] += pp.T @ dox[:, h]
                out["dk_" + kind][:, g] += st.scale * (dss.T @ qx[:, h])
    return res


def useful_pairs(st) -> int:
    """Number of unmasked (query head, key) pairs, summed over all q heads.

    Main row r of sequence s: r - cu[s] + 1 keys.  Branch token j of branch b
    (anchor a in sequence s, depth D): a - cu[s] + 1 main keys plus j + 1
    (causal kinds) or D (block-bidirectional) branch keys.
    """
    dv = derive(st)
    main = int((np.arange(dv.n_main) - dv.cu[dv.main_seq] + 1).sum())
    anchors = np.asarray(st.anchors, dtype=np.int64)
    depth = dv.cu_branch[1:] - dv.cu_branch[:-1]
    pre = anchors - dv.cu[dv.branch_seq] + 1 if anchors.size else np.zeros(0, dtype=np.int64)
    if st.mask_kind == MASK_BLOCK_BIDIR:
        loc = depth * depth
    else:
        loc = depth * (depth + 1) // 2
    branch = int((pre * depth + loc).sum())
    return (main + branch) * st.hq


def visible_counts(st, dv: Derived = None) -> Tuple[np.ndarray, np.ndarray]:
    """Number of keys each main row and each branch row sees (mask definition):
    main row r of sequence s sees r - cu[s] + 1 keys; branch token j of branch
    b (anchor a, depth D) sees a - cu[s] + 1 main keys plus j + 1 (causal
    kinds) or D (block-bidirectional) keys of its branch."""
    dv = dv or derive(st)
    n_m = np.arange(dv.n_main) - dv.cu[dv.main_seq] + 1
    anchors = np.asarray(st.anchors, dtype=np.int64)
    b = dv.row_branch
    j = np.arange(dv.n_branch_tokens) - dv.cu_branch[b]
    depth = dv.cu_branch[b + 1] - dv.cu_branch[b]
    pre = anchors[b] - dv.cu[dv.branch_seq[b]] + 1 if b.size else np.zeros(0, dtype=np.int64)
    loc = depth if st.mask_kind == MASK_BLOCK_BIDIR else j + 1
    return n_m.astype(np.int64), (pre + loc).astype(np.int64)


def zero_query_dv(st, t, groups=None):
    """dV of every main and branch key when every query is zero.

    With q = 0 every visible score is 0, so P_ik = 1 / n_i over the n_i keys
    row i sees (visible_counts), and the backward definition gives
    dV_k = sum over the rows i that see key k of dO_i / n_i (summed over the q
    heads of k's kv group) and dK_k = scale sum_i dS_ik q_i = 0.
      * main key k of sequence s is seen by the main rows i >= k of s and by
        every token of the branches of s anchored at a position >= k, so its
        dV is a suffix sum over the positions of s of w_i = dO_i / n_i plus,
        at each anchor position, the branch tokens' w;
      * branch key (b, j') is seen by the tokens (b, j) with j >= j' (causal
        kinds: a suffix sum within the branch) or by every token of b
        (block-bidirectional: the branch total).
    Only kv heads in `groups` (default all) are filled; returns dv_m [N, Hkv, d]
    and dv_b [Nb, Hkv, d] in fp64.
    """
    dv = derive(st)
    hq, hkv, d = st.hq, st.hkv, st.head_dim
    grp = hq // hkv
    groups = list(range(hkv)) if groups is None else [int(g) for g in groups]
    n_m, n_b = visible_counts(st, dv)
    n, nb = dv.n_main, dv.n_branch_tokens
    anchors = np.asarray(st.anchors, dtype=np.int64)
    seq_end = dv.cu[dv.main_seq + 1]                  # end of each main token's sequence
    out_m = np.zeros((n, hkv, d))
    out_b = np.zeros((nb, hkv, d))
    for g in groups:
        for h in range(g * grp, (g + 1) * grp):
            w_m = to64(t["do_m"][:, h]) / n_m[:, None]
            w_b = to64(t["do_b"][:, h]) / n_b[:, None] if nb else np.zeros((0, d))
            tot = w_m.copy()
            if nb:
                per_branch = np.zeros((anchors.size, d))
                np.add.at(per_branch, dv.row_branch, w_b)
                np.add.at(tot, anchors, per_branch)
            # G[k] = sum_{i >= k} tot_i; the suffix within k's sequence is G[k] - G[end]
            G = np.zeros((n + 1, d))
            G[:n] = np.cumsum(tot[::-1], axis=0)[::-1]
            out_m[:, g] += G[:n] - G[seq_end]
            if nb:
                if st.mask_kind == MASK_BLOCK_BIDIR:
                    out_b[:, g] += per_branch[dv.row_branch]
                else:
                    Gb = np.zeros((nb + 1, d))
                    Gb[:nb] = np.cumsum(w_b[::-1], axis=0)[::-1]
                    out_b[:, g] += Gb[:nb] - Gb[dv.cu_branch[dv.row_branch + 1]]
    return out_m, out_b
