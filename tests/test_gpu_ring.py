"""Zigzag ring across ranks on the GPU: ring plans and ring steps.

One GPU emulates the C ranks of the ring in one process: rank q's step t
reads the main K/V of shard (q - t) mod C from a local copy of that shard,
which is what the ring's exchange delivers.  Checked against the oracle:
- every ring plan's per-row key intervals, bit-exactly, against the oracle's
  brute-force intervals (oracle/ring.py);
- the ring's outputs, gathered back to the batch's rows, against the fp64
  forward on small batches and against the monolithic forward of the library
  (and the oracle's sampled rows) on the 20K and 32K batches and on a 32K
  prefix of the 256K sequence.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from oracle import ring as oring

from test_gpu_parity import check, check_lse, cpu, run, _sample_rows

pytestmark = pytest.mark.gpu

KINDS = (wl.MASK_TTT_CAUSAL, wl.MASK_BLOCK_BIDIR, wl.MASK_BLOCK_CAUSAL)


def _long_enough(seed, C, kind, n_seqs=3, max_len=300, hq=4, hkv=2, d=64, p=0.5):
    st = wl.random_structure(seed, n_seqs=n_seqs, max_len=max_len, max_depth=6, hq=hq, hkv=hkv,
                             head_dim=d, mask_kind=kind, branch_prob=p)
    lens = np.maximum(np.diff(st.cu_seqlens), 2 * C)
    cu = np.concatenate([[0], np.cumsum(lens)])
    rng = np.random.default_rng(seed)
    anchors = np.sort(np.nonzero(rng.random(int(cu[-1])) < p)[0])
    depths = rng.integers(1, 7, size=anchors.shape[0])
    return wl.Structure(f"ring{seed}", cu, anchors, depths, hq, hkv, d, kind)


def _ranks(ba, st, C):
    return [ba.ZigzagRingAttention(st.cu_seqlens, st.anchors, st.depths, st.hq, st.hkv,
                                   st.head_dim, st.mask_kind, C, q, st.scale) for q in range(C)]


def _local(t, rank):
    mr = torch.as_tensor(rank.main_rows.astype(np.int64), device="cuda")
    br = torch.as_tensor(rank.branch_rows.astype(np.int64), device="cuda")
    return {k: v.index_select(0, mr if k.endswith("_m") else br).contiguous()
            for k, v in t.items()}


def emulate_ring(ba, st, t, C):
    ranks = _ranks(ba, st, C)
    loc = [_local(t, r) for r in ranks]
    outs = []
    for q, r in enumerate(ranks):
        r.plan()
        for step in range(C):
            j = (q - step) % C
            r.step(step, loc[q]["q_m"], loc[q]["q_b"], loc[j]["k_m"], loc[j]["v_m"])
        outs.append(r.finish(loc[q]["q_m"], loc[q]["q_b"], loc[q]["k_b"], loc[q]["v_b"]))
    torch.cuda.synchronize()
    for r in ranks:
        assert r.plan_status() == [0] * C
    o_m, o_b = torch.empty_like(t["q_m"]), torch.empty_like(t["q_b"])
    lse_m = torch.empty((st.hq, st.n_main), dtype=torch.float32, device="cuda")
    lse_b = torch.empty((st.hq, st.n_branch_tokens), dtype=torch.float32, device="cuda")
    for r, out in zip(ranks, outs):
        mr = torch.as_tensor(r.main_rows.astype(np.int64), device="cuda")
        br = torch.as_tensor(r.branch_rows.astype(np.int64), device="cuda")
        o_m[mr] = out["o_m"]
        lse_m[:, mr] = out["lse_m"]
        if br.numel():
            o_b[br] = out["o_b"]
            lse_b[:, br] = out["lse_b"]
    return {"o_m": o_m, "o_b": o_b, "lse_m": lse_m, "lse_b": lse_b}


def _row_iv(ba, rank, step):
    L = ba.ba_plan_layout_query(rank.local)
    raw = rank.plan_ws[step].cpu().numpy().view(np.int32)
    rows = rank.local.c.n_main + rank.local.c.n_branch_tokens
    return raw[L["off_row_iv"] // 4: L["off_row_iv"] // 4 + 4 * rows].reshape(rows, 4)


@pytest.mark.parametrize("C", [2, 3, 4])
@pytest.mark.parametrize("kind", KINDS)
def test_ring_plan_matches_oracle(cuda_lib, C, kind):
    st = _long_enough(50 + C, C, kind, max_len=120)
    for q, r in enumerate(_ranks(cuda_lib, st, C)):
        r.plan()
        torch.cuda.synchronize()
        assert r.plan_status() == [0] * C
        for step in range(1, C):
            got = _row_iv(cuda_lib, r, step)[:, :2].astype(np.int64)
            ref = oring.step_intervals(st, C, q, step)
            empty_g, empty_r = got[:, 1] < got[:, 0], ref[:, 1] < ref[:, 0]
            np.testing.assert_array_equal(empty_g, empty_r, err_msg=f"q={q} step={step}")
            np.testing.assert_array_equal(got[~empty_g], ref[~empty_r],
                                          err_msg=f"q={q} step={step}")


@pytest.mark.parametrize("C", [2, 3, 4])
@pytest.mark.parametrize("kind", KINDS)
def test_ring_forward_matches_oracle(cuda_lib, C, kind):
    """Several query / key tiles per shard, ragged tails, varlen, GQA."""
    st = _long_enough(60 + C, C, kind)
    t = wl.tensors(st, 9, "cuda")
    out = emulate_ring(cuda_lib, st, t, C)
    o_m, o_b, lse_m, lse_b = oracle.forward_dense(st, t)
    check("o_m (ring)", cpu(out["o_m"]), o_m)
    check("o_b (ring)", cpu(out["o_b"]), o_b)
    check_lse("lse_m (ring)", cpu(out["lse_m"]), lse_m)
    check_lse("lse_b (ring)", cpu(out["lse_b"]), lse_b)


def _ring_vs_monolithic(ba, st, t, C, n_rand=8):
    _, mono, _ = run(ba, st, t, bwd=False)
    out = emulate_ring(ba, st, t, C)
    for key in ("o_m", "o_b"):
        check(f"{key} ring C={C} vs monolithic", cpu(out[key]), cpu(mono[key]))
    for key in ("lse_m", "lse_b"):
        check_lse(f"{key} ring C={C} vs monolithic", cpu(out[key]), cpu(mono[key]))
    mr, br = _sample_rows(st, n_rand, np.random.default_rng(C))
    ref = oracle.rows_forward(st, t, mr, br)
    R = len(mr)
    check(f"o_m rows (ring C={C})", cpu(out["o_m"][mr]), ref["o"][:R])
    check(f"o_b rows (ring C={C})", cpu(out["o_b"][br]), ref["o"][R:])


@pytest.mark.parametrize("name,C", [("ttt_20k", 4), ("dflash_32k", 8)])
def test_ring_full_size_batches(cuda_lib, name, C):
    st = wl.structure(name)
    _ring_vs_monolithic(cuda_lib, st, wl.tensors(st, wl.workload_seed(name), "cuda"), C)


def test_ring_256k_prefix(cuda_lib):
    """First 32,768 tokens of the 256K sequence (and their branches), C = 8."""
    full = wl.structure("ttt_256k")
    st = dataclasses.replace(wl.truncate(full, 32768), zigzag_C=1)
    t_full = wl.tensors(full, wl.workload_seed("ttt_256k"), "cuda")
    t = {k: v.contiguous() for k, v in wl.slice_tensors(full, st, t_full).items()}
    del t_full
    torch.cuda.empty_cache()
    _ring_vs_monolithic(cuda_lib, st, t, 8)
