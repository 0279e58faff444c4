"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (fp32 accumulation over bf16 inputs, P and dS rounded to bf16 for
the tensor-core products, bf16 outputs): O, dQ, dK, dV elementwise
|x - ref| <= 2e-2 + 1e-2 |ref| (max abs error 2e-2, relative 1e-2) and
relative L2 error <= 1e-2 per tensor; LSE max abs error <= 1e-3; tile
metadata bit-exact.  The relative part of the elementwise bound is what makes
the bound attainable for bf16 outputs: rounding a value of magnitude >= 4 to
bf16 alone moves it by up to 2^-9 |x| >= 7.8e-3.  That this relative part is
spent on output rounding only, not on kernel error, is checked as well: the
error in excess of the best bf16 output, max(|x - ref| - |bf16(ref) - ref|),
must be <= 2e-2 everywhere.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

ABS, REL, LSE_ABS = 2e-2, 1e-2, 1e-3
KINDS = (wl.MASK_TTT_CAUSAL, wl.MASK_BLOCK_BIDIR, wl.MASK_BLOCK_CAUSAL)
FAMILIES = (0, 1)   # backward: 0 = split dK/dV + dQ kernels (default), 1 = fused kernel


def bf16_rounding(ref):
    """|bf16(ref) - ref|: the error of the best bf16 output (round to nearest even)."""
    r = torch.from_numpy(np.ascontiguousarray(ref, dtype=np.float64))
    return np.abs(r.to(torch.bfloat16).double().numpy() - ref)


def check(name, got, ref, abs_tol=ABS, rel_tol=REL, beyond_tol=ABS, beyond_rel=0.0):
    """Spec bound (elementwise and relative L2) and, unless beyond_tol is
    None, the error beyond bf16 output rounding: at most beyond_tol +
    beyond_rel |ref| at every element."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    if got.size == 0:
        return
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    diff = np.abs(got - ref)
    excess = (diff - (abs_tol + rel_tol * np.abs(ref))).max()
    beyond = diff - bf16_rounding(ref)
    worst = int(np.argmax(beyond))
    beyond_rounding = beyond.flat[worst]
    beyond_excess = (beyond - beyond_rel * np.abs(ref)).max()
    # the relative L2 bound applies when the reference is not within the
    # absolute tolerance of zero (e.g. dQ of a query that sees only itself is 0)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref) if np.abs(ref).max() > abs_tol else 0.0
    print(f"{name}: max abs {diff.max():.3e}, beyond bf16 output rounding {beyond_rounding:.3e} "
          f"(|ref| {abs(ref.flat[worst]):.3e} there), rel L2 {rel:.3e}")
    assert excess <= 0 and rel <= rel_tol and (beyond_tol is None or beyond_excess <= beyond_tol), \
        f"{name}: max abs {diff.max():.3e}, worst excess over 2e-2+1e-2|ref| {excess:.3e}, " \
        f"error beyond bf16 output rounding {beyond_rounding:.3e}, rel L2 {rel:.3e}"


def check_lse(name, got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    if got.size == 0:
        return
    err = np.abs(got - ref).max()
    assert err <= LSE_ABS, f"{name}: LSE max abs {err:.3e}"


def cpu(x):
    return x.detach().float().cpu().numpy()


def run(ba, st, t, family=0, bwd=True, zigzag_C=None):
    ba.ba_set_kernel_family(family)
    try:
        prob = ba.Problem.from_structure(st, zigzag_C=zigzag_C)
        runner = ba.BranchAttention(prob)
        runner.plan()
        assert runner.plan_status() == 0
        out = runner.forward(t)
        grads = runner.backward(t, out) if bwd else None
        torch.cuda.synchronize()
        # raises BranchAttnError(BA_ERR_DEVICE_TIMEOUT) if a bounded wait gave up
        assert runner.plan_status() == 0
    finally:
        ba.ba_set_kernel_family(0)
    return runner, out, grads


def full_parity(ba, st, seed, family):
    t = wl.tensors(st, seed, "cuda")
    _, out, g = run(ba, st, t, family)
    o_m, o_b, lse_m, lse_b = oracle.forward_dense(st, t)
    check("o_m", cpu(out["o_m"]), o_m)
    check("o_b", cpu(out["o_b"]), o_b)
    check_lse("lse_m", cpu(out["lse_m"]), lse_m)
    check_lse("lse_b", cpu(out["lse_b"]), lse_b)
    ref = oracle.backward_dense(st, t)
    for name, r in zip(("dq_m", "dk_m", "dv_m", "dq_b", "dk_b", "dv_b"), ref):
        check(name, cpu(g[name]), r)


# ------------------------------------------------------------ metadata
def _plan_equal(ba, st):
    prob = ba.Problem.from_structure(st)
    runner = ba.BranchAttention(prob)
    runner.plan()
    assert runner.plan_status() == 0
    got = runner.read_plan()
    ref = oracle.plan(st)
    assert got["status"] == 0
    for key, r in ref.items():
        np.testing.assert_array_equal(got[key], r, err_msg=key)


@pytest.mark.parametrize("name", wl.WORKLOADS)
def test_plan_bit_exact_workloads(cuda_lib, name):
    _plan_equal(cuda_lib, wl.structure(name))


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("kind", KINDS)
def test_plan_bit_exact_random(cuda_lib, seed, kind):
    st = wl.random_structure(seed, n_seqs=1 + seed, max_len=700, max_depth=64 if seed % 2 else 7,
                             head_dim=64, mask_kind=kind, branch_prob=0.3, zigzag_C=1 + seed % 4)
    _plan_equal(cuda_lib, st)


def test_plan_reports_bad_metadata(cuda_lib):
    ba = cuda_lib
    dev = "cuda"
    cases = {
        0x10: ([0, 10, 20], [5, 3], [2, 2]),     # anchors decrease
        0x08: ([0, 10, 20], [5, 20], [2, 2]),    # anchor out of range
        0x20: ([0, 10, 20], [5, 6], [0, 4]),     # depth 0
        0x02: ([0, 10, 10], [5, 6], [2, 2]),     # empty sequence
    }
    for bit, (cu, an, de) in cases.items():
        prob = ba.Problem(torch.tensor(cu, dtype=torch.int32, device=dev),
                          torch.tensor(an, dtype=torch.int32, device=dev),
                          torch.tensor(de, dtype=torch.int32, device=dev), 4, 2, 1, 64)
        runner = ba.BranchAttention(prob)
        runner.plan()
        status = runner.plan_status()
        assert status & bit, (bit, status)
        # kernels reading a bad plan return without touching their outputs
        st = wl.Structure("bad", np.array(cu), np.array(an), np.array([2, 2]), 2, 1, 64, 0)
        t = wl.tensors(st, 0, dev)
        out = runner.alloc_outputs()
        for v in out.values():
            v.fill_(7.0)
        runner.forward(t, out)
        torch.cuda.synchronize()
        assert bool((out["o_m"] == 7.0).all()) and bool((out["lse_m"] == 7.0).all())


# ------------------------------------------------------------ full parity
@pytest.mark.parametrize("family", FAMILIES)
def test_tiny_ttt_full(cuda_lib, family):
    st = wl.structure("tiny_ttt")
    full_parity(cuda_lib, st, wl.workload_seed("tiny_ttt"), family)


@pytest.mark.parametrize("family", FAMILIES)
@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("d,hq,hkv", [(64, 4, 2), (128, 4, 1), (128, 2, 2)])
def test_random_full(cuda_lib, family, kind, d, hq, hkv):
    """Several query and key tiles, ragged tails, varlen packing, GQA."""
    st = wl.random_structure(10 + d + hq, n_seqs=3, max_len=330, max_depth=9, hq=hq, hkv=hkv,
                             head_dim=d, mask_kind=kind, branch_prob=0.45)
    full_parity(cuda_lib, st, 7, family)


EDGE = {
    "one_token": (np.array([0, 1]), np.array([0]), np.array([1])),
    "no_branches": (np.array([0, 130, 131, 300]), np.zeros(0, int), np.zeros(0, int)),
    "unit_sequences": (np.arange(0, 41), np.arange(0, 40, 3), np.full(14, 2)),
    "depth64": (np.array([0, 70, 200]), np.array([0, 69, 70, 150, 199]), np.full(5, 64)),
    "same_anchor": (np.array([0, 257]), np.full(9, 256), np.array([1, 2, 3, 4, 5, 6, 7, 8, 9])),
    "first_positions": (np.array([0, 129, 258, 387]), np.array([0, 129, 258]),
                        np.array([16, 16, 16])),
}


@pytest.mark.parametrize("family", FAMILIES)
@pytest.mark.parametrize("case", sorted(EDGE))
@pytest.mark.parametrize("kind", KINDS)
def test_edge_cases(cuda_lib, family, case, kind):
    cu, an, de = EDGE[case]
    st = wl.Structure(case, cu, an, de, 4, 2, 64, kind)
    full_parity(cuda_lib, st, 3, family)


@pytest.mark.parametrize("C", [2, 3, 5])
def test_zigzag_small_matches_oracle(cuda_lib, C):
    """The virtual zigzag ring (C shards, LSE-merged) equals the monolithic result."""
    st = wl.random_structure(21 + C, n_seqs=3, max_len=500, max_depth=5, hq=4, hkv=2,
                             head_dim=64, branch_prob=0.5, zigzag_C=C)
    t = wl.tensors(st, 5, "cuda")
    _, out, _ = run(cuda_lib, st, t, bwd=False)
    o_m, o_b, lse_m, lse_b = oracle.zigzag_forward(st, t, C)
    check("o_m", cpu(out["o_m"]), o_m)
    check("o_b", cpu(out["o_b"]), o_b)
    check_lse("lse_m", cpu(out["lse_m"]), lse_m)
    check_lse("lse_b", cpu(out["lse_b"]), lse_b)


# ------------------------------------------------------------ lse_merge
@pytest.mark.parametrize("fp32", [True, False])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("inplace", [False, True])
def test_lse_merge(cuda_lib, fp32, d, inplace):
    ba = cuda_lib
    rows, heads = 1000, 3
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1)
    dt = torch.float32 if fp32 else torch.bfloat16
    oa = torch.randn(rows, heads, d, generator=gen, device="cuda").to(dt)
    ob = torch.randn(rows, heads, d, generator=gen, device="cuda").to(dt)
    la = torch.randn(heads, rows, generator=gen, device="cuda") * 5
    lb = torch.randn(heads, rows, generator=gen, device="cuda") * 5
    la[0, :50] = -float("inf")
    lb[1, :50] = -float("inf")
    la[2, :20] = -float("inf")
    lb[2, :20] = -float("inf")
    la[2, 20:40] = 80.0
    lb[2, 20:40] = 80.5
    ref_o, ref_l = oracle.lse_merge(cpu(oa).transpose(1, 0, 2), cpu(la),
                                    cpu(ob).transpose(1, 0, 2), cpu(lb))
    if inplace:
        oo, lo = oa, la
    else:
        oo, lo = torch.empty_like(oa), torch.empty_like(la)
    ba.lse_merge(oa, la, ob, lb, oo, lo)
    torch.cuda.synchronize()
    got_l = cpu(lo)
    assert np.array_equal(np.isneginf(got_l), np.isneginf(ref_l))
    fin = np.isfinite(ref_l)
    assert np.abs(got_l[fin] - ref_l[fin]).max() <= 1e-5 * 100
    tol = 1e-5 if fp32 else 1e-2
    np.testing.assert_allclose(cpu(oo).transpose(1, 0, 2), ref_o, atol=tol, rtol=tol)


# ------------------------------------------------------------ full-size workloads
def _sample_rows(st, n_rand, rng):
    dv = oracle.derive(st)
    n, nb = dv.n_main, dv.n_branch_tokens
    main = set()
    for s in range(st.n_seqs):
        main.update({int(dv.cu[s]), int(dv.cu[s + 1]) - 1})
    main.update({127, 128, n - 1})
    main.update(int(x) for x in rng.integers(0, n, n_rand))
    branch = {0, nb - 1, min(127, nb - 1), min(128, nb - 1)}
    branch.update(int(x) for x in rng.integers(0, nb, n_rand))
    return sorted(x for x in main if 0 <= x < n), sorted(x for x in branch if 0 <= x < nb)


def _count_visible(st):
    iv = oracle.row_intervals(st)
    cnt = (iv[:, 1] - iv[:, 0] + 1) + np.maximum(iv[:, 3] - iv[:, 2] + 1, 0)
    return cnt[:st.n_main], cnt[st.n_main:]


def check_head_keys(ba, st, t, g, groups, name):
    """dK / dV of the first 128 main keys of the longest sequence against the
    oracle.  Every later query of that sequence and every branch anchored in
    it visits these keys, so they are the key tiles with the longest walks
    (every visiting query tile of every q head of the group, accumulated in
    TMEM over the whole walk)."""
    lens = np.diff(st.cu_seqlens)
    s = int(np.argmax(lens))
    lo = int(st.cu_seqlens[s])
    keys = list(range(lo, lo + min(128, int(lens[s]))))
    gs = list(groups)
    km, km_op = oracle.keys_backward_both(st, t, main_keys=keys, groups=gs)
    # against the exact gradients: the benchmark spec's bound.  Over these walks the
    # bf16 rounding of the P and dS operands of the tensor-core products (each
    # within 2^-9 relative) adds up beyond what output rounding explains, so
    # the second comparison takes those operands (and the O that D is formed
    # from) in bf16 and holds the kernel to 2e-2 beyond output rounding against
    # that.  dV meets it with room (~1e-3); dK stays about one bf16 rounding of
    # |ref| beyond the model (relative L2 ~2.2e-3), which is allowed on top
    for key, rel in (("dk_m", 2.0 ** -8), ("dv_m", 0.0)):
        got = cpu(g[key][keys][:, gs])
        check(f"{key} first keys ({name})", got, km[key][:, gs], beyond_tol=None)
        check(f"{key} first keys, bf16 P / dS operands ({name})", got, km_op[key][:, gs],
              beyond_rel=rel)


def check_zero_query_grads(ba, runner, st, t, groups, name):
    """Every key at full size, by a closed form: with Q = 0, P is uniform over
    each row's visible keys, dV_k = sum_i dO_i / n_i over the rows that see k,
    and dK = 0 exactly."""
    tz = dict(t)
    tz["q_m"] = torch.zeros_like(t["q_m"])
    tz["q_b"] = torch.zeros_like(t["q_b"])
    zout = runner.forward(tz)
    zg = runner.backward(tz, zout)
    torch.cuda.synchronize()
    assert runner.plan_status() == 0
    assert int(torch.count_nonzero(zg["dk_m"])) == 0, f"{name}: dK of main keys is not 0"
    assert int(torch.count_nonzero(zg["dk_b"])) == 0, f"{name}: dK of branch keys is not 0"
    gs = list(groups)
    ref_m, ref_b = oracle.zero_query_dv(st, {"do_m": t["do_m"].cpu(), "do_b": t["do_b"].cpu()},
                                        groups=gs)
    check(f"dv_m all keys, Q = 0 ({name})", cpu(zg["dv_m"][:, gs]), ref_m[:, gs])
    check(f"dv_b all keys, Q = 0 ({name})", cpu(zg["dv_b"][:, gs]), ref_b[:, gs])
    return zout


def workload_check(ba, st, seed, n_rand=24, tail_keys=128, groups=None, zigzag=False,
                   head_keys=True, family=0):
    groups = (0, st.hkv - 1) if groups is None else groups
    rng = np.random.default_rng(seed)
    t = wl.tensors(st, seed, "cuda")
    runner, out, g = run(ba, st, t, family)
    # 1) sampled rows: O, LSE and dQ over all heads
    mr, br = _sample_rows(st, n_rand, rng)
    ref = oracle.rows_backward_dq(st, t, mr, br)
    R = len(mr)
    check("o_m rows", cpu(out["o_m"][mr]), ref["o"][:R])
    check("o_b rows", cpu(out["o_b"][br]), ref["o"][R:])
    check_lse("lse_m rows", cpu(out["lse_m"][:, mr]), ref["lse"][:, :R])
    check_lse("lse_b rows", cpu(out["lse_b"][:, br]), ref["lse"][:, R:])
    check("dq_m rows", cpu(g["dq_m"][mr]), ref["dq"][:R])
    check("dq_b rows", cpu(g["dq_b"][br]), ref["dq"][R:])
    # 2) branch keys of a few branches (each seen by <= 64 queries)
    dv = oracle.derive(st)
    gs = list(groups)
    bsel = sorted({0, st.n_branches - 1, *rng.integers(0, st.n_branches, 3).tolist()})
    bkeys = [k for b in bsel for k in range(int(dv.cu_branch[b]), int(dv.cu_branch[b + 1]))]
    kb = oracle.keys_backward(st, t, branch_keys=bkeys, groups=gs)
    check("dk_b keys", cpu(g["dk_b"][bkeys][:, gs]), kb["dk_b"][:, gs])
    check("dv_b keys", cpu(g["dv_b"][bkeys][:, gs]), kb["dv_b"][:, gs])
    # 3) tail window of main keys of the shortest sequence (few visitors)
    if tail_keys:
        lens = np.diff(st.cu_seqlens)
        s = int(np.argmin(lens))
        hi = int(st.cu_seqlens[s + 1])
        mkeys = list(range(max(int(st.cu_seqlens[s]), hi - tail_keys), hi))
        km = oracle.keys_backward(st, t, main_keys=mkeys, groups=gs)
        check("dk_m tail", cpu(g["dk_m"][mkeys][:, gs]), km["dk_m"][:, gs])
        check("dv_m tail", cpu(g["dv_m"][mkeys][:, gs]), km["dv_m"][:, gs])
    # 4) head keys of the longest sequence (the longest walks)
    if head_keys:
        check_head_keys(ba, st, t, g, gs, st.name)
    # 5) every key with Q = 0 (closed form), and every row's LSE = ln(#visible keys)
    ba.ba_set_kernel_family(family)
    try:
        zout = check_zero_query_grads(ba, runner, st, t, gs, st.name)
    finally:
        ba.ba_set_kernel_family(0)
    cm, cb = oracle.visible_counts(st)
    check_lse("lse_m (Q=0, all rows)", cpu(zout["lse_m"]), np.log(cm)[None].repeat(st.hq, 0))
    check_lse("lse_b (Q=0, all rows)", cpu(zout["lse_b"]), np.log(cb)[None].repeat(st.hq, 0))
    # 6) zigzag virtual shards agree with the monolithic run
    if zigzag:
        _, zo, _ = run(ba, st, t, 0, bwd=False, zigzag_C=st.zigzag_C)
        for key in ("o_m", "o_b"):
            check(f"{key} zigzag vs monolithic", cpu(zo[key]), cpu(out[key]))
        for key in ("lse_m", "lse_b"):
            check_lse(f"{key} zigzag vs monolithic", cpu(zo[key]), cpu(out[key]))
        check("o_m rows (zigzag)", cpu(zo["o_m"][mr]), ref["o"][:R])
        check("o_b rows (zigzag)", cpu(zo["o_b"][br]), ref["o"][R:])
    return t


@pytest.mark.parametrize("name", ["ttt_20k", "dflash_32k"])
def test_workload_full_size(cuda_lib, name):
    st = wl.structure(name)
    workload_check(cuda_lib, st, wl.workload_seed(name))


def test_workload_ttt_20k_fused_backward(cuda_lib):
    """The fused backward (family 1) at full size, same checks."""
    st = wl.structure("ttt_20k")
    workload_check(cuda_lib, st, wl.workload_seed("ttt_20k"), family=1)


def test_workload_dspark_64k(cuda_lib):
    """One 64K sequence: exact head keys would take the oracle minutes (every
    one of the 80K rows scores up to 64K keys), so the longest walks are
    checked on a 12,288-token prefix below and here every key by the Q = 0
    closed form."""
    st = wl.structure("dspark_64k")
    workload_check(cuda_lib, st, wl.workload_seed("dspark_64k"), head_keys=False)


def test_workload_ttt_256k_and_zigzag(cuda_lib):
    st = wl.structure("ttt_256k")
    workload_check(cuda_lib, st, wl.workload_seed("ttt_256k"), n_rand=8, tail_keys=0,
                   zigzag=True, head_keys=False)


def _prefix(name, n_tokens):
    full = wl.structure(name)
    st = dataclasses.replace(wl.truncate(full, n_tokens), zigzag_C=1)
    t_full = wl.tensors(full, wl.workload_seed(name), "cuda")
    t = {k: v.contiguous() for k, v in wl.slice_tensors(full, st, t_full).items()}
    del t_full
    torch.cuda.empty_cache()
    return st, t


def test_workload_dspark_64k_prefix_head_keys(cuda_lib):
    """First 12,288 tokens of the 64K sequence (same data): the first key tile
    is walked by 96 main and 24 branch query tiles x 8 q heads."""
    st, t = _prefix("dspark_64k", 12288)
    _, _, g = run(cuda_lib, st, t, 0)
    check_head_keys(cuda_lib, st, t, g, (0, st.hkv - 1), "dspark 12K prefix")


@pytest.mark.parametrize("C", [1, 8])
def test_workload_ttt_256k_truncated_prefix(cuda_lib, C):
    """First 8,192 tokens (and their branches) of the 256K batch, same data,
    monolithic and with the forward as 8 virtual zigzag shards (the backward
    then reads the LSE that the ring produced)."""
    st, t = _prefix("ttt_256k", 8192)
    _, out, g = run(cuda_lib, st, t, 0, zigzag_C=C)
    rng = np.random.default_rng(0)
    mr, br = _sample_rows(st, 16, rng)
    ref = oracle.rows_backward_dq(st, t, mr, br)
    R = len(mr)
    check("o_m", cpu(out["o_m"][mr]), ref["o"][:R])
    check("o_b", cpu(out["o_b"][br]), ref["o"][R:])
    check("dq_m", cpu(g["dq_m"][mr]), ref["dq"][:R])
    check("dq_b", cpu(g["dq_b"][br]), ref["dq"][R:])
    mkeys = list(range(8192 - 128, 8192))
    km = oracle.keys_backward(st, t, main_keys=mkeys, groups=[0, 7])
    check("dk_m tail", cpu(g["dk_m"][mkeys][:, [0, 7]]), km["dk_m"][:, [0, 7]])
    check("dv_m tail", cpu(g["dv_m"][mkeys][:, [0, 7]]), km["dv_m"][:, [0, 7]])
    check_head_keys(cuda_lib, st, t, g, (0, 7), f"256K 8K prefix, C={C}")


# ------------------------------------------------------------ exponential
def test_exp2_polynomial_against_exact(cuda_lib):
    """The FMA-pipe 2^x: relative error <= 1e-4 against exact 2^x (fp64) on the
    softmax's input range, exactly 0 below -125, and the hardware ex2 within
    about 2^-22 (checked at 1e-6) for reference."""
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_001),
                   torch.tensor([-125.0, -124.5, -0.5, -0.25, 0.0, 0.5, 1.0, 7.5, 8.0]),
                   torch.tensor([-126.0, -200.0, -1e30, float("-inf")])]).float().cuda()
    y_fma, y_hw = cuda_lib.ba_exp2_check(x)
    xs = x.double().cpu().numpy()
    exact = np.exp2(xs)
    got = y_fma.double().cpu().numpy()
    inside = xs >= -125.0
    rel = np.abs(got[inside] / exact[inside] - 1.0)
    assert rel.max() <= 1e-4, rel.max()
    assert np.all(got[~inside] == 0.0)
    hw = y_hw.double().cpu().numpy()
    rel_hw = np.abs(hw[inside & (xs > -120)] / exact[inside & (xs > -120)] - 1.0)
    assert rel_hw.max() <= 1e-6
