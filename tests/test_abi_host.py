"""Host-only checks of the C ABI: exports match the header, and every invalid
argument is rejected with its documented status before anything launches.

No call here reaches a kernel: every argument set is one the host-side
validation rejects (fake device addresses are never dereferenced)."""
import ctypes
import os
import re

import pytest

import speculative_draft_branch_b200 as ba

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "branch_attn.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^BA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("ba_plan", "branch_attn_fwd", "branch_attn_bwd", "lse_merge",
                     "ba_workspace_size", "ba_plan_status", "ba_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(ba.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(ba.EXPORTS) <= set(_declared())


def _problem(**kw):
    base = dict(n_seqs=2, n_main=256, n_branches=256, n_branch_tokens=768, hq=4, hkv=2,
                head_dim=64, scale=0.125, mask=0, zigzag_C=1, cu_seqlens=0x10000,
                branch_anchor=0x20000, branch_depth=0x30000)
    base.update(kw)
    return ba.BAProblem(**base)


def _sizes(p):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    st = ba.lib.ba_workspace_size(ctypes.byref(p), ctypes.byref(a), ctypes.byref(b),
                                  ctypes.byref(c))
    return st, a.value, b.value, c.value


@pytest.mark.parametrize("kw,code", [
    (dict(n_seqs=0), -1), (dict(n_main=0), -1), (dict(n_seqs=300), -1),
    (dict(n_branches=-1), -1), (dict(n_branch_tokens=100), -1),  # < n_branches
    (dict(n_branch_tokens=256 * 65), -1),                         # depth > 64
    (dict(hq=6, hkv=4), -1), (dict(hkv=0), -1), (dict(head_dim=96), -2),
    (dict(head_dim=256), -2), (dict(mask=3), -1), (dict(mask=-1), -1),
    (dict(zigzag_C=0), -1), (dict(zigzag_C=65), -1), (dict(scale=0.0), -1),
    (dict(scale=float("nan")), -1), (dict(scale=float("inf")), -1),
])
def test_invalid_problem_rejected(kw, code):
    st, *_ = _sizes(_problem(**kw))
    assert st == code
    assert ba.lib.ba_last_error().decode() != ""


def test_workspace_sizes_follow_the_layout():
    p = _problem()
    st, plan_b, fwd_b, bwd_b = _sizes(p)
    assert st == 0
    L = ba.BAPlanLayout()
    assert ba.lib.ba_plan_layout_query(ctypes.byref(p), ctypes.byref(L)) == 0
    assert L.total_bytes == plan_b
    assert (L.n_qtiles_main, L.n_qtiles_branch, L.n_kv_main, L.n_kv_branch) == (2, 6, 2, 6)
    assert fwd_b == 0
    rows = 256 + 768
    rows_pad = 256 + 768          # both kinds already multiples of 128
    # D [Hq, rows], records [Hq, rows_pad] x {LSE, D} fp32, fp32 dQ accumulator
    assert bwd_b == 4 * rows * 4 + 8 * rows_pad * 4 + 4 * rows * 4 * 64
    # arrays are 256-byte aligned and do not overlap
    offs = sorted(getattr(L, f) for f, _ in ba.BAPlanLayout._fields_ if f.startswith("off_"))
    assert all(o % 256 == 0 for o in offs)
    assert L.off_row_iv - L.off_branch_seq >= 4 * 256
    pz = _problem(zigzag_C=8)
    _, _, fwd_z, _ = _sizes(pz)
    assert fwd_z >= 4 * rows * 4 * 64 + 4 * rows * 4


def test_plan_rejects_bad_pointers_and_small_workspace():
    p = _problem()
    st, plan_b, _, _ = _sizes(p)
    # NULL index arrays
    q = _problem(cu_seqlens=None)
    assert ba.lib.ba_plan(ctypes.byref(q), 0x100000, plan_b, None) == -1
    # misaligned index array
    q = _problem(branch_anchor=0x20002)
    assert ba.lib.ba_plan(ctypes.byref(q), 0x100000, plan_b, None) == -3
    # NULL / misaligned workspace
    assert ba.lib.ba_plan(ctypes.byref(p), None, plan_b, None) == -1
    assert ba.lib.ba_plan(ctypes.byref(p), 0x100008, plan_b, None) == -3
    # workspace too small
    assert ba.lib.ba_plan(ctypes.byref(p), 0x100000, plan_b - 1, None) == -4
    assert "too small" in ba.lib.ba_last_error().decode()


def test_fwd_bwd_reject_misaligned_or_missing_tensors():
    p = _problem()
    good = [0x200000 + i * 0x100000 for i in range(10)]
    args = [ctypes.byref(p), 0x100000, None, 0] + good[:6] + good[6:8] + [0x900000, 0xa00000]
    bad = list(args)
    bad[4] = 0x200001  # q_m misaligned
    assert ba.lib.branch_attn_fwd(*bad, None) == -3
    bad = list(args)
    bad[7] = None      # q_b missing while branch tokens exist
    assert ba.lib.branch_attn_fwd(*bad, None) == -1
    bad = list(args)
    bad[12] = 0x900002  # lse_m not 4-byte aligned
    assert ba.lib.branch_attn_fwd(*bad, None) == -3
    # zigzag needs a workspace
    pz = _problem(zigzag_C=4)
    zargs = [ctypes.byref(pz), 0x100000, None, 0] + args[4:]
    assert ba.lib.branch_attn_fwd(*zargs, None) == -1
    zargs[2] = 0x5000000
    zargs[3] = 16
    assert ba.lib.branch_attn_fwd(*zargs, None) == -4
    # backward: workspace too small, a gradient pointer missing
    st, _, _, bwd_b = _sizes(p)
    bargs = [ctypes.byref(p), 0x100000, 0x6000000, bwd_b - 256] + \
        [0x200000 + i * 0x100000 for i in range(8)] + [0x900000, 0xa00000] + \
        [0xb00000 + i * 0x100000 for i in range(8)]
    assert ba.lib.branch_attn_bwd(*bargs, None) == -4
    bargs[3] = bwd_b
    bargs[16] = None  # dq_m
    assert ba.lib.branch_attn_bwd(*bargs, None) == -1


def test_step_host_sizes_and_rejections():
    """The host-buffer step: its staging holds every workspace and tensor, and
    bad arguments are refused before any copy or launch."""
    p = _problem()
    n = ctypes.c_size_t()
    assert ba.lib.ba_step_host_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    _, plan_b, fwd_b, bwd_b = _sizes(p)
    d = 64
    tensors = 2 * d * (3 * 256 * 4 + 2 * 256 * 2 + 3 * 768 * 4 + 2 * 768 * 2)  # q, o, dq / k, v
    tensors += 2 * 2 * d * (256 * 4 + 768 * 4)                                 # dO, dK / dV extra
    assert n.value >= plan_b + fwd_b + bwd_b + tensors
    bad = _problem(head_dim=96)
    assert ba.lib.ba_step_host_workspace_size(ctypes.byref(bad), ctypes.byref(n)) == -2
    host = [0x7000000 + i * 0x100000 for i in range(18)]
    step = ba.lib.branch_attn_step_host
    need = ctypes.c_size_t()
    ba.lib.ba_step_host_workspace_size(ctypes.byref(p), ctypes.byref(need))
    assert step(None, 0x100000, need.value, *host, None) == -1
    assert step(ctypes.byref(p), None, need.value, *host, None) == -1
    assert step(ctypes.byref(p), 0x100000, need.value - 1, *host, None) == -4
    assert step(ctypes.byref(p), 0x100080, need.value, *host, None) == -3
    missing = list(host)
    missing[7] = None   # do_b while branch tokens exist
    assert step(ctypes.byref(p), 0x100000, need.value, *missing, None) == -1
    assert "null host buffer" in ba.lib.ba_last_error().decode()
    nometa = _problem(cu_seqlens=None)
    assert step(ctypes.byref(nometa), 0x100000, need.value, *host, None) == -1


def test_lse_merge_rejections():
    f = ba.lib.lse_merge
    assert f(-1, 4, 64, 1, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None) == -1
    assert f(10, 0, 64, 1, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None) == -1
    assert f(10, 4, 80, 1, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None) == -2
    assert f(10, 4, 64, 1, 0x1008, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None) == -3
    assert f(10, 4, 64, 1, None, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None) == -1
    assert f(10, 4, 64, 0, 0x1000, 0x2002, 0x3000, 0x4000, 0x5000, 0x6000, None) == -3
    # zero rows is a no-op that touches nothing
    assert f(0, 4, 64, 1, None, None, None, None, None, None, None) == 0


def test_kernel_family_switch():
    old = ba.ba_get_kernel_family()
    try:
        for fam in (0, 1):
            ba.ba_set_kernel_family(fam)
            assert ba.ba_get_kernel_family() == fam
        for bad in (2, 3, -1):
            with pytest.raises(ba.BranchAttnError):
                ba.ba_set_kernel_family(bad)
    finally:
        ba.ba_set_kernel_family(old)


def test_binding_refuses_host_memory_where_the_library_reads_the_device():
    """Host tensors passed where the library dereferences device memory (the
    index arrays at plan time, the workspaces, the operands) are refused by the
    binding before any library call, and the host step refuses a host staging
    buffer."""
    import torch
    import workloads as wl
    st = wl.structure("tiny_ttt")
    prob = ba.Problem.from_structure(st, device="cpu")
    ws = torch.zeros(4096, dtype=torch.uint8)
    with pytest.raises(ValueError, match="cu_seqlens must be a CUDA tensor"):
        ba.ba_plan(prob, ws)
    with pytest.raises(ValueError, match="plan_ws must be a CUDA tensor"):
        ba.ba_plan_status(ws)
    t = wl.tensors(st, 1, "cpu")
    sh = prob.shapes()
    o_m, o_b = torch.empty_like(t["q_m"]), torch.empty_like(t["q_b"])
    lse_m = torch.empty(sh["lse_m"], dtype=torch.float32)
    lse_b = torch.empty(sh["lse_b"], dtype=torch.float32)
    fwd_in = (t["q_m"], t["k_m"], t["v_m"], t["q_b"], t["k_b"], t["v_b"])
    with pytest.raises(ValueError, match="plan_ws must be a CUDA tensor"):
        ba.branch_attn_fwd(prob, ws, None, *fwd_in, o_m, o_b, lse_m, lse_b)
    grads = [torch.empty_like(t[k]) for k in ("q_m", "k_m", "v_m", "q_b", "k_b", "v_b")]
    with pytest.raises(ValueError, match="plan_ws must be a CUDA tensor"):
        ba.branch_attn_bwd(prob, ws, ws, *fwd_in, o_m, o_b, lse_m, lse_b, t["do_m"], t["do_b"],
                           *grads)
    with pytest.raises(ValueError, match="plan_ws must be a CUDA tensor"):
        ba.branch_attn_bwd_static_scratch(prob, ws, *fwd_in, o_m, o_b, lse_m, lse_b, t["do_m"],
                                          t["do_b"], *grads)
    with pytest.raises(ValueError, match="staging must be a CUDA tensor"):
        ba.branch_attn_step_host(prob, ws, *fwd_in, t["do_m"], t["do_b"], o_m, o_b, lse_m,
                                 lse_b, *grads)
    oa = torch.zeros(8, 2, 64)
    la = torch.zeros(2, 8)
    with pytest.raises(ValueError, match="o_a must be a CUDA tensor"):
        ba.lse_merge(oa, la, oa.clone(), la.clone(), oa.clone(), la.clone())


def test_package_fails_loudly_without_the_library():
    """The binding without libbranch_attn.so does not import: there is no
    fallback path to take instead."""
    import shutil
    import subprocess
    import sys
    import tempfile
    os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
    with tempfile.TemporaryDirectory(dir=os.path.join(ROOT, "_build")) as tmp:
        pkg = os.path.join(tmp, "speculative_draft_branch_b200")
        os.mkdir(pkg)
        src = os.path.join(ROOT, "speculative_draft_branch_b200")
        for f in ("__init__.py", "runner.py"):
            shutil.copy(os.path.join(src, f), os.path.join(pkg, f))
        r = subprocess.run([sys.executable, "-c", "import speculative_draft_branch_b200"],
                           cwd=tmp, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "build.py" in r.stderr


def test_product_sources_do_not_reach_the_oracle():
    """Neither the package nor the C interface imports, links or names the
    CPU oracle: it is test infrastructure only."""
    for base in (os.path.join(ROOT, "speculative_draft_branch_b200"), os.path.join(ROOT, "include")):
        for dirpath, _, files in os.walk(base):
            for f in files:
                if f.endswith((".py", ".cu", ".cuh", ".h", ".c", ".cpp")):
                    text = open(os.path.join(dirpath, f)).read()
                    assert not re.search(r"\boracle\b", text, flags=re.I), os.path.join(dirpath, f)


def test_wait_check_rejections():
    """The failure-detection self-check refuses a missing or misaligned plan
    workspace and an unknown mode before launching."""
    f = ba.lib.ba_wait_check
    assert f(None, 0, None) == -1
    assert f(0x100008, 0, None) == -3
    assert f(0x100000, 2, None) == -1
    assert "arrive" in ba.lib.ba_last_error().decode()


def test_struct_layouts_match_the_header():
    """The binding's ctypes mirrors of ba_problem and ba_plan_layout have the
    header's size and field offsets, as the host C compiler lays them out."""
    import shutil
    import subprocess
    import tempfile
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    mirrors = {"ba_problem": ba.BAProblem, "ba_plan_layout": ba.BAPlanLayout}
    src = ["#include <stdio.h>", "#include <stddef.h>", '#include "branch_attn.h"',
           "int main(void) {"]
    for name, cls in mirrors.items():
        src.append(f'  printf("{name} sizeof %zu\\n", sizeof({name}));')
        for field, _ in cls._fields_:
            src.append(f'  printf("{name} {field} %zu\\n", offsetof({name}, {field}));')
    src += ["  return 0;", "}"]
    os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
    with tempfile.TemporaryDirectory(dir=os.path.join(ROOT, "_build")) as tmp:
        c_file, exe = os.path.join(tmp, "layout.c"), os.path.join(tmp, "layout")
        with open(c_file, "w") as f:
            f.write("\n".join(src) + "\n")
        subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        c_file, "-o", exe], check=True, timeout=120)
        out = subprocess.run([exe], check=True, capture_output=True, text=True,
                             timeout=60).stdout
    seen = 0
    for line in out.splitlines():
        name, field, value = line.split()
        cls = mirrors[name]
        if field == "sizeof":
            assert ctypes.sizeof(cls) == int(value), name
        else:
            assert getattr(cls, field).offset == int(value), (name, field)
        seen += 1
    assert seen == sum(len(c._fields_) + 1 for c in mirrors.values())


def test_binding_argument_counts_match_the_header():
    """Every entry point's ctypes argtypes has as many entries as the header
    declares parameters."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    decls = re.findall(r"BA_API\s+[\w\s\*]+?\b(\w+)\s*\(([^)]*)\)\s*;", text, flags=re.S)
    assert decls
    for name, params in decls:
        params = params.strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        fn = getattr(ba.lib, name)
        assert fn.argtypes is not None, name
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)


def test_plain_c_caller_links_and_runs():
    """A C program (tests/c/host_caller.c) compiles against the header, links
    the shared library and gets the documented results from the calls that
    need no GPU."""
    import shutil
    import subprocess
    import tempfile
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    lib_dir = os.path.dirname(ba.LIB_PATH)
    os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
    with tempfile.TemporaryDirectory(dir=os.path.join(ROOT, "_build")) as tmp:
        exe = os.path.join(tmp, "host_caller")
        subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c", "host_caller.c"), "-o", exe,
                        "-L", lib_dir, "-lbranch_attn", f"-Wl,-rpath,{lib_dir}"],
                       check=True, timeout=120)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
