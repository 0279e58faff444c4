"""Branch attention for online draft co-training on B200 (sm_100a).

Thin ctypes binding of ``libbranch_attn.so`` (C ABI in include/branch_attn.h).
The functions below carry the same names as the C entry points and only
marshal arguments: torch tensors become device pointers, the current CUDA
stream becomes the ``stream`` argument.  Shapes and dtypes are checked here so
that a mismatched tensor is rejected on the host instead of being read out of
bounds on the device.  Every step of the computation runs in the library's
CUDA kernels; there is no fallback.  Importing this package fails loudly when
the library has not been built (``python speculative_draft_branch_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbranch_attn.so")

MASK_TTT_CAUSAL = 0
MASK_BLOCK_BIDIR = 1
MASK_BLOCK_CAUSAL = 2
TILE_M = 128
TILE_N = 128

STATUS_NAMES = {0: "BA_OK", -1: "BA_ERR_INVALID_ARG", -2: "BA_ERR_UNSUPPORTED",
                -3: "BA_ERR_MISALIGNED", -4: "BA_ERR_WORKSPACE_TOO_SMALL", -5: "BA_ERR_CUDA",
                -6: "BA_ERR_DEVICE_TIMEOUT", -7: "BA_ERR_BAD_METADATA"}

EXPORTS = ("ba_workspace_size", "ba_plan_layout_query", "ba_plan", "ba_plan_status",
           "branch_attn_fwd", "branch_attn_bwd", "lse_merge", "ba_set_kernel_family",
           "ba_get_kernel_family", "ba_set_kernel_events", "ba_launch_count", "ba_last_error",
           "ba_version", "branch_attn_bwd_static_scratch", "ba_exp2_check",
           "ba_step_host_workspace_size", "branch_attn_step_host", "ba_wait_check",
           "ba_zigzag_shard", "ba_ring_workspace_size", "ba_ring_plan", "branch_attn_ring_step",
           "branch_attn_ring_finish", "ba_tap_mailbox_size", "ba_tap_create", "ba_tap_attach",
           "ba_tap_send", "ba_tap_wait", "ba_tap_release", "ba_tap_close")


class BAProblem(ctypes.Structure):
    _fields_ = [("n_seqs", ctypes.c_int32), ("n_main", ctypes.c_int32),
                ("n_branches", ctypes.c_int32), ("n_branch_tokens", ctypes.c_int32),
                ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("scale", ctypes.c_float), ("mask", ctypes.c_int32), ("zigzag_C", ctypes.c_int32),
                ("cu_seqlens", ctypes.c_void_p), ("branch_anchor", ctypes.c_void_p),
                ("branch_depth", ctypes.c_void_p)]


class BAPlanLayout(ctypes.Structure):
    _fields_ = [("total_bytes", ctypes.c_size_t)] + [
        (name, ctypes.c_size_t) for name in (
            "off_status", "off_cu_branch", "off_branch_seq", "off_row_iv", "off_qtile",
            "off_kv_main", "off_kv_branch", "off_fwd_order", "off_bwd_order", "off_fwd_cost",
            "off_bwd_cost", "off_zz_tiles", "off_key_iv", "off_bwd_prefix")] + [
        (name, ctypes.c_int32) for name in (
            "n_qtiles_main", "n_qtiles_branch", "n_kv_main", "n_kv_branch")]


class BranchAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python speculative_draft_branch_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, S, I32, I64, VP = (ctypes.POINTER(BAProblem), ctypes.c_size_t, ctypes.c_int32,
                          ctypes.c_int64, ctypes.c_void_p)
    sig = {
        "ba_workspace_size": [P, ctypes.POINTER(S), ctypes.POINTER(S), ctypes.POINTER(S)],
        "ba_plan_layout_query": [P, ctypes.POINTER(BAPlanLayout)],
        "ba_plan": [P, VP, S, VP],
        "ba_plan_status": [VP, VP, ctypes.POINTER(I32)],
        "branch_attn_fwd": [P, VP, VP, S] + [VP] * 10 + [VP],
        "branch_attn_bwd": [P, VP, VP, S] + [VP] * 18 + [VP],
        "branch_attn_bwd_static_scratch": [P, VP] + [VP] * 18 + [VP],
        "lse_merge": [I64, I32, I32, I32, VP, VP, VP, VP, VP, VP, VP],
        "ba_set_kernel_family": [I32],
        "ba_get_kernel_family": [],
        "ba_set_kernel_events": [I32, VP, VP],
        "ba_exp2_check": [VP, VP, VP, I64, VP],
        "ba_wait_check": [VP, I32, VP],
        "ba_step_host_workspace_size": [P, ctypes.POINTER(S)],
        "branch_attn_step_host": [P, VP, S] + [VP] * 18 + [VP],
        "ba_zigzag_shard": [VP, I32, VP, VP, I32, I32, I32] + [VP] * 8,
        "ba_ring_workspace_size": [P, I32, ctypes.POINTER(S), ctypes.POINTER(S)],
        "ba_ring_plan": [P, I32, I32, I32, VP, VP, VP, S, VP],
        "branch_attn_ring_step": [P, I32, I32, VP, VP, S, I32, VP, VP, VP, VP, VP],
        "branch_attn_ring_finish": [P, I32, VP, VP, S] + [VP] * 8 + [VP],
        "ba_tap_mailbox_size": [I32, I32, I64, ctypes.POINTER(S)],
        "ba_tap_create": [VP, S, I32, I32, I64, VP, S, ctypes.POINTER(VP)],
        "ba_tap_attach": [VP, S, I32, ctypes.POINTER(VP)],
        "ba_tap_send": [VP, I64, VP, I64, I64, VP],
        "ba_tap_wait": [VP, I32, I64, I64, ctypes.POINTER(VP)],
        "ba_tap_release": [VP, I32, I64, VP],
        "ba_tap_close": [VP],
        "ba_launch_count": [],
        "ba_last_error": [],
        "ba_version": [],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int32
    lib.ba_launch_count.restype = ctypes.c_int64
    lib.ba_last_error.restype = ctypes.c_char_p
    lib.ba_version.restype = ctypes.c_char_p
    return lib


lib = _load()


def _check(status: int) -> None:
    if status != 0:
        raise BranchAttnError(status, lib.ba_last_error().decode())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr() if t.numel() > 0 else None


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


class Problem:
    """A packed batch: sizes plus device index arrays (kept alive here)."""

    def __init__(self, cu_seqlens, branch_anchor, branch_depth, n_branch_tokens: int, hq: int,
                 hkv: int, head_dim: int, mask: int = MASK_TTT_CAUSAL,
                 scale: Optional[float] = None, zigzag_C: int = 1):
        import torch
        for name, t in (("cu_seqlens", cu_seqlens), ("branch_anchor", branch_anchor),
                        ("branch_depth", branch_depth)):
            if t.dtype != torch.int32 or not t.is_contiguous() or t.dim() != 1:
                raise ValueError(f"{name} must be a contiguous 1-D int32 tensor")
        if branch_anchor.numel() != branch_depth.numel():
            raise ValueError("branch_anchor and branch_depth differ in length")
        self.cu_seqlens, self.branch_anchor, self.branch_depth = (
            cu_seqlens, branch_anchor, branch_depth)
        n_main = int(cu_seqlens[-1].item()) if cu_seqlens.numel() else 0
        self.c = BAProblem(
            n_seqs=cu_seqlens.numel() - 1, n_main=n_main, n_branches=branch_anchor.numel(),
            n_branch_tokens=n_branch_tokens, hq=hq, hkv=hkv, head_dim=head_dim,
            scale=(head_dim ** -0.5) if scale is None else scale, mask=mask, zigzag_C=zigzag_C,
            cu_seqlens=_ptr(cu_seqlens), branch_anchor=_ptr(branch_anchor),
            branch_depth=_ptr(branch_depth))

    @classmethod
    def from_structure(cls, st, device="cuda", zigzag_C: Optional[int] = None):
        """From a host-side structure with numpy cu_seqlens / anchors / depths."""
        import torch
        cu = torch.as_tensor(st.cu_seqlens, dtype=torch.int32).to(device)
        an = torch.as_tensor(st.anchors, dtype=torch.int32).to(device)
        de = torch.as_tensor(st.depths, dtype=torch.int32).to(device)
        return cls(cu, an, de, int(st.depths.sum()), st.hq, st.hkv, st.head_dim, st.mask_kind,
                   st.scale, st.zigzag_C if zigzag_C is None else zigzag_C)

    def __getattr__(self, name):
        return getattr(self.c, name)

    def shapes(self):
        c = self.c
        return {"q_m": (c.n_main, c.hq, c.head_dim), "k_m": (c.n_main, c.hkv, c.head_dim),
                "v_m": (c.n_main, c.hkv, c.head_dim),
                "q_b": (c.n_branch_tokens, c.hq, c.head_dim),
                "k_b": (c.n_branch_tokens, c.hkv, c.head_dim),
                "v_b": (c.n_branch_tokens, c.hkv, c.head_dim),
                "lse_m": (c.hq, c.n_main), "lse_b": (c.hq, c.n_branch_tokens)}


def _on_current_device(t, name):
    """The library launches on the current CUDA device and dereferences every
    pointer there: a host tensor or one on another device is refused here
    instead of faulting in a kernel."""
    import torch
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (got one on {t.device})")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, but the current device is "
                         f"cuda:{torch.cuda.current_device()}")


def _expect(t, shape, dtype, name):
    if t is None:
        if 0 in shape:
            return
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")
    if t.numel():
        _on_current_device(t, name)


def _expect_ws(t, name):
    """A workspace: any dtype, contiguous, on the current device."""
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel():
        _on_current_device(t, name)


def _expect_index_arrays(problem, where):
    """ba_plan reads the index arrays on the device; the host step copies them
    from the host itself."""
    for name in ("cu_seqlens", "branch_anchor", "branch_depth"):
        t = getattr(problem, name)
        if t.numel() == 0:
            continue
        if where == "device":
            _on_current_device(t, name)
        elif t.is_cuda:
            raise ValueError(f"{name} must be a host tensor for branch_attn_step_host")


def ba_workspace_size(problem: Problem):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.ba_workspace_size(ctypes.byref(problem.c), ctypes.byref(a), ctypes.byref(b),
                                 ctypes.byref(c)))
    return a.value, b.value, c.value


def ba_plan_layout_query(problem: Problem) -> dict:
    L = BAPlanLayout()
    _check(lib.ba_plan_layout_query(ctypes.byref(problem.c), ctypes.byref(L)))
    return {name: getattr(L, name) for name, _ in BAPlanLayout._fields_}


def ba_plan(problem: Problem, plan_ws, stream=None) -> None:
    import torch
    _expect_index_arrays(problem, "device")
    _expect(plan_ws, (plan_ws.numel(),), torch.uint8, "plan_ws")
    _check(lib.ba_plan(ctypes.byref(problem.c), _ptr(plan_ws), plan_ws.numel(), _stream(stream)))


def ba_plan_status(plan_ws, stream=None) -> int:
    _expect_ws(plan_ws, "plan_ws")
    word = ctypes.c_int32()
    st = lib.ba_plan_status(_ptr(plan_ws), _stream(stream), ctypes.byref(word))
    if st not in (0, -7):
        _check(st)  # BA_ERR_DEVICE_TIMEOUT or a CUDA error raises
    return word.value


def branch_attn_fwd(problem: Problem, plan_ws, fwd_ws, q_m, k_m, v_m, q_b, k_b, v_b, o_m, o_b,
                    lse_m, lse_b, stream=None) -> None:
    import torch
    _expect_ws(plan_ws, "plan_ws")
    if fwd_ws is not None:
        _expect_ws(fwd_ws, "fwd_ws")
    sh = problem.shapes()
    for name, t in (("q_m", q_m), ("k_m", k_m), ("v_m", v_m), ("q_b", q_b), ("k_b", k_b),
                    ("v_b", v_b)):
        _expect(t, sh[name], torch.bfloat16, name)
    _expect(o_m, sh["q_m"], torch.bfloat16, "o_m")
    _expect(o_b, sh["q_b"], torch.bfloat16, "o_b")
    _expect(lse_m, sh["lse_m"], torch.float32, "lse_m")
    _expect(lse_b, sh["lse_b"], torch.float32, "lse_b")
    nbytes = fwd_ws.numel() * fwd_ws.element_size() if fwd_ws is not None else 0
    _check(lib.branch_attn_fwd(ctypes.byref(problem.c), _ptr(plan_ws), _ptr(fwd_ws), nbytes,
                               _ptr(q_m), _ptr(k_m), _ptr(v_m), _ptr(q_b), _ptr(k_b), _ptr(v_b),
                               _ptr(o_m), _ptr(o_b), _ptr(lse_m), _ptr(lse_b), _stream(stream)))


def branch_attn_bwd(problem: Problem, plan_ws, bwd_ws, q_m, k_m, v_m, q_b, k_b, v_b, o_m, o_b,
                    lse_m, lse_b, do_m, do_b, dq_m, dk_m, dv_m, dq_b, dk_b, dv_b,
                    stream=None) -> None:
    import torch
    _expect_ws(plan_ws, "plan_ws")
    _expect_ws(bwd_ws, "bwd_ws")
    sh = problem.shapes()
    pairs = (("q_m", q_m, "q_m"), ("k_m", k_m, "k_m"), ("v_m", v_m, "v_m"), ("q_b", q_b, "q_b"),
             ("k_b", k_b, "k_b"), ("v_b", v_b, "v_b"), ("o_m", o_m, "q_m"), ("o_b", o_b, "q_b"),
             ("do_m", do_m, "q_m"), ("do_b", do_b, "q_b"), ("dq_m", dq_m, "q_m"),
             ("dk_m", dk_m, "k_m"), ("dv_m", dv_m, "v_m"), ("dq_b", dq_b, "q_b"),
             ("dk_b", dk_b, "k_b"), ("dv_b", dv_b, "v_b"))
    for name, t, like in pairs:
        _expect(t, sh[like], torch.bfloat16, name)
    _expect(lse_m, sh["lse_m"], torch.float32, "lse_m")
    _expect(lse_b, sh["lse_b"], torch.float32, "lse_b")
    nbytes = bwd_ws.numel() * bwd_ws.element_size()
    _check(lib.branch_attn_bwd(ctypes.byref(problem.c), _ptr(plan_ws), _ptr(bwd_ws), nbytes,
                               _ptr(q_m), _ptr(k_m), _ptr(v_m), _ptr(q_b), _ptr(k_b), _ptr(v_b),
                               _ptr(o_m), _ptr(o_b), _ptr(lse_m), _ptr(lse_b), _ptr(do_m),
                               _ptr(do_b), _ptr(dq_m), _ptr(dk_m), _ptr(dv_m), _ptr(dq_b),
                               _ptr(dk_b), _ptr(dv_b), _stream(stream)))


def branch_attn_bwd_static_scratch(problem: Problem, plan_ws, q_m, k_m, v_m, q_b, k_b, v_b, o_m,
                                   o_b, lse_m, lse_b, do_m, do_b, dq_m, dk_m, dv_m, dq_b, dk_b,
                                   dv_b, stream=None) -> None:
    """branch_attn_bwd without a workspace argument, for callers that cannot
    allocate device memory: the scratch lives in a fixed 32 MiB array inside
    the library (larger problems are rejected).  Calls that overlap on the GPU
    share that array and must not run concurrently."""
    import torch
    _expect_ws(plan_ws, "plan_ws")
    sh = problem.shapes()
    pairs = (("q_m", q_m, "q_m"), ("k_m", k_m, "k_m"), ("v_m", v_m, "v_m"), ("q_b", q_b, "q_b"),
             ("k_b", k_b, "k_b"), ("v_b", v_b, "v_b"), ("o_m", o_m, "q_m"), ("o_b", o_b, "q_b"),
             ("do_m", do_m, "q_m"), ("do_b", do_b, "q_b"), ("dq_m", dq_m, "q_m"),
             ("dk_m", dk_m, "k_m"), ("dv_m", dv_m, "v_m"), ("dq_b", dq_b, "q_b"),
             ("dk_b", dk_b, "k_b"), ("dv_b", dv_b, "v_b"))
    for name, t, like in pairs:
        _expect(t, sh[like], torch.bfloat16, name)
    _expect(lse_m, sh["lse_m"], torch.float32, "lse_m")
    _expect(lse_b, sh["lse_b"], torch.float32, "lse_b")
    _check(lib.branch_attn_bwd_static_scratch(
        ctypes.byref(problem.c), _ptr(plan_ws), _ptr(q_m), _ptr(k_m), _ptr(v_m), _ptr(q_b),
        _ptr(k_b), _ptr(v_b), _ptr(o_m), _ptr(o_b), _ptr(lse_m), _ptr(lse_b), _ptr(do_m),
        _ptr(do_b), _ptr(dq_m), _ptr(dk_m), _ptr(dv_m), _ptr(dq_b), _ptr(dk_b), _ptr(dv_b),
        _stream(stream)))


def _expect_host(t, shape, dtype, name):
    if t is None:
        if 0 in shape:
            return
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous() or t.is_cuda:
        raise ValueError(f"{name}: expected contiguous host {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


def ba_step_host_workspace_size(problem: Problem) -> int:
    """Device staging bytes branch_attn_step_host needs for this problem."""
    n = ctypes.c_size_t()
    _check(lib.ba_step_host_workspace_size(ctypes.byref(problem.c), ctypes.byref(n)))
    return n.value


def branch_attn_step_host(problem: Problem, staging, q_m, k_m, v_m, q_b, k_b, v_b, do_m, do_b,
                          o_m, o_b, lse_m, lse_b, dq_m, dk_m, dv_m, dq_b, dk_b, dv_b,
                          stream=None) -> None:
    """One fwd+bwd step on host tensors (pinned for overlap): the problem's
    index arrays and every tensor are on the host, `staging` is a device
    uint8 buffer of ba_step_host_workspace_size bytes.  Asynchronous on
    `stream`; the host outputs are final once the stream reaches this point."""
    import torch
    sh = problem.shapes()
    for name, t, like in (("q_m", q_m, "q_m"), ("k_m", k_m, "k_m"), ("v_m", v_m, "v_m"),
                          ("q_b", q_b, "q_b"), ("k_b", k_b, "k_b"), ("v_b", v_b, "v_b"),
                          ("do_m", do_m, "q_m"), ("do_b", do_b, "q_b"), ("o_m", o_m, "q_m"),
                          ("o_b", o_b, "q_b"), ("dq_m", dq_m, "q_m"), ("dk_m", dk_m, "k_m"),
                          ("dv_m", dv_m, "v_m"), ("dq_b", dq_b, "q_b"), ("dk_b", dk_b, "k_b"),
                          ("dv_b", dv_b, "v_b")):
        _expect_host(t, sh[like], torch.bfloat16, name)
    _expect_host(lse_m, sh["lse_m"], torch.float32, "lse_m")
    _expect_host(lse_b, sh["lse_b"], torch.float32, "lse_b")
    _expect_index_arrays(problem, "host")
    _expect_ws(staging, "staging")
    nbytes = staging.numel() * staging.element_size()
    _check(lib.branch_attn_step_host(
        ctypes.byref(problem.c), _ptr(staging), nbytes, _ptr(q_m), _ptr(k_m), _ptr(v_m),
        _ptr(q_b), _ptr(k_b), _ptr(v_b), _ptr(do_m), _ptr(do_b), _ptr(o_m), _ptr(o_b),
        _ptr(lse_m), _ptr(lse_b), _ptr(dq_m), _ptr(dk_m), _ptr(dv_m), _ptr(dq_b), _ptr(dk_b),
        _ptr(dv_b), _stream(stream)))


def lse_merge(o_a, lse_a, o_b, lse_b, o_out, lse_out, stream=None) -> None:
    """o_* [rows, heads, d] fp32 or bf16; lse_* [heads, rows] fp32; in place allowed."""
    import torch
    rows, heads, d = o_a.shape
    for name, t in (("o_a", o_a), ("o_b", o_b), ("o_out", o_out)):
        _expect(t, o_a.shape, o_a.dtype, name)
    for name, t in (("lse_a", lse_a), ("lse_b", lse_b), ("lse_out", lse_out)):
        _expect(t, (heads, rows), torch.float32, name)
    if o_a.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("o_a must be fp32 or bf16")
    _check(lib.lse_merge(rows, heads, d, 1 if o_a.dtype == torch.float32 else 0, _ptr(o_a),
                         _ptr(lse_a), _ptr(o_b), _ptr(lse_b), _ptr(o_out), _ptr(lse_out),
                         _stream(stream)))


# ---- zigzag ring across ranks ------------------------------------------------
def ba_zigzag_shard(cu_seqlens, branch_anchor, branch_depth, C: int, shard: int) -> dict:
    """Local problem of one zigzag shard, from host int32 arrays of the whole
    batch: {"cu_local", "anchor_local", "depth_local", "main_rows",
    "branch_rows"} as numpy int32 arrays (see the C declaration)."""
    import numpy as np
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    an = np.ascontiguousarray(branch_anchor, dtype=np.int32)
    de = np.ascontiguousarray(branch_depth, dtype=np.int32)
    n_seqs, n_br = cu.shape[0] - 1, an.shape[0]
    if de.shape[0] != n_br:
        raise ValueError("branch_anchor and branch_depth differ in length")
    nm, nb, nbt = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    args = (cu.ctypes.data, n_seqs, an.ctypes.data if n_br else None,
            de.ctypes.data if n_br else None, n_br, C, shard,
            ctypes.byref(nm), ctypes.byref(nb), ctypes.byref(nbt))
    _check(lib.ba_zigzag_shard(*args, None, None, None, None, None))
    out = {"cu_local": np.zeros(n_seqs + 1, np.int32), "anchor_local": np.zeros(nb.value, np.int32),
           "depth_local": np.zeros(nb.value, np.int32), "main_rows": np.zeros(nm.value, np.int32),
           "branch_rows": np.zeros(nbt.value, np.int32)}
    ptrs = [out[k].ctypes.data if out[k].size else None
            for k in ("cu_local", "anchor_local", "depth_local", "main_rows", "branch_rows")]
    _check(lib.ba_zigzag_shard(*args, *ptrs))
    return out


def ba_ring_workspace_size(local: Problem, C: int):
    """(plan_bytes, acc_bytes) of one ring rank."""
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.ba_ring_workspace_size(ctypes.byref(local.c), C, ctypes.byref(a),
                                      ctypes.byref(b)))
    return a.value, b.value


def ba_ring_plan(local: Problem, C: int, shard: int, step: int, cu_global, cu_visit, plan_ws,
                 stream=None) -> None:
    import torch
    _expect_index_arrays(local, "device")
    _expect(plan_ws, (plan_ws.numel(),), torch.uint8, "plan_ws")
    for name, t in (("cu_global", cu_global), ("cu_visit", cu_visit)):
        if step > 0:
            _expect(t, (local.c.n_seqs + 1,), torch.int32, name)
    _check(lib.ba_ring_plan(ctypes.byref(local.c), C, shard, step,
                            _ptr(cu_global) if step > 0 else None,
                            _ptr(cu_visit) if step > 0 else None, _ptr(plan_ws), plan_ws.numel(),
                            _stream(stream)))


def branch_attn_ring_step(local: Problem, C: int, step: int, plan_ws, acc_ws, q_m, k_m_visit,
                          v_m_visit, q_b, stream=None) -> None:
    import torch
    _expect_ws(plan_ws, "plan_ws")
    _expect_ws(acc_ws, "acc_ws")
    sh = local.shapes()
    _expect(q_m, sh["q_m"], torch.bfloat16, "q_m")
    _expect(q_b, sh["q_b"], torch.bfloat16, "q_b")
    n_visit = k_m_visit.shape[0]
    for name, t in (("k_m_visit", k_m_visit), ("v_m_visit", v_m_visit)):
        _expect(t, (n_visit, local.c.hkv, local.c.head_dim), torch.bfloat16, name)
    _check(lib.branch_attn_ring_step(ctypes.byref(local.c), C, step, _ptr(plan_ws), _ptr(acc_ws),
                                     acc_ws.numel() * acc_ws.element_size(), n_visit, _ptr(q_m),
                                     _ptr(k_m_visit), _ptr(v_m_visit), _ptr(q_b), _stream(stream)))


def branch_attn_ring_finish(local: Problem, C: int, plan_ws, acc_ws, q_m, q_b, k_b, v_b, o_m, o_b,
                            lse_m, lse_b, stream=None) -> None:
    import torch
    _expect_ws(plan_ws, "plan_ws")
    _expect_ws(acc_ws, "acc_ws")
    sh = local.shapes()
    for name, t, like in (("q_m", q_m, "q_m"), ("q_b", q_b, "q_b"), ("k_b", k_b, "k_b"),
                          ("v_b", v_b, "v_b"), ("o_m", o_m, "q_m"), ("o_b", o_b, "q_b")):
        _expect(t, sh[like], torch.bfloat16, name)
    _expect(lse_m, sh["lse_m"], torch.float32, "lse_m")
    _expect(lse_b, sh["lse_b"], torch.float32, "lse_b")
    _check(lib.branch_attn_ring_finish(
        ctypes.byref(local.c), C, _ptr(plan_ws), _ptr(acc_ws),
        acc_ws.numel() * acc_ws.element_size(), _ptr(q_m), _ptr(q_b), _ptr(k_b), _ptr(v_b),
        _ptr(o_m), _ptr(o_b), _ptr(lse_m), _ptr(lse_b), _stream(stream)))


# ---- TapChannel ---------------------------------------------------------------
TAP_HANDLE_BYTES = 128


def ba_tap_mailbox_size(n_producers: int, n_slots: int, slot_bytes: int) -> int:
    n = ctypes.c_size_t()
    _check(lib.ba_tap_mailbox_size(n_producers, n_slots, slot_bytes, ctypes.byref(n)))
    return n.value


class TapConsumer:
    """The draft stage's end of a TapChannel: owns the mailbox (device memory
    allocated here with torch) and hands out `handle`, the bytes producers
    attach with."""

    def __init__(self, n_producers: int, n_slots: int, slot_bytes: int, device="cuda"):
        import torch
        self.n_producers, self.n_slots, self.slot_bytes = n_producers, n_slots, slot_bytes
        nbytes = ba_tap_mailbox_size(n_producers, n_slots, slot_bytes)
        self.mailbox = torch.empty(nbytes, dtype=torch.uint8, device=device)
        blob = ctypes.create_string_buffer(TAP_HANDLE_BYTES)
        t = ctypes.c_void_p()
        _check(lib.ba_tap_create(self.mailbox.data_ptr(), nbytes, n_producers, n_slots,
                                 slot_bytes, blob, TAP_HANDLE_BYTES, ctypes.byref(t)))
        self._t, self.handle = t, blob.raw

    def wait(self, producer: int, seq: int, timeout_s: float = 10.0):
        """Message `seq` of `producer` as a uint8 view of its slot."""
        p = ctypes.c_void_p()
        _check(lib.ba_tap_wait(self._t, producer, seq, int(timeout_s * 1e9), ctypes.byref(p)))
        off = p.value - self.mailbox.data_ptr()
        return self.mailbox[off:off + self.slot_bytes]

    def release(self, producer: int, seq: int, stream=None) -> None:
        _check(lib.ba_tap_release(self._t, producer, seq, _stream(stream)))

    def close(self) -> None:
        if self._t:
            _check(lib.ba_tap_close(self._t))
            self._t = None


class TapProducer:
    """A producer stage's end: maps the consumer's mailbox from its handle."""

    def __init__(self, handle: bytes, producer: int):
        t = ctypes.c_void_p()
        buf = ctypes.create_string_buffer(bytes(handle), len(handle))
        _check(lib.ba_tap_attach(buf, len(handle), producer, ctypes.byref(t)))
        self._t, self.producer = t, producer

    def send(self, seq: int, src, timeout_s: float = 10.0, stream=None) -> None:
        """Message `seq` from the CUDA tensor `src` (contiguous, current device)."""
        _expect_ws(src, "src")
        _check(lib.ba_tap_send(self._t, seq, src.data_ptr(), src.numel() * src.element_size(),
                               int(timeout_s * 1e9), _stream(stream)))

    def close(self) -> None:
        if self._t:
            _check(lib.ba_tap_close(self._t))
            self._t = None


def ba_set_kernel_family(family: int) -> None:
    _check(lib.ba_set_kernel_family(family))


def ba_get_kernel_family() -> int:
    return lib.ba_get_kernel_family()


def ba_set_kernel_events(which: int, start=None, stop=None) -> None:
    """Record torch.cuda.Event `start`/`stop` around the fwd (0) / bwd (1) kernel."""
    _check(lib.ba_set_kernel_events(which, start.cuda_event if start is not None else None,
                                    stop.cuda_event if stop is not None else None))


def ba_exp2_check(x, stream=None):
    """(polynomial 2^x, hardware ex2) of a CUDA fp32 tensor, computed on the device."""
    import torch
    _expect(x, (x.numel(),), torch.float32, "x")
    y_fma, y_hw = torch.empty_like(x), torch.empty_like(x)
    _check(lib.ba_exp2_check(_ptr(x), _ptr(y_fma), _ptr(y_hw), x.numel(), _stream(stream)))
    return y_fma, y_hw


def ba_wait_check(plan_ws, arrive: bool, stream=None) -> None:
    """Failure-detection self-check: a bounded device wait on a barrier that is
    (arrive=True) or is not (arrive=False) arrived on; in the second case the
    wait gives up after 2 s and ba_plan_status(plan_ws) then reports
    BA_ERR_DEVICE_TIMEOUT.  Asynchronous on `stream`."""
    _expect_ws(plan_ws, "plan_ws")
    _check(lib.ba_wait_check(_ptr(plan_ws), 1 if arrive else 0, _stream(stream)))


def ba_launch_count() -> int:
    return lib.ba_launch_count()


def ba_version() -> str:
    return lib.ba_version().decode()


from .runner import BranchAttention  # noqa: E402,F401
from . import ring  # noqa: E402,F401
from .ring import RingSchedule, ZigzagRingAttention  # noqa: E402,F401
