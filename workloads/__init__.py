"""Seeded synthetic workloads for branch attention (structure + tensors).

This module only draws random numbers and lays out index arrays; it holds none
of the attention arithmetic. Both the fp64 oracle tests and the CUDA path take
their inputs from here, so the two sides see bit-identical data.

Structure (which tokens exist, which main positions anchor a branch, how deep
each branch is) follows the workload descriptions of "Online Draft Co-Training"
(the EAGLE-3 TTT, DFlash block and DSpark block-causal draft layers named in the
key-results and experiment-design sections of the paper summary pages):

  tiny_ttt     2 packed sequences (96, 160 tokens), 4 q / 2 kv heads, d=64,
               a depth-3 branch at every main position, TTT-causal.
  ttt_20k      20,480 packed main tokens, lengths uniform in [1024, 8192] with
               the last one cut to fit, 32 q / 8 kv heads, d=128, depth-3
               branch at every position, TTT-causal.
  dflash_32k   32,768 packed main tokens, lengths round(2048 * 8**U) (log-
               uniform 2K..16K) with the last one cut to fit, 32/8 heads,
               d=128, 2,048 distinct anchors drawn uniformly without
               replacement, 16-token blocks, bidirectional inside a block.
  dspark_64k   one 65,536-token sequence, 32 q / 4 kv heads, d=128, an 8-token
               branch anchored at 0-based positions 32k+31, block-causal.
  ttt_256k     one 262,144-token sequence, 32/8 heads, d=128, depth-3 branch
               at every position, TTT-causal; also run as C=8 virtual zigzag
               shards.

Tensors are N(0, 1) drawn in fp32 with torch.randn and rounded to bf16, in the
fixed order q_m, k_m, v_m, q_b, k_b, v_b, do_m, do_b, from a torch generator
seeded 100 + workload id.  Structure uses numpy.random.default_rng(workload id).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

MASK_TTT_CAUSAL = 0
MASK_BLOCK_BIDIR = 1
MASK_BLOCK_CAUSAL = 2
MASK_NAMES = {MASK_TTT_CAUSAL: "ttt_causal", MASK_BLOCK_BIDIR: "block_bidir",
              MASK_BLOCK_CAUSAL: "block_causal"}


@dataclasses.dataclass
class Structure:
    """Index structure of one packed branch-attention batch (host numpy, int64)."""
    name: str
    cu_seqlens: np.ndarray      # [S+1], cu[0]=0, strictly increasing
    anchors: np.ndarray         # [n_br], packed main index, non-decreasing
    depths: np.ndarray          # [n_br], 1..64
    hq: int
    hkv: int
    head_dim: int
    mask_kind: int
    zigzag_C: int = 1
    scale: Optional[float] = None

    def __post_init__(self):
        self.cu_seqlens = np.asarray(self.cu_seqlens, dtype=np.int64)
        self.anchors = np.asarray(self.anchors, dtype=np.int64)
        self.depths = np.asarray(self.depths, dtype=np.int64)
        if self.scale is None:
            self.scale = 1.0 / float(np.sqrt(self.head_dim))

    @property
    def n_seqs(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def n_main(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def n_branches(self) -> int:
        return int(self.anchors.shape[0])

    @property
    def n_branch_tokens(self) -> int:
        return int(self.depths.sum())

    def with_mask(self, mask_kind: int) -> "Structure":
        return dataclasses.replace(self, mask_kind=mask_kind)


WORKLOADS = ("tiny_ttt", "ttt_20k", "dflash_32k", "dspark_64k", "ttt_256k")
WORKLOAD_ID = {name: i + 1 for i, name in enumerate(WORKLOADS)}


def _pack_lengths(rng, target, draw):
    lengths = []
    total = 0
    while total < target:
        ln = int(draw(rng))
        if total + ln >= target:
            ln = target - total
        lengths.append(ln)
        total += ln
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


def structure(name: str) -> Structure:
    """Structure of a named workload (deterministic)."""
    wid = WORKLOAD_ID[name]
    rng = np.random.default_rng(wid)
    if name == "tiny_ttt":
        cu = np.array([0, 96, 256], dtype=np.int64)
        n = 256
        return Structure(name, cu, np.arange(n), np.full(n, 3), 4, 2, 64, MASK_TTT_CAUSAL)
    if name == "ttt_20k":
        cu = _pack_lengths(rng, 20480, lambda r: r.integers(1024, 8192, endpoint=True))
        n = 20480
        return Structure(name, cu, np.arange(n), np.full(n, 3), 32, 8, 128, MASK_TTT_CAUSAL)
    if name == "dflash_32k":
        cu = _pack_lengths(rng, 32768, lambda r: round(2048.0 * 8.0 ** r.random()))
        anchors = np.sort(rng.choice(32768, size=2048, replace=False))
        return Structure(name, cu, anchors, np.full(2048, 16), 32, 8, 128, MASK_BLOCK_BIDIR)
    if name == "dspark_64k":
        cu = np.array([0, 65536], dtype=np.int64)
        anchors = 32 * np.arange(2048) + 31
        return Structure(name, cu, anchors, np.full(2048, 8), 32, 4, 128, MASK_BLOCK_CAUSAL)
    if name == "ttt_256k":
        n = 262144
        cu = np.array([0, n], dtype=np.int64)
        return Structure(name, cu, np.arange(n), np.full(n, 3), 32, 8, 128, MASK_TTT_CAUSAL,
                         zigzag_C=8)
    raise KeyError(name)


def random_structure(seed: int, n_seqs: int = 3, max_len: int = 40, max_depth: int = 5,
                     hq: int = 2, hkv: int = 1, head_dim: int = 8, mask_kind: int = 0,
                     branch_prob: float = 0.5, zigzag_C: int = 1) -> Structure:
    """Small random packed batch for brute-force checks."""
    rng = np.random.default_rng(seed)
    lengths = rng.integers(1, max_len, size=n_seqs, endpoint=True)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    n = int(cu[-1])
    sel = np.nonzero(rng.random(n) < branch_prob)[0]
    anchors = np.sort(sel).astype(np.int64)
    depths = rng.integers(1, max_depth, size=anchors.shape[0], endpoint=True)
    return Structure(f"random{seed}", cu, anchors, depths, hq, hkv, head_dim, mask_kind,
                     zigzag_C=zigzag_C)


def truncate(st: Structure, n_tokens: int) -> Structure:
    """First n_tokens main tokens of a batch and the branches anchored in them."""
    cu = st.cu_seqlens
    keep = cu[cu < n_tokens]
    cu_new = np.concatenate([keep, [n_tokens]]).astype(np.int64)
    sel = st.anchors < n_tokens
    return dataclasses.replace(st, name=f"{st.name}[:{n_tokens}]", cu_seqlens=cu_new,
                               anchors=st.anchors[sel], depths=st.depths[sel])


TENSOR_ORDER = ("q_m", "k_m", "v_m", "q_b", "k_b", "v_b", "do_m", "do_b")


def tensor_shapes(st: Structure) -> Dict[str, tuple]:
    n, nb, hq, hkv, d = st.n_main, st.n_branch_tokens, st.hq, st.hkv, st.head_dim
    return {"q_m": (n, hq, d), "k_m": (n, hkv, d), "v_m": (n, hkv, d),
            "q_b": (nb, hq, d), "k_b": (nb, hkv, d), "v_b": (nb, hkv, d),
            "do_m": (n, hq, d), "do_b": (nb, hq, d)}


def tensors(st: Structure, seed: int, device="cpu"):
    """bf16 N(0,1) tensors in the fixed draw order (torch generator on `device`)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = {}
    for key, shape in tensor_shapes(st).items():
        x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        out[key] = x.to(torch.bfloat16)
    return out


def workload_seed(name: str) -> int:
    return 100 + WORKLOAD_ID[name]


def slice_tensors(st_full: Structure, st_trunc: Structure, t: dict) -> dict:
    """Restrict full-batch tensors to a truncated batch (prefix rows)."""
    n = st_trunc.n_main
    nb = st_trunc.n_branch_tokens
    out = {}
    for key, x in t.items():
        out[key] = x[:n] if key.endswith("_m") else x[:nb]
    return out


def truncate_each(st: Structure, k: int, parts: int):
    """Every sequence of a batch cut to its first floor(k L / parts) tokens (L its
    length; sequences cut to nothing are dropped) with the branches anchored in
    what is kept.  Returns the structure and the kept main rows and branch rows
    of the original batch, in order, for gather_tensors."""
    cu = st.cu_seqlens
    lens = np.diff(cu)
    keep_len = (k * lens) // parts
    main_rows, new_cu = [], [0]
    for s in range(st.n_seqs):
        if keep_len[s] > 0:
            main_rows.append(np.arange(cu[s], cu[s] + keep_len[s]))
            new_cu.append(new_cu[-1] + int(keep_len[s]))
    main_rows = np.concatenate(main_rows) if main_rows else np.zeros(0, dtype=np.int64)
    new_index = np.full(st.n_main, -1, dtype=np.int64)
    new_index[main_rows] = np.arange(main_rows.shape[0])
    cu_branch = np.concatenate([[0], np.cumsum(st.depths)])
    sel = np.nonzero(new_index[st.anchors] >= 0)[0] if st.n_branches else np.zeros(0, np.int64)
    branch_rows = (np.concatenate([np.arange(cu_branch[b], cu_branch[b + 1]) for b in sel])
                   if sel.size else np.zeros(0, dtype=np.int64))
    out = dataclasses.replace(st, name=f"{st.name}[{k}/{parts} of each sequence]",
                              cu_seqlens=np.asarray(new_cu, dtype=np.int64),
                              anchors=new_index[st.anchors[sel]], depths=st.depths[sel])
    return out, main_rows, branch_rows


def gather_tensors(t: dict, main_rows, branch_rows) -> dict:
    """Rows of a batch's tensors picked by truncate_each (contiguous copies)."""
    import torch
    out = {}
    for key, x in t.items():
        rows = main_rows if key.endswith("_m") else branch_rows
        idx = torch.as_tensor(np.asarray(rows, dtype=np.int64), device=x.device)
        out[key] = x.index_select(0, idx).contiguous()
    return out
