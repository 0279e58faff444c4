"""Builds libbranch_attn.so in-tree with nvcc for sm_100a.

    python speculative_draft_branch_b200/build.py [--force] [--verbose]

Every .cu file under csrc/ is compiled separately (parallel) and linked into
one shared library next to this file.  Rebuilds only what changed, as
decided by a content hash of each output's sources, headers and command line.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libbranch_attn.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps() -> list:
    out = [os.path.join(INCLUDE, "branch_attn.h")]
    out += sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h")))
    return out


def _digest(paths, cmd) -> str:
    """Content hash of the files an output depends on and of the command that
    makes it: an output is rebuilt whenever this changes, whatever the files'
    modification times say (a checkout or a copy can leave a built library
    newer than sources it was not built from)."""
    h = hashlib.sha256()
    h.update("\0".join(cmd).encode())
    for p in paths:
        h.update(p.encode())
        with open(p, "rb") as f:
            h.update(hashlib.sha256(f.read()).digest())
    return h.hexdigest()


def _fresh(target: str, digest: str) -> bool:
    stamp = target + ".sha256"
    if not (os.path.exists(target) and os.path.exists(stamp)):
        return False
    with open(stamp) as f:
        return f.read().strip() == digest


def _stamp(target: str, digest: str) -> None:
    with open(target + ".sha256", "w") as f:
        f.write(digest + "\n")


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    os.makedirs(OBJ, exist_ok=True)
    cu = sorted(f for f in os.listdir(CSRC) if f.endswith(".cu"))
    deps = _deps()
    jobs = []
    objs = []
    for f in cu:
        src = os.path.join(CSRC, f)
        obj = os.path.join(OBJ, f[:-3] + ".o")
        objs.append(obj)
        cmd = [nvcc()] + ARCH + FLAGS + list(extra) + ["-c", src, "-o", obj]
        digest = _digest([src] + deps, cmd[1:])
        if force or not _fresh(obj, digest):
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            jobs.append((cmd, obj, digest))

    def run(job):
        cmd, obj, digest = job
        r = subprocess.run(cmd, capture_output=True, text=True)
        return job, r

    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for (cmd, obj, digest), r in ex.map(run, jobs):
            if verbose or r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode != 0:
                raise RuntimeError("nvcc failed: " + " ".join(cmd))
            _stamp(obj, digest)
    link = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", LIB] + objs
    lib_digest = _digest(objs, link[1:])
    if force or jobs or not _fresh(LIB, lib_digest):
        r = subprocess.run(link, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("link failed")
        _stamp(LIB, lib_digest)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose))


if __name__ == "__main__":
    main()
