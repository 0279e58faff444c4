"""The allocation-free backward entry point.

Callers that manage all device memory themselves (their own pool, no
cudaMalloc after start-up) use branch_attn_bwd_static_scratch, which keeps
the backward scratch in a fixed array inside the library.  This file is named
so that pytest collects it last.  It checks, through the C ABI, that two calls
in a row each match the workspace-taking branch_attn_bwd, and that a problem
too large for the fixed scratch is refused before anything runs.
"""
import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu

ABS, REL = 2e-2, 1e-2
NAMES = ("dq_m", "dk_m", "dv_m", "dq_b", "dk_b", "dv_b")


def _close(name, got, ref):
    got = got.detach().double().cpu().numpy()
    ref = ref.detach().double().cpu().numpy()
    diff = np.abs(got - ref)
    assert (diff <= ABS + REL * np.abs(ref)).all(), f"{name}: max abs {diff.max():.3e}"
    if np.abs(ref).max() > ABS:
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel <= REL, f"{name}: rel L2 {rel:.3e}"


@pytest.mark.parametrize("family", [0, 1])
def test_static_scratch_backward_matches_workspace_backward(cuda_lib, family):
    """Same kernels, same inputs, only the scratch memory differs, so the
    results must be bit-identical wherever the backward is deterministic: every
    gradient of the split backward (family 0, the default), and dK / dV of the
    fused one (family 1), whose dQ sums fp32 partials in an order that varies
    from run to run and is compared within the parity tolerance instead."""
    ba = cuda_lib
    st = wl.structure("tiny_ttt")
    t = wl.tensors(st, wl.workload_seed("tiny_ttt"), "cuda")
    prob = ba.Problem.from_structure(st)
    runner = ba.BranchAttention(prob)
    runner.plan()
    assert runner.plan_status() == 0
    ba.ba_set_kernel_family(family)
    try:
        out = runner.forward(t)
        ref = runner.backward(t, out)
        torch.cuda.synchronize()
        for call in range(2):
            g = runner.alloc_grads()
            for v in g.values():
                v.fill_(123.0)
            ba.branch_attn_bwd_static_scratch(
                prob, runner.plan_ws, t["q_m"], t["k_m"], t["v_m"], t["q_b"], t["k_b"], t["v_b"],
                out["o_m"], out["o_b"], out["lse_m"], out["lse_b"], t["do_m"], t["do_b"],
                g["dq_m"], g["dk_m"], g["dv_m"], g["dq_b"], g["dk_b"], g["dv_b"])
            torch.cuda.synchronize()
            assert runner.plan_status() == 0
            for name in NAMES:
                label = f"{name} (family {family}, call {call + 1})"
                if family == 1 and name.startswith("dq"):
                    _close(label, g[name], ref[name])
                else:
                    assert torch.equal(g[name], ref[name]), f"{label}: not bit-identical"
    finally:
        ba.ba_set_kernel_family(0)


def test_static_scratch_rejects_oversized_problem(cuda_lib):
    ba = cuda_lib
    st = wl.structure("ttt_20k")
    prob = ba.Problem.from_structure(st)
    _, _, need = ba.ba_workspace_size(prob)
    assert need > 32 << 20
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    # the size check runs before any pointer is used: pass raw C calls with
    # placeholder addresses so nothing large has to be allocated
    rc = ba.lib.branch_attn_bwd_static_scratch(
        ba.ctypes.byref(prob.c), dummy.data_ptr(), *([dummy.data_ptr()] * 18), None)
    assert rc == -4
    assert "static scratch" in ba.lib.ba_last_error().decode()
