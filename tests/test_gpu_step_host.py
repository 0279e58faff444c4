"""The host-buffer step (branch_attn_step_host) against the device path.

The step stages host tensors through a device workspace and runs the same
plan / forward / backward kernels, which are deterministic (no atomics), so
its host outputs must equal the device path's outputs bit for bit.  Two steps
issued on two streams with their own staging (the pipelined use the
interface is made for) must each still match.
"""
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu

OUTS = ("o_m", "o_b", "lse_m", "lse_b")
GRADS = ("dq_m", "dk_m", "dv_m", "dq_b", "dk_b", "dv_b")
INS = ("q_m", "k_m", "v_m", "q_b", "k_b", "v_b", "do_m", "do_b")


def device_path(ba, st, t):
    prob = ba.Problem.from_structure(st)
    runner = ba.BranchAttention(prob)
    runner.plan()
    assert runner.plan_status() == 0
    out = runner.forward(t)
    grads = runner.backward(t, out)
    torch.cuda.synchronize()
    assert runner.plan_status() == 0
    res = dict(out)
    res.update(grads)
    return {k: v.cpu() for k, v in res.items()}


def host_step(ba, st, t, stream=None, staging=None):
    prob = ba.Problem.from_structure(st, device="cpu")
    hin = {k: t[k].cpu().pin_memory() for k in INS}
    sh = prob.shapes()
    like = {"o_m": "q_m", "o_b": "q_b", "dq_m": "q_m", "dk_m": "k_m", "dv_m": "v_m",
            "dq_b": "q_b", "dk_b": "k_b", "dv_b": "v_b"}
    hout = {k: torch.empty(sh[like[k]], dtype=torch.bfloat16, pin_memory=True) for k in like}
    hout["lse_m"] = torch.empty(sh["lse_m"], dtype=torch.float32, pin_memory=True)
    hout["lse_b"] = torch.empty(sh["lse_b"], dtype=torch.float32, pin_memory=True)
    if staging is None:
        staging = torch.empty(ba.ba_step_host_workspace_size(prob), dtype=torch.uint8,
                              device="cuda")
    ba.branch_attn_step_host(prob, staging, *(hin[k] for k in INS),
                             *(hout[k] for k in OUTS), *(hout[k] for k in GRADS), stream=stream)
    return prob, hin, hout, staging


def assert_same(got, ref):
    for k in OUTS + GRADS:
        assert got[k].shape == ref[k].shape, k
        assert torch.equal(got[k], ref[k]), f"{k} differs from the device path"


@pytest.mark.parametrize("case", ["tiny", "random", "no_branches"])
def test_step_host_matches_device_path(cuda_lib, case):
    if case == "tiny":
        st = wl.structure("tiny_ttt")
    elif case == "random":
        st = wl.random_structure(5, n_seqs=3, max_len=300,
                                 hq=8, hkv=2, head_dim=128, mask_kind=wl.MASK_TTT_CAUSAL)
    else:
        st = wl.random_structure(6, n_seqs=2, max_len=200,
                                 hq=4, hkv=4, head_dim=64, mask_kind=wl.MASK_TTT_CAUSAL,
                                 branch_prob=0.0)
    t = wl.tensors(st, 31, "cuda")
    ref = device_path(cuda_lib, st, t)
    prob, _, hout, staging = host_step(cuda_lib, st, t)
    torch.cuda.synchronize()
    assert cuda_lib.ba_plan_status(staging) == 0
    assert_same(hout, ref)


def test_step_host_two_streams_pipelined(cuda_lib):
    st = wl.random_structure(8, n_seqs=4, max_len=400,
                             hq=8, hkv=2, head_dim=128, mask_kind=wl.MASK_BLOCK_CAUSAL)
    ts = [wl.tensors(st, 40 + i, "cuda") for i in range(2)]
    refs = [device_path(cuda_lib, st, t) for t in ts]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    results = [host_step(cuda_lib, st, t, stream=s) for t, s in zip(ts, streams)]
    torch.cuda.synchronize()
    for (_, _, hout, staging), ref in zip(results, refs):
        assert cuda_lib.ba_plan_status(staging) == 0
        assert_same(hout, ref)


def test_step_host_rejects_small_staging(cuda_lib):
    st = wl.structure("tiny_ttt")
    t = wl.tensors(st, 3, "cuda")
    prob = cuda_lib.Problem.from_structure(st, device="cpu")
    need = cuda_lib.ba_step_host_workspace_size(prob)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(cuda_lib.BranchAttnError) as e:
        host_step(cuda_lib, st, t, staging=small)
    assert e.value.status == -4
