"""Failure detection on the device without a fault.

Every wait in the tcgen05 kernels is bounded; on expiry the kernel returns and
reports through the plan workspace's device-timeout word.  ba_wait_check runs
that same bounded wait on a barrier nothing arrives on (a flag that is never
set): the wait must give up after its limit, the host must read
BA_ERR_DEVICE_TIMEOUT, and the context must stay usable for the next step.
"""
import time

import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu


def _step(ba, runner, t):
    runner.plan()
    out = runner.forward(t)
    grads = runner.backward(t, out)
    torch.cuda.synchronize()
    assert runner.plan_status() == 0
    return {k: v.cpu() for k, v in {**out, **grads}.items()}


def test_bounded_wait_gives_up_and_the_context_stays_usable(cuda_lib):
    ba = cuda_lib
    st = wl.structure("tiny_ttt")
    t = wl.tensors(st, 11, "cuda")
    runner = ba.BranchAttention(ba.Problem.from_structure(st))
    before = _step(ba, runner, t)

    # a wait whose barrier is arrived on completes and reports nothing
    ba.ba_wait_check(runner.plan_ws, True)
    torch.cuda.synchronize()
    assert runner.plan_status() == 0

    # nothing arrives: the wait gives up after its 2 s limit
    t0 = time.perf_counter()
    ba.ba_wait_check(runner.plan_ws, False)
    with pytest.raises(ba.BranchAttnError) as e:
        runner.plan_status()
    assert e.value.status == -6
    assert "0x8000" in str(e.value)
    assert time.perf_counter() - t0 >= 1.9

    # the next plan clears the word and the same step gives the same results
    after = _step(ba, runner, t)
    for k in before:
        assert torch.equal(before[k], after[k]), k
