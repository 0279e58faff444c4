"""TapChannel on the GPU: producers in other processes fan messages into the
consumer's mailbox through CUDA IPC.

Two producer processes each send 10 messages through a 3-slot mailbox (so
every slot is reused and producers must wait for releases); the consumer
checks every payload and stamp in order, and releases each slot after
reading it.  A wait for a message nobody sends gives up after its limit.
(CUDA IPC handles open only in other processes, so producers always run in
processes of their own.)  All processes share this GPU: no kernel of the
channel waits for another process (waits are host polls), so that is safe.
"""
import multiprocessing as mp

import pytest
import torch

pytestmark = pytest.mark.gpu

SLOT = 1 << 20
N_MSG = 10


def _pattern(producer, seq, n):
    # a payload that differs per producer, message and position
    base = torch.arange(n, dtype=torch.int32, device="cuda")
    return ((base * 7 + producer * 1000003 + seq * 131) % 251).to(torch.uint8)


def _producer(handle, producer, q):
    import os
    import sys
    sys.path.insert(0, os.environ["BA_ROOT"])
    import speculative_draft_branch_b200 as ba
    torch.cuda.set_device(0)
    try:
        tx = ba.TapProducer(handle, producer)
        for seq in range(N_MSG):
            n = SLOT - 4096 * (seq % 3)          # payloads of varying length
            tx.send(seq, _pattern(producer, seq, n), timeout_s=60)
            torch.cuda.current_stream().synchronize()
        tx.close()
        q.put((producer, "ok"))
    except Exception as e:  # reported to the test
        q.put((producer, repr(e)))


def test_fan_in_through_reused_slots(cuda_lib, monkeypatch):
    import os
    ba = cuda_lib
    monkeypatch.setenv("BA_ROOT", os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    rx = ba.TapConsumer(2, 3, SLOT)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_producer, args=(rx.handle, p, q)) for p in range(2)]
    for p in procs:
        p.start()
    try:
        for seq in range(N_MSG):
            for p in range(2):
                slot = rx.wait(p, seq, timeout_s=120)
                n = SLOT - 4096 * (seq % 3)
                assert torch.equal(slot[:n], _pattern(p, seq, n)), (p, seq)
                rx.release(p, seq)
        results = sorted(q.get(timeout=120) for _ in procs)
        assert results == [(0, "ok"), (1, "ok")], results
    finally:
        for p in procs:
            p.join(timeout=60)
        rx.close()
    assert all(p.exitcode == 0 for p in procs)


def test_wait_gives_up_and_channel_stays_usable(cuda_lib):
    """A wait for a message nobody sends ends with BA_ERR_DEVICE_TIMEOUT after
    its limit; the channel can still be released from and closed, and a new
    one made."""
    ba = cuda_lib
    rx = ba.TapConsumer(1, 2, 4096)
    with pytest.raises(ba.BranchAttnError) as e:
        rx.wait(0, 0, timeout_s=0.2)
    assert e.value.status == -6
    rx.release(0, 0)
    torch.cuda.synchronize()
    rx.close()
    again = ba.TapConsumer(1, 2, 4096)
    again.close()
