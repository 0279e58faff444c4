"""TapChannel host side (no GPU): mailbox sizes and argument checks that run
before any CUDA call."""
import ctypes

import pytest

import speculative_draft_branch_b200 as ba


def test_mailbox_size_layout():
    # stamps and acks: 2 x P x S int64 rounded up to 256 bytes, then the slots
    assert ba.ba_tap_mailbox_size(1, 1, 16) == 256 + 16
    assert ba.ba_tap_mailbox_size(2, 3, 1 << 20) == 256 + 6 * (1 << 20)
    assert ba.ba_tap_mailbox_size(16, 16, 64) == 4096 + 256 * 64


@pytest.mark.parametrize("p,s,b", [(0, 1, 16), (257, 1, 16), (1, 0, 16), (1, 1025, 16),
                                   (1, 1, 8), (1, 1, 24)])
def test_mailbox_size_rejects(p, s, b):
    with pytest.raises(ba.BranchAttnError) as e:
        ba.ba_tap_mailbox_size(p, s, b)
    assert e.value.status == -1


def test_attach_rejects_foreign_bytes():
    with pytest.raises(ba.BranchAttnError) as e:
        ba.TapProducer(b"\0" * 128, 0)
    assert e.value.status == -1 and "not a mailbox handle" in str(e.value)
    t = ctypes.c_void_p()
    assert ba.lib.ba_tap_attach(None, 0, 0, ctypes.byref(t)) == -1


def test_create_rejects_missing_memory():
    t = ctypes.c_void_p()
    blob = ctypes.create_string_buffer(128)
    assert ba.lib.ba_tap_create(None, 1 << 20, 1, 1, 16, blob, 128, ctypes.byref(t)) == -1
    assert ba.lib.ba_tap_create(0x1010, 1 << 20, 1, 1, 16, blob, 128, ctypes.byref(t)) == -3
    assert ba.lib.ba_tap_create(0x1000, 100, 1, 1, 16, blob, 128, ctypes.byref(t)) == -4
    assert ba.lib.ba_tap_create(0x1000, 1 << 20, 1, 1, 16, blob, 64, ctypes.byref(t)) == -4


def test_side_checks():
    # send on a consumer-side or missing channel, wait / release on a producer side
    assert ba.lib.ba_tap_send(None, 0, 0x1000, 16, 0, None) == -1
    assert ba.lib.ba_tap_wait(None, 0, 0, 0, None) == -1
    assert ba.lib.ba_tap_release(None, 0, 0, None) == -1
    assert ba.lib.ba_tap_close(None) == 0
