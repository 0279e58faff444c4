"""Host logic of bench.py's HBM-step measurement, run on the CPU with fake
CUDA events and a fake library, so every line executes and the byte
accounting is checked against hand-computed figures."""
import os
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class _Clock:
    t = 0.0


class _FakeEvent:
    """Records a tick of a shared clock; elapsed_time is the tick difference (ms)."""

    def __init__(self, enable_timing=True):
        self.stamp = None
        self.cuda_event = 1

    def record(self, stream=None):
        _Clock.t += 1.0
        self.stamp = _Clock.t

    def elapsed_time(self, other):
        return other.stamp - self.stamp


def test_hbm_steps_byte_accounting(monkeypatch):
    import torch
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    calls = {"merge": 0, "bwd": 0, "events": []}
    ks_ke = {}

    def lse_merge(o_a, l_a, o_b, l_b, o_o, l_o, stream=None):
        assert o_a.shape == o_b.shape == o_o.shape and l_a.shape == (o_a.shape[1], o_a.shape[0])
        calls["merge"] += 1

    def set_events(which, start=None, stop=None):
        assert which == 2                          # the preprocess kernel's own events
        calls["events"].append(start is not None)
        ks_ke["pair"] = (start, stop)

    ba = types.SimpleNamespace(lse_merge=lse_merge, ba_set_kernel_events=set_events,
                               ba_get_kernel_family=lambda: family[0])

    class Runner:
        problem = types.SimpleNamespace(c=types.SimpleNamespace(
            n_main=1000, n_branch_tokens=3000, hq=4, head_dim=64))

        def backward(self, t, out, grads):
            # the library records the preprocess events right around its kernel
            calls["bwd"] += 1
            start, stop = ks_ke["pair"]
            start.record()
            _Clock.t += 1.0                       # the kernel itself: 2 ticks apart
            stop.record()

    for fam, zero in ((0, 0), (1, 4 * 64)):
        family = [fam]
        calls.update(merge=0, bwd=0, events=[])
        res = bench.hbm_steps(ba, Runner(), {}, {}, {}, None, "cpu", hbm_gbs=1000.0,
                              max_rows=2500)
        assert calls["merge"] == 13 and calls["bwd"] == 5
        assert calls["events"][-1] is False           # events switched off afterwards
        m = res["lse_merge"]
        assert m["rows"] == 2500                      # capped at max_rows
        assert m["bytes_per_launch"] == 2500 * 4 * (3 * 64 * 4 + 3 * 4)
        assert m["ms"] == pytest.approx(0.1)          # 10 calls between two ticks
        p = res["bwd_preprocess"]
        assert p["ms"] == pytest.approx(2.0)
        # O, dO, LSE read, D and the {LSE, D} record written per row-head (plus
        # the zeroed fp32 dQ accumulator of the fused backward)
        assert p["bytes_per_launch"] == 4000 * 4 * (2 * 64 * 2 + 4 + 4 + 8 + zero)
        assert p["frac"] == pytest.approx(p["achieved"] / 1000.0)
        assert p["achieved"] == pytest.approx(p["bytes_per_launch"] / 2e-3 / 1e9)


def test_clock_sampler_parses_samples_and_reasons(monkeypatch):
    """ClockSampler against a stand-in nvidia-smi printing three samples: the
    median SM clock is taken over the samples under load, throttle reasons are
    the ones reported Active, and the sampler cleans up after itself."""
    import stat
    import tempfile
    sys.path.insert(0, ROOT)
    import bench
    lines = ["0, 1500, 1965, 900.5, 0x4, Not Active, Not Active, Not Active, Active",
             "0, 300, 1965, 100.0, 0x0, Not Active, Not Active, Not Active, Not Active",
             "0, 1520, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active"]
    os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
    with tempfile.TemporaryDirectory(dir=os.path.join(ROOT, "_build")) as tmp:
        fake = os.path.join(tmp, "nvidia-smi")
        with open(fake, "w") as f:
            f.write("#!/usr/bin/env python3\nimport time\n")
            for ln in lines:
                f.write(f"print({ln!r}, flush=True)\n")
            f.write("time.sleep(60)\n")
        os.chmod(fake, os.stat(fake).st_mode | stat.S_IXUSR)
        monkeypatch.setenv("PATH", tmp + os.pathsep + os.environ["PATH"])
        cs = bench.ClockSampler(0)
        cs.start()
        import time
        time.sleep(1.0)
        clk = cs.stop()
        assert not os.path.exists(cs.path) and cs.out.closed
    assert clk["samples"] == 3
    assert clk["sm_mhz"] == pytest.approx(1510.0)
    assert clk["sm_max_mhz"] == pytest.approx(1965.0)
    assert clk["reasons"] == ["sw_power_cap"]
    assert clk["power_w_max"] == pytest.approx(950.0)


def test_clock_sampler_without_nvidia_smi(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("PATH", os.path.join(ROOT, "no-such-dir"))
    cs = bench.ClockSampler(0)
    cs.start()
    clk = cs.stop()
    assert clk["reasons"] == ["nvidia-smi unavailable"] and not os.path.exists(cs.path)


def test_profiled_traffic_only_for_the_profiled_sources(monkeypatch):
    """The traffic figure of a profile summary is used only while its source
    hash matches the current kernel sources; every profile kind hashes its own
    list of sources, and every listed file exists."""
    import tempfile
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setattr(bench, "kernel_source_sha", lambda kernel="bwd_attention": "00c0ffee00c0ffee")
    os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
    with tempfile.TemporaryDirectory(dir=os.path.join(ROOT, "_build")) as tmp:
        os.mkdir(os.path.join(tmp, "profiles"))
        monkeypatch.setattr(bench, "ROOT", tmp)
        with open(os.path.join(tmp, "profiles", "bwd_attention_w.md"), "w") as f:
            f.write("traffic_bytes_per_launch: 2.5e9\nsource_sha: 00c0ffee00c0ffee\n")
        with open(os.path.join(tmp, "profiles", "fwd_attention_w.md"), "w") as f:
            f.write("traffic_bytes_per_launch: 1.0e9\nsource_sha: 1111111111111111\n")
        assert bench.profiled_traffic("bwd_attention", "w") == 2.5e9
        assert bench.profiled_traffic("fwd_attention", "w") is None     # stale profile
        assert bench.profiled_traffic("bwd_attention", "other") is None  # no profile
    monkeypatch.undo()
    for kind in bench.PROFILED_SOURCES:
        assert len(bench.kernel_source_sha(kind)) == 16
