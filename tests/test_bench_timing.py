"""The benchmark's timing protocol, checked on the CPU with fakes for the CUDA
events, the synchronisation and the NVML clock sampler: W untimed warm-up
steps, then exactly K steps between one event pair each and a region pair
around all of them, with the clock sampler created (NVML initialised) before
the warm-up, so that nothing slow separates the warm-up from the timed steps.
"""
import importlib.util
import os

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_warmup_and_timed_steps_and_sampler_order(monkeypatch):
    bench = _bench()
    log = []

    class Event:
        n = 0

        def __init__(self, enable_timing=False):
            assert enable_timing
            Event.n += 1
            self.id = Event.n
            self.t = None

        def record(self):
            log.append(("record", self.id))
            self.t = len(log)

        def elapsed_time(self, other):
            return float(other.t - self.t)

    class Sampler:
        def __init__(self, index):
            log.append(("sampler_init", index))

        def __enter__(self):
            log.append(("sampler_start",))
            return self

        def __exit__(self, *a):
            log.append(("sampler_stop",))

        def summary(self):
            return {"sm_mhz": 1, "sm_max_mhz": 1, "reasons": []}

    monkeypatch.setattr(torch.cuda, "Event", Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: log.append(("sync",)))
    monkeypatch.setattr(bench, "ClockSampler", Sampler)
    monkeypatch.setattr(bench, "nvtx_range", lambda name: _Null())

    steps, warmup = 7, 4
    total, per, clk = bench.time_steps(lambda: log.append(("step",)), steps, warmup,
                                       dist_on=False, device_index=3)
    kinds = [e[0] for e in log]
    init = kinds.index("sampler_init")
    first_step = kinds.index("step")
    assert init < first_step, "NVML must initialise before the warm-up"
    start = kinds.index("sampler_start")
    # exactly W steps before the timed region, K inside it
    assert kinds[:start].count("step") == warmup
    assert kinds[start:].count("step") == steps
    # between the last warm-up step and the region: synchronisations only
    last_warm = max(i for i in range(start) if kinds[i] == "step")
    assert set(kinds[last_warm + 1:start]) <= {"sync"}
    # the region: t0, then (a, step, b) K times, then t1 and a synchronisation
    body = kinds[start + 1:]
    assert body[0] == "record"
    assert body[1:1 + 3 * steps] == ["record", "step", "record"] * steps
    assert body[1 + 3 * steps:1 + 3 * steps + 2] == ["record", "sync"]
    assert clk["sm_mhz"] == 1
    # the per-step mean spans only the step between its own events
    assert per == 2.0
    assert total == 3.0 * steps + 1.0


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def test_clock_sampler_with_a_fake_nvml(monkeypatch):
    """The sampler reads the SM clock and ORs the clock-event reasons while the
    region runs; `gpu_idle` is not reported; an NVML without the newer reasons
    call falls back to the older one."""
    import sys
    import time
    import types
    bench = _bench()
    state = {"calls": 0}
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByIndex=lambda i: ("h", i),
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetClockInfo=lambda h, c: 1965 if state["calls"] % 2 else 1900,
    )

    def reasons(h):
        state["calls"] += 1
        return 0x1 | (0x4 if state["calls"] > 3 else 0)

    fake.nvmlDeviceGetCurrentClocksThrottleReasons = reasons  # older NVML only
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    s = bench.ClockSampler(0, period_s=0.001)
    assert s.ok and s.max_mhz == 1965 and not s.samples
    with s:
        time.sleep(0.05)
    out = s.summary()
    assert out["samples"] >= 3 and out["sm_max_mhz"] == 1965
    assert out["sm_mhz"] in (1900, 1932.5, 1965)
    assert out["reasons"] == ["sw_power_cap"]
