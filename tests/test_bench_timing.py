"""Host logic of the bench's timed region: the per-step events and their
percentiles (no GPU: CUDA events are replaced by a fake clock)."""
import numpy as np

import bench


class _FakeEvent:
    clock = 0.0
    step_ms = []

    def __init__(self, enable_timing=True):
        self.at = None

    def record(self, stream=None):
        # each record lands after the step that preceded it
        if self.at is None and _FakeEvent.step_ms:
            _FakeEvent.clock += _FakeEvent.step_ms.pop(0)
        self.at = _FakeEvent.clock

    def synchronize(self):
        pass

    def elapsed_time(self, other):
        return other.at - self.at


def test_timed_steps_brackets_every_step(monkeypatch):
    import torch
    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    durations = [2.0, 2.5, 1.5, 3.0]
    _FakeEvent.clock = 0.0
    _FakeEvent.step_ms = [0.0] + list(durations)     # nothing before the first event
    ran = []
    total, per = bench.timed_steps(lambda: ran.append(1), len(durations), stream=None)
    assert len(ran) == len(durations)
    assert per == durations
    assert total == sum(durations)


def test_step_percentiles():
    x = [2.0, 2.1, 1.9, 2.05, 2.2, 2.0, 1.95, 2.3, 2.1, 2.0]
    s = bench.step_percentiles(x)
    assert s["n"] == len(x)
    assert s["median"] == float(np.median(x))
    assert s["p10"] <= s["median"] <= s["p90"]
    assert s["p10"] == float(np.percentile(x, 10)) and s["p90"] == float(np.percentile(x, 90))
    assert bench.step_percentiles([]) is None
