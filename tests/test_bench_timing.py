"""bench.device_times on CPU with a stand-in for torch.cuda: the order of
event records, calls and the one synchronisation at the end."""

import bench


class _FakeEvent:
    def __init__(self, log, enable_timing=False):
        self.log = log
        self.t = None
        self.synced = False

    def record(self, stream):
        self.t = len(self.log)
        self.log.append(("record", id(self)))

    def synchronize(self):
        self.synced = True
        self.log.append(("sync", id(self)))

    def elapsed_time(self, other):
        return float(other.t - self.t)


class _FakeTorch:
    def __init__(self):
        self.log = []
        outer = self

        class _Cuda:
            @staticmethod
            def Event(enable_timing=False):
                return _FakeEvent(outer.log, enable_timing)

        self.cuda = _Cuda()


def test_device_times_brackets_each_call_and_syncs_once():
    t = _FakeTorch()
    calls = []
    f = lambda: (calls.append("f"), t.log.append(("call", "f")))
    g = lambda: (calls.append("g"), t.log.append(("call", "g")))
    flush = lambda: t.log.append(("call", "flush"))
    tf, tg = bench.device_times(t, None, [f, g], reps=3, before=flush)
    assert calls == ["f", "g"] * 3
    assert len(tf) == len(tg) == 3
    # Per repetition: flush, record, f, record, g, record; each timed interval
    # spans exactly its own call (record -> call -> record: 2 log entries).
    assert all(x == 2.0 for x in tf + tg)
    kinds = [k for k, _ in t.log]
    assert kinds.count("sync") == 1 and kinds[-1] == "sync"
    for r in range(3):
        seg = t.log[r * 6:(r + 1) * 6]
        assert [k for k, _ in seg] == ["call", "record", "call", "record", "call", "record"]
        assert seg[0][1] == "flush"


def test_device_times_without_before():
    t = _FakeTorch()
    (ts,) = bench.device_times(t, None, [lambda: t.log.append(("call", "f"))], reps=2)
    assert ts == [2.0, 2.0]
    assert [k for k, _ in t.log].count("sync") == 1
