"""bench.time_steps against a fake torch.cuda that records what each CUDA
graph captures and logs every replay, event record, synchronize and barrier.
The timed window (start event to end event) must hold exactly the timed
steps; every graph replayed after the barrier must have been replayed once
before it (no first-replay upload inside the window); the start event must
follow at least one untimed step and sit on a forked branch (so the first
timed step keeps its place in the launch chain); and at least `warmup` steps
must run before the barrier."""
import contextlib
import types

import pytest

import bench


def _fake_torch(log):
    state = {"stream": "default", "capturing": None}

    class Stream:
        _n = 0

        def __init__(self):
            Stream._n += 1
            self.name = f"s{Stream._n}"

        def wait_stream(self, other):
            if state["capturing"] is not None:
                state["capturing"].nodes.append(("wait", self.name, other.name))

    class _Current:
        def __init__(self, name):
            self.name = name

        def wait_stream(self, other):
            if state["capturing"] is not None:
                state["capturing"].nodes.append(("wait", self.name, other.name))

    def current_stream():
        return _Current(state["stream"])

    @contextlib.contextmanager
    def stream(s):
        prev = state["stream"]
        state["stream"] = s.name
        try:
            yield
        finally:
            state["stream"] = prev

    class CUDAGraph:
        _n = 0

        def __init__(self):
            CUDAGraph._n += 1
            self.gid = CUDAGraph._n
            self.nodes = []

        def replay(self):
            log.append(("replay", self.gid))
            for n in self.nodes:
                log.append(n)

    @contextlib.contextmanager
    def graph(g):
        prev = state["stream"]
        state["stream"] = f"capture{g.gid}"
        state["capturing"] = g
        try:
            yield
        finally:
            state["capturing"] = None
            state["stream"] = prev

    class Event:
        def __init__(self, enable_timing=False, external=False):
            assert enable_timing and external
            self.eid = id(self)

        def record(self):
            assert state["capturing"] is not None, "timing events are graph nodes"
            state["capturing"].nodes.append(("record", self.eid, state["stream"]))

        def elapsed_time(self, other):
            return 1.0

    cuda = types.SimpleNamespace(CUDAGraph=CUDAGraph, graph=graph, Event=Event, Stream=Stream, stream=stream,
                                 current_stream=current_stream, synchronize=lambda: log.append(("sync",)))
    return types.SimpleNamespace(cuda=cuda), state


def _run(steps, warmup, period):
    log = []
    torch, state = _fake_torch(log)

    def fn(i):
        g = state["capturing"]
        if g is not None:
            g.nodes.append(("step", i))
        else:
            log.append(("eager_step", i))

    ms = bench.time_steps(torch, fn, steps, warmup, period, lambda: log.append(("barrier",)))
    return log, ms


@pytest.mark.parametrize("steps,warmup,period", [(20, 5, 48), (10, 3, 10), (4000, 480, 48), (100, 3, 48),
                                                 (48, 3, 48), (3, 3, 3), (7, 50, 4), (2000, 5, 48)])
def test_timed_window_holds_exactly_the_timed_steps(steps, warmup, period):
    log, ms = _run(steps, warmup, period)
    barriers = [i for i, e in enumerate(log) if e == ("barrier",)]
    assert len(barriers) == 2
    b0 = barriers[0]
    assert log[b0 - 1] == ("sync",)
    timed = log[b0 + 1:barriers[1]]
    records = [i for i, e in enumerate(timed) if e[0] == "record"]
    assert len(records) == 2
    i_start, i_end = records
    # exactly the timed steps between the two events
    assert sum(1 for e in timed[i_start + 1:i_end] if e[0] == "step") == steps
    # at least one untimed step before the start event, none after the end event
    assert any(e[0] == "step" for e in timed[:i_start])
    assert not any(e[0] == "step" for e in timed[i_end + 1:])
    # the start event is recorded on a forked branch, not on the capture stream
    start_stream = timed[i_start][2]
    assert not start_stream.startswith("capture")
    # no host synchronize between the replays of the window
    assert ("sync",) not in timed[:i_end]
    # every graph replayed in the window was replayed once before the barrier
    before = log[:b0]
    replayed_before = {e[1] for e in before if e[0] == "replay"}
    for e in timed:
        if e[0] == "replay":
            assert e[1] in replayed_before
    # warm-up: at least `warmup` steps before the barrier
    assert sum(1 for e in before if e[0] in ("step", "eager_step")) >= warmup
    assert ms == 1.0


def test_graphs_are_bounded():
    """Large step counts are split over several graphs, each at most
    MAX_GRAPH_STEPS timed steps (plus the lead in the first)."""
    log, _ = _run(5000, 5, 48)
    b0 = log.index(("barrier",))
    counts, cur = [], None
    for e in log[b0 + 1:]:
        if e[0] == "replay":
            cur = 0
            counts.append(0)
        elif e[0] == "step":
            counts[-1] += 1
    assert len(counts) >= 5
    assert max(counts[1:]) <= bench.MAX_GRAPH_STEPS
    assert counts[0] <= bench.MAX_GRAPH_STEPS + 48
