"""Host logic of fit.run, without a GPU: a fake library records the calls
and a fake graph capture records what a chunk would replay.  The replayed
schedule must issue exactly the eager schedule's calls, in order, and the
number of propagation passes must follow the schedule's definition
(iteration t propagates iff t is an event or (t - 1) mod U == 0; an update
outside an event runs Q passes)."""
import contextlib
import types

import pytest

from soft_voronoi_render_b200 import fit


class FakeLib(types.SimpleNamespace):
    SAD_STATS = 1

    def __init__(self):
        super().__init__()
        self.log, self.capture = [], None

    def _rec(self, name):
        (self.capture if self.capture is not None else self.log).append(name)

    def adam_cfg(self, **kw):
        return ("adam", tuple(sorted(kw.items())))

    def densify_cfg(self, **kw):
        return ("densify", tuple(sorted(kw.items())))

    def __getattr__(self, name):
        if name.startswith("sad_"):
            return lambda *a, **k: self._rec(name)
        raise AttributeError(name)


class FakeGraph:
    def __init__(self, lib):
        self.lib, self.calls = lib, None

    def replay(self):
        assert self.calls is not None
        self.lib.log.extend(self.calls)


def fake_sad(lib):
    @contextlib.contextmanager
    def graph(g):
        lib.capture = []
        yield
        g.calls, lib.capture = lib.capture, None

    cuda = types.SimpleNamespace(CUDAGraph=lambda: FakeGraph(lib), graph=graph, current_stream=lambda: "capture")
    return types.SimpleNamespace(ctx=1, stream="main", torch=types.SimpleNamespace(cuda=cuda))


def run(monkeypatch, sched, graphs):
    lib = FakeLib()
    monkeypatch.setattr(fit, "_lib", lib)
    events = []
    info = fit.run(fake_sad(lib), sched, on_event=events.append, graphs=graphs)
    return lib.log, info, events


@pytest.mark.parametrize("T,events,U,Q", [(40, (), 1, 1), (60, (30,), 1, 1), (100, (17, 50, 51), 4, 2),
                                          (33, (), 8, 3), (16, (), 16, 1), (5, (3,), 2, 1), (200, (100,), 6, 1)])
def test_replayed_schedule_issues_the_eager_calls(monkeypatch, T, events, U, Q):
    sched = fit.Schedule(iterations=T, events=events, update_every=U, passes_per_update=Q)
    eager, ie, ev_e = run(monkeypatch, sched, graphs=False)
    replay, ir, ev_r = run(monkeypatch, sched, graphs=True)
    assert replay == eager
    assert ev_e == ev_r == sorted(events)
    assert ie["graph_replays"] == 0 and ie["eager_iterations"] == T - len(events)
    assert ir["eager_iterations"] + ir["chunk"] * ir["graph_replays"] + len(events) == T
    # jump-1 passes per iteration (fused or separate; refreshes not counted)
    passes = eager.count("sad_fit_iteration") + eager.count("sad_propagate")
    want = 0
    for t in range(1, T + 1):
        if t in events:
            want += 1
        elif (t - 1) % U == 0:
            want += Q
    assert passes == want
    assert eager.count("sad_adam_step") + eager.count("sad_fit_iteration") == T
    assert eager.count("sad_refresh") == 1 + len(events)


def test_chunk_is_a_multiple_of_update_every(monkeypatch):
    for U in (1, 3, 5, 16, 20):
        _, info, _ = run(monkeypatch, fit.Schedule(iterations=64, events=(), update_every=U), graphs=True)
        assert info["chunk"] % U == 0 and info["chunk"] >= 16


def test_bad_schedule_is_rejected(monkeypatch):
    with pytest.raises(ValueError):
        run(monkeypatch, fit.Schedule(iterations=4, update_every=0), graphs=False)
    with pytest.raises(ValueError):
        run(monkeypatch, fit.Schedule(iterations=4, passes_per_update=0), graphs=False)
