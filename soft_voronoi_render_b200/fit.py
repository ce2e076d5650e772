"""Host-side fitting schedule: every step is a C-ABI call on the device.

A fit starts with a full candidate refresh, then runs fitting iterations.
An iteration that precedes a budget-control event accumulates the
statistics (propagate, backward with SAD_STATS, Adam), runs the
densify/prune event and refreshes the candidate lists; every other
iteration is one sad_fit_iteration (fused pass + Adam).  With
``update_every`` = U > 1 the lists are propagated only on iterations 1,
1 + U, 1 + 2U, ... (and event iterations); in between the pass renders and
differentiates the cached lists (sad_fit_pass_cached), the infrequent
candidate update of the pages' section B.3; ``passes_per_update`` jump-1
passes run at each such update (the last one fused with the render).  The
site count stays on the device.
"""
from __future__ import annotations

from dataclasses import dataclass, field

from . import _lib


@dataclass
class Schedule:
    iterations: int = 2000
    G: int = 2
    events: tuple = field(default_factory=lambda: tuple(range(100, 1601, 100)))
    grow: int = 2500
    prune_frac: float = 0.005
    update_every: int = 1
    passes_per_update: int = 1
    lr: dict = field(default_factory=lambda: dict(lr_pos=1e-3, lr_log_tau=1e-3, lr_r=1e-3, lr_color=5e-3,
                                                  lr_theta=1e-3, lr_a=1e-3))


def _iteration(ctx, sched: Schedule, cfg, st, update: bool) -> None:
    if update:
        for _ in range(sched.passes_per_update - 1):
            _lib.sad_propagate(ctx, 1, sched.G, st)
        _lib.sad_fit_iteration(ctx, sched.G, cfg, st)
    else:
        _lib.sad_fit_pass_cached(ctx, st)
        _lib.sad_adam_step(ctx, cfg, st)


def run(sad, sched: Schedule, on_event=None, graphs: bool = True) -> dict:
    """Fit the bound target with the context's sites (``sad`` is a ``Sad``).

    With ``graphs`` the plain iterations between events run as replays of
    one captured CUDA graph of ``chunk`` iterations (a multiple of
    update_every, at least 16), which starts on an update iteration; the
    device-resident counters make every replay advance the schedule.
    Returns how many iterations ran eagerly and how many graph replays ran.
    """
    ctx, st = sad.ctx, sad.stream
    cfg = _lib.adam_cfg(**sched.lr)
    dcfg = _lib.densify_cfg(grow=sched.grow, prune_frac=sched.prune_frac)
    events = set(sched.events)
    U = sched.update_every
    if U < 1 or sched.passes_per_update < 1:
        raise ValueError("update_every and passes_per_update must be >= 1")
    chunk = U * -(-16 // U)
    graph = None
    eager = replays = 0
    _lib.sad_refresh(ctx, sched.G, st)
    it = 1
    while it <= sched.iterations:
        if it in events:
            _lib.sad_propagate(ctx, 1, sched.G, st)
            _lib.sad_backward(ctx, _lib.SAD_STATS, st)
            _lib.sad_adam_step(ctx, cfg, st)
            _lib.sad_densify_prune(ctx, dcfg, st)
            _lib.sad_refresh(ctx, sched.G, st)
            if on_event is not None:
                on_event(it)
            it += 1
            continue
        last = it + chunk - 1
        if (graphs and (it - 1) % U == 0 and last <= sched.iterations
                and not any(e in events for e in range(it, last + 1))):
            if graph is None:
                torch = sad.torch
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    gst = torch.cuda.current_stream()
                    for q in range(chunk):
                        _iteration(ctx, sched, cfg, gst, q % U == 0)
            graph.replay()
            replays += 1
            it += chunk
            continue
        _iteration(ctx, sched, cfg, st, (it - 1) % U == 0)
        eager += 1
        it += 1
    return {"eager_iterations": eager, "graph_replays": replays, "chunk": chunk}
