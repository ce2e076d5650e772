"""GPU parity of the refresh variants ("Soft Anisotropic Diagrams for
Differentiable Image Representation", summary B.3): the 3x3 JFA prepass,
bit-exact against the oracle's flood passes, and the pass on cached lists
(no propagation) used between candidate updates, against the oracle's
render + backward on the same lists.

Tolerances as in the main parity file: tables bit-exact, loss 1e-5
relative, render 1e-5 absolute, gradients 1e-4 relative with a 1e-6 floor."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

SENT = 0xFFFFFFFF
RENDER_ATOL = 1e-5
GRAD_RTOL, GRAD_ATOL = 1e-4, 1e-6
LOSS_RTOL = 1e-5


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _ctx(H, W, N, prm, tgt=None, seed=1):
    from soft_voronoi_render_b200 import Sad
    s = Sad(H, W, N, seed=seed)
    s.set_sites(prm)
    if tgt is not None:
        s.set_target(tgt)
    return s


def _assert_grads(g_gpu, g_orc, what=""):
    err = np.abs(g_gpu.astype(np.float64) - g_orc)
    tol = np.maximum(GRAD_RTOL * np.abs(g_orc), GRAD_ATOL)
    bad = err > tol
    assert not bad.any(), (what, int(bad.sum()), float((err / tol).max()))


@pytest.mark.parametrize("wl,H,W,N", [("c1", None, None, None), ("c2", None, None, None),
                                      ("c1", 37, 70, 400), ("c1", 1, 1, 1), ("c1", 5, 300, 40)])
def test_jfa_prepass_bit_exact(torch_cuda, wl, H, W, N):
    tgt, prm, w = synth.make_workload(wl, seed=3, H=H, W=W, N=N)
    H, W, N = tgt.shape[1], tgt.shape[2], prm.shape[1]
    prm = prm.copy()
    if N > 10:
        prm[0, ::10] = -1.0
    s = _ctx(H, W, N, prm, seed=17)
    s.jfa_prepass()
    ref = oracle.jfa_prepass(H, W, prm)
    got = s.get_table()
    np.testing.assert_array_equal(got, ref)
    assert np.all(got[:, 4:] == SENT)
    n = len(oracle.flood_schedule(H, W))
    assert s.stats()["pass_counter"] == n
    # ordinary propagation passes then fill the lists, counter-hashed
    # injections keyed on the pass counter
    s.propagate(1, 2)
    ref = oracle.propagate(H, W, oracle.records(H, W, prm), ref, 1, 2, seed=17, pass_index=n)
    np.testing.assert_array_equal(s.get_table(), ref)


@pytest.mark.parametrize("wl,H,W,N", [("c1", None, None, None), ("c2", None, None, None),
                                      ("c1", 37, 70, 400), ("c1", 8, 33, 50)])
def test_fit_pass_cached_matches_backward(torch_cuda, wl, H, W, N):
    tgt, prm, w = synth.make_workload(wl, seed=5, H=H, W=W, N=N)
    H, W, N = tgt.shape[1], tgt.shape[2], prm.shape[1]
    prm = prm.copy()
    prm[0, 3] = -1.0
    t0, _ = oracle.refresh(H, W, prm, 2, seed=8)
    t0 = t0.copy()
    t0[::5, 6] = t0[::5, 2]       # the same id twice in one list counts twice
    t0[::13, 7] = N + 4           # an id beyond capacity is dropped
    s = _ctx(H, W, N, prm, tgt, seed=8)
    s.set_table(t0)
    s.fit_pass_cached()
    np.testing.assert_array_equal(s.get_table(), t0)
    L, g, img = oracle.loss_backward(H, W, prm, t0, tgt, want_image=True)
    assert abs(s.loss() - L) <= LOSS_RTOL * L
    assert np.abs(s.image.cpu().numpy() - img).max() <= RENDER_ATOL
    _assert_grads(s.grads.cpu().numpy(), g, "cached")
    st = s.stats()
    assert st["pass_counter"] == 0 and st["current_table"] == 0
    assert st["dropped_ids"] == (H * W + 12) // 13
    # the standalone backward on the same lists agrees
    s.grads.zero_()
    s.backward()
    _assert_grads(s.grads.cpu().numpy(), g, "backward")


def test_fit_pass_cached_crowded_tiles(torch_cuda):
    """Random lists with far more than 128 distinct sites per tile: the
    cached pass takes the generic path and still matches the oracle."""
    H, W, N = 40, 70, 30000
    prm = synth.uniform_sites(H, W, N, 14)
    tgt = synth.make_image(H, W, 8, 0, 14)
    st = synth.Stream(14, "crowded-cached")
    t0 = st.integers(H * W * 8, N).astype(np.uint32).reshape(H * W, 8)
    t0[st.uniform(H * W * 8).reshape(H * W, 8) < 0.1] = SENT
    s = _ctx(H, W, N, prm, tgt, seed=3)
    s.set_table(t0)
    s.fit_pass_cached()
    L, g = oracle.loss_backward(H, W, prm, t0, tgt)
    assert abs(s.loss() - L) <= LOSS_RTOL * L
    _assert_grads(s.grads.cpu().numpy(), g, "crowded")
    assert s.stats()["hash_overflow"] > 0


def test_infrequent_updates_step_by_step(torch_cuda):
    """Propagating only every 3rd iteration (summary B.3): each iteration,
    checked against the oracle on the GPU's own state before it, gives the
    oracle's propagated table (or leaves the cached one alone) and its loss."""
    from soft_voronoi_render_b200 import _lib, adam_cfg
    H, W, N, G, U = 64, 96, 600, 2, 3
    tgt = synth.make_image(H, W, 8, 0, 41)
    prm = synth.gradient_sites(tgt, N, 41)
    s = _ctx(H, W, N, prm, tgt, seed=4)
    cfg = adam_cfg(lr_color=5e-3)
    s.refresh(G)
    npass = len(oracle.jump_schedule(H, W))
    for it in range(1, 8):
        P, T = s.get_sites(), s.get_table()
        if (it - 1) % U == 0:
            s.fit_pass(G)
            T = oracle.propagate(H, W, oracle.records(H, W, P), T, 1, G, seed=4, pass_index=npass)
            npass += 1
        else:
            s.fit_pass_cached()
        np.testing.assert_array_equal(s.get_table(), T)
        L, g = oracle.loss_backward(H, W, P, T, tgt)
        assert abs(s.loss() - L) <= LOSS_RTOL * L
        _assert_grads(s.grads.cpu().numpy(), g, f"iteration {it}")
        _lib.sad_adam_step(s.ctx, cfg, s.stream)
    assert s.stats()["pass_counter"] == npass


def test_infrequent_updates_schedule(torch_cuda):
    """fit.run with update_every = 4 and two passes per update against the
    oracle's schedule: the same propagation passes, and the same outcome
    within 0.2 dB PSNR.  The two agree step for step (previous test), but
    not along a whole fit: Adam's
    first steps divide gradients of order 1e-8 by |g| + eps, which turns
    float32 rounding into position differences of a few hundredths of a
    pixel that the following iterations carry on."""
    import math
    from soft_voronoi_render_b200 import fit
    H, W, N, G = 64, 96, 600, 2
    tgt = synth.make_image(H, W, 8, 0, 41)
    prm = synth.gradient_sites(tgt, N, 41)
    s = _ctx(H, W, N, prm, tgt, seed=4)
    sched = fit.Schedule(iterations=12, G=G, events=(), update_every=4, passes_per_update=2)
    fit.run(s, sched)
    lr = dict(pos=1e-3, log_tau=1e-3, r=1e-3, color=5e-3, theta=1e-3, a=1e-3)
    lr32 = {k: float(np.float32(x)) for k, x in lr.items()}
    _, L_orc, npass = oracle.fit(H, W, prm, tgt, N, 12, (), 0, 0.0, lr32, G, 4, update_every=4,
                                 passes_per_update=2)
    assert s.stats()["pass_counter"] == npass == len(oracle.jump_schedule(H, W)) + 6
    assert s.stats()["adam_step"] == 12
    psnr = lambda L: 10 * math.log10(3.0 / L)
    assert abs(psnr(s.loss()) - psnr(L_orc)) <= 0.2, (s.loss(), L_orc)


@pytest.mark.parametrize("H,W,N,cell", [(96, 128, 800, 2), (37, 70, 400, 3), (64, 64, 300, 4), (9, 33, 40, 8)])
def test_candidate_grid_parity(torch_cuda, H, W, N, cell):
    """Lists on a ceil(H/s) x ceil(W/s) grid scored at the cell centres
    (summary B.3): refresh, exact top-K, the JFA prepass and a fitting pass
    bit-exact on the grid; render, loss and gradients with every pixel using
    its cell's list; tau diffusion on the site's cell list."""
    tgt, prm, _ = synth.make_workload("c1", seed=7, H=H, W=W, N=N)
    prm = prm.copy()
    prm[0, 4] = -1.0
    G = 2
    s = _ctx(H, W, N, prm, tgt, seed=31)
    s.set_candidate_grid(cell)
    GH, GW = oracle.grid_dims(H, W, cell)
    assert s.get_table().shape == (GH * GW, 8) and np.all(s.get_table() == SENT)
    rec = oracle.records(H, W, prm)
    s.refresh(G)
    t0, npass = oracle.refresh(H, W, prm, G, seed=31, cell=cell)
    np.testing.assert_array_equal(s.get_table(), t0)
    ex = s.topk_exact().cpu().numpy().view(np.uint32)
    np.testing.assert_array_equal(ex, oracle.topk_exact(H, W, rec, cell=cell))
    # one fitting pass: propagation on the grid, backward per pixel
    s.fit_pass(G)
    t1 = oracle.propagate(H, W, rec, t0, 1, G, seed=31, pass_index=npass, cell=cell)
    np.testing.assert_array_equal(s.get_table(), t1)
    L, g, img = oracle.loss_backward(H, W, prm, oracle.expand_table(H, W, t1, cell), tgt, want_image=True)
    assert abs(s.loss() - L) <= LOSS_RTOL * L
    assert np.abs(s.image.cpu().numpy() - img).max() <= RENDER_ATOL
    _assert_grads(s.grads.cpu().numpy(), g, "grid fit pass")
    # the cached pass on the grid and tau diffusion on the site's cell list
    s.grads.zero_()
    s.fit_pass_cached()
    _assert_grads(s.grads.cpu().numpy(), g, "grid cached pass")
    gr = synth.random_gradients(N, 8)
    s.grads.copy_(torch_cuda.from_numpy(gr))
    s.tau_diffuse(0.5)
    ref = oracle.tau_diffuse(H, W, prm, oracle.expand_table(H, W, t1, cell), gr.astype(np.float64), 0.5)
    np.testing.assert_allclose(s.grads.cpu().numpy().astype(np.float64), ref, rtol=1e-6, atol=1e-12)
    # the prepass on the grid
    s.jfa_prepass()
    np.testing.assert_array_equal(s.get_table(), oracle.jfa_prepass(H, W, prm, cell=cell))
    # back to the pixel grid
    s.set_candidate_grid(1)
    s.refresh(G)
    assert s.get_table().shape == (H * W, 8)


@pytest.mark.parametrize("U", [1, 4])
def test_fit_graph_replay_matches_eager(torch_cuda, U):
    """fit.run replaying captured CUDA graphs of 16 iterations gives what the
    eager schedule gives.  With zero learning rates every step is
    deterministic (integer list decisions on fixed records, a fixed-order
    loss sum), so lists, counters and loss must agree exactly."""
    from soft_voronoi_render_b200 import fit
    H, W, N = 64, 96, 600
    tgt = synth.make_image(H, W, 8, 0, 43)
    prm = synth.gradient_sites(tgt, N, 43)
    zero = dict(lr_pos=0.0, lr_log_tau=0.0, lr_r=0.0, lr_color=0.0, lr_theta=0.0, lr_a=0.0)
    out = {}
    for graphs in (True, False):
        s = _ctx(H, W, N, prm, tgt, seed=6)
        sched = fit.Schedule(iterations=40, G=2, events=(), update_every=U, lr=zero)
        info = fit.run(s, sched, graphs=graphs)
        st = s.stats()
        out[graphs] = (info, s.get_table(), st["pass_counter"], st["adam_step"], s.loss())
    (gi, gt, gp, ga, gl), (ei, et, ep, ea, el) = out[True], out[False]
    assert gi["graph_replays"] == 2 and gi["eager_iterations"] == 8 and ei["graph_replays"] == 0
    np.testing.assert_array_equal(gt, et)
    assert (gp, ga, gl) == (ep, ea, el) and ga == 40


def test_fit_graph_replay_with_an_event(torch_cuda):
    """With a densify event between the replays the device counters still
    advance exactly as in the eager schedule (the loss is not compared:
    float32 atomics order the statistics differently from run to run, which
    can flip near-tied densify selections)."""
    from soft_voronoi_render_b200 import fit
    H, W, N, N_cap = 64, 96, 600, 900
    tgt = synth.make_image(H, W, 8, 0, 43)
    prm = synth.gradient_sites(tgt, N, 43)
    out = {}
    for graphs in (True, False):
        s = _ctx(H, W, N_cap, prm, tgt, seed=6)
        sched = fit.Schedule(iterations=60, G=2, events=(30,), grow=100, prune_frac=0.01)
        info = fit.run(s, sched, graphs=graphs)
        st = s.stats()
        out[graphs] = (info, st["pass_counter"], st["adam_step"], st["n_active"], s.loss())
    (gi, gp, ga, gn, gl), (ei, ep, ea, en, el) = out[True], out[False]
    assert gi["graph_replays"] == 2 and gi["eager_iterations"] == 27 and ei["graph_replays"] == 0
    assert (gp, ga, gn) == (ep, ea, en) and ga == 60 and gn == 600  # active before the event
    assert np.isfinite(gl) and np.isfinite(el)
