"""Pins of the oracle's budget-control statistics and densify/prune step
("Soft Anisotropic Diagrams for Differentiable Image Representation",
summary B.4-B.5; reading notes, key design 4).

Independent checks: partition-of-unity sums, the removal delta against a
render with the site actually removed, second moments by brute force over
the oracle's softmax weights, and the densify decisions and split geometry
re-derived with numpy (argsort, eigh)."""
import math

import numpy as np

import synth

SENT = 0xFFFFFFFF


def _case(orc, H=14, W=18, N=24, seed=3, log10_tau=(0.8, 1.4)):
    st = synth.Stream(seed, "budget")
    prm = np.zeros((9, N))
    prm[0] = st.uniform(N, 0, W)
    prm[1] = st.uniform(N, 0, H)
    prm[2] = synth.LN10 * st.uniform(N, *log10_tau)
    prm[3] = st.uniform(N, 0, 2)
    prm[4:7] = st.uniform(3 * N).reshape(3, N)
    prm[7] = st.uniform(N, 0, math.pi)
    prm[8] = st.normal(N, 0, 0.6)
    prm = prm.astype(np.float32)
    tgt = synth.make_image(H, W, 3, 0, seed)
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    return H, W, prm, tgt, tab


def test_stats_partition_sums(orc):
    H, W, prm, tgt, tab = _case(orc)
    L, g, st = orc.loss_backward_stats(H, W, prm, tab, tgt)
    L2, g2 = orc.loss_backward(H, W, prm, tab, tgt)
    assert L == L2 and np.array_equal(g, g2)
    # sum_i w_i = 1 per pixel, so sum_i m_i = P and sum_i E_i = sum_x e(x) = P L
    np.testing.assert_allclose(st[0].sum(), H * W, rtol=1e-12)
    np.testing.assert_allclose(st[1].sum(), H * W * L, rtol=1e-12)


def test_removal_delta_equals_render_without_the_site(orc):
    H, W, prm, tgt, tab = _case(orc)
    _, _, st = orc.loss_backward_stats(H, W, prm, tab, tgt)
    base = orc.render(H, W, prm, tab)
    err = ((base - tgt) ** 2).sum(0).ravel()
    w = orc.weights(H, W, prm, tab)
    assert w.max() < 1 - 1e-6  # the renormalisation never hits the floor here
    for i in range(prm.shape[1]):
        has = (tab == i).any(1)
        if not has.any():
            assert st[5, i] == 0.0
            continue
        t2 = np.where(tab == i, SENT, tab).astype(np.uint32)
        img = orc.render(H, W, prm, t2)
        err2 = ((img - tgt) ** 2).sum(0).ravel()
        np.testing.assert_allclose(st[5, i], (err2 - err)[has].sum(), rtol=1e-9, atol=1e-12)


def test_second_moments_brute_force(orc):
    H, W, prm, tgt, tab = _case(orc, seed=5)
    _, _, st = orc.loss_backward_stats(H, W, prm, tab, tgt)
    w = orc.weights(H, W, prm, tab)
    img = orc.render(H, W, prm, tab)
    e = ((img - tgt) ** 2).sum(0).ravel()
    jj, ii = np.mgrid[0:H, 0:W]
    x = ii.ravel() + 0.5
    y = jj.ravel() + 0.5
    N = prm.shape[1]
    ref = np.zeros((5, N))
    for q in range(8):
        ids = tab[:, q].astype(np.int64)
        ok = ids < N
        i = ids[ok]
        dx = x[ok] - prm[0, i].astype(np.float64)
        dy = y[ok] - prm[1, i].astype(np.float64)
        we = w[ok, q] * e[ok]
        np.add.at(ref[0], i, w[ok, q])
        np.add.at(ref[1], i, we)
        np.add.at(ref[2], i, we * dx * dx)
        np.add.at(ref[3], i, we * dx * dy)
        np.add.at(ref[4], i, we * dy * dy)
    np.testing.assert_allclose(st[:5], ref, rtol=1e-10, atol=1e-12)


def test_densify_decisions_and_children(orc):
    H, W, N = 40, 56, 120
    tgt = synth.make_image(H, W, 6, 0, 8)
    prm = synth.uniform_sites(H, W, N, 8)
    prm[0, 100:] = -1.0                      # 20 free slots
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    _, _, st64 = orc.loss_backward_stats(H, W, prm, tab, tgt)
    st = st64.astype(np.float32)
    st[1, 7] = st[1].max() * 10              # selected for splitting, but
    st[2:5, 7] = 0.0                         # a zero second moment: fallback axis
    cfg = orc.densify_cfg(grow=6, prune_frac=0.05, alpha=0.5, eps=1e-6)
    m = np.full((9, N), 0.5, np.float32)
    v = np.full((9, N), 0.25, np.float32)
    P2, M2, V2, n_split, n_pruned = orc.densify_prune(H, W, prm, m, v, st, tgt, cfg)
    active = prm[0] >= 0
    n_active = int(active.sum())
    # 1. prune: the floor(0.05 n_active) smallest removal deltas (ties: id)
    assert n_pruned == int(0.05 * n_active)
    ids = np.nonzero(active)[0]
    order = ids[np.lexsort((ids, st[5, ids]))]
    pruned = set(order[:n_pruned].tolist())
    # 2. split: largest float32 score E / sqrt(max(m, eps)) among the rest
    rest = np.array(sorted(set(ids.tolist()) - pruned))
    score = st[1, rest] / np.sqrt(np.maximum(st[0, rest], np.float32(1e-6)))
    assert score.dtype == np.float32
    sel = rest[np.lexsort((rest, -score))][:n_split]
    free = np.array(sorted(set(np.nonzero(~active)[0].tolist()) | pruned))
    assert n_split == min(n_pruned + 6, free.size, rest.size)
    parents = np.sort(sel)
    kids = free[:n_split]
    # pruned slots that took no child stay inactive; untouched sites keep all
    untouched = sorted(set(range(N)) - set(parents.tolist()) - set(kids.tolist()))
    for i in untouched:
        if i in pruned:
            assert P2[0, i] == -1.0
        else:
            assert np.array_equal(P2[:, i], prm[:, i])
            assert np.array_equal(M2[:, i], m[:, i]) and np.array_equal(V2[:, i], v[:, i])
    # 3. children
    for a_id, b_id in zip(parents, kids):
        E = float(st[1, a_id])
        C = np.array([[st[2, a_id], st[3, a_id]], [st[3, a_id], st[4, a_id]]], np.float64) / max(E, 1e-300)
        lam, vec = np.linalg.eigh(C)
        if E > 0 and lam[1] > 0:
            e1 = vec[:, 1]
            if e1[0] < 0 or (e1[0] == 0 and e1[1] < 0):
                e1 = -e1
            d = 0.5 * math.sqrt(lam[1]) * e1
        else:
            th, a = float(prm[7, a_id]), float(prm[8, a_id])
            ax = np.array([-math.sin(th), math.cos(th)]) if a > 0 else np.array([math.cos(th), math.sin(th)])
            d = 0.5 * ax
        for dst, sg in ((a_id, 1.0), (b_id, -1.0)):
            want = np.clip(prm[:2, a_id].astype(np.float64) + sg * d, 0, [W - 1e-4, H - 1e-4])
            np.testing.assert_allclose(P2[:2, dst], want, rtol=0, atol=1e-4)
            px, py = int(np.floor(P2[0, dst])), int(np.floor(P2[1, dst]))
            np.testing.assert_array_equal(P2[4:7, dst], tgt[:, py, px])
            assert P2[3, dst] == np.float32(prm[3, a_id] * np.float32(0.85))
            assert P2[2, dst] == np.float32(prm[2, a_id] - np.float32(math.log(2)))
            assert P2[7, dst] == prm[7, a_id] and P2[8, dst] == prm[8, a_id]
            assert np.all(M2[:, dst] == 0) and np.all(V2[:, dst] == 0)
    assert 7 in parents  # the fallback axis was exercised
    assert int((P2[0] >= 0).sum()) == n_active - n_pruned + n_split


# --------------------------------------------------------------------------
# frozen sites (summary section 7) and tau diffusion (summary B.6)
# --------------------------------------------------------------------------

def test_adam_frozen_sites_untouched(orc):
    H, W, N = 20, 30, 40
    prm = synth.uniform_sites(H, W, N, 61).astype(np.float64)
    g = synth.random_gradients(N, 61).astype(np.float64)
    frozen = np.zeros(N, np.uint8)
    frozen[::3] = 1
    lr = [1e-3] * 9
    P1, M1, V1 = orc.adam(H, W, prm, np.zeros_like(prm), np.zeros_like(prm), g, lr, 1, frozen=frozen)
    P0, M0, V0 = orc.adam(H, W, prm, np.zeros_like(prm), np.zeros_like(prm), g, lr, 1)
    f = frozen.astype(bool)
    assert np.array_equal(P1[:, f], prm[:, f]) and np.all(M1[:, f] == 0) and np.all(V1[:, f] == 0)
    assert np.array_equal(P1[:, ~f], P0[:, ~f]) and np.array_equal(M1[:, ~f], M0[:, ~f])


def test_tau_diffusion_against_numpy(orc):
    H, W, prm, tgt, tab = _case(orc, seed=7)
    prm = prm.copy()
    prm[0, 4] = -1.0
    N = prm.shape[1]
    g = synth.random_gradients(N, 7).astype(np.float64)
    for lam in (0.0, 0.3, 1.0):
        out = orc.tau_diffuse(H, W, prm, tab, g, lam)
        ref = g.copy()
        for i in range(N):
            if prm[0, i] < 0:
                continue
            px, py = int(np.floor(prm[0, i])), int(np.floor(prm[1, i]))
            nb = [int(j) for j in tab[py * W + px] if j != SENT and j < N and j != i and prm[0, j] >= 0]
            if nb:
                ref[2, i] = (1 - lam) * g[2, i] + lam * np.mean(g[2, nb])
        np.testing.assert_allclose(out, ref, rtol=1e-15, atol=0)
        assert np.array_equal(np.delete(out, 2, 0), np.delete(g, 2, 0))  # only the ln tau plane moves
    # a constant gradient field is a fixed point
    gc = np.zeros_like(g)
    gc[2] = 0.25
    np.testing.assert_allclose(orc.tau_diffuse(H, W, prm, tab, gc, 0.7)[2], 0.25, rtol=1e-15)
