"""Pins of the oracle's downscaled candidate grid ("Soft Anisotropic Diagrams
for Differentiable Image Representation", summary B.3 "Candidate field"):
lists on a ceil(W/s) x ceil(H/s) grid, integer cell mapping, candidates
scored at the centres of their cells.

Independent checks: exact top-K at the cell centres against scipy's k-d
tree; one propagation pass against a numpy restatement scored at the cell
centres; the seed pass and the pixel-to-cell expansion against direct
indexing; cell = 1 against the pixel-grid functions."""
import numpy as np
import pytest
from scipy.spatial import cKDTree

import synth
from test_oracle_pins import SENT, _params


def _centres(GH, GW, cell):
    jj, ii = np.mgrid[0:GH, 0:GW]
    return np.stack([(ii.ravel() + 0.5) * cell, (jj.ravel() + 0.5) * cell], 1).astype(np.float64)


def test_grid_dims_and_expansion(orc):
    assert orc.grid_dims(37, 50, 4) == (10, 13)
    assert orc.grid_dims(32, 32, 8) == (4, 4)
    assert orc.grid_dims(5, 7, 1) == (5, 7)
    H, W, c = 9, 11, 4
    GH, GW = orc.grid_dims(H, W, c)
    t = np.arange(GH * GW * 8, dtype=np.uint32).reshape(GH * GW, 8)
    e = orc.expand_table(H, W, t, c)
    assert e.shape == (H * W, 8)
    for (x, y) in ((0, 0), (3, 3), (4, 3), (10, 8), (7, 4)):
        np.testing.assert_array_equal(e[y * W + x], t[(y // c) * GW + x // c])
    t1 = np.arange(H * W * 8, dtype=np.uint32).reshape(H * W, 8)
    np.testing.assert_array_equal(orc.expand_table(H, W, t1, 1), t1)


def test_grid_topk_euclidean_is_knn_at_cell_centres(orc):
    """a = 0, r = 0, uniform tau: a cell's exact top-8 are the 8 Euclidean
    nearest sites to its centre (not to its corner)."""
    H, W, N, c = 37, 50, 200, 4
    prm = _params(N, H, W, 91)
    rec = orc.records(H, W, prm)
    tab = orc.topk_exact(H, W, rec, cell=c)
    GH, GW = orc.grid_dims(H, W, c)
    assert tab.shape == (GH * GW, 8)
    P = np.stack([prm[0], prm[1]], 1).astype(np.float64)
    _, nn = cKDTree(P).query(_centres(GH, GW, c), k=8)
    assert np.mean(np.all(tab.astype(np.int64) == nn, axis=1)) > 0.99
    # the corner-evaluated answer differs on many cells: the centring matters
    _, nn_corner = cKDTree(P).query(_centres(GH, GW, c) - 0.5 * c, k=1)
    assert np.mean(tab[:, 0].astype(np.int64) != nn_corner) > 0.1
    # cell = 1 is the pixel grid
    np.testing.assert_array_equal(orc.topk_exact(H, W, rec, cell=1), orc.topk_exact(H, W, rec))


def _union_top8_cells(orc, H, W, c, rec, tin, jump, G, seed, pas):
    """One pass restated on the cell grid: union of the own and the four
    jump-k neighbour lists plus the injections keyed on the cell index,
    scored at the cell centre, selected by a lexicographic sort."""
    GH, GW = orc.grid_dims(H, W, c)
    N = rec.shape[0]
    out = np.full((GH * GW, 8), SENT, dtype=np.uint32)
    for j in range(GH):
        for i in range(GW):
            p = j * GW + i
            cand = [tin[p]]
            for (ni, nj) in ((i - jump, j), (i + jump, j), (i, j - jump), (i, j + jump)):
                if 0 <= ni < GW and 0 <= nj < GH:
                    cand.append(tin[nj * GW + ni])
            if G > 0:
                cand.append(orc.inject_ids(seed, pas, p, N, G))
            ids = np.unique(np.concatenate(cand).astype(np.int64))
            ids = ids[(ids != SENT) & (ids < N)]
            ids = ids[rec[ids, 0] >= 0]
            fx, fy = (i + 0.5) * c, (j + 0.5) * c
            sc = np.array([orc.score32_at(rec, int(q), fx, fy) for q in ids], dtype=np.float64)
            keep = ~np.isnan(sc)
            ids, sc = ids[keep], sc[keep]
            order = np.lexsort((ids, -sc))[:8]
            out[p, :order.size] = ids[order]
    return out


@pytest.mark.parametrize("c,jump,G", [(2, 1, 0), (3, 1, 2), (4, 2, 3)])
def test_grid_propagate_equals_union_top8(orc, c, jump, G):
    H, W, N = 29, 34, 70
    prm = _params(N, H, W, 93 + c, a_sd=0.8, r_max=4, log10_tau=(1.5, 3))
    prm[0, 5] = -1.0
    rec = orc.records(H, W, prm)
    GH, GW = orc.grid_dims(H, W, c)
    st = synth.Stream(c * 100 + jump, "grid-tables")
    tin = st.integers(GH * GW * 8, N + 6).astype(np.uint32).reshape(GH * GW, 8)
    tin[st.uniform(GH * GW * 8).reshape(GH * GW, 8) < 0.2] = SENT
    got = orc.propagate(H, W, rec, tin, jump, G, seed=12, pass_index=3, cell=c)
    np.testing.assert_array_equal(got, _union_top8_cells(orc, H, W, c, rec, tin, jump, G, 12, 3))


def test_grid_seed_pass(orc):
    H, W, N, c = 19, 26, 90, 4
    prm = _params(N, H, W, 95)
    prm[0, 2] = -1.0
    t = orc.seed_table(H, W, prm, cell=c)
    GH, GW = orc.grid_dims(H, W, c)
    assert t.shape == (GH * GW, 8) and np.all(t[:, 1:] == SENT)
    ref = np.full(GH * GW, SENT, dtype=np.uint32)
    for i in range(N - 1, -1, -1):
        if prm[0, i] >= 0:
            ref[(int(np.floor(prm[1, i])) // c) * GW + int(np.floor(prm[0, i])) // c] = i
    np.testing.assert_array_equal(t[:, 0], ref)


def test_grid_refresh_then_passes_reach_exact(orc):
    """Refresh plus jump-1 passes on a cell grid converge to the exact top-8
    at the cell centres on almost every cell, and the prepass works on the
    grid too."""
    H, W, N, c = 48, 64, 150, 2
    prm = _params(N, H, W, 97, a_sd=0.5, r_max=2, log10_tau=(1.5, 2.5))
    rec = orc.records(H, W, prm)
    t, n = orc.refresh(H, W, prm, 2, seed=5, cell=c)
    assert n == len(orc.jump_schedule(*orc.grid_dims(H, W, c)))
    for q in range(6):
        t = orc.propagate(H, W, rec, t, 1, 2, seed=5, pass_index=n + q, cell=c)
    ex = orc.topk_exact(H, W, rec, cell=c)
    assert np.mean(np.all(t == ex, axis=1)) > 0.95
    tj = orc.jfa_prepass(H, W, prm, cell=c)
    assert tj.shape == ex.shape and np.all(tj[:, 4:] == SENT)
    assert np.mean(tj[:, 0] == ex[:, 0]) > 0.9
