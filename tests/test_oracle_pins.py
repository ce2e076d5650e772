"""Pins of the CPU oracle against what the pages and mathematics fix.

Every check here is independent of the oracle's own formulas: closed forms,
library routines (scipy distances and softmax, torch.optim.Adam, numpy
eigendecomposition), invariants stated on the pages, published test vectors,
brute force on tiny inputs, and central finite differences.

Page references (by title and section):
  [P1] "Soft Anisotropic Diagrams for Differentiable Image Representation"
       (paperlayer summary), sections 3, 4, B.2-B.4.
  [P2] reading notes on the paper, key designs 1-4.
  [P4] "SAD: Soft Anisotropic Diagrams" project page, Method.
  [P5] Chinese news article on SAD, section 3 (propagation accuracy).
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
from scipy.spatial import cKDTree
from scipy.spatial.distance import cdist

import synth

SENT = 0xFFFFFFFF
HERE = os.path.dirname(os.path.abspath(__file__))


def _grid(H, W):
    jj, ii = np.mgrid[0:H, 0:W]
    return np.stack([ii.ravel() + 0.5, jj.ravel() + 0.5], axis=1)


def _params(N, H, W, seed, *, a_sd=0.0, r_max=0.0, log10_tau=(3.0, 3.0)):
    st = synth.Stream(seed, "pins")
    prm = np.zeros((9, N))
    prm[0] = st.uniform(N, 0, W)
    prm[1] = st.uniform(N, 0, H)
    prm[2] = synth.LN10 * st.uniform(N, *log10_tau)
    prm[3] = st.uniform(N, 0, r_max) if r_max > 0 else 0.0
    prm[4:7] = st.uniform(3 * N).reshape(3, N)
    prm[7] = st.uniform(N, 0, math.pi)
    prm[8] = st.normal(N, 0, a_sd) if a_sd > 0 else 0.0
    return prm.astype(np.float32)


def _check_valid_topk(table, ref_score, tol):
    """table (P, 8) must be a top-8 of each row of ref_score (P, N), ranked by
    descending score, up to near-ties within tol."""
    P, N = ref_score.shape
    n_valid = min(8, N)
    assert np.all(table[:, :n_valid] != SENT)
    assert np.all(table[:, n_valid:] == SENT)
    ids = table[:, :n_valid].astype(np.int64)
    for row in ids:
        assert len(set(row.tolist())) == n_valid
    sel = np.take_along_axis(ref_score, ids, axis=1)
    assert np.all(sel[:, :-1] >= sel[:, 1:] - tol), "slots out of order"
    mask = np.ones_like(ref_score, dtype=bool)
    np.put_along_axis(mask, ids, False, axis=1)
    if N > n_valid:
        best_out = np.where(mask, ref_score, -np.inf).max(axis=1)
        assert np.all(sel[:, -1] >= best_out - tol), "a better site was left out"


# --------------------------------------------------------------------------
# metric and records ([P2] key design 1; [P1] section 4 "det(G_i) = 1")
# --------------------------------------------------------------------------

def test_records_metric_det_one_and_eigenframe(orc):
    H, W, N = 64, 48, 200
    prm = _params(N, H, W, 3, a_sd=0.8, r_max=4.0, log10_tau=(2, 4))
    r32, r64 = orc.records(H, W, prm, with64=True)
    s = 1.0 / max(H, W)
    tau = np.exp(prm[2].astype(np.float64))
    k = tau * s
    np.testing.assert_allclose(r64[:, 6], k, rtol=1e-14)
    np.testing.assert_allclose(r64[:, 5], k * prm[3], rtol=1e-14)
    # G' = k^2 G with det G = 1  =>  A C - B^2 = k^4
    A, B, C = r64[:, 2], r64[:, 3], r64[:, 4]
    np.testing.assert_allclose((A * C - B * B) / k ** 4, 1.0, rtol=1e-12)
    # eigenvalues e^{+a}, e^{-a}; the e^{+a} eigenvector is (cos theta, sin theta)
    for i in range(N):
        G = np.array([[A[i], B[i]], [B[i], C[i]]]) / k[i] ** 2
        ev, vec = np.linalg.eigh(G)
        a = float(prm[8, i])
        np.testing.assert_allclose(sorted(ev), sorted([math.exp(a), math.exp(-a)]), rtol=1e-12)
        big = vec[:, np.argmin(np.abs(ev - math.exp(a)))]
        u = np.array([math.cos(prm[7, i]), math.sin(prm[7, i])])
        if abs(a) > 1e-3:
            assert abs(abs(big @ u) - 1.0) < 1e-9
    # float32 records are the double records rounded once
    assert np.array_equal(r32, r64.astype(np.float32))
    # det-1 survives float32 rounding to float32 accuracy
    A32, B32, C32 = (r32[:, q].astype(np.float64) for q in (2, 3, 4))
    assert np.all(np.abs((A32 * C32 - B32 * B32) / k ** 4 - 1.0) < 2e-5)


def test_inactive_site_records(orc):
    prm = _params(4, 8, 8, 1)
    prm[0, 1] = -1.0
    prm[0, 2] = np.nan
    r32 = orc.records(8, 8, prm)
    assert r32[1, 0] < 0 and r32[2, 0] < 0 and r32[0, 0] >= 0
    tab = orc.topk_exact(8, 8, r32)
    assert not np.isin(tab, [1, 2]).any()


# --------------------------------------------------------------------------
# exact top-K: the special cases of [P1] section 3 reduce to textbook routines
# --------------------------------------------------------------------------

def test_topk_euclidean_special_case_is_knn(orc):
    """a = 0, r = 0, uniform tau: top-8 = the 8 Euclidean nearest sites."""
    H, W, N = 40, 56, 300
    prm = _params(N, H, W, 11)
    rec = orc.records(H, W, prm)
    tab = orc.topk_exact(H, W, rec)
    X = _grid(H, W)
    P = np.stack([prm[0], prm[1]], 1).astype(np.float64)
    d, nn = cKDTree(P).query(X, k=8)
    same = np.all(tab.astype(np.int64) == nn, axis=1)
    assert same.mean() > 0.999
    _check_valid_topk(tab, -cdist(X, P), tol=1e-4)


def test_topk_apollonius_special_case(orc):
    """a = 0, r != 0, uniform tau: ranking by ||x - p|| - r (Apollonius)."""
    H, W, N = 32, 32, 120
    prm = _params(N, H, W, 12, r_max=5.0)
    rec = orc.records(H, W, prm)
    tab = orc.topk_exact(H, W, rec)
    X = _grid(H, W)
    P = np.stack([prm[0], prm[1]], 1).astype(np.float64)
    ref = -(cdist(X, P) - prm[3].astype(np.float64)[None, :])
    _check_valid_topk(tab, ref, tol=1e-4)
    assert np.mean(tab[:, 0] == np.argmax(ref, axis=1)) > 0.999


def test_topk_anisotropic_special_case(orc):
    """r = 0, uniform tau: ranking by the per-site Mahalanobis-type norm."""
    H, W, N = 24, 24, 48
    prm = _params(N, H, W, 13, a_sd=0.9)
    rec = orc.records(H, W, prm)
    tab = orc.topk_exact(H, W, rec)
    X = _grid(H, W)
    ref = np.empty((H * W, N))
    for i in range(N):
        a, th = float(prm[8, i]), float(prm[7, i])
        R = np.array([[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]])
        G = R @ np.diag([math.exp(a), math.exp(-a)]) @ R.T
        ref[:, i] = -cdist(X, prm[0:2, i:i + 1].T.astype(np.float64), "mahalanobis", VI=G)[:, 0]
    _check_valid_topk(tab, ref, tol=1e-4)


def test_topk_temperature_weighting(orc):
    """a = 0, r = 0, varying tau: ranking by tau_i ||x - p_i|| (the logit is
    -tau_i s n_i, so hotter sites lose faster with distance)."""
    H, W, N = 30, 20, 80
    prm = _params(N, H, W, 14, log10_tau=(1.0, 3.0))
    rec = orc.records(H, W, prm)
    tab = orc.topk_exact(H, W, rec)
    X = _grid(H, W)
    P = np.stack([prm[0], prm[1]], 1).astype(np.float64)
    ref = -cdist(X, P) * np.exp(prm[2].astype(np.float64))[None, :] / max(H, W)
    _check_valid_topk(tab, ref, tol=1e-4)


def test_topk_ties_break_by_smaller_id(orc):
    H, W = 4, 4
    prm = _params(3, H, W, 15)
    prm[:, 2] = prm[:, 0]  # site 2 duplicates site 0 exactly
    rec = orc.records(H, W, prm)
    tab = orc.topk_exact(H, W, rec)
    for row in tab:
        ids = row[:3].tolist()
        assert ids.index(0) < ids.index(2)
        assert abs(ids.index(0) - ids.index(2)) == 1
    assert np.all(tab[:, 3:] == SENT)


# --------------------------------------------------------------------------
# render: partition of unity and closed forms ([P2] key design 2, [P4])
# --------------------------------------------------------------------------

def _full_logits(prm, H, W):
    """l_i(x) = -tau_i (s n_i(x) - s r_i) with n_i from scipy's Mahalanobis."""
    X = _grid(H, W)
    N = prm.shape[1]
    s = 1.0 / max(H, W)
    out = np.empty((H * W, N))
    for i in range(N):
        a, th = float(prm[8, i]), float(prm[7, i])
        R = np.array([[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]])
        G = R @ np.diag([math.exp(a), math.exp(-a)]) @ R.T
        n = cdist(X, prm[0:2, i:i + 1].T.astype(np.float64), "mahalanobis", VI=G)[:, 0]
        out[:, i] = -math.exp(float(prm[2, i])) * (s * n - s * float(prm[3, i]))
    return out


def test_render_partition_of_unity(orc):
    H, W, N = 32, 40, 90
    prm = _params(N, H, W, 21, a_sd=0.7, r_max=4, log10_tau=(1, 3))
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    prm[4:7] = 1.0
    img = orc.render(H, W, prm, tab)
    np.testing.assert_allclose(img, 1.0, atol=1e-12)
    w = orc.weights(H, W, prm, tab)
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-12)
    assert np.all(w >= 0)


def test_render_single_site_is_its_colour(orc):
    H, W = 12, 9
    prm = _params(1, H, W, 22, a_sd=1.0, r_max=3, log10_tau=(1, 3))
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    img = orc.render(H, W, prm, tab)
    for ch in range(3):
        np.testing.assert_allclose(img[ch], prm[4 + ch, 0], atol=0, rtol=1e-15)


def test_render_two_sites_logistic(orc):
    """Two sites, uniform tau: w_0 = sigmoid(tau s ((n_1 - r_1) - (n_0 - r_0)))."""
    H, W = 16, 16
    prm = _params(2, H, W, 23, r_max=3.0, log10_tau=(1.5, 1.5))
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    img = orc.render(H, W, prm, tab)
    X = _grid(H, W)
    P = np.stack([prm[0], prm[1]], 1).astype(np.float64)
    d = cdist(X, P) - prm[3].astype(np.float64)[None, :]
    tau = math.exp(float(prm[2, 0]))
    w0 = scipy.special.expit(tau / 16.0 * (d[:, 1] - d[:, 0]))
    for ch in range(3):
        ref = w0 * prm[4 + ch, 0] + (1 - w0) * prm[4 + ch, 1]
        np.testing.assert_allclose(img[ch].ravel(), ref, atol=1e-13)


def test_render_k_covers_all_sites_equals_full_softmax(orc):
    H, W, N = 20, 14, 7
    prm = _params(N, H, W, 24, a_sd=0.8, r_max=4, log10_tau=(1, 2.5))
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    img = orc.render(H, W, prm, tab)
    w = scipy.special.softmax(_full_logits(prm, H, W), axis=1)
    ref = w @ prm[4:7].T.astype(np.float64)
    for ch in range(3):
        np.testing.assert_allclose(img[ch].ravel(), ref[:, ch], atol=1e-12)


def test_render_large_tau_is_hard_apollonius(orc):
    """Large tau reproduces the hard arg-min ownership ([P1] section 3)."""
    H, W, N = 40, 40, 30
    prm = _params(N, H, W, 25, r_max=4.0, log10_tau=(6, 6))
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    img = orc.render(H, W, prm, tab)
    X = _grid(H, W)
    d = cdist(X, np.stack([prm[0], prm[1]], 1).astype(np.float64)) - prm[3].astype(np.float64)
    srt = np.sort(d, axis=1)
    margin = srt[:, 1] - srt[:, 0]
    tau_s = 1e6 / max(H, W)
    far = tau_s * margin >= 30
    assert far.mean() > 0.9
    own = np.argmin(d, axis=1)
    for ch in range(3):
        np.testing.assert_allclose(img[ch].ravel()[far], prm[4 + ch, own[far]], atol=1e-6)


def test_render_shift_invariance(orc):
    """Adding the same offset to every radius under uniform tau shifts all
    logits equally; max-subtracted softmax weights are unchanged ([P1] B.4)."""
    H, W, N = 24, 24, 60
    prm = _params(N, H, W, 26, a_sd=0.5, r_max=3, log10_tau=(2, 2))
    prm[3] = np.round(prm[3] * 1024) / 1024   # so that r + 8 is exact in float32
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    img0 = orc.render(H, W, prm, tab)
    prm2 = prm.copy()
    prm2[3] += np.float32(8.0)
    img1 = orc.render(H, W, prm2, tab)
    np.testing.assert_allclose(img0, img1, atol=1e-12)


def test_render_skips_invalid_slots(orc):
    H, W, N = 8, 8, 10
    prm = _params(N, H, W, 27)
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    bad = tab.copy()
    bad[:, 7] = 5000           # out-of-range id
    bad[0, :] = SENT           # empty pixel
    prm2 = prm.copy()
    img = orc.render(H, W, prm2, bad)
    assert np.all(img[:, 0, 0] == 0.0)
    ref = orc.render(H, W, prm2, np.where(np.arange(8) == 7, SENT, tab))
    np.testing.assert_allclose(img[:, 1:, :], ref[:, 1:, :], atol=0)


# --------------------------------------------------------------------------
# loss and analytic backward ([P1] B.4, [P2] key design 4)
# --------------------------------------------------------------------------

def test_loss_is_per_pixel_normalised_mse(orc):
    H, W, N = 16, 20, 30
    prm = _params(N, H, W, 31, a_sd=0.5, r_max=2, log10_tau=(1, 2))
    tgt = synth.make_image(H, W, 3, 0, 5)
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    L, _, img = orc.loss_backward(H, W, prm, tab, tgt, want_image=True)
    np.testing.assert_allclose(L, np.sum((img - tgt) ** 2) / (H * W), rtol=1e-13)
    np.testing.assert_allclose(img, orc.render(H, W, prm, tab), atol=0)


def _fd_grad(orc, H, W, prm, tab, tgt, plane, site, h):
    def loss_at(delta):
        p2 = prm.copy()
        p2[plane, site] = np.float32(prm[plane, site] + delta)
        assert float(p2[plane, site]) - float(prm[plane, site]) == delta
        return orc.loss_backward(H, W, p2, tab, tgt)[0]

    def D(hh):
        return (loss_at(hh) - loss_at(-hh)) / (2 * hh)

    return (4 * D(h / 2) - D(h)) / 3  # Richardson extrapolation


@pytest.mark.parametrize("seed", [41, 42])
def test_backward_matches_central_differences(orc, seed):
    H, W, N = 16, 16, 24
    prm = _params(N, H, W, seed, a_sd=0.7, r_max=3, log10_tau=(0.8, 1.6))
    tgt = synth.make_image(H, W, 4, 0, seed)
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    _, g = orc.loss_backward(H, W, prm, tab, tgt)
    h = 2.0 ** -11
    checked = 0
    for site in range(0, N, 3):
        for plane in range(9):
            fd = _fd_grad(orc, H, W, prm, tab, tgt, plane, site, h)
            an = g[plane, site]
            assert abs(fd - an) <= 1e-6 * max(abs(an), 1e-4) + 1e-11, (plane, site, fd, an)
            checked += 1
    assert checked == 8 * 9


def test_backward_no_nan_at_site_centre(orc):
    H, W = 8, 8
    prm = _params(3, H, W, 43, a_sd=0.5, r_max=1, log10_tau=(1, 1.5))
    prm[0, 0], prm[1, 0] = 3.5, 4.5   # exactly on a pixel centre
    tgt = synth.make_image(H, W, 1, 0, 1)
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    L, g = orc.loss_backward(H, W, prm, tab, tgt)
    assert np.isfinite(L) and np.all(np.isfinite(g))


def test_inactive_sites_get_no_gradient(orc):
    H, W, N = 12, 12, 20
    prm = _params(N, H, W, 44, a_sd=0.5, r_max=2, log10_tau=(1, 2))
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    prm2 = prm.copy()
    prm2[0, 5] = -1.0
    tgt = synth.make_image(H, W, 2, 0, 2)
    _, g = orc.loss_backward(H, W, prm2, tab, tgt)
    assert np.all(g[:, 5] == 0.0)


# --------------------------------------------------------------------------
# Adam ([P2] key design 4) against torch.optim.Adam
# --------------------------------------------------------------------------

def test_adam_matches_torch_adam(orc):
    import torch
    H, W, N = 64, 32, 50
    s = 1.0 / max(H, W)
    prm = _params(N, H, W, 51, a_sd=0.5, r_max=3, log10_tau=(2, 4)).astype(np.float64)
    prm[0, 7] = -1.0  # inactive: untouched
    lr = {"pos": 1e-3, "log_tau": 2e-3, "r": 3e-3, "color": 5e-3, "theta": 4e-3, "a": 6e-3}
    lrv = np.array([lr[g] for g in orc.ADAM_PLANE_GROUP])
    sig = np.ones(9)
    sig[[0, 1, 3]] = 1.0 / s
    # torch reference on the scaled variables z = param / sigma
    z = torch.tensor(prm / sig[:, None], dtype=torch.float64)
    rows = [torch.nn.Parameter(z[j].clone()) for j in range(9)]
    opt = torch.optim.Adam([{"params": [rows[j]], "lr": float(lrv[j])} for j in range(9)],
                           betas=(0.9, 0.999), eps=1e-8)
    P, M, V = prm.copy(), np.zeros_like(prm), np.zeros_like(prm)
    active = prm[0] >= 0
    for t in range(1, 4):
        g = synth.random_gradients(N, 100 + t).astype(np.float64)
        P, M, V = orc.adam(H, W, P, M, V, g, lr, t)
        for j in range(9):
            gj = torch.tensor(g[j] * sig[j])
            gj[~torch.tensor(active)] = 0.0
            rows[j].grad = gj
        opt.step()
        with torch.no_grad():  # the step keeps positions inside the image
            rows[0].clamp_(0.0, float(np.nextafter(np.float32(W), np.float32(0))) / sig[0])
            rows[1].clamp_(0.0, float(np.nextafter(np.float32(H), np.float32(0))) / sig[1])
        ref = np.stack([rows[j].detach().numpy() * sig[j] for j in range(9)])
        np.testing.assert_allclose(P[:, active], ref[:, active], rtol=1e-13, atol=1e-13)
        assert np.array_equal(P[:, ~active], prm[:, ~active])


def test_adam_first_step_closed_form(orc):
    H, W, N = 16, 16, 10
    prm = _params(N, H, W, 52).astype(np.float64)
    g = synth.random_gradients(N, 7).astype(np.float64)
    lr = [1e-3] * 9
    P, _, _ = orc.adam(H, W, prm, np.zeros_like(prm), np.zeros_like(prm), g, lr, 1)
    sig = np.ones(9)
    sig[[0, 1, 3]] = 16.0
    gh = g * sig[:, None]
    ref = prm - 1e-3 * sig[:, None] * gh / (np.abs(gh) + 1e-8)
    np.testing.assert_allclose(P, ref, rtol=1e-12, atol=1e-15)


# --------------------------------------------------------------------------
# candidate propagation ([P2] key design 3, [P1] B.3) and its RNG
# --------------------------------------------------------------------------

def test_fmix32_published_vectors(orc):
    """MurmurHash3_x86_32 of an empty key is fmix32(seed): SMHasher's
    verification values for seeds 0, 1 and 0xffffffff."""
    assert orc.fmix32(0) == 0
    assert orc.fmix32(1) == 0x514E28B7
    assert orc.fmix32(0xFFFFFFFF) == 0x81F16F39


def test_xorshift32_matches_gf2_matrix_form(orc):
    """Marsaglia's xorshift is x -> x T with T = (I + L^a)(I + R^b)(I + L^c)
    over GF(2); check the (13, 17, 5) generator through that matrix form."""
    n = 32
    I = np.eye(n, dtype=np.int64)
    L = np.zeros((n, n), dtype=np.int64)   # left shift by one bit: bit q -> q + 1
    for q in range(n - 1):
        L[q + 1, q] = 1
    Rm = L.T.copy()                         # right shift
    mp = np.linalg.matrix_power
    # x ^= x << 13; x ^= x >> 17; x ^= x << 5  as column-vector maps
    T = ((I + mp(L, 5)) % 2) @ ((I + mp(Rm, 17)) % 2) % 2 @ ((I + mp(L, 13)) % 2) % 2
    st = synth.Stream(9, "xs")
    for x in st.bits(64):
        x = int(x) & 0xFFFFFFFF
        if x == 0:
            continue
        bits = np.array([(x >> q) & 1 for q in range(n)], dtype=np.int64)
        y = T @ bits % 2
        ref = sum(int(b) << q for q, b in enumerate(y))
        assert orc.xorshift32(x) == ref


def test_injection_ids_in_range_and_uniform(orc):
    N = 1000
    ids = np.concatenate([orc.inject_ids(7, 3, p, N, 4) for p in range(20000)])
    assert ids.min() >= 0 and ids.max() < N
    counts = np.bincount(ids, minlength=N)
    chi2 = ((counts - ids.size / N) ** 2 / (ids.size / N)).sum()
    # 999 dof: mean 999, sd ~ 44.7; accept within 5 sd
    assert abs(chi2 - (N - 1)) < 5 * math.sqrt(2 * (N - 1))
    # different passes and seeds give different draws
    assert not np.array_equal(orc.inject_ids(7, 3, 5, N, 4), orc.inject_ids(7, 4, 5, N, 4))
    assert not np.array_equal(orc.inject_ids(7, 3, 5, N, 4), orc.inject_ids(8, 3, 5, N, 4))


def _union_top8_reference(orc, H, W, rec, tin, jump, G, seed, pas):
    """Independent restatement of one pass: gather the candidate union with
    numpy, score each unique valid id with the pinned float32 score, select
    with a lexicographic sort."""
    N = rec.shape[0]
    out = np.full((H * W, 8), SENT, dtype=np.uint32)
    for j in range(H):
        for i in range(W):
            p = j * W + i
            cand = [tin[p]]
            for (ni, nj) in ((i - jump, j), (i + jump, j), (i, j - jump), (i, j + jump)):
                if 0 <= ni < W and 0 <= nj < H:
                    cand.append(tin[nj * W + ni])
            if G > 0:
                cand.append(orc.inject_ids(seed, pas, p, N, G))
            ids = np.unique(np.concatenate(cand).astype(np.int64))
            ids = ids[(ids != SENT) & (ids < N)]
            ids = ids[rec[ids, 0] >= 0]
            sc = np.array([orc.score32(rec, int(q), i, j) for q in ids], dtype=np.float64)
            keep = ~np.isnan(sc)
            ids, sc = ids[keep], sc[keep]
            order = np.lexsort((ids, -sc))[:8]
            out[p, :order.size] = ids[order]
    return out


@pytest.mark.parametrize("jump,G", [(1, 0), (1, 3), (4, 2), (16, 1)])
def test_propagate_equals_union_top8(orc, jump, G):
    H, W, N = 14, 11, 60
    prm = _params(N, H, W, 61 + jump, a_sd=0.8, r_max=4, log10_tau=(1.5, 3))
    prm[0, 3] = -1.0   # one inactive site
    rec = orc.records(H, W, prm)
    st = synth.Stream(jump * 10 + G, "tables")
    tin = st.integers(H * W * 8, N + 8).astype(np.uint32).reshape(H * W, 8)
    tin[st.uniform(H * W * 8).reshape(H * W, 8) < 0.2] = SENT
    tout = orc.propagate(H, W, rec, tin, jump, G, seed=77, pass_index=5)
    ref = _union_top8_reference(orc, H, W, rec, tin, jump, G, 77, 5)
    np.testing.assert_array_equal(tout, ref)
    # a pass's lists hold no id twice, whatever its input held (the refresh's
    # later passes rely on it: they read only lists written by a pass)
    for row in tout:
        v = row[row != SENT]
        assert v.size == np.unique(v).size


def test_propagate_with_rich_injection_converges_to_exact(orc):
    H, W, N = 16, 16, 40
    prm = _params(N, H, W, 71, a_sd=0.6, r_max=3, log10_tau=(1, 3))
    rec = orc.records(H, W, prm)
    t = np.full((H * W, 8), SENT, dtype=np.uint32)
    for pas in range(6):
        t = orc.propagate(H, W, rec, t, 1, 64, seed=3, pass_index=pas)
    np.testing.assert_array_equal(t, orc.topk_exact(H, W, rec))


def test_seed_pass(orc):
    H, W, N = 10, 12, 80
    prm = _params(N, H, W, 72)
    prm[0, 0] = -1.0
    t = orc.seed_table(H, W, prm)
    assert np.all(t[:, 1:] == SENT)
    ref = np.full(H * W, SENT, dtype=np.uint32)
    for i in range(N - 1, -1, -1):
        if prm[0, i] >= 0:
            ref[int(np.floor(prm[1, i])) * W + int(np.floor(prm[0, i]))] = i
    np.testing.assert_array_equal(t[:, 0], ref)


def test_jump_schedule(orc):
    assert orc.jump_schedule(512, 768) == [256, 128, 64, 32, 16, 8, 4, 2, 1]
    assert orc.jump_schedule(4096, 4096)[0] == 2048 and len(orc.jump_schedule(4096, 4096)) == 12


def test_refresh_reaches_pages_accuracy_at_1024(orc):
    """[P5] section 3: after 12-16 propagation rounds at 1024^2 more than 96%
    of pixels hold exactly the right top-8 list."""
    claim = json.load(open(os.path.join(HERE, "golden", "pages_claims.json")))["propagation_exact_top8"]
    H = W = claim["resolution"]
    N = 65536
    tgt = synth.make_image(H, W, 60, 4, 9)
    prm = synth.gradient_sites(tgt, N, 9)
    rec = orc.records(H, W, prm)
    t = orc.seed_table(H, W, prm)
    sched = orc.jump_schedule(H, W)
    rounds = claim["rounds"][1]
    sched = sched + [1] * (rounds - len(sched))
    for pas, k in enumerate(sched):
        t = orc.propagate(H, W, rec, t, k, 2, seed=1, pass_index=pas)
    pix = synth.Stream(1, "sample").integers(4096, H * W)
    ex = orc.topk_exact(H, W, rec, pix)
    exact = np.all(np.sort(t[pix], 1) == np.sort(ex, 1), axis=1)
    assert exact.mean() > claim["min_fraction_exact"]


def test_jfa3x3_prepass(orc):
    """The optional 3x3 flood prepass ([P1] B.3): each pass keeps the 4 best
    distinct candidates of the 9 lists at jump k, re-scored at the pixel
    (checked against an independent restatement); on Euclidean sites the
    prepass finds the nearest site on most pixels (jump flooding is
    approximate) and only ever fills slots 0-3."""
    H, W, N = 48, 40, 90
    prm = _params(N, H, W, 81)                  # a = 0, r = 0, uniform tau
    rec = orc.records(H, W, prm)
    assert orc.flood_schedule(48, 40) == [32, 16, 8, 4, 2, 1]
    t = orc.jfa_prepass(H, W, prm)
    assert np.all(t[:, 4:] == SENT)
    ex = orc.topk_exact(H, W, rec)
    assert np.mean(t[:, 0] == ex[:, 0]) > 0.95
    # one pass against an independent restatement
    st = synth.Stream(5, "jfa")
    tin = st.integers(H * W * 8, N + 3).astype(np.uint32).reshape(H * W, 8)
    for k in (1, 3, 7):
        got = orc.jfa3x3(H, W, rec, tin, k)
        for p in range(0, H * W, 37):
            j, i = divmod(p, W)
            cand = [tin[(j + b * k) * W + i + a * k] for b in (-1, 0, 1) for a in (-1, 0, 1)
                    if 0 <= i + a * k < W and 0 <= j + b * k < H]
            ids = np.unique(np.concatenate(cand).astype(np.int64))
            ids = ids[ids < N]
            sc = np.array([orc.score32(rec, int(q), i, j) for q in ids])
            order = np.lexsort((ids, -sc))[:4]
            want = np.full(8, SENT, np.uint32)
            want[:order.size] = ids[order]
            np.testing.assert_array_equal(got[p], want)
