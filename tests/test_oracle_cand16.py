"""Pins of the oracle's packed candidate-site mode ("Soft Anisotropic
Diagrams for Differentiable Image Representation", paperlayer summary B.2:
candidate-update kernels score from a 16-byte buffer of float16 pairs).

The mode ranks candidates on score coefficients rounded to binary16 and
re-scores the kept 8 in float32.  Pinned here against numpy's own binary16
conversion, against the float32 mode where the rounding is exact, and
against a numpy restatement of the selection and the final order."""
import math

import numpy as np
import pytest

import synth
from test_oracle_pins import SENT, _params, _union_top8_reference


def test_binary16_rounding_matches_numpy(orc):
    st = synth.Stream(16, "binary16")
    mags = 10.0 ** st.uniform(4000, -9.0, 5.2)
    vals = (mags * np.where(st.uniform(4000) < 0.5, -1.0, 1.0)).astype(np.float32)
    # ties, the largest finite value, the overflow threshold, subnormals
    edge = np.array([0.0, -0.0, 1.0, 2049.0, 2051.0, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 65504.0, 65519.99,
                     65520.0, 1e6, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14, 6.0e-5, math.inf, -math.inf],
                    dtype=np.float32)
    for x in np.concatenate([vals, edge]):
        with np.errstate(over="ignore"):
            want = float(np.float16(x))
        got = orc.to_binary16(float(x))
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), (float(x), got, want)
    assert math.isnan(orc.to_binary16(math.nan))


def test_selection_record_rounds_the_coefficients_only(orc):
    H, W, N = 20, 30, 50
    prm = _params(N, H, W, 5, a_sd=0.7, r_max=3, log10_tau=(1.5, 3.5))
    rec = orc.records(H, W, prm)
    sel = orc.cand16_record(rec)
    keep = [f for f in range(16) if f not in (2, 3, 4, 5)]
    assert np.array_equal(sel[:, keep].view(np.uint32), rec[:, keep].view(np.uint32))
    want = rec[:, 2:6].astype(np.float16).astype(np.float32)
    assert np.array_equal(sel[:, 2:6].view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("jump,G", [(1, 2), (4, 0)])
def test_exact_coefficients_give_the_float32_lists(orc, jump, G):
    """Sites with a = 0, theta = 0, r = 0 and k = tau s a power of two have
    A = C = k^2, B = b = 0, all binary16 values: both modes agree bit for bit."""
    H, W, N = 16, 16, 70
    st = synth.Stream(jump, "exact16")
    prm = np.zeros((9, N), np.float32)
    prm[0] = st.uniform(N, 0, W)
    prm[1] = st.uniform(N, 0, H)
    prm[2] = np.log(2.0 ** st.integers(N, 4).astype(np.float64) * max(H, W))  # k = 1, 2, 4, 8
    prm[4:7] = st.uniform(3 * N).reshape(3, N)
    rec = orc.records(H, W, prm)
    assert np.array_equal(orc.cand16_record(rec).view(np.uint32), rec.view(np.uint32))
    tin = orc.topk_exact(H, W, rec)
    tin[::3, 4:] = SENT
    a = orc.propagate(H, W, rec, tin, jump, G, seed=3, pass_index=1)
    b = orc.propagate(H, W, rec, tin, jump, G, seed=3, pass_index=1, cand16=True)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("jump,G", [(1, 3), (2, 1), (8, 2)])
def test_cand16_pass_equals_restatement(orc, jump, G):
    """Union top-8 under the binary16-coefficient score (the pinned float32
    score on the selection record), then the kept ids ordered by the float32
    score with ties to the smaller id."""
    H, W, N = 12, 13, 55
    prm = _params(N, H, W, 70 + jump, a_sd=0.9, r_max=4, log10_tau=(1.5, 3.5))
    prm[0, 7] = -1.0
    rec = orc.records(H, W, prm)
    sel = orc.cand16_record(rec)
    st = synth.Stream(jump * 7 + G, "tables16")
    tin = st.integers(H * W * 8, N + 4).astype(np.uint32).reshape(H * W, 8)
    tin[st.uniform(H * W * 8).reshape(H * W, 8) < 0.25] = SENT
    got = orc.propagate(H, W, rec, tin, jump, G, seed=9, pass_index=4, cand16=True)
    kept = _union_top8_reference(orc, H, W, sel, tin, jump, G, 9, 4)
    want = np.full_like(kept, SENT)
    for p in range(H * W):
        ids = kept[p][kept[p] != SENT].astype(np.int64)
        sc = np.array([orc.score32(rec, int(q), p % W, p // W) for q in ids])
        order = np.lexsort((ids, -sc))
        want[p, :ids.size] = ids[order]
    np.testing.assert_array_equal(got, want)
    # the rounding does change decisions somewhere on this workload
    plain = orc.propagate(H, W, rec, tin, jump, G, seed=9, pass_index=4)
    assert (np.sort(plain, 1) != np.sort(got, 1)).any() or jump == 1


def test_cand16_refresh_reaches_high_recall(orc):
    """A refresh ranked on the packed record, then jump-1 passes, holds
    nearly the exact top-8 (the float32 mode's recall on this workload is
    checked elsewhere)."""
    H, W, N = 96, 128, 1500
    tgt = synth.make_image(H, W, 10, 0, 3)
    prm = synth.gradient_sites(tgt, N, 3)
    t, n = orc.refresh(H, W, prm, 2, seed=5, cand16=True)
    rec = orc.records(H, W, prm)
    for k in range(8):
        t = orc.propagate(H, W, rec, t, 1, 2, seed=5, pass_index=n + k, cand16=True)
    ex = orc.topk_exact(H, W, rec)
    hit = np.mean([len(set(a.tolist()) & set(b.tolist()) - {SENT}) / max(1, int((b != SENT).sum()))
                   for a, b in zip(t, ex)])
    assert hit >= 0.99, hit
