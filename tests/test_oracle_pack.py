"""Pins of the oracle's 16-byte evaluation record ("Soft Anisotropic
Diagrams for Differentiable Image Representation", summary B.2 "Packed
storage for evaluation": ten semantic values in four 32-bit words, quantised,
with per-image min/scale for ln tau and radius).

Independent checks: the bit layout read back with Python integers, the
round-trip error of every field against half a quantisation step, the
per-image ranges against numpy, the rendered image of decoded sites against
the original, and the bitrate against the pages' Kodak figure."""
import json
import math
import os

import numpy as np

import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def _sites(H, W, N, seed):
    st = synth.Stream(seed, "pack")
    prm = np.zeros((9, N))
    prm[0] = st.uniform(N, 0, W)
    prm[1] = st.uniform(N, 0, H)
    prm[2] = synth.LN10 * st.uniform(N, 1.5, 4.0)
    prm[3] = st.uniform(N, 0, 5)
    prm[4:7] = st.uniform(3 * N, -0.1, 1.1).reshape(3, N)   # a few out of [0, 1]
    prm[7] = st.uniform(N, -7, 7)                           # any angle
    prm[8] = st.normal(N, 0, 0.8)
    prm[0, ::17] = -1.0
    return prm.astype(np.float32)


def _field(words, name, fields):
    big = sum(int(w) << (32 * q) for q, w in enumerate(words))
    off, n = fields[name]
    return (big >> off) & ((1 << n) - 1)


def test_ranges_are_min_max_of_active_sites(orc):
    prm = _sites(40, 60, 500, 1)
    lohi = orc.pack_ranges(prm)
    act = prm[0] >= 0
    for f, plane in enumerate((2, 3, 8)):
        assert lohi[f] == prm[plane, act].min() and lohi[3 + f] == prm[plane, act].max()
    none = prm.copy()
    none[0] = -1.0
    assert np.all(orc.pack_ranges(none) == 0)


def test_layout_and_endpoints(orc):
    H, W = 64, 96
    prm = _sites(H, W, 300, 2)
    packed, lohi = orc.pack_sites(H, W, prm)
    F = orc.PACK_FIELDS
    assert packed.shape == (300, 4) and packed.dtype == np.uint32
    assert sum(n for _, n in F.values()) <= 128
    for i in range(300):
        w = packed[i]
        if prm[0, i] < 0:
            assert np.all(w == 0)
            continue
        assert _field(w, "active", F) == 1
        assert (int(w[3]) >> 28) & 0x7 == 0            # spare bits 124-126
        assert _field(w, "x", F) == min(int(math.floor(prm[0, i] / W * 2 ** 18)), 2 ** 18 - 1)
    # fields at known values: colours 1, 0, 1/2 and the axis pi/2 (= -pi/2)
    q = prm.copy()
    q[0, 0], q[4, 0], q[5, 0], q[6, 0], q[7, 0] = 10.0, 1.0, 0.0, 0.5, -math.pi / 2
    w0 = orc.pack_sites(H, W, q, lohi)[0][0]
    assert (_field(w0, "cr", F), _field(w0, "cg", F), _field(w0, "cb", F)) == (1023, 0, 512)
    assert _field(w0, "theta", F) == 2 ** 13
    # the site holding the range minimum packs to 0, the maximum to 2^b - 1,
    # and both decode exactly to the stored range ends
    dec = orc.unpack_sites(H, W, packed, lohi)
    act = np.nonzero(prm[0] >= 0)[0]
    for f, (plane, name) in enumerate(((2, "ln_tau"), (3, "r"), (8, "a"))):
        lo_i = act[np.argmin(prm[plane, act])]
        hi_i = act[np.argmax(prm[plane, act])]
        assert _field(packed[lo_i], name, F) == 0
        assert _field(packed[hi_i], name, F) == 2 ** F[name][1] - 1
        assert dec[plane, lo_i] == lohi[f] and dec[plane, hi_i] == lohi[3 + f]


def test_round_trip_within_half_a_step(orc):
    H, W = 512, 768
    prm = _sites(H, W, 4000, 3)
    packed, lohi = orc.pack_sites(H, W, prm)
    dec = orc.unpack_sites(H, W, packed, lohi)
    act = prm[0] >= 0
    np.testing.assert_array_equal(dec[0] >= 0, act)
    assert np.all(dec[:, ~act][1:] == 0) and np.all(dec[0, ~act] == -1)
    p, d = prm[:, act].astype(np.float64), dec[:, act].astype(np.float64)
    ulp = lambda v: np.spacing(np.abs(v).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(d[0] - p[0]) <= W / 2 ** 19 + ulp(p[0]))
    assert np.all(np.abs(d[1] - p[1]) <= H / 2 ** 19 + ulp(p[1]))
    c = np.clip(p[4:7], 0, 1)
    assert np.all(np.abs(d[4:7] - c) <= 0.5 / 1023 + 1e-7)
    for f, (plane, bits) in enumerate(((2, 16), (3, 14), (8, 14))):
        step = (float(lohi[3 + f]) - float(lohi[f])) / (2 ** bits - 1)
        assert np.all(np.abs(d[plane] - p[plane]) <= 0.5 * step + 2 * ulp(p[plane]))
    # theta is an axis: compare modulo pi
    dt = np.abs(np.mod(d[7] - p[7] + np.pi / 2, np.pi) - np.pi / 2)
    assert np.all(dt <= np.pi / 2 ** 15 + 1e-6)
    assert np.all((d[7] >= 0) & (d[7] < np.pi))


def test_decoded_sites_render_like_the_originals(orc):
    """Quantisation moves the rendered image by far less than a fit's error:
    the decoded sites' render is within 45 dB PSNR of the original render
    (same lists, colours inside [0, 1])."""
    H, W, N = 96, 128, 1500
    tgt = synth.make_image(H, W, 10, 0, 4)
    prm = synth.gradient_sites(tgt, N, 4)
    tab = orc.topk_exact(H, W, orc.records(H, W, prm))
    packed, lohi = orc.pack_sites(H, W, prm)
    dec = orc.unpack_sites(H, W, packed, lohi)
    a = orc.render(H, W, prm, tab)
    b = orc.render(H, W, dec, tab)
    mse = float(np.mean((a - b) ** 2))
    assert 10 * math.log10(1.0 / mse) > 45.0


def test_bitrate_matches_the_pages_kodak_figure(orc):
    claim = json.load(open(os.path.join(HERE, "golden", "pages_claims.json")))["kodak_bits_per_pixel"]
    N, H, W = claim["N"], claim["H"], claim["W"]
    prm = _sites(H, W, 64, 5)
    packed, _ = orc.pack_sites(H, W, prm)
    bits_per_site = packed.itemsize * packed.shape[1] * 8
    assert bits_per_site == 128
    bpp = bits_per_site * N / (H * W)
    assert abs(bpp - claim["value"]) / claim["value"] < 0.05, bpp
