"""Seeded synthetic inputs for Soft Anisotropic Diagrams (SAD) workloads.

This module only draws numbers and paints test images.  It holds none of the
method's arithmetic (no metric, score, softmax, gradient or optimiser step), so
both the CPU oracle and the CUDA library may consume what it produces.

Random numbers come from SplitMix64 (Steele, Lea & Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) used as a counter-based
generator: draw k of a stream is mix64(base + (k + 1) * 0x9E3779B97F4A7C15),
where mix64 is SplitMix64's output function and base identifies the stream.
Uniform floats take the top 53 bits; normals use the Box-Muller transform.

Workloads (pixel counts P = H * W, site capacity N, K = 8 candidates):

* ``c1`` 256 x 256, N = 1024: uniform sites, 40 ellipses.
* ``c2`` 768 x 512, N = 50,000: uniform sites, 120 ellipses (Kodak-shaped).
* ``c3`` 2048 x 2048, N = 131,072: gradient-weighted sites, 300 ellipses and
  24 sinusoidal texture patches.
* ``c4`` 4096 x 4096, N = 524,288: gradient-weighted sites, then perturbed
  (p jittered by N(0, 3 px), a ~ N(0, 1), log10 tau ~ U[2, 4.5]).
* ``c5`` 768 x 512, N from 10,000 upward: gradient-weighted start.

Site parameters are returned as a float32 array of shape (9, N) in the plane
order ``PARAM_NAMES``; positions and radii are in pixels, the temperature is
stored as its natural logarithm.  Distribution notation N(mu, sd) takes a
standard deviation.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

PARAM_NAMES = ("x", "y", "log_tau", "r", "cr", "cg", "cb", "theta", "a")
N_PARAMS = 9
LN10 = math.log(10.0)

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wrapping arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _stream_base(seed: int, tag: str) -> np.uint64:
    h = np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    with np.errstate(over="ignore"):
        for ch in tag.encode():
            h = _mix64(h ^ np.uint64(ch)) + _GAMMA
        return _mix64(h)[0]


class Stream:
    """One counter-based SplitMix64 stream identified by (seed, tag)."""

    def __init__(self, seed: int, tag: str):
        self.base = _stream_base(seed, tag)
        self.counter = 0

    def bits(self, n: int) -> np.ndarray:
        k = np.arange(self.counter + 1, self.counter + 1 + n, dtype=np.uint64)
        self.counter += n
        with np.errstate(over="ignore"):
            return _mix64(self.base + k * _GAMMA)

    def uniform(self, n: int, lo: float = 0.0, hi: float = 1.0) -> np.ndarray:
        u = (self.bits(n) >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
        return lo + (hi - lo) * u

    def normal(self, n: int, mu: float = 0.0, sd: float = 1.0) -> np.ndarray:
        u1 = self.uniform(n)
        u2 = self.uniform(n)
        z = np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * math.pi * u2)
        return mu + sd * z

    def integers(self, n: int, hi: int) -> np.ndarray:
        """Integers in [0, hi) by 64-bit multiply-high of the top 32 bits."""
        b = self.bits(n) >> np.uint64(32)
        return ((b * np.uint64(hi)) >> np.uint64(32)).astype(np.int64)


# --------------------------------------------------------------------------
# target images
# --------------------------------------------------------------------------

def make_image(H: int, W: int, n_ellipses: int, n_patches: int, seed: int,
               noise_sd: float = 0.01) -> np.ndarray:
    """Procedural linear-RGB target of shape (3, H, W), float32, in [0, 1].

    Sum of three linear colour ramps (random direction, random endpoint
    colours, weights summing to one), then ``n_ellipses`` opaque hard-edged
    ellipses painted in order (centre uniform, semi-axes U(4, 0.15 max(H, W))
    px, angle U[0, pi), flat colour U[0, 1]^3), then ``n_patches`` discs of
    radius U(32, 256) px carrying an added sinusoid A_ch sin(2 pi f (x . w) +
    phi) with f ~ U(0.05, 0.3) cycles/px, random unit w and A_ch ~
    U(0.05, 0.25) per channel, then i.i.d. N(0, noise_sd) noise; clipped.
    """
    st = Stream(seed, f"image/{H}x{W}/{n_ellipses}/{n_patches}")
    yy = (np.arange(H, dtype=np.float64) + 0.5)[:, None]
    xx = (np.arange(W, dtype=np.float64) + 0.5)[None, :]
    img = np.zeros((3, H, W), dtype=np.float64)

    wts = st.uniform(3) + 1e-3
    wts = wts / wts.sum()
    for g in range(3):
        phi = st.uniform(1, 0.0, 2.0 * math.pi)[0]
        c0 = st.uniform(3)
        c1 = st.uniform(3)
        d = np.array([math.cos(phi), math.sin(phi)])
        extent = abs(W * d[0]) + abs(H * d[1])
        t = ((xx - 0.5 * W) * d[0] + (yy - 0.5 * H) * d[1]) / extent + 0.5
        t = np.clip(t, 0.0, 1.0)
        for ch in range(3):
            img[ch] += wts[g] * (c0[ch] + t * (c1[ch] - c0[ch]))

    big = 0.15 * max(H, W)
    for _ in range(n_ellipses):
        cx, cy = st.uniform(1, 0, W)[0], st.uniform(1, 0, H)[0]
        ea, eb = st.uniform(2, 4.0, max(big, 4.0 + 1e-6))
        ang = st.uniform(1, 0.0, math.pi)[0]
        col = st.uniform(3)
        rr = max(ea, eb)
        x0, x1 = max(int(cx - rr) - 1, 0), min(int(cx + rr) + 2, W)
        y0, y1 = max(int(cy - rr) - 1, 0), min(int(cy + rr) + 2, H)
        if x0 >= x1 or y0 >= y1:
            continue
        lx = xx[:, x0:x1] - cx
        ly = yy[y0:y1, :] - cy
        ca, sa = math.cos(ang), math.sin(ang)
        u = lx * ca + ly * sa
        v = -lx * sa + ly * ca
        inside = (u / ea) ** 2 + (v / eb) ** 2 <= 1.0
        for ch in range(3):
            blk = img[ch, y0:y1, x0:x1]
            blk[inside] = col[ch]

    for _ in range(n_patches):
        cx, cy = st.uniform(1, 0, W)[0], st.uniform(1, 0, H)[0]
        rad = st.uniform(1, 32.0, 256.0)[0]
        f = st.uniform(1, 0.05, 0.3)[0]
        om = st.uniform(1, 0.0, 2.0 * math.pi)[0]
        ph = st.uniform(1, 0.0, 2.0 * math.pi)[0]
        amp = st.uniform(3, 0.05, 0.25)
        x0, x1 = max(int(cx - rad) - 1, 0), min(int(cx + rad) + 2, W)
        y0, y1 = max(int(cy - rad) - 1, 0), min(int(cy + rad) + 2, H)
        if x0 >= x1 or y0 >= y1:
            continue
        lx = xx[:, x0:x1] - cx
        ly = yy[y0:y1, :] - cy
        inside = lx * lx + ly * ly <= rad * rad
        wave = np.sin(2.0 * math.pi * f * (xx[:, x0:x1] * math.cos(om) + yy[y0:y1, :] * math.sin(om)) + ph)
        for ch in range(3):
            blk = img[ch, y0:y1, x0:x1]
            blk[inside] += (amp[ch] * wave)[inside]

    if noise_sd > 0:
        img += st.normal(3 * H * W, 0.0, noise_sd).reshape(3, H, W)
    return np.clip(img, 0.0, 1.0).astype(np.float32)


# --------------------------------------------------------------------------
# sites
# --------------------------------------------------------------------------

def uniform_sites(H: int, W: int, N: int, seed: int, *, a_sd: float = 0.5,
                  log10_tau: tuple = (2.0, 4.0), r_max: float = 4.0) -> np.ndarray:
    """Sites with p ~ U[0,W) x U[0,H), a ~ N(0, a_sd), theta ~ U[0, pi),
    r ~ U(0, r_max) px, log10 tau ~ U[lo, hi], c ~ U[0, 1]^3."""
    st = Stream(seed, f"sites/uniform/{H}x{W}/{N}")
    prm = np.empty((N_PARAMS, N), dtype=np.float64)
    prm[0] = st.uniform(N, 0.0, W)
    prm[1] = st.uniform(N, 0.0, H)
    prm[2] = LN10 * st.uniform(N, *log10_tau)
    prm[3] = st.uniform(N, 0.0, r_max)
    prm[4:7] = st.uniform(3 * N).reshape(3, N)
    prm[7] = st.uniform(N, 0.0, math.pi)
    prm[8] = st.normal(N, 0.0, a_sd)
    out = prm.astype(np.float32)
    # float32 rounding must not push a position onto the far image edge
    out[0] = np.minimum(out[0], np.nextafter(np.float32(W), np.float32(0)))
    out[1] = np.minimum(out[1], np.nextafter(np.float32(H), np.float32(0)))
    return out


def _sobel_magnitude(lum: np.ndarray) -> np.ndarray:
    p = np.pad(lum, 1, mode="edge")
    gx = (p[:-2, 2:] + 2 * p[1:-1, 2:] + p[2:, 2:]) - (p[:-2, :-2] + 2 * p[1:-1, :-2] + p[2:, :-2])
    gy = (p[2:, :-2] + 2 * p[2:, 1:-1] + p[2:, 2:]) - (p[:-2, :-2] + 2 * p[:-2, 1:-1] + p[:-2, 2:])
    return np.sqrt(gx * gx + gy * gy)


def gradient_sites(target: np.ndarray, N: int, seed: int, *, mix: float = 0.5,
                   a_sd: float = 0.5, log10_tau: tuple = (2.0, 4.0),
                   r_max: float = 4.0) -> np.ndarray:
    """Gradient-weighted initial layout: pixels drawn with probability
    mix * |Sobel(luma)| / sum + (1 - mix) / P, positions jittered uniformly
    inside the drawn pixel, colours read from the target at that pixel; the
    other parameters follow ``uniform_sites``."""
    _, H, W = target.shape
    st = Stream(seed, f"sites/gradient/{H}x{W}/{N}")
    lum = 0.2126 * target[0] + 0.7152 * target[1] + 0.0722 * target[2]
    mag = _sobel_magnitude(lum.astype(np.float64)).ravel()
    tot = mag.sum()
    prob = (mix * mag / tot if tot > 0 else 0.0) + (1.0 - mix) / mag.size
    cdf = np.cumsum(prob)
    cdf /= cdf[-1]
    pick = np.searchsorted(cdf, st.uniform(N), side="right")
    pick = np.minimum(pick, mag.size - 1)
    py, px = np.divmod(pick, W)
    prm = np.empty((N_PARAMS, N), dtype=np.float64)
    prm[0] = px + st.uniform(N)
    prm[1] = py + st.uniform(N)
    prm[2] = LN10 * st.uniform(N, *log10_tau)
    prm[3] = st.uniform(N, 0.0, r_max)
    for ch in range(3):
        prm[4 + ch] = target[ch].ravel()[pick]
    prm[7] = st.uniform(N, 0.0, math.pi)
    prm[8] = st.normal(N, 0.0, a_sd)
    out = prm.astype(np.float32)
    out[0] = np.minimum(out[0], np.nextafter(np.float32(W), np.float32(0)))
    out[1] = np.minimum(out[1], np.nextafter(np.float32(H), np.float32(0)))
    return out


def perturbed_sites(target: np.ndarray, N: int, seed: int) -> np.ndarray:
    """A fitted-like layout disturbed for a full refresh: gradient-weighted
    positions jittered by N(0, 3 px) (kept inside the image), a ~ N(0, 1),
    log10 tau ~ U[2, 4.5]."""
    _, H, W = target.shape
    prm = gradient_sites(target, N, seed).astype(np.float64)
    st = Stream(seed, f"sites/perturb/{H}x{W}/{N}")
    prm[0] = np.clip(prm[0] + st.normal(N, 0.0, 3.0), 0.0, W)
    prm[1] = np.clip(prm[1] + st.normal(N, 0.0, 3.0), 0.0, H)
    prm[8] = st.normal(N, 0.0, 1.0)
    prm[2] = LN10 * st.uniform(N, 2.0, 4.5)
    out = prm.astype(np.float32)
    out[0] = np.minimum(out[0], np.nextafter(np.float32(W), np.float32(0)))
    out[1] = np.minimum(out[1], np.nextafter(np.float32(H), np.float32(0)))
    return out


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    W: int
    N: int
    n_ellipses: int
    n_patches: int
    sites: str          # "uniform" | "gradient" | "perturbed"
    G: int              # stochastic injections per pixel per propagation pass
    description: str


WORKLOADS = {
    "c1": Workload("c1", 256, 256, 1024, 40, 0, "uniform", 2,
                   "256x256, N=1024: exact top-K, render, backward, one Adam step"),
    "c2": Workload("c2", 512, 768, 50_000, 120, 0, "uniform", 2,
                   "768x512, N=50,000: seed + refresh 256..1, fit iterations"),
    "c3": Workload("c3", 2048, 2048, 131_072, 300, 24, "gradient", 2,
                   "2048x2048, N=131,072: steady-state fit iterations (k=1, G=2)"),
    "c4": Workload("c4", 4096, 4096, 524_288, 300, 24, "perturbed", 4,
                   "4096x4096, N=524,288: full refresh 2048..1 (G=4) + render"),
    "c5": Workload("c5", 512, 768, 10_000, 120, 0, "gradient", 2,
                   "768x512, N from 10,000: end-to-end fit with densify/prune"),
}


def make_workload(name: str, seed: int = 1, N: int | None = None,
                  H: int | None = None, W: int | None = None):
    """Return (target (3,H,W) float32, params (9,N) float32, Workload)."""
    wl = WORKLOADS[name]
    H = wl.H if H is None else H
    W = wl.W if W is None else W
    N = wl.N if N is None else N
    salt = {"c1": 101, "c2": 202, "c3": 303, "c4": 404, "c5": 505}[name]
    tgt = make_image(H, W, wl.n_ellipses, wl.n_patches, seed * 1000 + salt)
    if wl.sites == "uniform":
        prm = uniform_sites(H, W, N, seed * 1000 + salt)
    elif wl.sites == "gradient":
        prm = gradient_sites(tgt, N, seed * 1000 + salt)
    else:
        prm = perturbed_sites(tgt, N, seed * 1000 + salt)
    return tgt, prm, wl


def random_gradients(N: int, seed: int, scale: float = 1e-4) -> np.ndarray:
    """Synthetic per-site gradient planes (9, N) for optimiser tests: a mix of
    normal values across several magnitudes, exact zeros and a few tiny ones."""
    st = Stream(seed, f"grads/{N}")
    g = st.normal(N_PARAMS * N, 0.0, 1.0).reshape(N_PARAMS, N)
    mag = 10.0 ** st.uniform(N_PARAMS * N, -3.0, 1.0).reshape(N_PARAMS, N)
    g = g * mag * scale
    z = st.uniform(N_PARAMS * N).reshape(N_PARAMS, N)
    g[z < 0.05] = 0.0
    return g.astype(np.float32)
