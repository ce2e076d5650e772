"""CPU oracle for one Soft Anisotropic Diagrams fitting iteration.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA library never
imports, links or runs anything here, and this package imports nothing from
the CUDA library.

Thin ctypes wrappers over ``sad_oracle.c`` (plain C, fp64 render / backward /
Adam, fp32 top-K decisions).  Tables are (P, 8) uint32 arrays of site ids,
images (3, H, W), site parameters (9, N) float32 planes in the order
x, y, ln tau, r, cr, cg, cb, theta, a.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from . import build as _build

SENTINEL = 0xFFFFFFFF
K = 8
REC = 16

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c_int, c_i64, c_u32, c_dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_uint32, ctypes.c_double
        vp = ctypes.c_void_p
        L.orc_records.argtypes = [c_int, c_int, c_int, vp, vp, vp]
        L.orc_score32.argtypes = [vp, c_int, c_int, c_int]
        L.orc_score32.restype = ctypes.c_float
        L.orc_topk_exact.argtypes = [c_int, c_int, c_int, vp, vp, c_i64, vp]
        L.orc_topk_exact_cell.argtypes = [c_int, c_int, c_int, c_int, vp, vp, c_i64, vp]
        L.orc_propagate_cell.argtypes = [c_int, c_int, c_int, c_int, vp, vp, vp, c_int, c_int, c_u32, c_u32]
        L.orc_seed_cell.argtypes = [c_int, c_int, c_int, c_int, vp, vp]
        L.orc_jfa3x3_cell.argtypes = [c_int, c_int, c_int, c_int, vp, vp, vp, c_int]
        L.orc_score32_at.argtypes = [vp, c_int, ctypes.c_float, ctypes.c_float]
        L.orc_score32_at.restype = ctypes.c_float
        L.orc_fmix32.argtypes = [c_u32]
        L.orc_fmix32.restype = c_u32
        L.orc_xorshift32.argtypes = [c_u32]
        L.orc_xorshift32.restype = c_u32
        L.orc_inject_ids.argtypes = [c_u32, c_u32, c_u32, c_int, c_int, vp]
        L.orc_propagate.argtypes = [c_int, c_int, c_int, vp, vp, vp, c_int, c_int, c_u32, c_u32]
        L.orc_seed.argtypes = [c_int, c_int, c_int, vp, vp]
        L.orc_render.argtypes = [c_int, c_int, c_int, vp, vp, vp]
        L.orc_weights.argtypes = [c_int, c_int, c_int, vp, vp, vp]
        L.orc_loss_backward.argtypes = [c_int, c_int, c_int, vp, vp, vp, vp, vp]
        L.orc_loss_backward.restype = c_dbl
        L.orc_adam.argtypes = [c_int, c_int, c_int, vp, vp, vp, vp, vp, c_dbl, c_dbl, c_dbl, c_int]
        L.orc_loss_backward_stats.argtypes = [c_int, c_int, c_int, vp, vp, vp, vp, vp, vp, vp]
        L.orc_loss_backward_stats.restype = c_dbl
        L.orc_split_score.argtypes = [ctypes.c_float] * 4
        L.orc_split_score.restype = ctypes.c_float
        L.orc_densify_prune.argtypes = [c_int, c_int, c_int, vp, vp, vp, vp, vp, vp, vp]
        L.orc_densify_prune.restype = c_int
        L.orc_adam_frozen.argtypes = [c_int, c_int, c_int, vp, vp, vp, vp, vp, c_dbl, c_dbl, c_dbl, c_int, vp]
        L.orc_tau_diffuse.argtypes = [c_int, c_int, c_int, vp, vp, vp, c_dbl]
        L.orc_jfa3x3.argtypes = [c_int, c_int, c_int, vp, vp, vp, c_int]
        L.orc_pack_ranges.argtypes = [c_int, vp, vp]
        L.orc_pack_sites.argtypes = [c_int, c_int, c_int, vp, vp, vp]
        L.orc_unpack_sites.argtypes = [c_int, c_int, c_int, vp, vp, vp]
        L.orc_to_binary16.argtypes = [ctypes.c_float]
        L.orc_to_binary16.restype = ctypes.c_float
        L.orc_cand16_record.argtypes = [c_int, vp, vp]
        L.orc_rescore_sort_cell.argtypes = [c_int, c_int, c_int, c_int, vp, vp]
        L.orc_num_threads.restype = c_int
        L.orc_set_threads.argtypes = [c_int]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _u32(a):
    return np.ascontiguousarray(a, dtype=np.uint32)


def num_threads() -> int:
    return lib().orc_num_threads()


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def records(H: int, W: int, params: np.ndarray, with64: bool = False):
    """Per-site score records (N, 16) float32 (and float64 if ``with64``)."""
    params = _f32(params)
    N = params.shape[1]
    r32 = np.empty((N, REC), dtype=np.float32)
    r64 = np.empty((N, REC), dtype=np.float64) if with64 else None
    lib().orc_records(H, W, N, _p(params), _p(r32), _p(r64) if with64 else None)
    return (r32, r64) if with64 else r32


def score32(rec32: np.ndarray, site: int, i: int, j: int) -> float:
    rec32 = _f32(rec32)
    return float(lib().orc_score32(_p(rec32), int(site), int(i), int(j)))


def score32_at(rec32: np.ndarray, site: int, fx: float, fy: float) -> float:
    rec32 = _f32(rec32)
    return float(lib().orc_score32_at(_p(rec32), int(site), float(fx), float(fy)))


def grid_dims(H: int, W: int, cell: int = 1):
    """Candidate grid of an H x W image with cells of cell x cell pixels
    ("Candidate field", summary B.3): (ceil(H / cell), ceil(W / cell))."""
    return (H + cell - 1) // cell, (W + cell - 1) // cell


def expand_table(H: int, W: int, table: np.ndarray, cell: int) -> np.ndarray:
    """Per-pixel view of a candidate-grid table: pixel (x, y) takes the list
    of cell (x // cell, y // cell)."""
    GH, GW = grid_dims(H, W, cell)
    tab = _u32(table).reshape(GH * GW, K)
    jj, ii = np.mgrid[0:H, 0:W]
    return np.ascontiguousarray(tab[((jj // cell) * GW + ii // cell).ravel()])


def topk_exact(H: int, W: int, rec32: np.ndarray, pixels: np.ndarray | None = None, cell: int = 1) -> np.ndarray:
    """Brute-force top-8 over all active sites at each requested pixel (cell
    centre when cell > 1); (n_pix, 8) uint32."""
    rec32 = _f32(rec32)
    N = rec32.shape[0]
    GH, GW = grid_dims(H, W, cell)
    if pixels is None:
        n = GH * GW
        out = np.empty((n, K), dtype=np.uint32)
        lib().orc_topk_exact_cell(GH, GW, cell, N, _p(rec32), None, n, _p(out))
    else:
        pix = np.ascontiguousarray(pixels, dtype=np.int64)
        out = np.empty((pix.size, K), dtype=np.uint32)
        lib().orc_topk_exact_cell(GH, GW, cell, N, _p(rec32), _p(pix), pix.size, _p(out))
    return out


def fmix32(h: int) -> int:
    return int(lib().orc_fmix32(h & 0xFFFFFFFF))


def xorshift32(h: int) -> int:
    return int(lib().orc_xorshift32(h & 0xFFFFFFFF))


def inject_ids(seed: int, pass_index: int, pixel: int, N: int, G: int) -> np.ndarray:
    out = np.empty(max(G, 1), dtype=np.uint32)
    lib().orc_inject_ids(seed & 0xFFFFFFFF, pass_index & 0xFFFFFFFF, pixel & 0xFFFFFFFF, N, G, _p(out))
    return out[:G]


def to_binary16(x: float) -> float:
    """x rounded to the nearest IEEE binary16 value (ties to even), as a float."""
    return float(lib().orc_to_binary16(float(x)))


def cand16_record(rec32: np.ndarray) -> np.ndarray:
    """The candidate-selection record of the packed candidate-site mode:
    the float32 record with A, B, C and b rounded to binary16."""
    rec32 = _f32(rec32)
    out = np.empty_like(rec32)
    lib().orc_cand16_record(rec32.shape[0], _p(rec32), _p(out))
    return out


def rescore_sort(H: int, W: int, rec32: np.ndarray, table: np.ndarray, cell: int = 1) -> np.ndarray:
    """Each list re-scored with the float32 record, in (logit desc, id asc) order."""
    rec32 = _f32(rec32)
    GH, GW = grid_dims(H, W, cell)
    t = _u32(table).reshape(GH * GW, K).copy()
    lib().orc_rescore_sort_cell(GH, GW, cell, rec32.shape[0], _p(rec32), _p(t))
    return t


def propagate(H: int, W: int, rec32: np.ndarray, table: np.ndarray, jump: int, G: int,
              seed: int, pass_index: int, cell: int = 1, cand16: bool = False) -> np.ndarray:
    """One Jacobi propagation pass on the candidate grid of an H x W image;
    returns the new (cells, 8) table.  With cand16 the candidates are ranked
    on the packed candidate-site record (cand16_record) and the kept 8 are
    re-scored in float32 (rescore_sort)."""
    rec32 = _f32(rec32)
    GH, GW = grid_dims(H, W, cell)
    tin = _u32(table).reshape(GH * GW, K)
    tout = np.empty_like(tin)
    sel = cand16_record(rec32) if cand16 else rec32
    lib().orc_propagate_cell(GH, GW, cell, rec32.shape[0], _p(sel), _p(tin), _p(tout), int(jump), int(G),
                             seed & 0xFFFFFFFF, pass_index & 0xFFFFFFFF)
    if cand16:
        lib().orc_rescore_sort_cell(GH, GW, cell, rec32.shape[0], _p(rec32), _p(tout))
    return tout


def seed_table(H: int, W: int, params: np.ndarray, cell: int = 1) -> np.ndarray:
    params = _f32(params)
    GH, GW = grid_dims(H, W, cell)
    out = np.empty((GH * GW, K), dtype=np.uint32)
    lib().orc_seed_cell(H, W, cell, params.shape[1], _p(params), _p(out))
    return out


def jump_schedule(H: int, W: int) -> list:
    """B/2, B/4, ..., 1 with B the largest power of two <= max(H, W)."""
    B = 1
    while B * 2 <= max(H, W):
        B *= 2
    out = []
    k = B // 2
    while k >= 1:
        out.append(k)
        k //= 2
    return out


def refresh(H: int, W: int, params: np.ndarray, G: int, seed: int, first_pass: int = 0, cell: int = 1,
            cand16: bool = False):
    """Seed pass then one propagation pass per jump of ``jump_schedule`` of
    the candidate grid.  Returns (table, number of passes run)."""
    rec = records(H, W, params)
    t = seed_table(H, W, params, cell)
    n = 0
    for k in jump_schedule(*grid_dims(H, W, cell)):
        t = propagate(H, W, rec, t, k, G, seed, first_pass + n, cell, cand16=cand16)
        n += 1
    return t, n


def render(H: int, W: int, params: np.ndarray, table: np.ndarray) -> np.ndarray:
    params = _f32(params)
    tab = _u32(table).reshape(H * W, K)
    img = np.empty((3, H, W), dtype=np.float64)
    lib().orc_render(H, W, params.shape[1], _p(params), _p(tab), _p(img))
    return img


def weights(H: int, W: int, params: np.ndarray, table: np.ndarray) -> np.ndarray:
    params = _f32(params)
    tab = _u32(table).reshape(H * W, K)
    w = np.empty((H * W, K), dtype=np.float64)
    lib().orc_weights(H, W, params.shape[1], _p(params), _p(tab), _p(w))
    return w


def loss_backward(H: int, W: int, params: np.ndarray, table: np.ndarray, target: np.ndarray,
                  want_image: bool = False):
    """Returns (loss, grads (9, N) float64[, image (3, H, W) float64])."""
    params = _f32(params)
    tab = _u32(table).reshape(H * W, K)
    tgt = _f32(target).reshape(3, H * W)
    N = params.shape[1]
    g = np.empty((9, N), dtype=np.float64)
    img = np.empty((3, H, W), dtype=np.float64) if want_image else None
    L = lib().orc_loss_backward(H, W, N, _p(params), _p(tab), _p(tgt), _p(g),
                                _p(img) if want_image else None)
    return (L, g, img) if want_image else (L, g)


ADAM_PLANE_GROUP = ("pos", "pos", "log_tau", "r", "color", "color", "color", "theta", "a")


def adam(H: int, W: int, params, m, v, grads, lr, t: int, b1: float = 0.9, b2: float = 0.999,
         eps: float = 1e-8, frozen=None):
    """One Adam step in double.  ``lr`` is a dict keyed by ADAM_PLANE_GROUP
    names or a length-9 sequence; ``frozen`` an optional per-site uint8 mask
    of sites left untouched.  Returns new (params, m, v) float64."""
    P = np.array(params, dtype=np.float64, order="C", copy=True)
    M = np.array(m, dtype=np.float64, order="C", copy=True)
    V = np.array(v, dtype=np.float64, order="C", copy=True)
    G = np.ascontiguousarray(grads, dtype=np.float64)
    if isinstance(lr, dict):
        lrv = np.array([lr[gname] for gname in ADAM_PLANE_GROUP], dtype=np.float64)
    else:
        lrv = np.ascontiguousarray(lr, dtype=np.float64)
    if frozen is None:
        lib().orc_adam(H, W, P.shape[1], _p(P), _p(M), _p(V), _p(G), _p(lrv), b1, b2, eps, int(t))
    else:
        fz = np.ascontiguousarray(frozen, dtype=np.uint8)
        lib().orc_adam_frozen(H, W, P.shape[1], _p(P), _p(M), _p(V), _p(G), _p(lrv), b1, b2, eps, int(t), _p(fz))
    return P, M, V


STAT_NAMES = ("mass", "energy", "sxx", "sxy", "syy", "removal")


def loss_backward_stats(H: int, W: int, params, table, target, want_abs: bool = False):
    """Returns (loss, grads (9, N), stats (6, N)[, stats_abs (6, N)]) in
    float64; stats rows are STAT_NAMES, stats_abs the sums of the terms'
    absolute values."""
    params = _f32(params)
    tab = _u32(table).reshape(H * W, K)
    tgt = _f32(target).reshape(3, H * W)
    N = params.shape[1]
    g = np.empty((9, N), dtype=np.float64)
    st = np.empty((6, N), dtype=np.float64)
    sa = np.empty((6, N), dtype=np.float64) if want_abs else None
    L = lib().orc_loss_backward_stats(H, W, N, _p(params), _p(tab), _p(tgt), _p(g), None, _p(st),
                                      _p(sa) if want_abs else None)
    return (L, g, st, sa) if want_abs else (L, g, st)


class DensifyCfg(ctypes.Structure):
    _fields_ = [("grow", ctypes.c_int), ("prune_frac", ctypes.c_float), ("alpha", ctypes.c_float),
                ("eps", ctypes.c_float), ("r_scale", ctypes.c_float), ("log_tau_shift", ctypes.c_float),
                ("offset_scale", ctypes.c_float), ("fallback_offset", ctypes.c_float)]


def densify_cfg(grow=2500, prune_frac=0.005, alpha=0.5, eps=1e-6, r_scale=0.85, log_tau_shift=0.6931471805599453,
                offset_scale=0.5, fallback_offset=0.5) -> DensifyCfg:
    return DensifyCfg(grow, prune_frac, alpha, eps, r_scale, log_tau_shift, offset_scale, fallback_offset)


def split_score(m, E, alpha=0.5, eps=1e-6) -> float:
    return float(lib().orc_split_score(m, E, alpha, eps))


def densify_prune(H: int, W: int, params, m, v, stats, target, cfg: DensifyCfg):
    """One densify/prune event on float32 state (copies).  Returns
    (params, m, v, n_split, n_pruned)."""
    P_ = np.array(params, dtype=np.float32, order="C", copy=True)
    M = np.array(m, dtype=np.float32, order="C", copy=True)
    V = np.array(v, dtype=np.float32, order="C", copy=True)
    S = np.ascontiguousarray(stats, dtype=np.float32)
    T = _f32(target).reshape(3, H * W)
    npr = ctypes.c_int(0)
    ns = lib().orc_densify_prune(H, W, P_.shape[1], _p(P_), _p(M), _p(V), _p(S), _p(T), ctypes.byref(cfg),
                                 ctypes.byref(npr))
    return P_, M, V, int(ns), int(npr.value)


def fit(H: int, W: int, params, target, N_cap: int, iterations: int, events, grow: int, prune_frac: float,
        lr: dict, G: int, seed: int, on_event=None, update_every: int = 1, passes_per_update: int = 1):
    """The oracle's fitting schedule, step for step the device driver's: a
    refresh, then iterations of (propagate k=1, loss + backward, Adam in
    double stored as float32, records); an event iteration also accumulates
    the statistics, densifies/prunes and refreshes.  With update_every = U
    the lists are propagated only on iterations 1, 1 + U, 1 + 2U, ... and on
    event iterations; the others reuse the cached lists (summary B.3).  An
    update outside an event runs passes_per_update jump-1 passes.
    Returns (params float32 (9, N_cap), last loss, number of propagation
    passes run)."""
    prm = np.zeros((9, N_cap), dtype=np.float32)
    n0 = params.shape[1]
    prm[:, :n0] = params
    prm[0, n0:] = -1.0
    m = np.zeros((9, N_cap), dtype=np.float32)
    v = np.zeros((9, N_cap), dtype=np.float32)
    tab, npass = refresh(H, W, prm, G, seed, 0)
    rec = records(H, W, prm)
    dcfg = densify_cfg(grow=grow, prune_frac=prune_frac)
    events = set(events)
    step = 0
    L = None
    for it in range(1, iterations + 1):
        if it in events or (it - 1) % update_every == 0:
            for _ in range(1 if it in events else passes_per_update):
                tab = propagate(H, W, rec, tab, 1, G, seed, npass)
                npass += 1
        if it in events:
            L, g, st = loss_backward_stats(H, W, prm, tab, target)
        else:
            L, g = loss_backward(H, W, prm, tab, target)
        step += 1
        P64, M64, V64 = adam(H, W, prm, m, v, g, lr, step, float(np.float32(0.9)), float(np.float32(0.999)),
                             float(np.float32(1e-8)))
        prm, m, v = P64.astype(np.float32), M64.astype(np.float32), V64.astype(np.float32)
        if it in events:
            prm, m, v, _, _ = densify_prune(H, W, prm, m, v, st.astype(np.float32), target, dcfg)
            tab, n = refresh(H, W, prm, G, seed, npass)
            npass += n
            if on_event is not None:
                on_event(it, prm)
        rec = records(H, W, prm)
    return prm, L, npass


def tau_diffuse(H: int, W: int, params, table, grads, lam: float):
    """One Jacobi tau-diffusion step; returns new grads (9, N) float64."""
    params = _f32(params)
    tab = _u32(table).reshape(H * W, K)
    G = np.array(grads, dtype=np.float64, order="C", copy=True)
    lib().orc_tau_diffuse(H, W, params.shape[1], _p(params), _p(tab), _p(G), float(lam))
    return G


def jfa3x3(H: int, W: int, rec32, table, jump: int, cell: int = 1):
    """One 3x3 flood pass keeping the 4 best ids in slots 0-3."""
    rec32 = _f32(rec32)
    GH, GW = grid_dims(H, W, cell)
    tin = _u32(table).reshape(GH * GW, K)
    tout = np.empty_like(tin)
    lib().orc_jfa3x3_cell(GH, GW, cell, rec32.shape[0], _p(rec32), _p(tin), _p(tout), int(jump))
    return tout


def flood_schedule(H: int, W: int) -> list:
    """ceil(log2 max(W, H)) jumps: 2^(n-1), ..., 1."""
    n = max(1, math.ceil(math.log2(max(H, W))))
    return [1 << (n - 1 - q) for q in range(n)]


def jfa_prepass(H: int, W: int, params, cell: int = 1):
    """Seed pass, then one 3x3 flood pass per jump of flood_schedule of the
    candidate grid."""
    rec = records(H, W, params)
    t = seed_table(H, W, params, cell)
    for k in flood_schedule(*grid_dims(H, W, cell)):
        t = jfa3x3(H, W, rec, t, k, cell)
    return t


PACK_FIELDS = {"x": (0, 18), "y": (18, 18), "cr": (36, 10), "cg": (46, 10), "cb": (56, 10), "ln_tau": (66, 16),
               "r": (82, 14), "theta": (96, 14), "a": (110, 14), "active": (127, 1)}


def pack_ranges(params) -> np.ndarray:
    """Per-image (lo, hi) of ln tau, r and a over the active sites, as
    float32 (lo_lt, lo_r, lo_a, hi_lt, hi_r, hi_a)."""
    params = _f32(params)
    out = np.empty(6, dtype=np.float32)
    lib().orc_pack_ranges(params.shape[1], _p(params), _p(out))
    return out


def pack_sites(H: int, W: int, params, lohi=None):
    """16-byte evaluation records (N, 4) uint32 and the ranges they use."""
    params = _f32(params)
    lohi = pack_ranges(params) if lohi is None else np.ascontiguousarray(lohi, dtype=np.float32)
    out = np.empty((params.shape[1], 4), dtype=np.uint32)
    lib().orc_pack_sites(H, W, params.shape[1], _p(params), _p(lohi), _p(out))
    return out, lohi


def unpack_sites(H: int, W: int, packed, lohi) -> np.ndarray:
    """Decode 16-byte records to float32 parameters (9, N)."""
    packed = _u32(packed).reshape(-1, 4)
    lohi = np.ascontiguousarray(lohi, dtype=np.float32)
    out = np.empty((9, packed.shape[0]), dtype=np.float32)
    lib().orc_unpack_sites(H, W, packed.shape[0], _p(packed), _p(lohi), _p(out))
    return out
