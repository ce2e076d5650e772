"""ctypes binding of libsad (include/sad.h): same names, marshalling only.

Every function here converts Python arguments (torch tensors, numpy arrays,
ints, stream handles) into the plain pointers and sizes of the C ABI and
raises ``SadError`` on a non-zero status.  No step of the computation runs in
Python: a missing or unloadable library is an error, never a fallback.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

SAD_OK = 0
SAD_ERR_INVALID_ARG = 1
SAD_ERR_UNSUPPORTED = 2
SAD_ERR_CUDA = 3
SAD_ERR_CAPACITY = 4
SAD_ERR_NOT_BOUND = 5
SAD_K = 8
SAD_MAX_INJECT = 64
SAD_EMPTY = 0xFFFFFFFF

_STATUS = {0: "SAD_OK", 1: "SAD_ERR_INVALID_ARG", 2: "SAD_ERR_UNSUPPORTED", 3: "SAD_ERR_CUDA",
           4: "SAD_ERR_CAPACITY", 5: "SAD_ERR_NOT_BOUND"}


class SadError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


class sad_buffers(ctypes.Structure):
    _fields_ = [("params", ctypes.c_void_p), ("grads", ctypes.c_void_p), ("adam_m", ctypes.c_void_p),
                ("adam_v", ctypes.c_void_p), ("records", ctypes.c_void_p), ("table", ctypes.c_void_p),
                ("target", ctypes.c_void_p), ("image", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("stats", ctypes.c_void_p), ("frozen", ctypes.c_void_p),
                ("cand16", ctypes.c_void_p)]


class sad_densify_cfg(ctypes.Structure):
    _fields_ = [("grow", ctypes.c_int), ("prune_frac", ctypes.c_float), ("alpha", ctypes.c_float),
                ("eps", ctypes.c_float), ("r_scale", ctypes.c_float), ("log_tau_shift", ctypes.c_float),
                ("offset_scale", ctypes.c_float), ("fallback_offset", ctypes.c_float)]


SAD_STATS = 1
SAD_DETERMINISTIC = 2
SAD_STAGING_LOADS = 0
SAD_STAGING_TMA = 1


def densify_cfg(grow=2500, prune_frac=0.005, alpha=0.5, eps=1e-6, r_scale=0.85, log_tau_shift=0.6931471805599453,
                offset_scale=0.5, fallback_offset=0.5) -> sad_densify_cfg:
    return sad_densify_cfg(grow, prune_frac, alpha, eps, r_scale, log_tau_shift, offset_scale, fallback_offset)


class sad_adam_cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_float) for n in
                ("lr_pos", "lr_log_tau", "lr_r", "lr_color", "lr_theta", "lr_a", "beta1", "beta2", "eps")]


class sad_stats(ctypes.Structure):
    _fields_ = [("hash_overflow", ctypes.c_uint64), ("nonfinite_pixels", ctypes.c_uint64),
                ("empty_pixels", ctypes.c_uint64), ("dropped_ids", ctypes.c_uint64),
                ("pass_counter", ctypes.c_uint32), ("adam_step", ctypes.c_uint32),
                ("current_table", ctypes.c_uint32), ("staging_fallbacks", ctypes.c_uint32), ("loss", ctypes.c_double),
                ("n_active", ctypes.c_uint32), ("n_split", ctypes.c_uint32), ("n_pruned", ctypes.c_uint32),
                ("check_failures", ctypes.c_uint32)]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_ if not n.startswith("reserved")}


class sad_fit_state(ctypes.Structure):
    _fields_ = [("pass_counter", ctypes.c_uint32), ("adam_step", ctypes.c_uint32), ("seed", ctypes.c_uint32),
                ("reserved", ctypes.c_uint32)]


EXPORTED = (
    "sad_workspace_bytes", "sad_create", "sad_destroy", "sad_bind", "sad_reset", "sad_set_sites",
    "sad_get_sites", "sad_set_target", "sad_prep_records", "sad_topk_exact", "sad_refresh", "sad_jfa_prepass",
    "sad_propagate", "sad_fit_pass_cached", "sad_set_candidate_grid", "sad_pack_sites", "sad_unpack_sites", "sad_bind_target", "sad_set_target_u8",
    "sad_render", "sad_backward", "sad_densify_prune", "sad_tau_diffuse", "sad_adam_step", "sad_fit_pass", "sad_fit_iteration", "sad_get_table", "sad_set_table",
    "sad_get_stats", "sad_get_loss", "sad_copy_loss", "sad_last_error", "sad_backward_noalloc",
    "sad_get_fit_state", "sad_set_fit_state", "sad_set_candidate_precision", "sad_set_list_staging",
)

_lib = None


def library_path() -> str:
    """libsad.so, or with SAD_CHECKS=1 in the environment the debug build
    libsad_checks.so (device-side bounds checks counted in sad_stats)."""
    return _build.LIB_CHECKS if os.environ.get("SAD_CHECKS") == "1" else _build.LIB


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load the library from the package's build folder (building it first
    if it is absent and nvcc is available).  Raises if it cannot be loaded."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if build_if_missing:
        _build.build()
    if not os.path.exists(path):
        raise ImportError(f"libsad is not built: {path} is missing")
    L = ctypes.CDLL(path)
    vp, ci, cu32, ci64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint32, ctypes.c_int64
    sig = {
        "sad_workspace_bytes": [ci, ci, ci, ctypes.POINTER(ctypes.c_size_t)],
        "sad_create": [ci, ci, ci, ci, ctypes.POINTER(vp)],
        "sad_destroy": [vp],
        "sad_bind": [vp, ctypes.POINTER(sad_buffers)],
        "sad_reset": [vp, cu32, vp],
        "sad_set_sites": [vp, vp, ci, vp],
        "sad_get_sites": [vp, vp, ci, vp],
        "sad_set_target": [vp, vp, vp],
        "sad_prep_records": [vp, vp],
        "sad_topk_exact": [vp, vp, ci64, vp, vp],
        "sad_refresh": [vp, ci, vp],
        "sad_propagate": [vp, ci, ci, vp],
        "sad_jfa_prepass": [vp, vp],
        "sad_fit_pass_cached": [vp, vp],
        "sad_set_candidate_grid": [vp, ci, vp],
        "sad_pack_sites": [vp, vp, vp, vp],
        "sad_bind_target": [vp, vp],
        "sad_set_target_u8": [vp, vp, vp],
        "sad_unpack_sites": [vp, vp, vp, vp],
        "sad_render": [vp, vp, vp],
        "sad_backward": [vp, cu32, vp],
        "sad_adam_step": [vp, ctypes.POINTER(sad_adam_cfg), vp],
        "sad_densify_prune": [vp, ctypes.POINTER(sad_densify_cfg), vp],
        "sad_tau_diffuse": [vp, ctypes.c_float, vp],
        "sad_fit_pass": [vp, ci, vp],
        "sad_fit_iteration": [vp, ci, ctypes.POINTER(sad_adam_cfg), vp],
        "sad_get_table": [vp, vp, vp],
        "sad_set_table": [vp, vp, vp],
        "sad_get_stats": [vp, ctypes.POINTER(sad_stats), vp],
        "sad_get_loss": [vp, ctypes.POINTER(ctypes.c_double), vp],
        "sad_copy_loss": [vp, vp, vp],
        "sad_last_error": [vp],
        "sad_backward_noalloc": [ci, ci, ci, vp, vp, vp, vp, vp, vp, vp],
        "sad_get_fit_state": [vp, ctypes.POINTER(sad_fit_state), vp],
        "sad_set_fit_state": [vp, ctypes.POINTER(sad_fit_state), vp],
        "sad_set_candidate_precision": [vp, ci, vp],
        "sad_set_list_staging": [vp, ci, vp],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_char_p if name == "sad_last_error" else ci
    _lib = L
    return L


def _ptr(x):
    """Device/host address of a torch tensor, numpy array or int (None -> NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)}")


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(ctx, status: int):
    if status != SAD_OK:
        msg = load().sad_last_error(ctx).decode() if ctx else ""
        raise SadError(status, msg)


# ---- the C ABI, one wrapper per entry point --------------------------------

def sad_workspace_bytes(H: int, W: int, N_cap: int) -> int:
    out = ctypes.c_size_t(0)
    _check(None, load().sad_workspace_bytes(H, W, N_cap, ctypes.byref(out)))
    return out.value


def sad_create(H: int, W: int, N_cap: int, K: int = SAD_K) -> int:
    h = ctypes.c_void_p(0)
    _check(None, load().sad_create(H, W, N_cap, K, ctypes.byref(h)))
    return h.value


def sad_destroy(ctx: int) -> None:
    _check(None, load().sad_destroy(ctx))


def sad_bind(ctx: int, *, params, grads, adam_m, adam_v, records, table, target, workspace,
             workspace_bytes: int, image=None, stats=None, frozen=None, cand16=None) -> None:
    b = sad_buffers(_ptr(params), _ptr(grads), _ptr(adam_m), _ptr(adam_v), _ptr(records), _ptr(table),
                    _ptr(target), _ptr(image), _ptr(workspace), workspace_bytes, _ptr(stats), _ptr(frozen),
                    _ptr(cand16))
    _check(ctx, load().sad_bind(ctx, ctypes.byref(b)))


def sad_reset(ctx: int, seed: int, stream=None) -> None:
    _check(ctx, load().sad_reset(ctx, seed & 0xFFFFFFFF, _stream(stream)))


def sad_set_sites(ctx: int, params_9xn, n: int, stream=None) -> None:
    _check(ctx, load().sad_set_sites(ctx, _ptr(params_9xn), n, _stream(stream)))


def sad_get_sites(ctx: int, dst_9xn, n: int, stream=None) -> None:
    _check(ctx, load().sad_get_sites(ctx, _ptr(dst_9xn), n, _stream(stream)))


def sad_set_target(ctx: int, target_3xp, stream=None) -> None:
    _check(ctx, load().sad_set_target(ctx, _ptr(target_3xp), _stream(stream)))


def sad_prep_records(ctx: int, stream=None) -> None:
    _check(ctx, load().sad_prep_records(ctx, _stream(stream)))


def sad_topk_exact(ctx: int, pixels, n_pix: int, out, stream=None) -> None:
    _check(ctx, load().sad_topk_exact(ctx, _ptr(pixels), n_pix, _ptr(out), _stream(stream)))


def sad_refresh(ctx: int, G: int, stream=None) -> None:
    _check(ctx, load().sad_refresh(ctx, G, _stream(stream)))


def sad_jfa_prepass(ctx: int, stream=None) -> None:
    _check(ctx, load().sad_jfa_prepass(ctx, _stream(stream)))


def sad_set_target_u8(ctx: int, src, stream=None) -> None:
    _check(ctx, load().sad_set_target_u8(ctx, _ptr(src), _stream(stream)))


def sad_bind_target(ctx: int, target) -> None:
    _check(ctx, load().sad_bind_target(ctx, _ptr(target)))


def sad_pack_sites(ctx: int, packed, range_out=None, stream=None) -> None:
    _check(ctx, load().sad_pack_sites(ctx, _ptr(packed), _ptr(range_out) if range_out is not None else None,
                                      _stream(stream)))


def sad_unpack_sites(ctx: int, packed, range_in, stream=None) -> None:
    _check(ctx, load().sad_unpack_sites(ctx, _ptr(packed), _ptr(range_in), _stream(stream)))


def sad_set_candidate_grid(ctx: int, cell: int, stream=None) -> None:
    _check(ctx, load().sad_set_candidate_grid(ctx, cell, _stream(stream)))


def sad_fit_pass_cached(ctx: int, stream=None) -> None:
    _check(ctx, load().sad_fit_pass_cached(ctx, _stream(stream)))


def sad_propagate(ctx: int, jump: int, G: int, stream=None) -> None:
    _check(ctx, load().sad_propagate(ctx, jump, G, _stream(stream)))


def sad_render(ctx: int, image=None, stream=None) -> None:
    _check(ctx, load().sad_render(ctx, _ptr(image), _stream(stream)))


def sad_backward(ctx: int, flags: int = 0, stream=None) -> None:
    _check(ctx, load().sad_backward(ctx, flags, _stream(stream)))


def adam_cfg(lr_pos=1e-3, lr_log_tau=1e-3, lr_r=1e-3, lr_color=1e-3, lr_theta=1e-3, lr_a=1e-3,
             beta1=0.9, beta2=0.999, eps=1e-8) -> sad_adam_cfg:
    return sad_adam_cfg(lr_pos, lr_log_tau, lr_r, lr_color, lr_theta, lr_a, beta1, beta2, eps)


def sad_densify_prune(ctx: int, cfg: sad_densify_cfg, stream=None) -> None:
    _check(ctx, load().sad_densify_prune(ctx, ctypes.byref(cfg), _stream(stream)))


def sad_tau_diffuse(ctx: int, lam: float, stream=None) -> None:
    _check(ctx, load().sad_tau_diffuse(ctx, lam, _stream(stream)))


def sad_adam_step(ctx: int, cfg: sad_adam_cfg, stream=None) -> None:
    _check(ctx, load().sad_adam_step(ctx, ctypes.byref(cfg), _stream(stream)))


def sad_fit_pass(ctx: int, G: int, stream=None) -> None:
    _check(ctx, load().sad_fit_pass(ctx, G, _stream(stream)))


def sad_fit_iteration(ctx: int, G: int, cfg: sad_adam_cfg, stream=None) -> None:
    _check(ctx, load().sad_fit_iteration(ctx, G, ctypes.byref(cfg), _stream(stream)))


def sad_get_table(ctx: int, dst, stream=None) -> None:
    _check(ctx, load().sad_get_table(ctx, _ptr(dst), _stream(stream)))


def sad_set_table(ctx: int, src, stream=None) -> None:
    _check(ctx, load().sad_set_table(ctx, _ptr(src), _stream(stream)))


def sad_get_stats(ctx: int, stream=None) -> dict:
    s = sad_stats()
    _check(ctx, load().sad_get_stats(ctx, ctypes.byref(s), _stream(stream)))
    return s.as_dict()


def sad_set_candidate_precision(ctx: int, bits: int, stream=None) -> None:
    _check(ctx, load().sad_set_candidate_precision(ctx, int(bits), _stream(stream)))


def sad_set_list_staging(ctx: int, mode: int, stream=None) -> None:
    _check(ctx, load().sad_set_list_staging(ctx, int(mode), _stream(stream)))


def sad_get_fit_state(ctx: int, stream=None) -> dict:
    s = sad_fit_state()
    _check(ctx, load().sad_get_fit_state(ctx, ctypes.byref(s), _stream(stream)))
    return {"pass_counter": s.pass_counter, "adam_step": s.adam_step, "seed": s.seed}


def sad_set_fit_state(ctx: int, pass_counter: int, adam_step: int, seed: int, stream=None, reserved: int = 0) -> None:
    s = sad_fit_state(pass_counter, adam_step, seed, reserved)
    _check(ctx, load().sad_set_fit_state(ctx, ctypes.byref(s), _stream(stream)))


def sad_copy_loss(ctx: int, dst, stream=None) -> None:
    _check(ctx, load().sad_copy_loss(ctx, _ptr(dst), _stream(stream)))


def sad_get_loss(ctx: int, stream=None) -> float:
    out = ctypes.c_double(0.0)
    _check(ctx, load().sad_get_loss(ctx, ctypes.byref(out), _stream(stream)))
    return out.value


def sad_last_error(ctx: int) -> str:
    return load().sad_last_error(ctx).decode()


def sad_backward_noalloc(H: int, W: int, N_cap: int, records, table, target, image, grads, loss,
                         stream=None) -> None:
    """Render + loss + backward without a context or workspace, for callers
    that cannot allocate device memory (see include/sad.h)."""
    _check(None, load().sad_backward_noalloc(H, W, N_cap, _ptr(records), _ptr(table), _ptr(target), _ptr(image),
                                             _ptr(grads), _ptr(loss), _stream(stream)))
