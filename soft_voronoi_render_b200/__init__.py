"""B200 (sm_100a) library for one Soft Anisotropic Diagrams fitting iteration.

The computation lives in ``libsad.so`` (CUDA kernels behind the C ABI of
``include/sad.h``).  ``_lib`` exposes every C entry point under its C name;
``Sad`` below owns the device buffers as PyTorch tensors (PyTorch is used for
memory and streams only) and forwards each call to the library.
"""
from __future__ import annotations

import numpy as np

from . import _lib
from ._lib import (SAD_DETERMINISTIC, SAD_STAGING_LOADS, SAD_STAGING_TMA, SAD_STATS, SadError,  # noqa: F401
                   adam_cfg, densify_cfg)

__all__ = ["Sad", "SadError", "adam_cfg", "densify_cfg", "SAD_STATS", "SAD_DETERMINISTIC", "SAD_STAGING_LOADS",
           "SAD_STAGING_TMA", "load"]


def load():
    """Load (building if needed) the CUDA library; raises if unavailable."""
    return _lib.load()


class Sad:
    """A context plus its caller-owned device buffers.

    Buffers (torch tensors on ``device``): params/grads/adam_m/adam_v
    (9, N) float32, records (N, 16) float32, table (2, 2, P, 4) int32 view of
    uint32 ids, target/image (3, H, W) float32, site_stats (6, N) float32,
    frozen (N,) uint8 (non-zero: Adam leaves the site alone), workspace bytes.
    """

    def __init__(self, H: int, W: int, N_cap: int, device="cuda", with_image: bool = True, seed: int = 1,
                 with_stats: bool = True):
        import torch

        if not torch.cuda.is_available():
            raise SadError(_lib.SAD_ERR_CUDA, "no CUDA device is available")
        self.torch = torch
        self.H, self.W, self.N = int(H), int(W), int(N_cap)
        self.P = self.H * self.W
        self.cell, self.PT = 1, self.P  # candidate grid (set_candidate_grid)
        self.device = torch.device(device)
        _lib.load()
        f32 = dict(dtype=torch.float32, device=self.device)
        self.params = torch.zeros((9, self.N), **f32)
        self.grads = torch.zeros((9, self.N), **f32)
        self.adam_m = torch.zeros((9, self.N), **f32)
        self.adam_v = torch.zeros((9, self.N), **f32)
        self.records = torch.zeros((self.N, 16), **f32)
        self.table = torch.full((2, 2, self.P, 4), -1, dtype=torch.int32, device=self.device)
        self.target = torch.zeros((3, self.H, self.W), **f32)
        self.image = torch.zeros((3, self.H, self.W), **f32) if with_image else None
        self.site_stats = torch.zeros((6, self.N), **f32) if with_stats else None
        self.frozen = torch.zeros((self.N,), dtype=torch.uint8, device=self.device)
        self.cand16 = torch.zeros((self.N, 4), dtype=torch.int32, device=self.device)
        self.ws_bytes = _lib.sad_workspace_bytes(self.H, self.W, self.N)
        self.workspace = torch.zeros(((self.ws_bytes + 255) // 256 * 256,), dtype=torch.uint8, device=self.device)
        self.ctx = _lib.sad_create(self.H, self.W, self.N, _lib.SAD_K)
        _lib.sad_bind(self.ctx, params=self.params, grads=self.grads, adam_m=self.adam_m, adam_v=self.adam_v,
                      records=self.records, table=self.table, target=self.target, image=self.image,
                      workspace=self.workspace, workspace_bytes=self.workspace.numel(), stats=self.site_stats,
                      frozen=self.frozen, cand16=self.cand16)
        _lib.sad_reset(self.ctx, seed, self.stream)

    # the stream every call is issued on: torch's current stream
    @property
    def stream(self):
        return self.torch.cuda.current_stream(self.device)

    def close(self):
        if getattr(self, "ctx", None):
            _lib.sad_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---- data in / out ------------------------------------------------------
    def _dev(self, x, dtype):
        t = self.torch
        if isinstance(x, np.ndarray):
            x = t.from_numpy(np.ascontiguousarray(x))
        return x.to(device=self.device, dtype=dtype).contiguous()

    def set_sites(self, params):
        src = self._dev(params, self.torch.float32)
        _lib.sad_set_sites(self.ctx, src, src.shape[1], self.stream)
        self._keep = src  # the copy is asynchronous: keep the source alive

    def get_sites(self, n=None):
        n = self.N if n is None else n
        out = np.empty((9, n), dtype=np.float32)
        _lib.sad_get_sites(self.ctx, out, n, self.stream)
        return out

    def set_target(self, target):
        src = self._dev(target, self.torch.float32)
        _lib.sad_set_target(self.ctx, src, self.stream)
        self._keep_t = src

    def set_target_u8(self, rgb):
        """Target from an 8-bit RGB image (H, W, 3), converted on the device."""
        src = self._dev(rgb, self.torch.uint8)
        _lib.sad_set_target_u8(self.ctx, src, self.stream)
        self._keep_t = src

    def bind_target(self, target):
        """Point the context at another device target tensor (3, H, W) float32
        without copying; the caller keeps it alive while kernels read it."""
        _lib.sad_bind_target(self.ctx, target)

    def reset(self, seed: int = 1):
        _lib.sad_reset(self.ctx, seed, self.stream)

    def pack_sites(self):
        """16-byte evaluation records: (packed (N, 4) int32 device tensor,
        range (6,) float32 numpy array)."""
        t = self.torch
        packed = t.empty((self.N, 4), dtype=t.int32, device=self.device)
        rng = t.empty(6, dtype=t.float32, device=self.device)
        _lib.sad_pack_sites(self.ctx, packed, rng, self.stream)
        return packed, rng.cpu().numpy()

    def unpack_sites(self, packed, rng):
        t = self.torch
        src = self._dev(np.asarray(packed).view(np.int32) if isinstance(packed, np.ndarray) else packed, t.int32)
        r = self._dev(np.asarray(rng, dtype=np.float32), t.float32)
        _lib.sad_unpack_sites(self.ctx, src, r, self.stream)
        self.torch.cuda.current_stream(self.device).synchronize()

    def set_candidate_precision(self, bits: int):
        """32: candidates ranked by the float32 logit; 16: ranked on the
        packed candidate-site records (binary16 coefficients), the kept 8
        re-scored in float32."""
        _lib.sad_set_candidate_precision(self.ctx, bits, self.stream)

    def set_list_staging(self, mode: int):
        """SAD_STAGING_LOADS (default) or SAD_STAGING_TMA: how the fit pass
        brings each tile's lists on chip (see sad_set_list_staging)."""
        _lib.sad_set_list_staging(self.ctx, mode, self.stream)

    def set_candidate_grid(self, cell: int):
        """Lists on a ceil(H/cell) x ceil(W/cell) grid; the table starts empty."""
        _lib.sad_set_candidate_grid(self.ctx, cell, self.stream)
        self.cell = cell
        self.PT = ((self.H + cell - 1) // cell) * ((self.W + cell - 1) // cell)

    def get_table(self) -> np.ndarray:
        out = np.empty((self.PT, 8), dtype=np.uint32)
        _lib.sad_get_table(self.ctx, out, self.stream)
        return out

    def set_table(self, table: np.ndarray):
        src = np.ascontiguousarray(table, dtype=np.uint32).reshape(self.PT, 8)
        _lib.sad_set_table(self.ctx, src, self.stream)

    def checkpoint(self) -> dict:
        """Everything a fit needs to resume: site parameters, Adam moments,
        the current candidate lists and the fit state (pass counter, Adam
        step, injection seed), as host arrays."""
        t = self.torch
        t.cuda.current_stream(self.device).synchronize()
        return {"params": self.params.cpu().numpy().copy(), "adam_m": self.adam_m.cpu().numpy().copy(),
                "adam_v": self.adam_v.cpu().numpy().copy(), "table": self.get_table(),
                "state": _lib.sad_get_fit_state(self.ctx, self.stream)}

    def restore(self, ck: dict):
        """Resume from a checkpoint() of a context of the same sizes; the
        score records are rebuilt from the parameters."""
        t = self.torch
        for name in ("params", "adam_m", "adam_v"):
            getattr(self, name).copy_(t.from_numpy(np.ascontiguousarray(ck[name])).to(self.device))
        st = ck["state"]
        _lib.sad_set_fit_state(self.ctx, st["pass_counter"], st["adam_step"], st["seed"], self.stream)
        self.set_table(ck["table"])
        self.grads.zero_()
        self.prep_records()

    def stats(self) -> dict:
        return _lib.sad_get_stats(self.ctx, self.stream)

    def loss(self) -> float:
        return _lib.sad_get_loss(self.ctx, self.stream)

    # ---- the hot path ---------------------------------------------------------
    def prep_records(self):
        _lib.sad_prep_records(self.ctx, self.stream)

    def topk_exact(self, pixels=None):
        t = self.torch
        if pixels is None:
            out = t.empty((self.PT, 8), dtype=t.int32, device=self.device)
            _lib.sad_topk_exact(self.ctx, None, self.PT, out, self.stream)
        else:
            pix = self._dev(pixels, t.int64)
            out = t.empty((pix.numel(), 8), dtype=t.int32, device=self.device)
            _lib.sad_topk_exact(self.ctx, pix, pix.numel(), out, self.stream)
        return out

    def refresh(self, G: int):
        _lib.sad_refresh(self.ctx, G, self.stream)

    def jfa_prepass(self):
        _lib.sad_jfa_prepass(self.ctx, self.stream)

    def fit_pass_cached(self):
        _lib.sad_fit_pass_cached(self.ctx, self.stream)

    def propagate(self, jump: int, G: int):
        _lib.sad_propagate(self.ctx, jump, G, self.stream)

    def render(self, image=None):
        _lib.sad_render(self.ctx, image, self.stream)
        return image if image is not None else self.image

    def backward(self, flags: int = 0):
        _lib.sad_backward(self.ctx, flags, self.stream)

    def densify_prune(self, cfg):
        _lib.sad_densify_prune(self.ctx, cfg, self.stream)

    def tau_diffuse(self, lam: float):
        _lib.sad_tau_diffuse(self.ctx, lam, self.stream)

    def adam_step(self, cfg):
        _lib.sad_adam_step(self.ctx, cfg, self.stream)

    def fit_pass(self, G: int):
        _lib.sad_fit_pass(self.ctx, G, self.stream)

    def fit_iteration(self, G: int, cfg):
        _lib.sad_fit_iteration(self.ctx, G, cfg, self.stream)
