"""The C-ABI library loads and exports every entry point include/sad.h
declares; host-side argument checks work without a GPU (no compute calls)."""
import ctypes
import os
import re

import pytest

from soft_voronoi_render_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "sad.h")).read()
    return sorted(set(re.findall(r"^\s*(?:int|const char \*)\s*(sad_\w+)\s*\(", txt, flags=re.M)))


def test_header_declares_the_abi():
    names = _declared()
    assert set(names) == set(_lib.EXPORTED), set(names) ^ set(_lib.EXPORTED)


def test_library_exports_every_declared_symbol():
    L = _lib.load()
    for name in _declared():
        assert hasattr(L, name), name
    # the bounds-checked debug build exports the same ABI
    from soft_voronoi_render_b200 import build as _build
    Lc = ctypes.CDLL(_build.LIB_CHECKS)
    for name in _declared():
        assert hasattr(Lc, name), name


def test_create_validates_arguments():
    L = _lib.load()
    h = ctypes.c_void_p(0)
    assert L.sad_create(0, 4, 4, 8, ctypes.byref(h)) == _lib.SAD_ERR_INVALID_ARG
    assert L.sad_create(4, 4, 0, 8, ctypes.byref(h)) == _lib.SAD_ERR_INVALID_ARG
    assert L.sad_create(65536, 65536, 4, 8, ctypes.byref(h)) == _lib.SAD_ERR_INVALID_ARG
    assert L.sad_create(4, 4, 4, 4, ctypes.byref(h)) == _lib.SAD_ERR_UNSUPPORTED
    assert L.sad_create(4, 4, 4, 8, None) == _lib.SAD_ERR_INVALID_ARG
    ctx = _lib.sad_create(16, 24, 100)
    try:
        assert ctx
    finally:
        _lib.sad_destroy(ctx)


def test_workspace_bytes():
    b = _lib.sad_workspace_bytes(2048, 2048, 131072)
    assert b >= 256 + 8 * (2048 // 32) * (2048 // 8)
    with pytest.raises(_lib.SadError):
        _lib.sad_workspace_bytes(0, 1, 1)


def test_bind_checks_alignment_and_sizes_without_touching_memory():
    ctx = _lib.sad_create(8, 8, 16)
    ws = _lib.sad_workspace_bytes(8, 8, 16)
    fake = dict(params=0x10000, grads=0x20000, adam_m=0x30000, adam_v=0x40000, records=0x50000,
                table=0x60000, target=0x70000, workspace=0x80000, workspace_bytes=ws)
    try:
        # calls that need bound buffers fail before binding
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_render(ctx)
        assert e.value.status == _lib.SAD_ERR_NOT_BOUND
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_set_fit_state(ctx, 0, 0, 1)
        assert e.value.status == _lib.SAD_ERR_NOT_BOUND
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_bind(ctx, **{**fake, "records": 0x50004})
        assert e.value.status == _lib.SAD_ERR_INVALID_ARG and "aligned" in str(e.value)
        # records are read in 32-byte loads: 16-byte alignment is not enough
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_bind(ctx, **{**fake, "records": 0x50010})
        assert e.value.status == _lib.SAD_ERR_INVALID_ARG and "32-byte" in str(e.value)
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_bind(ctx, **{**fake, "target": None})
        assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_bind(ctx, **{**fake, "workspace_bytes": ws - 8})
        assert "workspace" in str(e.value)
        _lib.sad_bind(ctx, **fake)  # only checks; no memory is touched
        # argument checks that precede any launch
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_propagate(ctx, 0, 2)
        assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_propagate(ctx, 1, 65)
        assert e.value.status == _lib.SAD_ERR_CAPACITY
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_refresh(ctx, -1)
        assert e.value.status == _lib.SAD_ERR_CAPACITY
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_set_sites(ctx, 0x90000, 17)
        assert e.value.status == _lib.SAD_ERR_CAPACITY
        for flags in (4, _lib.SAD_STATS | _lib.SAD_DETERMINISTIC):
            with pytest.raises(_lib.SadError) as e:
                _lib.sad_backward(ctx, flags)
            assert e.value.status == _lib.SAD_ERR_UNSUPPORTED
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_backward(ctx, _lib.SAD_STATS)  # no stats buffer bound
        assert e.value.status == _lib.SAD_ERR_NOT_BOUND
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_densify_prune(ctx, _lib.densify_cfg())
        assert e.value.status == _lib.SAD_ERR_NOT_BOUND
        _lib.sad_bind(ctx, **fake, stats=0xA0000)
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_densify_prune(ctx, _lib.densify_cfg(prune_frac=1.5))
        assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_bind(ctx, **fake, stats=0xA0004)
        assert "stats" in str(e.value)
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_adam_step(ctx, _lib.adam_cfg(beta1=1.0))
        assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_adam_step(ctx, _lib.adam_cfg(lr_pos=-1.0))
        assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        # rebinding the target, the candidate grid and packed records check
        # their pointers and sizes before any launch
        for bad in (None, 0xB0004):
            with pytest.raises(_lib.SadError) as e:
                _lib.sad_bind_target(ctx, bad)
            assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        _lib.sad_bind_target(ctx, 0xB0000)
        for bad in (0, 65):
            with pytest.raises(_lib.SadError) as e:
                _lib.sad_set_candidate_grid(ctx, bad)
            assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_pack_sites(ctx, 0xC0008)
        assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_unpack_sites(ctx, 0xC0000, None)
        assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        # packed candidates need a bound cand16 buffer; only 32 and 16 bits
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_set_candidate_precision(ctx, 16)
        assert e.value.status == _lib.SAD_ERR_NOT_BOUND
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_set_candidate_precision(ctx, 8)
        assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        _lib.sad_set_candidate_precision(ctx, 32)
        for bad in (-1, 2):
            with pytest.raises(_lib.SadError) as e:
                _lib.sad_set_list_staging(ctx, bad)
            assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        _lib.sad_set_list_staging(ctx, _lib.SAD_STAGING_TMA)
        _lib.sad_set_list_staging(ctx, _lib.SAD_STAGING_LOADS)
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_bind(ctx, **fake, cand16=0xD0008)
        assert "cand16" in str(e.value)
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_set_fit_state(ctx, 1, 1, 1, reserved=3)
        assert e.value.status == _lib.SAD_ERR_INVALID_ARG
        assert _lib.load().sad_get_fit_state(ctx, None, None) == _lib.SAD_ERR_INVALID_ARG
    finally:
        _lib.sad_destroy(ctx)


def test_product_path_has_no_oracle_dependency():
    """The CUDA package never imports the oracle (test infrastructure)."""
    pkg = os.path.join(ROOT, "soft_voronoi_render_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c", ".cpp")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "sad_oracle" not in txt and "orc_" not in txt, f


def test_backward_noalloc_rejects_sizes_before_any_cuda_call():
    """The allocation-free backward checks sizes and pointers on the host and
    returns before touching the GPU: too many tiles for its fixed scratch, or
    more tile rows than a launch allows, give SAD_ERR_CAPACITY."""
    fake = [0x10000, 0x20000, 0x30000, None, 0x40000, 0x50000]  # records, table, target, image, grads, loss
    for H, W, want in ((8200, 4200, _lib.SAD_ERR_CAPACITY),      # 131,200 tiles of 32 x 8
                       (600_000, 1, _lib.SAD_ERR_CAPACITY),      # 75,000 tiles but 75,000 tile rows
                       (0, 8, _lib.SAD_ERR_INVALID_ARG)):
        with pytest.raises(_lib.SadError) as e:
            _lib.sad_backward_noalloc(H, W, 16, *fake)
        assert e.value.status == want, (H, W)
    with pytest.raises(_lib.SadError) as e:
        _lib.sad_backward_noalloc(64, 64, 16, 0x10004, *fake[1:])  # misaligned records
    assert e.value.status == _lib.SAD_ERR_INVALID_ARG
    with pytest.raises(_lib.SadError) as e:
        _lib.sad_backward_noalloc(64, 64, 16, 0x10010, *fake[1:])  # records 16- but not 32-byte aligned
    assert e.value.status == _lib.SAD_ERR_INVALID_ARG
