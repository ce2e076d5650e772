"""Checkpoint and resume of a fit through the C ABI.

A checkpoint is the site parameters, the Adam moments, the current candidate
lists and the fit state (pass counter, Adam step, injection seed).  A fit
resumed from one in a fresh context must continue exactly as the original:
with the order-independent (fixed-point) backward every step is
deterministic, so the two continuations agree bit for bit."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _steps(s, n, G, cfg):
    from soft_voronoi_render_b200 import SAD_DETERMINISTIC
    for _ in range(n):
        s.propagate(1, G)
        s.backward(SAD_DETERMINISTIC)
        s.adam_step(cfg)


def test_resume_from_checkpoint_is_bit_exact(torch_cuda):
    from soft_voronoi_render_b200 import Sad, adam_cfg
    tgt, prm, w = synth.make_workload("c1", seed=5)
    cfg = adam_cfg(lr_color=5e-3)
    a = Sad(w.H, w.W, w.N, seed=9)
    a.set_sites(prm)
    a.set_target(tgt)
    a.refresh(2)
    _steps(a, 4, 2, cfg)
    ck = a.checkpoint()
    assert ck["state"]["adam_step"] == 4 and ck["state"]["seed"] == 9
    _steps(a, 3, 2, cfg)
    want = a.checkpoint()

    b = Sad(w.H, w.W, w.N, seed=1)  # a different seed: the state overrides it
    b.set_target(tgt)
    b.restore(ck)
    assert b.checkpoint()["state"] == ck["state"]
    _steps(b, 3, 2, cfg)
    got = b.checkpoint()
    assert got["state"] == want["state"]
    for k in ("params", "adam_m", "adam_v", "table"):
        assert np.array_equal(got[k].view(np.uint32), want[k].view(np.uint32)), k
    assert b.loss() == a.loss()
    # and the resumed context keeps fitting
    assert not np.array_equal(want["params"], ck["params"])


def test_set_fit_state_checks_its_argument(torch_cuda):
    from soft_voronoi_render_b200 import Sad, _lib
    s = Sad(8, 8, 4)
    with pytest.raises(_lib.SadError) as e:
        _lib.sad_set_fit_state(s.ctx, 1, 2, 3, s.stream, reserved=1)
    assert e.value.status == _lib.SAD_ERR_INVALID_ARG
    _lib.sad_set_fit_state(s.ctx, 7, 5, 11, s.stream)
    assert _lib.sad_get_fit_state(s.ctx, s.stream) == {"pass_counter": 7, "adam_step": 5, "seed": 11}
    st = s.stats()
    assert st["pass_counter"] == 7 and st["adam_step"] == 5
