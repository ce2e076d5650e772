"""The allocation-free backward entry point gives the oracle's loss, image
and gradients, as sad_backward does.

sad_backward_noalloc serves callers that cannot allocate device memory (a
fixed memory budget owned by another framework, a plugin interface that
passes only inputs and outputs).  It keeps its scratch in a library-owned
device array, so this checks two calls in a row: the second must not see
the first call's leftovers.  Collected last so that a stop-at-first-failure
run has already run every other test.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

GRAD_RTOL, GRAD_ATOL = 1e-4, 1e-6   # the per-site gradient tolerance of the parity tests
LOSS_RTOL = 1e-5
RENDER_ATOL = 1e-5


def _close_grads(g, ref):
    return np.all(np.abs(g - ref) <= np.maximum(GRAD_RTOL * np.abs(ref), GRAD_ATOL))


@pytest.mark.parametrize("H,W,N", [(None, None, None), (37, 70, 400)])
def test_backward_noalloc_matches_oracle_on_two_calls(H, W, N):
    """The 256 x 256 workload and a ragged 37 x 70 image (partial tiles on
    both edges): both calls agree with the oracle and with sad_backward."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from soft_voronoi_render_b200 import Sad, _lib

    tgt, prm, w = synth.make_workload("c1", seed=2, H=H, W=W, N=N)
    H, W, N = tgt.shape[1], tgt.shape[2], prm.shape[1]
    table = oracle.topk_exact(H, W, oracle.records(H, W, prm))
    L_orc, g_orc, img_orc = oracle.loss_backward(H, W, prm, table, tgt, want_image=True)
    s = Sad(H, W, N, seed=3)
    s.set_sites(prm)
    s.set_target(tgt)
    s.set_table(table)  # table 0 is current
    s.backward()
    g_ref = s.grads.cpu().numpy().astype(np.float64)
    img_ref = s.image.cpu().numpy()
    L_ref = s.loss()
    assert _close_grads(g_ref, g_orc)
    assert np.abs(img_ref - img_orc).max() <= RENDER_ATOL
    assert abs(L_ref - L_orc) <= LOSS_RTOL * L_orc

    grads = torch.zeros_like(s.grads)
    image = torch.empty_like(s.image)
    loss = torch.zeros(1, dtype=torch.float64, device=s.device)
    for call in range(2):
        grads.zero_()
        image.fill_(-1.0)
        loss.fill_(-1.0)
        _lib.sad_backward_noalloc(H, W, N, s.records, s.table[0], s.target, image, grads, loss, s.stream)
        torch.cuda.synchronize()
        g = grads.cpu().numpy().astype(np.float64)
        assert _close_grads(g, g_orc) and _close_grads(g, g_ref), call
        img = image.cpu().numpy()
        assert np.abs(img - img_orc).max() <= RENDER_ATOL and np.abs(img - img_ref).max() <= RENDER_ATOL, call
        assert abs(float(loss.item()) - L_orc) <= LOSS_RTOL * L_orc, call
        assert abs(float(loss.item()) - L_ref) <= LOSS_RTOL * L_ref, call
    with pytest.raises(_lib.SadError) as e:
        _lib.sad_backward_noalloc(8200, 4200, N, s.records, s.table[0], s.target, None, grads, loss, s.stream)
    assert e.value.status == _lib.SAD_ERR_CAPACITY
