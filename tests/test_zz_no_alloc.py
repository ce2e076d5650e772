"""The allocation-free backward entry point gives what sad_backward gives.

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


def test_backward_noalloc_matches_backward_on_two_calls():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from soft_voronoi_render_b200 import Sad, _lib

    tgt, prm, w = synth.make_workload("c1", seed=2)
    s = Sad(w.H, w.W, w.N, seed=3)
    s.set_sites(prm)
    s.set_target(tgt)
    s.set_table(oracle.topk_exact(w.H, w.W, oracle.records(w.H, w.W, prm)))  # table 0 is current
    s.backward()
    g_ref = s.grads.cpu().numpy().astype(np.float64)
    img_ref = s.image.cpu().numpy()
    L_ref = s.loss()

    grads = torch.zeros_like(s.grads)
    image = torch.empty_like(s.image)
    loss = torch.zeros(1, dtype=torch.float64, device=s.device)
    for call in range(2):
        grads.zero_()
        image.fill_(-1.0)
        loss.fill_(-1.0)
        _lib.sad_backward_noalloc(w.H, w.W, w.N, s.records, s.table[0], s.target, image, grads, loss, s.stream)
        torch.cuda.synchronize()
        g = grads.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - g_ref) <= np.maximum(GRAD_RTOL * np.abs(g_ref), GRAD_ATOL)), call
        assert np.abs(image.cpu().numpy() - img_ref).max() <= RENDER_ATOL, call
        assert abs(float(loss.item()) - L_ref) <= LOSS_RTOL * L_ref, call
    with pytest.raises(_lib.SadError) as e:
        _lib.sad_backward_noalloc(8200, 4200, w.N, s.records, s.table[0], s.target, None, grads, loss, s.stream)
    assert e.value.status == _lib.SAD_ERR_CAPACITY
