"""Randomized parity sweep of the tile kernel's forms against the oracle.

Each case draws an image size (1..90 x 1..120), a site count (dense and
sparse, so that both tile heights and the generic path for crowded tiles
occur), an injection count, inactive sites, and a table that is either the
exact top-8 or random ids with empty slots.  On the same inputs the fused
pass must give the oracle's propagated table bit for bit and its gradients;
propagation passes at jumps 1 and 2 must give the oracle's tables bit for
bit; the order-independent backward must agree with the oracle's gradients
and be bit-identical on a second call."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

GRAD_RTOL, GRAD_ATOL = 1e-4, 1e-6
LOSS_RTOL = 1e-5
SENT = 0xFFFFFFFF
CASES = 12


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _draw(k):
    rng = np.random.default_rng(7000 + k)
    H = int(rng.integers(1, 91))
    W = int(rng.integers(1, 121))
    if k % 4 == 3:  # thin images: one partial row of tiles, halos cut on every side
        H = int(rng.integers(1, 6))
        W = int(rng.integers(1, 50))
    P = H * W
    dense = bool(rng.integers(0, 2))
    N = int(rng.integers(max(1, P // 3), 3 * P + 2)) if dense else int(rng.integers(1, max(2, P // 6)))
    N = max(1, min(N, 5000))
    G = int(rng.integers(0, 9))
    exact = bool(rng.integers(0, 2))
    return rng, H, W, N, G, exact


def _inputs(k):
    rng, H, W, N, G, exact = _draw(k)
    prm = synth.uniform_sites(H, W, N, 100 + k)
    if N > 3:
        prm[0, rng.choice(N, size=max(1, N // 10), replace=False)] = -1.0  # inactive sites
    tgt = synth.make_image(H, W, 6, 0, 100 + k)
    if exact:
        table = oracle.topk_exact(H, W, oracle.records(H, W, prm))
    else:
        table = rng.integers(0, N, size=(H * W, 8)).astype(np.uint32)
        table[rng.random((H * W, 8)) < 0.3] = SENT
    return H, W, N, G, prm, tgt, table


def _ctx(H, W, N, prm, tgt, seed):
    from soft_voronoi_render_b200 import Sad
    s = Sad(H, W, N, seed=seed)
    s.set_sites(prm)
    s.set_target(tgt)
    return s


def _close(g, ref):
    return np.all(np.abs(g.astype(np.float64) - ref) <= np.maximum(GRAD_RTOL * np.abs(ref), GRAD_ATOL))


@pytest.mark.parametrize("k", range(CASES))
def test_fuzz_fit_pass_and_propagation(torch_cuda, k):
    H, W, N, G, prm, tgt, table = _inputs(k)
    rec = oracle.records(H, W, prm)
    s = _ctx(H, W, N, prm, tgt, 31 + k)
    s.set_table(table)
    s.fit_pass(G)
    t1 = oracle.propagate(H, W, rec, table, 1, G, seed=31 + k, pass_index=0)
    np.testing.assert_array_equal(s.get_table(), t1, err_msg=f"fit pass {H}x{W} N={N} G={G}")
    L, g = oracle.loss_backward(H, W, prm, t1, tgt)
    assert abs(s.loss() - L) <= LOSS_RTOL * max(L, 1e-30)
    assert _close(s.grads.cpu().numpy(), g), (H, W, N, G)
    for n, jump in enumerate((2, 1)):
        s.propagate(jump, G)
        t1 = oracle.propagate(H, W, rec, t1, jump, G, seed=31 + k, pass_index=n + 1)
        np.testing.assert_array_equal(s.get_table(), t1, err_msg=f"jump {jump} {H}x{W} N={N} G={G}")


@pytest.mark.parametrize("k", range(CASES))
def test_fuzz_deterministic_backward(torch_cuda, k):
    from soft_voronoi_render_b200 import SAD_DETERMINISTIC
    H, W, N, G, prm, tgt, table = _inputs(k)
    s = _ctx(H, W, N, prm, tgt, 51 + k)
    s.set_table(table)
    runs = []
    for _ in range(2):
        s.grads.zero_()
        s.backward(SAD_DETERMINISTIC)
        runs.append(s.grads.cpu().numpy().copy())
    assert np.array_equal(runs[0].view(np.uint32), runs[1].view(np.uint32))
    clean = table.copy()
    clean[clean >= N] = SENT
    L, g = oracle.loss_backward(H, W, prm, clean, tgt)
    assert abs(s.loss() - L) <= LOSS_RTOL * max(L, 1e-30)
    assert _close(runs[0], g), (H, W, N)
