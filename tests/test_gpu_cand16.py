"""Packed candidate-site records through the C ABI against the oracle
("Soft Anisotropic Diagrams for Differentiable Image Representation",
paperlayer summary B.2: candidate-update kernels score from a 16-byte
buffer of float16 pairs).

With sad_set_candidate_precision(16) every candidate update ranks on x, y
(float32) and (A, B), (C, b) rounded to binary16, then orders the kept 8 by
the float32 logit.  Tolerances as for the float32 mode: the records and the
lists bit-exact, render 1e-5, gradients 1e-4 relative with a 1e-6 floor."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

SENT = 0xFFFFFFFF


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _ctx(H, W, N, prm, tgt=None, seed=1, cell=1):
    from soft_voronoi_render_b200 import Sad
    s = Sad(H, W, N, seed=seed)
    s.set_sites(prm)
    if tgt is not None:
        s.set_target(tgt)
    if cell != 1:
        s.set_candidate_grid(cell)
    s.set_candidate_precision(16)
    return s


def test_packed_records_bitwise(torch_cuda):
    tgt, prm, w = synth.make_workload("c1", seed=3)
    prm = prm.copy()
    prm[0, 4] = -1.0
    s = _ctx(w.H, w.W, w.N, prm, seed=2)
    s.propagate(1, 0)  # packs the records first
    got = s.cand16.cpu().numpy().view(np.uint32)
    rec = oracle.records(w.H, w.W, prm)
    assert np.array_equal(got[:, :2], rec[:, :2].view(np.uint32))
    halves = got[:, 2:].copy().view(np.float16).reshape(-1, 4)
    sel = oracle.cand16_record(rec)
    assert np.array_equal(halves.astype(np.float32).view(np.uint32), sel[:, 2:6].view(np.uint32))


@pytest.mark.parametrize("H,W,N,jump,G", [(256, 256, 1024, 1, 2), (256, 256, 1024, 8, 3), (37, 53, 300, 2, 1)])
def test_propagate_cand16_bit_exact(torch_cuda, H, W, N, jump, G):
    prm = synth.uniform_sites(H, W, N, 40 + jump)
    prm[0, ::9] = -1.0
    s = _ctx(H, W, N, prm, seed=12)
    t0 = oracle.topk_exact(H, W, oracle.records(H, W, prm))
    t0[::5, 3:] = SENT
    s.set_table(t0)
    s.propagate(jump, G)
    ref = oracle.propagate(H, W, oracle.records(H, W, prm), t0, jump, G, seed=12, pass_index=0, cand16=True)
    np.testing.assert_array_equal(s.get_table(), ref)


@pytest.mark.parametrize("cell", [1, 2])
def test_refresh_cand16_c2_bit_exact(torch_cuda, cell):
    tgt, prm, w = synth.make_workload("c2", seed=1)
    s = _ctx(w.H, w.W, w.N, prm, seed=31, cell=cell)
    s.refresh(w.G)
    ref, npass = oracle.refresh(w.H, w.W, prm, w.G, seed=31, cell=cell, cand16=True)
    np.testing.assert_array_equal(s.get_table(), ref)


def test_fit_pass_cand16(torch_cuda):
    """The fitting pass with packed candidates: the propagation pass ranked
    on the packed records, then render + backward on the new lists."""
    tgt, prm, w = synth.make_workload("c1", seed=4)
    s = _ctx(w.H, w.W, w.N, prm, tgt, seed=8)
    t0, n = oracle.refresh(w.H, w.W, prm, 2, seed=8, cand16=True)
    s.set_table(t0)
    s.fit_pass(2)
    ref = oracle.propagate(w.H, w.W, oracle.records(w.H, w.W, prm), t0, 1, 2, seed=8, pass_index=0, cand16=True)
    np.testing.assert_array_equal(s.get_table(), ref)
    L, g = oracle.loss_backward(w.H, w.W, prm, ref, tgt)
    assert abs(s.loss() - L) <= 1e-5 * L
    gg = s.grads.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(gg - g) <= np.maximum(1e-4 * np.abs(g), 1e-6))


def test_recall_after_convergence_cand16_c2(torch_cuda):
    """Lists ranked on the packed records still reach recall@8 >= 0.99
    against the exact float32 top-K after convergence on the 768 x 512
    workload (params frozen; k = 1 passes until no slot changes, cap 64)."""
    tgt, prm, w = synth.make_workload("c2", seed=2)
    s = _ctx(w.H, w.W, w.N, prm, seed=5)
    s.refresh(w.G)
    prev = s.get_table()
    for _ in range(64):
        s.propagate(1, w.G)
        cur = s.get_table()
        if np.array_equal(cur, prev):
            break
        prev = cur
    pix = synth.Stream(2, "recall").integers(8192, w.H * w.W)
    ex = oracle.topk_exact(w.H, w.W, oracle.records(w.H, w.W, prm), pix)
    got = prev[pix]
    hit = [len(set(a.tolist()) & set(b.tolist()) - {SENT}) / max(1, int((b != SENT).sum()))
           for a, b in zip(got, ex)]
    assert np.mean(hit) >= 0.99, np.mean(hit)
