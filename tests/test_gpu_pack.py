"""GPU parity of the 16-byte evaluation record ("Soft Anisotropic Diagrams
for Differentiable Image Representation", summary B.2 "Packed storage for
evaluation"): packed words, ranges and decoded parameters bit-exact against
the oracle; a decode-only render (unpack, refresh, render) against the
oracle's render of the decoded sites on the same lists (1e-5 absolute)."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _ctx(H, W, N, prm, seed=1):
    from soft_voronoi_render_b200 import Sad
    s = Sad(H, W, N, seed=seed)
    s.set_sites(prm)
    return s


@pytest.mark.parametrize("wl", ["c1", "c2"])
def test_pack_bit_exact(torch_cuda, wl):
    tgt, prm, w = synth.make_workload(wl, seed=3)
    prm = prm.copy()
    st = synth.Stream(3, "pack-gpu")
    prm[0, ::13] = -1.0
    prm[4:7, ::7] += 0.3                                     # some colours above 1
    prm[7] = st.uniform(w.N, -9, 9).astype(np.float32)      # any angle
    prm[8, 5] = -0.0
    s = _ctx(w.H, w.W, w.N, prm)
    packed, rng = s.pack_sites()
    ref, ref_rng = oracle.pack_sites(w.H, w.W, prm)
    np.testing.assert_array_equal(rng.view(np.uint32), ref_rng.view(np.uint32))
    np.testing.assert_array_equal(packed.cpu().numpy().view(np.uint32), ref)
    # decode the oracle's words on the device
    s.unpack_sites(ref, ref_rng)
    dec = oracle.unpack_sites(w.H, w.W, ref, ref_rng)
    np.testing.assert_array_equal(s.params.cpu().numpy().view(np.uint32), dec.view(np.uint32))
    rec = s.records.cpu().numpy().copy()
    s.prep_records()
    assert np.array_equal(rec.view(np.uint32), s.records.cpu().numpy().view(np.uint32))


def test_pack_all_inactive(torch_cuda):
    H, W, N = 20, 30, 100
    prm = synth.uniform_sites(H, W, N, 4)
    prm[0] = -1.0
    s = _ctx(H, W, N, prm)
    packed, rng = s.pack_sites()
    assert np.all(packed.cpu().numpy() == 0) and np.all(rng == 0)
    s.unpack_sites(packed.cpu().numpy(), rng)
    p = s.params.cpu().numpy()
    assert np.all(p[0] == -1) and np.all(p[1:] == 0)


def test_decode_only_render(torch_cuda):
    """Sites rebuilt from their 16-byte records alone (no float parameters)
    render through a fresh refresh; the image equals the oracle's render of
    the decoded sites on the device's lists."""
    tgt, prm, w = synth.make_workload("c2", seed=5)
    s = _ctx(w.H, w.W, w.N, prm, seed=2)
    packed, rng = s.pack_sites()
    words = packed.cpu().numpy().view(np.uint32).copy()
    s2 = _ctx(w.H, w.W, w.N, np.full((9, 1), -1.0, np.float32), seed=2)
    s2.unpack_sites(words, rng)
    s2.refresh(w.G)
    s2.render()
    dec = oracle.unpack_sites(w.H, w.W, words, rng)
    img = oracle.render(w.H, w.W, dec, s2.get_table())
    assert np.abs(s2.image.cpu().numpy() - img).max() <= 1e-5
    # and the decoded image is close to the original sites' image
    s.refresh(w.G)
    s.render()
    d = s.image.cpu().numpy() - s2.image.cpu().numpy()
    assert 10 * np.log10(1.0 / float(np.mean(d ** 2))) > 40.0
