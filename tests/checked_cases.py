"""Cases run against the bounds-checked debug build (libsad_checks.so).

Run as a script in a process of its own with SAD_CHECKS=1 in the
environment (the library is chosen when it is first loaded).  Each case runs
the kernels whose indices rest on invariants rather than explicit guards --
the fused pass (tile index, masks, grouped entries), the cached-list pass,
the statistics backward, the standalone propagation and refresh -- on tiny
and ragged sizes, checks the result against the CPU oracle, and reads the
number of accesses the device-side checks refused; the fused pass runs
again with the TMA-staged list blocks (where its 32 x 16 tiles apply; the
other cases take the default form), and once more with every block's first
staging copy withheld (SAD_TEST_WITHHOLD_STAGING=1, read only by this
build): each block's bounded wait for the copy runs out, the block reads its
lists from global memory, the result is the same and staging_fallbacks
counts one fallback per block.  Last, the full-size workload runs the
same kinds of passes with the checks on.  Prints one JSON line."""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402


def main():
    assert os.environ.get("SAD_CHECKS") == "1"
    from soft_voronoi_render_b200 import SAD_STAGING_LOADS, SAD_STAGING_TMA, SAD_STATS, Sad, _lib
    assert _lib.library_path().endswith("libsad_checks.so")
    out = {"cases": 0, "check_failures": 0, "withheld_fallbacks": 0}
    for (H, W, N, seed) in ((1, 1, 3, 1), (9, 33, 40, 2), (37, 53, 300, 3), (16, 40, 200, 4), (24, 72, 6000, 5)):
        prm = synth.uniform_sites(H, W, N, seed)
        tgt = synth.make_image(H, W, 4, 0, seed)
        t0 = oracle.topk_exact(H, W, oracle.records(H, W, prm))
        if N == 200:
            t0[::3, 5] = t0[::3, 1]
            t0[::7, 7] = N + 11
        s = Sad(H, W, N, seed=seed)
        s.set_sites(prm)
        s.set_target(tgt)
        s.set_table(t0)
        s.fit_pass(2)
        t1 = oracle.propagate(H, W, oracle.records(H, W, prm), t0, 1, 2, seed=seed, pass_index=0)
        assert np.array_equal(s.get_table(), t1), (H, W, N)
        L, g = oracle.loss_backward(H, W, prm, t1, tgt)
        assert abs(s.loss() - L) <= 1e-5 * L
        gg = s.grads.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(gg - g) <= np.maximum(1e-4 * np.abs(g), 1e-6))
        # the same pass with the lists staged by TMA copies, from the same state
        _lib.sad_set_fit_state(s.ctx, 0, 0, seed, s.stream)
        s.set_table(t0)
        s.set_list_staging(SAD_STAGING_TMA)
        s.grads.zero_()
        s.fit_pass(2)
        assert np.array_equal(s.get_table(), t1), ("tma", H, W, N)
        assert abs(s.loss() - L) <= 1e-5 * L
        gg = s.grads.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(gg - g) <= np.maximum(1e-4 * np.abs(g), 1e-6))
        assert s.stats()["staging_fallbacks"] == 0
        # the first copy of every persistent block withheld: one persistent
        # block per tile at these sizes, each falling back once
        tall = H * W >= 4 * N
        n_tiles = ((W + 31) // 32) * ((H + 15) // 16)
        _lib.sad_set_fit_state(s.ctx, 0, 0, seed, s.stream)
        s.set_table(t0)
        s.grads.zero_()
        os.environ["SAD_TEST_WITHHOLD_STAGING"] = "1"
        try:
            s.fit_pass(2)  # the variable is read when the pass is launched
        finally:
            del os.environ["SAD_TEST_WITHHOLD_STAGING"]
        assert np.array_equal(s.get_table(), t1), ("withheld", H, W, N)
        assert abs(s.loss() - L) <= 1e-5 * L
        gg = s.grads.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(gg - g) <= np.maximum(1e-4 * np.abs(g), 1e-6))
        fb = s.stats()["staging_fallbacks"]
        assert fb == (n_tiles if tall else 0), (H, W, N, fb, n_tiles)
        out["withheld_fallbacks"] += fb
        s.set_list_staging(SAD_STAGING_LOADS)
        s.grads.zero_()
        s.fit_pass_cached()
        s.grads.zero_()
        s.backward(SAD_STATS)
        s.refresh(2)
        ref, _ = oracle.refresh(H, W, prm, 2, seed=seed, first_pass=1)
        assert np.array_equal(s.get_table(), ref), (H, W, N)
        st = s.stats()
        out["cases"] += 1
        out["check_failures"] += st["check_failures"]
        s.close()
    out["full_size"] = full_size_case()
    print(json.dumps(out), flush=True)


def full_size_case():
    """The 2048 x 2048, N = 131,072 workload in the checked build: a refresh,
    ten fitting iterations (where crowded tiles take the generic path), the
    TMA-staged pass, the cached-list, statistics and order-independent
    passes.  Returns the accesses the device-side checks refused."""
    from soft_voronoi_render_b200 import (SAD_DETERMINISTIC, SAD_STAGING_LOADS, SAD_STAGING_TMA, SAD_STATS, Sad,
                                          adam_cfg)
    tgt, prm, w = synth.make_workload("c3", seed=1)
    s = Sad(w.H, w.W, w.N, seed=1)
    s.set_sites(prm)
    s.set_target(tgt)
    s.refresh(w.G)
    cfg = adam_cfg(lr_pos=1e-3, lr_log_tau=1e-3, lr_r=1e-3, lr_color=5e-3, lr_theta=1e-3, lr_a=1e-3)
    for _ in range(10):
        s.fit_iteration(w.G, cfg)
    s.set_list_staging(SAD_STAGING_TMA)
    s.fit_pass(w.G)
    s.set_list_staging(SAD_STAGING_LOADS)
    s.grads.zero_()
    s.fit_pass_cached()
    s.grads.zero_()
    s.backward(SAD_STATS)
    s.grads.zero_()
    s.backward(SAD_DETERMINISTIC)
    st = s.stats()
    assert st["staging_fallbacks"] == 0 and np.isfinite(s.loss())
    s.close()
    return st["check_failures"]


if __name__ == "__main__":
    main()
