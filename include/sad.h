/*
 * sad.h -- C ABI of libsad, a B200 (sm_100a) implementation of one fitting
 * iteration of Soft Anisotropic Diagrams (SAD).
 *
 * Source pages (cited by title and section):
 *   [P1] "Soft Anisotropic Diagrams for Differentiable Image Representation"
 *        (paperlayer summary of arXiv:2604.21984v2), sections 4, 5, B.2-B.7.
 *   [P2] reading notes on the same paper, "key designs" 1-4 (formulas for
 *        G_i, d_mix, the softmax blend, the candidate update, budget control).
 *   [P4] "SAD: Soft Anisotropic Diagrams" project page, "Method".
 *
 * Model.  An image of H x W pixels is represented by up to N_cap sites.  Site
 * i has position p_i (pixels), log-temperature ln tau_i, radius r_i (pixels),
 * colour c_i (linear RGB), direction angle theta_i and anisotropy a_i.  With
 * s = 1 / max(H, W), u = (cos theta, sin theta), v = (-sin theta, cos theta),
 * G_i = e^a u u^T + e^-a v v^T (det G_i = 1) and n_i(x) = ||x - p_i||_{G_i},
 * the logit of site i at pixel centre x is
 *     l_i(x) = -tau_i (s n_i(x) - s r_i)                    ([P2] designs 1-2)
 * and the pixel colour is the softmax blend of the K = 8 sites held in the
 * pixel's candidate list ([P2] design 2, [P4] Method).  The candidate list is
 * maintained by Jacobi propagation passes ([P2] design 3, [P1] section 4).
 *
 * Memory.  The library allocates no device memory.  The caller owns every
 * device buffer (PyTorch tensors in the Python binding) and binds them with
 * sad_bind(); the library never frees them.  Layouts (all little-endian,
 * row-major, pixel id p = row * W + column, P = H * W):
 *   params   float32 [9][N_cap]  planes x, y, ln tau, r, cr, cg, cb, theta, a
 *                                ([P1] B.2 site buffer, with the direction
 *                                stored as one angle).  A site is active iff
 *                                x >= 0 (x < 0 or NaN marks an unused slot).
 *   grads    float32 [9][N_cap]  dL/d(param), same planes; accumulated by
 *                                sad_backward, consumed and zeroed by
 *                                sad_adam_step.
 *   adam_m, adam_v float32 [9][N_cap]  Adam moments.
 *   records  float32 [N_cap][16] derived per-site score record (64 bytes).
 *   table    uint32  [2][2][P][4]  two candidate tables (double buffer), each
 *                                two planes of uint4 (slots 0-3, slots 4-7)
 *                                ([P1] B.2: two four-channel uint32 textures,
 *                                K = 8, 0xffffffff = empty).
 *   target   float32 [3][P]      planar linear RGB.
 *   image    float32 [3][P]      planar rendered image (may be NULL).
 *   workspace bytes >= sad_workspace_bytes(); counters, statistics, loss,
 *                                scratch, and the refresh's score cache
 *                                (32 bytes per pixel).
 * Every pointer must be 16-byte aligned and records 32-byte aligned (the
 * kernels read a record's ranking fields in one 32-byte load); target and
 * image must not overlap other buffers.  Which of the two tables is current is kept in device
 * memory, so a captured CUDA graph of the calls below keeps alternating.
 *
 * Calls.  Every call except sad_get_stats, sad_get_loss, sad_get_table and
 * sad_get_sites is asynchronous on the given stream and returns a status.
 * Device-side anomalies (hash overflow, skipped non-finite pixels, empty
 * pixels, ids out of range) are counted in the statistics block; kernels
 * never trap and contain no waits.
 */
#ifndef SAD_H
#define SAD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *sad_stream_t; /* == cudaStream_t; NULL = legacy default stream */

enum {
    SAD_OK = 0,
    SAD_ERR_INVALID_ARG = 1, /* bad size, NULL where a buffer is required, misalignment */
    SAD_ERR_UNSUPPORTED = 2, /* K != 8, or a flag this build does not implement */
    SAD_ERR_CUDA = 3,        /* a CUDA call or kernel launch failed; see sad_last_error */
    SAD_ERR_CAPACITY = 4,    /* more sites than N_cap, too many injections, ... */
    SAD_ERR_NOT_BOUND = 5    /* buffers not bound yet */
};

#define SAD_K 8
#define SAD_N_PARAMS 9
#define SAD_RECORD_FLOATS 16
#define SAD_MAX_INJECT 64
#define SAD_EMPTY 0xFFFFFFFFu

typedef struct sad_ctx sad_ctx;

typedef struct sad_buffers {
    float *params;
    float *grads;
    float *adam_m;
    float *adam_v;
    float *records;
    uint32_t *table;
    float *target;
    float *image; /* optional */
    void *workspace;
    size_t workspace_bytes;
    float *stats; /* optional [6][N_cap]: budget-control statistics (SAD_STATS, sad_densify_prune) */
    const uint8_t *frozen; /* optional [N_cap]: non-zero = frozen site, left untouched by Adam
                              ([P1] section 7: boundary sites excluded from gradient updates) */
    void *cand16;          /* optional [N_cap] x 16 bytes, 16-byte aligned: packed candidate-site
                              records (sad_set_candidate_precision) */
} sad_buffers;

/* sad_backward flag: also accumulate the budget-control statistics into
 * stats ([P1] B.4-B.5): per site, mass m = sum w, energy E = sum w e,
 * second moments sum w e (dx^2, dx dy, dy^2) with (dx, dy) = x - p, and the
 * removal delta D = sum |(chat - w c) / max(1 - w, 1e-6) - t|^2 - e, where
 * e = |chat - t|^2 at each pixel holding the site. */
#define SAD_STATS 1u

/* sad_backward flag: gradients that do not depend on the order of the
 * atomic additions (bit-identical from run to run).  Every (pixel, slot)
 * contribution is rounded to a multiple of 2^-40 and summed in 64-bit fixed
 * point, per tile and then with integer atomics (exact, hence order-free),
 * then added to grads; the pages accumulate scaled integer gradients the
 * same way on WebGPU ([P1] B.4).  Magnitudes up to 2^23 per site and
 * parameter; terms below 2^-41 vanish.  Not combinable with SAD_STATS. */
#define SAD_DETERMINISTIC 2u

/* Densify / prune configuration ([P1] B.5, [P2] design 4). */
typedef struct sad_densify_cfg {
    int grow;              /* net sites added per event (2500 in the 768x512 schedule) */
    float prune_frac;      /* fraction of the active sites pruned (0.005) */
    float alpha;           /* score E / max(m, eps)^alpha (0.5) */
    float eps;             /* mass floor (1e-6) */
    float r_scale;         /* children's radius factor (0.85) */
    float log_tau_shift;   /* subtracted from the children's ln tau (ln 2) */
    float offset_scale;    /* child offset = offset_scale * sqrt(largest eigenvalue) (0.5) */
    float fallback_offset; /* offset in pixels along the metric's long axis when the moment is degenerate (0.5) */
} sad_densify_cfg;

/* Adam configuration ([P2] key design 4).  Learning rates per parameter
 * group; positions and radius are stepped in the resolution-free units s x
 * and s r in which the logit is written (their gradient is multiplied by
 * max(H, W) and their step by max(H, W)). */
typedef struct sad_adam_cfg {
    float lr_pos, lr_log_tau, lr_r, lr_color, lr_theta, lr_a;
    float beta1, beta2, eps;
} sad_adam_cfg;

typedef struct sad_stats {
    uint64_t hash_overflow;    /* pixels with a backward contribution that bypassed the tile
                                  index (a site outside it: crowded tiles, injected winners) */
    uint64_t nonfinite_pixels; /* always 0: a slot whose logit is not finite (NaN parameters)
                                  is not a candidate, so such a pixel renders from its other
                                  slots or counts in empty_pixels */
    uint64_t empty_pixels;     /* pixels without any valid candidate (render writes 0) */
    uint64_t dropped_ids;      /* table entries >= N_cap met by render/backward */
    uint32_t pass_counter;     /* propagation passes run (drives injection randomness) */
    uint32_t adam_step;        /* Adam steps taken (bias-correction t of the next step is +1) */
    uint32_t current_table;    /* 0 or 1: which table of the double buffer is current */
    uint32_t staging_fallbacks; /* fit passes: tile-list copies into shared memory that did not
                                   arrive within the wait bound, after which the block read the
                                   lists from global memory instead (expected 0) */
    double loss;               /* loss of the last sad_backward / sad_fit_iteration */
    uint32_t n_active;         /* active sites before the last densify event */
    uint32_t n_split;          /* sites split by the last densify event */
    uint32_t n_pruned;         /* sites pruned by the last densify event */
    uint32_t check_failures;   /* debug build (libsad_checks): accesses a bounds check refused */
} sad_stats;

/* Bytes of workspace the caller must bind for an H x W image and N_cap sites. */
int sad_workspace_bytes(int H, int W, int N_cap, size_t *bytes);

/* Create a context.  H, W >= 1, H * W < 2^31, N_cap >= 1, K must be 8
 * (SAD_ERR_UNSUPPORTED otherwise).  Allocates host memory for the handle
 * only.  *out is set on success. */
int sad_create(int H, int W, int N_cap, int K, sad_ctx **out);

/* Destroy a context.  Frees the handle only; bound buffers stay the caller's. */
int sad_destroy(sad_ctx *ctx);

/* Bind caller-owned device buffers (layouts above).  Checks non-NULL (except
 * image), 16-byte alignment and the workspace size.  Does not touch their
 * contents; call sad_reset before first use. */
int sad_bind(sad_ctx *ctx, const sad_buffers *buf);

/* Zero the counters, statistics, gradients and Adam moments, mark the first
 * table current and set the injection seed.  Asynchronous. */
int sad_reset(sad_ctx *ctx, uint32_t seed, sad_stream_t stream);

/* Copy n sites (host or device float32 [9][n] planes) into params slots
 * 0..n-1, mark slots n..N_cap-1 inactive and rebuild the score records
 * (step a1).  n <= N_cap else SAD_ERR_CAPACITY.  Asynchronous; a host source
 * must stay valid until the stream reaches the copy. */
int sad_set_sites(sad_ctx *ctx, const float *params_9xn, int n, sad_stream_t stream);

/* Copy params slots 0..n-1 into dst (host or device, [9][n]).  Synchronises
 * the stream when dst is host memory. */
int sad_get_sites(sad_ctx *ctx, float *dst_9xn, int n, sad_stream_t stream);

/* Copy a target image (host or device float32 [3][P]) into the bound target. */
int sad_set_target(sad_ctx *ctx, const float *target_3xp, sad_stream_t stream);

/* Convert an 8-bit RGB image into the bound target: src is DEVICE memory
 * holding H x W pixels of 3 interleaved bytes (row-major, the usual image
 * layout); channel c of pixel p becomes src[3 p + c] / 255 (IEEE float32
 * division) in the planar float32 target.  Streamed 8-bit inputs move a
 * quarter of the bytes of float32 ones.  Errors: SAD_ERR_INVALID_ARG for
 * NULL. */
int sad_set_target_u8(sad_ctx *ctx, const uint8_t *src_hw3, sad_stream_t stream);

/* Step a1: rebuild every score record from params.  Record of site i (fp32
 * values, each evaluated in double and rounded once): x, y, A, B, C, b, k, 0,
 * cr, cg, cb, cos theta, sin theta, k^2 e^a, k^2 e^-a, 0 where k = tau s,
 * (A, B, C) = k^2 (G11, G12, G22), b = k r ([P2] design 1; fields as in the
 * packed candidate-site buffer of [P1] B.2).  Inactive: x = -1, rest 0. */
int sad_prep_records(sad_ctx *ctx, sad_stream_t stream);

/* Step a8: exact top-K by brute force over all active sites ([P1] abstract:
 * the quantity the maintained list approximates).  pixels: device int64
 * pixel ids (NULL = all P pixels in order); out: device uint32 [n][8],
 * sorted by (logit desc, id asc), empty slots 0xffffffff.  The logit is
 * evaluated in float32 as l = b - sqrt(q), q = dx u1 + dy u2 with
 * u1 = A dx + B dy, u2 = C dy + B dx (fixed IEEE operation order, see the
 * records above), the pages' logit rearranged. */
int sad_topk_exact(sad_ctx *ctx, const int64_t *pixels, int64_t n_pix, uint32_t *out,
                   sad_stream_t stream);

/* Step a9: seed pass + full refresh ([P1] B.3: seed pass, then jump-flood
 * passes).  Clears the current table, writes each active site's id into slot
 * 0 of the pixel containing it (smallest id wins), then runs propagation
 * passes at jumps B/2, B/4, ..., 1 with B the largest power of two
 * <= max(H, W), each with G injections.  0 <= G <= 64.  The records do not
 * change during a refresh, so each pass keeps its lists' ranking scores in
 * the workspace and the next pass takes the pixel's own list's scores from
 * there instead of recomputing them (the same bits). */
int sad_refresh(sad_ctx *ctx, int G, sad_stream_t stream);

/* Rebind the target image to another caller-owned device buffer (float32
 * [3][H][W], 16-byte aligned) without copying: kernels launched after the
 * call read the new buffer, earlier launches keep the old one.  This lets a
 * caller stream targets in: copy the next target into a second buffer on
 * another stream while the current iteration runs, then bind it.  The
 * library never frees either buffer.  Errors: SAD_ERR_NOT_BOUND before
 * sad_bind, SAD_ERR_INVALID_ARG for NULL or misaligned pointers. */
int sad_bind_target(sad_ctx *ctx, const float *target);

/* 16-byte evaluation record ([P1] B.2, "Packed storage for evaluation": the
 * site's semantic values quantised into four 32-bit words, per-image
 * min/scale for ln tau and radius).  Field string, little-endian over the
 * four words, bit offset (width):
 *   x 0 (18), y 18 (18), cr 36 (10), cg 46 (10), cb 56 (10),
 *   ln tau 66 (16), r 82 (14), theta 96 (14), a 110 (14), active 127 (1).
 * x, y: cell floor(x / W 2^18) of 2^18 across the image (clamped), decoded
 * at the cell centre.  Colours: clamped to [0, 1], 1023 steps.  ln tau, r,
 * a: 2^b - 1 steps over the range [lo, hi] of the active sites.  theta: the
 * axis angle theta mod pi in 2^14 steps.  Rounding half up in double;
 * decoded values rounded once to float32.  Inactive sites pack to zeros.
 * 128 bits per site: 16.3 bits per pixel at 768 x 512 with 50,000 sites.
 *
 * sad_pack_sites: packed = device uint32 [N_cap][4] (16-byte aligned),
 * written in stream order; range = 6 floats (host or device, may be NULL)
 * receiving (lo ln tau, lo r, lo a, hi ln tau, hi r, hi a).
 * sad_unpack_sites: decodes packed + range into params and rebuilds the
 * records; grads, Adam moments and candidate lists are left alone (call
 * sad_reset and sad_refresh for a fresh fit or a decode-only render).
 * Errors: SAD_ERR_INVALID_ARG for NULL or misaligned pointers. */
int sad_pack_sites(sad_ctx *ctx, uint32_t *packed, float *range, sad_stream_t stream);
int sad_unpack_sites(sad_ctx *ctx, const uint32_t *packed, const float *range, sad_stream_t stream);

/* Candidate grid ([P1] B.3, "Candidate field"): keep the candidate lists on
 * a ceil(H/cell) x ceil(W/cell) grid of cell x cell pixel cells instead of
 * one list per pixel.  Cell (i, j) holds the pixels with floor(x/cell) = i,
 * floor(y/cell) = j (integer mapping, no interpolation); propagation, seed,
 * exact top-K and the JFA prepass work on the grid and score candidates at
 * the cell centre ((i + 0.5) cell, (j + 0.5) cell), as the pages score cells;
 * render and backward score each pixel's cell list at the pixel centre.
 * Injections are keyed on the cell index.  cell = 1 (the default) is the
 * pixel grid.  On a coarser grid sad_fit_pass runs a propagation pass on the
 * grid and then the tile pass of sad_fit_pass_cached, which reads each
 * pixel's cell list.  The table buffer bound for H x W holds any grid.
 * After the call the current table is empty (sentinels): call sad_refresh,
 * sad_jfa_prepass or sad_set_table next.  sad_get_table, sad_set_table and
 * sad_topk_exact (pixels = NULL, or cell indices) then use GH x GW lists.
 * Errors: SAD_ERR_INVALID_ARG when cell < 1 or cell > max(H, W).  May be
 * called before sad_bind (no launch then). */
int sad_set_candidate_grid(sad_ctx *ctx, int cell, sad_stream_t stream);

/* Optional JFA prepass ([P1] B.3, for reinitialisation or after large
 * edits): the seed pass, then ceil(log2 max(H, W)) flood passes at jumps
 * 2^(n-1), ..., 1, each taking for every pixel the 4 best distinct candidates
 * of the 9 lists at (i + a k, j + b k), a, b in {-1, 0, 1}, into slots 0-3
 * (the first of the two four-id planes; slots 4-7 empty).
 * Propagation passes then fill the lists. */
int sad_jfa_prepass(sad_ctx *ctx, sad_stream_t stream);

/* Steps a2/a3: one Jacobi propagation pass at jump >= 1 ([P2] design 3):
 * for every pixel the new list is the top 8 by (logit desc, id asc) of the
 * distinct valid ids among its own list, the lists of the four pixels at
 * (+-jump, 0) and (0, +-jump) that lie inside the image, and G injected ids.
 * Injection ([P1] B.3: an xorshift generator seeded per pass and pixel):
 * h = fmix32(p ^ fmix32(seed ^ pass * 0x9E3779B9)), 1 if zero, then G times
 * h = xorshift32(h) (13, 17, 5), id = (h * N_cap) >> 32.  Reads the current
 * table, writes the other one, makes it current, advances the pass counter. */
int sad_propagate(sad_ctx *ctx, int jump, int G, sad_stream_t stream);

/* Step a4: render the current table ([P2] design 2): w = softmax of the valid
 * slots' logits (max-subtracted), chat = sum w c; a pixel without a valid
 * slot gets 0.  image: device float32 [3][P], NULL = the bound image. */
int sad_render(sad_ctx *ctx, float *image, sad_stream_t stream);

/* Steps a4-a6: render, MSE loss L = (1/P) sum_x sum_ch (chat - t)^2 and the
 * analytic gradient ([P1] B.4), accumulated into grads per tile before the
 * global atomics ([P1] section 5 and B.4).  The pass is the tile pass on the
 * current lists (the work of sad_fit_pass_cached): the tile's site ids go
 * into a shared-memory hash keyed by site id (multiplicative hash, linear
 * probing capped at 8, compare-and-swap insert) that gives each a dense
 * tile-local index; the tile's (pixel, slot) entries are grouped by site and
 * summed in registers, with one global atomic per (site, parameter, run of
 * groups); entries of sites outside the index (more than 128 in a tile) go
 * straight to global atomics.  Writes the bound image when one is bound and
 * the loss into the statistics block.  flags: 0, SAD_STATS (needs the stats
 * buffer; carries the six statistics beside the nine gradients) or
 * SAD_DETERMINISTIC (the same pass with its sums in 64-bit fixed point:
 * order-independent).  SAD_ERR_UNSUPPORTED for other flags or both
 * together. */
int sad_backward(sad_ctx *ctx, uint32_t flags, sad_stream_t stream);

/* One budget-control event, on the device ([P1] B.5: split by the score
 * E / m^alpha along a covariance-estimated axis; prune by the removal score,
 * x = -1; [P2] design 4).  Reads the statistics accumulated by
 * sad_backward(ctx, SAD_STATS, ...) since the last event, then:
 *   1. prunes the floor(prune_frac * n_active) active sites with the smallest
 *      removal delta D (ties: smaller id);
 *   2. splits the min(n_pruned + grow, free slots, active sites left) active
 *      sites with the largest float32 score E / max(m, eps)^alpha (IEEE
 *      sqrt/division when alpha = 0.5; ties: smaller id); parents in
 *      ascending id take the free slots (x < 0) in ascending id;
 *   3. places the children at p +- d, d = offset_scale * sqrt(l) e with (l, e)
 *      the largest eigenpair of the second moment / E (e.x > 0, or e.x = 0
 *      and e.y > 0), or d = fallback_offset times the metric's long axis
 *      (v if a > 0, else u) when E or l is not positive; child A keeps the
 *      parent's slot, child B takes the free slot; both are clamped into the
 *      image, take the target colour at their pixel, r * r_scale,
 *      ln tau - log_tau_shift, the parent's theta and a, and zero Adam moments;
 *   4. zeroes the statistics and rebuilds the score records.
 * The candidate lists are stale afterwards: run sad_refresh before the next
 * pass.  Needs the stats buffer.  The number of sites never leaves the
 * device (see sad_get_stats). */
int sad_densify_prune(sad_ctx *ctx, const sad_densify_cfg *cfg, sad_stream_t stream);

/* Tau diffusion ([P1] B.6): one Jacobi step on the ln tau gradients,
 * g_i <- (1 - lambda) g_i + lambda mean_j g_j over the active sites j != i in
 * the candidate list of the pixel containing p_i (the site's local candidate
 * neighbourhood); all neighbours are read before any write; sites with no
 * such neighbour, or outside the image, keep g_i.  Call between the backward
 * pass and Adam.  0 <= lambda <= 1. */
int sad_tau_diffuse(sad_ctx *ctx, float lambda, sad_stream_t stream);

/* Step a7: one Adam step on every active site ([P2] design 4), reading and
 * zeroing grads, advancing the Adam step counter, and rebuilding the score
 * records (a1) in the same kernel.  Frozen sites (the optional frozen
 * buffer) are left untouched, like inactive ones.  The step keeps positions inside the
 * image, [0, W^-] x [0, H^-] with W^- the largest float below W (x < 0 is the
 * marker of a pruned site, not an optimiser outcome). */
int sad_adam_step(sad_ctx *ctx, const sad_adam_cfg *cfg, sad_stream_t stream);

/* Steps a2-a6 in one kernel: a propagation pass at jump 1 with G injections
 * (same result as sad_propagate(ctx, 1, G)), then render, loss and backward
 * on the new lists (same result as sad_backward, up to the summation order
 * of the gradients).  Each 32 x 16 tile (32 x 8 where there are fewer than
 * 4 pixels per site) gathers the distinct sites of its and
 * its halo's lists into a dense local index (at most 128 sites; tiles with
 * more take a slower generic path) that serves both to de-duplicate the
 * candidate union and to accumulate the tile's gradients ([P1] section 5 and
 * B.4: per-tile shared-memory reduction, one global atomic per site and
 * parameter).  Writes the bound image when one is bound. */
int sad_fit_pass(sad_ctx *ctx, int G, sad_stream_t stream);

/* Steps a4-a6 on the cached candidate lists, tiled like sad_fit_pass but
 * without the propagation: for the iterations between candidate updates
 * ([P1] B.3: updating every 8-16 iterations did not change the final PSNR).
 * Same results as sad_backward; the current table is not changed. */
int sad_fit_pass_cached(sad_ctx *ctx, sad_stream_t stream);

/* One steady-state fitting iteration: sad_fit_pass then sad_adam_step
 * (steps a2-a7, two kernels). */
int sad_fit_iteration(sad_ctx *ctx, int G, const sad_adam_cfg *cfg, sad_stream_t stream);

/* Copy the current table into dst (host or device uint32 [P][8], slot order).
 * Synchronises the stream. */
int sad_get_table(sad_ctx *ctx, uint32_t *dst, sad_stream_t stream);

/* Copy a table (host or device uint32 [P][8]) into the current table. */
int sad_set_table(sad_ctx *ctx, const uint32_t *src, sad_stream_t stream);

/* Read the statistics block (synchronises the stream). */
int sad_get_stats(sad_ctx *ctx, sad_stats *out, sad_stream_t stream);

/* Candidate precision ([P1] B.2: candidate-update kernels score from a
 * compact 16-byte per-site buffer of float16 pairs).  bits = 32 (the
 * default): candidates are ranked by the float32 logit of the score record.
 * bits = 16: every candidate update (sad_refresh, sad_propagate and the
 * propagation of sad_fit_pass / sad_fit_iteration, which then runs as a
 * propagation pass followed by the tile pass on the new lists) first packs
 * each site into the bound cand16 buffer -- x and y as float32, then the
 * binary16 pairs (A, B) and (C, b) (round to nearest even) -- ranks the
 * candidates by the float32 logit evaluated from those rounded coefficients
 * (the operation order of the score record), and re-scores the kept 8 with
 * the float32 record, storing them in (float32 logit desc, id asc) order.
 * The position stays float32 because binary16 steps by 1-2 px between 2048
 * and 4096 px.  The JFA prepass and the exact top-K stay float32.  Errors:
 * SAD_ERR_INVALID_ARG for other bits, SAD_ERR_NOT_BOUND for 16 without a
 * bound cand16 buffer. */
int sad_set_candidate_precision(sad_ctx *ctx, int bits, sad_stream_t stream);

/* How the propagating fit pass (sad_fit_pass, sad_fit_iteration) brings each
 * tile's candidate lists and their one-pixel halo on chip ([P1] section 5:
 * per-tile staging in shared memory).
 *   SAD_STAGING_LOADS (default): one block per 32 x 16 tile; every thread
 *     loads its own list and a share of the halo.
 *   SAD_STAGING_TMA: as many persistent blocks as fit the device take tiles
 *     from a ticket; while a block works on one tile, a TMA tensor copy
 *     brings the next tile's list block (both planes with the halo, 19.6 KB)
 *     into shared memory, signalled on a shared-memory barrier whose wait is
 *     bounded: a copy that does not arrive in time switches the block to
 *     plain loads and is counted in sad_stats.staging_fallbacks.
 * Both give the same lists bit for bit and the same sums.  The default is
 * the faster on B200: the co-resident block already hides the list loads'
 * latency, and a persistent block cannot begin its next tile before its
 * slowest warp has finished the current one.  The TMA form applies where
 * the pass uses 32 x 16 tiles (at least 4 pixels per site) on the pixel
 * grid; elsewhere the default runs.  The bounds-checked build of the
 * library (compiled with SAD_CHECKS) withholds every persistent block's
 * first copy when SAD_TEST_WITHHOLD_STAGING=1 is in the environment at the
 * launch, and bounds that wait at 1,024 polls, so that a test can run the
 * fallback; the normal build ignores the variable.  SAD_ERR_INVALID_ARG for
 * other modes. */
#define SAD_STAGING_LOADS 0
#define SAD_STAGING_TMA 1
int sad_set_list_staging(sad_ctx *ctx, int mode, sad_stream_t stream);

/* The fitting state that lives in the library's counter block: the pass
 * counter that keys the injection randomness ([P1] B.3: an xorshift
 * generator seeded per pass and pixel), Adam's step count (bias correction) and the
 * injection seed.  Everything else a fit needs is in caller-owned buffers:
 * the sites (sad_get_sites / sad_set_sites), the Adam moments (the bound
 * adam_m / adam_v) and the current candidate lists (sad_get_table /
 * sad_set_table).  Saved together, they are a checkpoint from which a fit
 * resumes as if it had not stopped (the pages keep the whole fit on the GPU
 * and move only site data across the host boundary, [P1] B.7/B.8). */
typedef struct sad_fit_state {
    uint32_t pass_counter; /* propagation passes run so far */
    uint32_t adam_step;    /* Adam steps taken so far */
    uint32_t seed;         /* injection seed (as given to sad_reset) */
    uint32_t reserved;     /* 0 */
} sad_fit_state;

/* Read the fit state (synchronises the stream).  SAD_ERR_INVALID_ARG for a
 * NULL destination, SAD_ERR_NOT_BOUND before sad_bind. */
int sad_get_fit_state(sad_ctx *ctx, sad_fit_state *out, sad_stream_t stream);

/* Write the fit state, in stream order (the values travel by value, so
 * *state may be released when the call returns).  Which table of the double
 * buffer is current is not part of the state: sad_set_table writes the
 * current one.  SAD_ERR_INVALID_ARG for NULL or a non-zero reserved field. */
int sad_set_fit_state(sad_ctx *ctx, const sad_fit_state *state, sad_stream_t stream);

/* Loss of the last backward pass, copied to host memory (synchronises). */
int sad_get_loss(sad_ctx *ctx, double *loss, sad_stream_t stream);

/* The same loss copied in stream order without synchronising: dst (one
 * double, host-pinned or device memory) holds it once the stream reaches the
 * copy.  Lets a caller read step k's loss while step k + 1 runs. */
int sad_copy_loss(sad_ctx *ctx, double *dst, sad_stream_t stream);

/* Message of the last failing call on this context ("" if none). */
const char *sad_last_error(const sad_ctx *ctx);

/* Render, loss and backward (the work of sad_backward) for callers that
 * cannot allocate device memory -- for example code running inside another
 * framework's fixed memory budget, or a plugin interface that receives only
 * input and output pointers and may not request a workspace.  This entry
 * point has no counterpart in the paper; it exists only for such callers.
 * It needs no context and no workspace: its scratch (a 256-byte counter block
 * plus one double per 32 x 8 tile) lives in a device array of
 * SAD_NOALLOC_SCRATCH_BYTES that the library holds on every GPU that loads
 * it, until the process exits.  It calls no cudaMalloc or cudaFree.
 *   records  float32 [N_cap][16] score records (as sad_prep_records writes)
 *   table    uint32  [2][P][4] the candidate table to render: plane 0 holds
 *            slots 0-3, plane 1 slots 4-7
 *   target   float32 [3][P];  image float32 [3][P] or NULL
 *   grads    float32 [9][N_cap], accumulated into (zero it first)
 *   loss     one device double, receives L
 * Pointers 16-byte aligned, records 32-byte (loss 8-byte).  Returns
 * SAD_ERR_CAPACITY when
 * ceil(W/32) * ceil(H/8) exceeds (SAD_NOALLOC_SCRATCH_BYTES - 256) / 8 =
 * 131,040 tiles (4096 x 8192 fits) or ceil(H/8) exceeds 65,535 (the launch
 * limit on tile rows), SAD_ERR_INVALID_ARG for bad sizes or pointers,
 * SAD_ERR_CUDA when a CUDA call fails.  The first call on a device looks up
 * the array's device address and keeps it for the process (a one-time
 * set-up): make that first call before capturing a stream, and do not call
 * this entry point on a device again after cudaDeviceReset, which leaves the
 * kept address stale.  All calls on a device share the one
 * array, which keeps the previous call's contents (each call clears what must
 * start at zero): calls that may overlap on the GPU -- on different streams,
 * or from several threads -- race on it and must be serialised by the
 * caller. */
#define SAD_NOALLOC_SCRATCH_BYTES (1u << 20)
int sad_backward_noalloc(int H, int W, int N_cap, const float *records, const uint32_t *table,
                         const float *target, float *image, float *grads, double *loss, sad_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SAD_H */
