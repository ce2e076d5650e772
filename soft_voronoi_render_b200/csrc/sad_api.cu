// sad_api.cu -- the C ABI of libsad (declared in include/sad.h).
//
// Argument checking, buffer binding, status codes and kernel sequencing.  The
// library allocates no device memory: every buffer is the caller's.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>

#include "sad.h"
#include "sad_device.cuh"
#include "sad_launch.h"

struct sad_ctx {
    int H, W, N, K;
    long long P;
    int cell, GH, GW;
    long long PT;
    bool bound;
    sad_buffers buf;
    sad::Dev dev;
    char err[512];
};

namespace {

int fail(sad_ctx *ctx, int code, const char *fmt, ...) {
    if (ctx) {
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(ctx->err, sizeof(ctx->err), fmt, ap);
        va_end(ap);
    }
    return code;
}

int cuda_status(sad_ctx *ctx, cudaError_t e, const char *what) {
    if (e == cudaSuccess) return SAD_OK;
    return fail(ctx, SAD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int need_bound(sad_ctx *ctx) {
    if (!ctx) return SAD_ERR_INVALID_ARG;
    if (!ctx->bound) return fail(ctx, SAD_ERR_NOT_BOUND, "buffers are not bound (call sad_bind)");
    return SAD_OK;
}

cudaStream_t cs(sad_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

int read_counters(sad_ctx *ctx, sad::Counters *out, cudaStream_t st) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_status(ctx, e, "stream synchronize");
    e = cudaMemcpy(out, ctx->buf.workspace, sizeof(sad::Counters), cudaMemcpyDeviceToHost);
    return cuda_status(ctx, e, "read counters");
}

// the packed candidate-site records follow the current score records: built
// at the start of every call that updates candidates in the binary16 mode
int pack_candidates(sad_ctx *ctx, cudaStream_t st) {
    if (!ctx->dev.f16) return SAD_OK;
    return cuda_status(ctx, sad::launch_pack_cand16(ctx->dev, st), "pack candidate records");
}

int run_refresh(sad_ctx *ctx, int G, cudaStream_t st) {
    int r = pack_candidates(ctx, st);
    if (r) return r;
    r = cuda_status(ctx, sad::launch_seed(ctx->dev, st), "seed");
    if (r) return r;
    int B = 1;
    const int m = ctx->GH > ctx->GW ? ctx->GH : ctx->GW;
    while (B * 2 <= m) B *= 2;
    // the records stay as they are during the refresh: the first pass stores
    // each new list's scores, every later pass takes its own list's from there
    for (int k = B / 2; k >= 1; k /= 2) {
        r = cuda_status(ctx, sad::launch_propagate(ctx->dev, k, G, st, k == B / 2 ? 1 : 2), "propagate");
        if (r) return r;
    }
    return SAD_OK;
}

// the fused propagating pass works on the pixel grid; on a coarser candidate
// grid the propagation runs on the grid, then the tile pass on the cached
// lists renders and differentiates every pixel from its cell's list
int run_fit_pass(sad_ctx *ctx, int G, cudaStream_t st) {
    if (ctx->cell == 1 && !ctx->dev.f16) return cuda_status(ctx, sad::launch_fit_tile(ctx->dev, G, st), "fit pass");
    // a coarser candidate grid, or candidates ranked on the packed records:
    // the propagation pass, then the tile pass on the new lists
    int r = pack_candidates(ctx, st);
    if (r) return r;
    r = cuda_status(ctx, sad::launch_propagate(ctx->dev, 1, G, st), "propagate");
    if (r) return r;
    return cuda_status(ctx, sad::launch_fit_tile_cached(ctx->dev, st), "fit pass (cached lists)");
}

int check_adam(sad_ctx *ctx, const sad_adam_cfg *cfg, sad::AdamHyper &h) {
    if (!cfg) return fail(ctx, SAD_ERR_INVALID_ARG, "adam config is NULL");
    if (!(cfg->beta1 >= 0.0f && cfg->beta1 < 1.0f) || !(cfg->beta2 >= 0.0f && cfg->beta2 < 1.0f) ||
        !(cfg->eps > 0.0f))
        return fail(ctx, SAD_ERR_INVALID_ARG, "adam betas must lie in [0, 1) and eps > 0");
    const float lr[9] = {cfg->lr_pos,   cfg->lr_pos,   cfg->lr_log_tau, cfg->lr_r, cfg->lr_color,
                         cfg->lr_color, cfg->lr_color, cfg->lr_theta,   cfg->lr_a};
    for (int k = 0; k < 9; ++k) {
        if (!(lr[k] >= 0.0f)) return fail(ctx, SAD_ERR_INVALID_ARG, "learning rates must be >= 0");
        h.lr[k] = lr[k];
    }
    h.beta1 = cfg->beta1;
    h.beta2 = cfg->beta2;
    h.eps = cfg->eps;
    return SAD_OK;
}

}  // namespace

extern "C" {

int sad_workspace_bytes(int H, int W, int N_cap, size_t *bytes) {
    if (!bytes || H < 1 || W < 1 || N_cap < 1 || (long long)H * W >= (1ll << 31)) return SAD_ERR_INVALID_ARG;
    *bytes = sad::workspace_bytes(H, W, N_cap);
    return SAD_OK;
}

int sad_create(int H, int W, int N_cap, int K, sad_ctx **out) {
    if (!out) return SAD_ERR_INVALID_ARG;
    *out = nullptr;
    if (H < 1 || W < 1 || N_cap < 1 || (long long)H * W >= (1ll << 31)) return SAD_ERR_INVALID_ARG;
    if (K != SAD_K) return SAD_ERR_UNSUPPORTED;
    sad_ctx *c = new (std::nothrow) sad_ctx();
    if (!c) return SAD_ERR_CAPACITY;
    c->H = H;
    c->W = W;
    c->N = N_cap;
    c->K = K;
    c->P = (long long)H * W;
    c->cell = 1;
    c->GH = H;
    c->GW = W;
    c->PT = c->P;
    c->bound = false;
    c->err[0] = 0;
    *out = c;
    return SAD_OK;
}

int sad_destroy(sad_ctx *ctx) {
    if (!ctx) return SAD_ERR_INVALID_ARG;
    delete ctx;
    return SAD_OK;
}

int sad_bind(sad_ctx *ctx, const sad_buffers *b) {
    if (!ctx) return SAD_ERR_INVALID_ARG;
    if (!b) return fail(ctx, SAD_ERR_INVALID_ARG, "buffers struct is NULL");
    const void *req[] = {b->params, b->grads, b->adam_m, b->adam_v, b->records, b->table, b->target, b->workspace};
    const char *names[] = {"params", "grads", "adam_m", "adam_v", "records", "table", "target", "workspace"};
    for (int q = 0; q < 8; ++q) {
        if (!req[q]) return fail(ctx, SAD_ERR_INVALID_ARG, "buffer %s is NULL", names[q]);
        if (!aligned16(req[q])) return fail(ctx, SAD_ERR_INVALID_ARG, "buffer %s is not 16-byte aligned", names[q]);
    }
    // the kernels read a record's ranking fields in one 32-byte load
    if ((reinterpret_cast<uintptr_t>(b->records) & 31u) != 0)
        return fail(ctx, SAD_ERR_INVALID_ARG, "buffer records is not 32-byte aligned");
    if (b->image && !aligned16(b->image)) return fail(ctx, SAD_ERR_INVALID_ARG, "buffer image is not 16-byte aligned");
    if (b->stats && !aligned16(b->stats)) return fail(ctx, SAD_ERR_INVALID_ARG, "buffer stats is not 16-byte aligned");
    if (b->cand16 && !aligned16(b->cand16))
        return fail(ctx, SAD_ERR_INVALID_ARG, "buffer cand16 is not 16-byte aligned");
    const size_t need = sad::workspace_bytes(ctx->H, ctx->W, ctx->N);
    if (b->workspace_bytes < need)
        return fail(ctx, SAD_ERR_INVALID_ARG, "workspace has %zu bytes, needs %zu", b->workspace_bytes, need);
    ctx->buf = *b;
    sad::Dev &d = ctx->dev;
    d.H = ctx->H;
    d.W = ctx->W;
    d.N = ctx->N;
    d.P = ctx->P;
    d.cell = ctx->cell;
    d.GH = ctx->GH;
    d.GW = ctx->GW;
    d.PT = ctx->PT;
    d.params = b->params;
    d.grads = b->grads;
    d.adam_m = b->adam_m;
    d.adam_v = b->adam_v;
    d.records = reinterpret_cast<float4 *>(b->records);
    d.table = b->table;
    d.target = b->target;
    d.image = b->image;
    d.stats = b->stats;
    d.frozen = b->frozen;
    d.cand16 = reinterpret_cast<uint4 *>(b->cand16);
    d.f16 = d.f16 && d.cand16;
    d.ws = b->workspace;
    // best effort: the launchers set the attributes themselves when this
    // fails (binding needs no device, only valid pointers)
    if (sad::prepare_fused() != cudaSuccess) (void)cudaGetLastError();
    ctx->bound = true;
    ctx->err[0] = 0;
    return SAD_OK;
}

int sad_reset(sad_ctx *ctx, uint32_t seed, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    cudaStream_t st = cs(stream);
    const size_t pn = sizeof(float) * 9 * (size_t)ctx->N;
    cudaError_t e = cudaMemsetAsync(ctx->buf.grads, 0, pn, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->buf.adam_m, 0, pn, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->buf.adam_v, 0, pn, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->buf.workspace, 0, ctx->buf.workspace_bytes, st);
    if (e == cudaSuccess && ctx->buf.stats) e = cudaMemsetAsync(ctx->buf.stats, 0, sizeof(float) * 6 * (size_t)ctx->N, st);
    if (e == cudaSuccess) e = sad::launch_init_counters(ctx->dev, seed, st);
    return cuda_status(ctx, e, "reset");
}

int sad_set_sites(sad_ctx *ctx, const float *src, int n, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (n < 0 || (n > 0 && !src)) return fail(ctx, SAD_ERR_INVALID_ARG, "bad site source (n=%d)", n);
    if (n > ctx->N) return fail(ctx, SAD_ERR_CAPACITY, "%d sites exceed the capacity %d", n, ctx->N);
    cudaStream_t st = cs(stream);
    cudaError_t e = cudaSuccess;
    if (n > 0)
        e = cudaMemcpy2DAsync(ctx->buf.params, sizeof(float) * (size_t)ctx->N, src, sizeof(float) * (size_t)n,
                              sizeof(float) * (size_t)n, 9, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = sad::launch_mark_inactive(ctx->dev, n, st);
    if (e == cudaSuccess) e = sad::launch_records(ctx->dev, st);
    return cuda_status(ctx, e, "set sites");
}

int sad_get_sites(sad_ctx *ctx, float *dst, int n, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (n < 0 || n > ctx->N || (n > 0 && !dst)) return fail(ctx, SAD_ERR_INVALID_ARG, "bad site destination");
    cudaStream_t st = cs(stream);
    if (n == 0) return SAD_OK;
    cudaError_t e = cudaMemcpy2DAsync(dst, sizeof(float) * (size_t)n, ctx->buf.params, sizeof(float) * (size_t)ctx->N,
                                      sizeof(float) * (size_t)n, 9, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return cuda_status(ctx, e, "get sites");
}

int sad_set_target(sad_ctx *ctx, const float *src, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!src) return fail(ctx, SAD_ERR_INVALID_ARG, "target source is NULL");
    cudaError_t e = cudaMemcpyAsync(ctx->buf.target, src, sizeof(float) * 3 * (size_t)ctx->P, cudaMemcpyDefault,
                                    cs(stream));
    return cuda_status(ctx, e, "set target");
}

int sad_set_target_u8(sad_ctx *ctx, const uint8_t *src, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!src) return fail(ctx, SAD_ERR_INVALID_ARG, "target source is NULL");
    return cuda_status(ctx, sad::launch_target_u8(ctx->dev, src, cs(stream)), "set target (8-bit)");
}

int sad_bind_target(sad_ctx *ctx, const float *target) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!target) return fail(ctx, SAD_ERR_INVALID_ARG, "target is NULL");
    if (!aligned16(target)) return fail(ctx, SAD_ERR_INVALID_ARG, "target is not 16-byte aligned");
    ctx->buf.target = const_cast<float *>(target);
    ctx->dev.target = const_cast<float *>(target);
    return SAD_OK;
}

int sad_prep_records(sad_ctx *ctx, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    return cuda_status(ctx, sad::launch_records(ctx->dev, cs(stream)), "records");
}

int sad_topk_exact(sad_ctx *ctx, const int64_t *pixels, int64_t n_pix, uint32_t *out, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!pixels) n_pix = ctx->PT;
    if (n_pix < 0 || (n_pix > 0 && !out)) return fail(ctx, SAD_ERR_INVALID_ARG, "bad top-K output");
    if (out && !aligned16(out)) return fail(ctx, SAD_ERR_INVALID_ARG, "top-K output is not 16-byte aligned");
    return cuda_status(ctx, sad::launch_topk_exact(ctx->dev, pixels, n_pix, out, cs(stream)), "topk_exact");
}

int sad_refresh(sad_ctx *ctx, int G, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (G < 0 || G > SAD_MAX_INJECT) return fail(ctx, SAD_ERR_CAPACITY, "G=%d outside [0, %d]", G, SAD_MAX_INJECT);
    return run_refresh(ctx, G, cs(stream));
}

int sad_jfa_prepass(sad_ctx *ctx, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    cudaStream_t st = cs(stream);
    r = cuda_status(ctx, sad::launch_seed(ctx->dev, st), "seed");
    if (r) return r;
    int n = 0;
    const int m = ctx->GH > ctx->GW ? ctx->GH : ctx->GW;
    while ((1 << n) < m) ++n;
    if (n == 0) n = 1;
    // the records stay as they are: each pass after the first starts from its
    // own list's stored scores
    for (int q = n - 1; q >= 0; --q) {
        r = cuda_status(ctx, sad::launch_jfa3x3(ctx->dev, 1 << q, st, q == n - 1 ? 1 : 2), "jfa pass");
        if (r) return r;
    }
    return SAD_OK;
}

int sad_propagate(sad_ctx *ctx, int jump, int G, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (jump < 1) return fail(ctx, SAD_ERR_INVALID_ARG, "jump must be >= 1");
    if (G < 0 || G > SAD_MAX_INJECT) return fail(ctx, SAD_ERR_CAPACITY, "G=%d outside [0, %d]", G, SAD_MAX_INJECT);
    r = pack_candidates(ctx, cs(stream));
    if (r) return r;
    return cuda_status(ctx, sad::launch_propagate(ctx->dev, jump, G, cs(stream)), "propagate");
}

int sad_set_candidate_precision(sad_ctx *ctx, int bits, sad_stream_t stream) {
    (void)stream;
    int r = need_bound(ctx);
    if (r) return r;
    if (bits != 32 && bits != 16) return fail(ctx, SAD_ERR_INVALID_ARG, "candidate precision must be 32 or 16 bits");
    if (bits == 16 && !ctx->dev.cand16) return fail(ctx, SAD_ERR_NOT_BOUND, "16-bit candidates need a bound cand16 buffer");
    ctx->dev.f16 = bits == 16;
    return SAD_OK;
}

int sad_set_list_staging(sad_ctx *ctx, int mode, sad_stream_t stream) {
    (void)stream;
    int r = need_bound(ctx);
    if (r) return r;
    if (mode != SAD_STAGING_LOADS && mode != SAD_STAGING_TMA)
        return fail(ctx, SAD_ERR_INVALID_ARG, "list staging mode must be SAD_STAGING_LOADS or SAD_STAGING_TMA");
    ctx->dev.tma_staging = mode == SAD_STAGING_TMA;
    return SAD_OK;
}

int sad_render(sad_ctx *ctx, float *image, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!image) image = ctx->buf.image;
    if (!image) return fail(ctx, SAD_ERR_INVALID_ARG, "no image buffer given or bound");
    if (!aligned16(image)) return fail(ctx, SAD_ERR_INVALID_ARG, "image is not 16-byte aligned");
    return cuda_status(ctx, sad::launch_render(ctx->dev, image, cs(stream)), "render");
}

int sad_backward(sad_ctx *ctx, uint32_t flags, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (flags & ~(SAD_STATS | SAD_DETERMINISTIC))
        return fail(ctx, SAD_ERR_UNSUPPORTED, "backward flags 0x%x not supported", flags);
    if ((flags & SAD_STATS) && (flags & SAD_DETERMINISTIC))
        return fail(ctx, SAD_ERR_UNSUPPORTED, "SAD_DETERMINISTIC carries the gradients only, not SAD_STATS");
    if (flags & SAD_DETERMINISTIC)
        return cuda_status(ctx, sad::launch_render_backward_det(ctx->dev, cs(stream)), "backward (deterministic)");
    if (flags & SAD_STATS) {
        if (!ctx->buf.stats) return fail(ctx, SAD_ERR_NOT_BOUND, "SAD_STATS needs a bound stats buffer");
        return cuda_status(ctx, sad::launch_fit_tile_cached_stats(ctx->dev, cs(stream)), "backward (stats)");
    }
    return cuda_status(ctx, sad::launch_fit_tile_cached(ctx->dev, cs(stream)), "backward");
}

int sad_densify_prune(sad_ctx *ctx, const sad_densify_cfg *cfg, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!cfg) return fail(ctx, SAD_ERR_INVALID_ARG, "densify config is NULL");
    if (!ctx->buf.stats) return fail(ctx, SAD_ERR_NOT_BOUND, "densify needs a bound stats buffer");
    if (!(cfg->prune_frac >= 0.0f && cfg->prune_frac <= 1.0f) || !(cfg->alpha >= 0.0f) || !(cfg->eps > 0.0f) ||
        !(cfg->r_scale >= 0.0f) || !(cfg->offset_scale >= 0.0f) || !(cfg->fallback_offset >= 0.0f) ||
        !(cfg->log_tau_shift == cfg->log_tau_shift))
        return fail(ctx, SAD_ERR_INVALID_ARG, "densify config out of range");
    sad::DensifyArgs a;
    a.grow = cfg->grow;
    a.prune_frac = cfg->prune_frac;
    a.alpha = cfg->alpha;
    a.eps = cfg->eps;
    a.r_scale = cfg->r_scale;
    a.log_tau_shift = cfg->log_tau_shift;
    a.offset_scale = cfg->offset_scale;
    a.fallback_offset = cfg->fallback_offset;
    cudaStream_t st = cs(stream);
    cudaError_t e = sad::launch_densify(ctx->dev, a, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->buf.stats, 0, sizeof(float) * 6 * (size_t)ctx->N, st);
    if (e == cudaSuccess) e = sad::launch_records(ctx->dev, st);
    return cuda_status(ctx, e, "densify");
}

int sad_tau_diffuse(sad_ctx *ctx, float lambda, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!(lambda >= 0.0f && lambda <= 1.0f)) return fail(ctx, SAD_ERR_INVALID_ARG, "lambda must lie in [0, 1]");
    return cuda_status(ctx, sad::launch_tau_diffuse(ctx->dev, lambda, cs(stream)), "tau diffusion");
}

int sad_adam_step(sad_ctx *ctx, const sad_adam_cfg *cfg, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    sad::AdamHyper h;
    r = check_adam(ctx, cfg, h);
    if (r) return r;
    return cuda_status(ctx, sad::launch_adam(ctx->dev, h, cs(stream)), "adam");
}

int sad_fit_iteration(sad_ctx *ctx, int G, const sad_adam_cfg *cfg, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (G < 0 || G > SAD_MAX_INJECT) return fail(ctx, SAD_ERR_CAPACITY, "G=%d outside [0, %d]", G, SAD_MAX_INJECT);
    sad::AdamHyper h;
    r = check_adam(ctx, cfg, h);
    if (r) return r;
    cudaStream_t st = cs(stream);
    if (ctx->cell == 1 && !ctx->dev.f16) {
        // the fused pass, then Adam, whose first block also finishes the pass
        unsigned tiles = 0;
        r = cuda_status(ctx, sad::launch_fit_tile(ctx->dev, G, st, &tiles), "fit pass");
        if (r) return r;
        return cuda_status(ctx, sad::launch_adam(ctx->dev, h, st, tiles), "adam");
    }
    r = run_fit_pass(ctx, G, st);
    if (r) return r;
    return cuda_status(ctx, sad::launch_adam(ctx->dev, h, st), "adam");
}

int sad_fit_pass_cached(sad_ctx *ctx, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    return cuda_status(ctx, sad::launch_fit_tile_cached(ctx->dev, cs(stream)), "fit pass (cached lists)");
}

int sad_fit_pass(sad_ctx *ctx, int G, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (G < 0 || G > SAD_MAX_INJECT) return fail(ctx, SAD_ERR_CAPACITY, "G=%d outside [0, %d]", G, SAD_MAX_INJECT);
    return run_fit_pass(ctx, G, cs(stream));
}

int sad_pack_sites(sad_ctx *ctx, uint32_t *packed, float *range, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!packed) return fail(ctx, SAD_ERR_INVALID_ARG, "packed destination is NULL");
    if (!aligned16(packed)) return fail(ctx, SAD_ERR_INVALID_ARG, "packed destination is not 16-byte aligned");
    cudaStream_t st = cs(stream);
    cudaError_t e = sad::launch_pack(ctx->dev, packed, st);
    if (e == cudaSuccess && range)
        e = cudaMemcpyAsync(range, sad::pack_range_device(ctx->dev), 6 * sizeof(float), cudaMemcpyDefault, st);
    return cuda_status(ctx, e, "pack sites");
}

int sad_unpack_sites(sad_ctx *ctx, const uint32_t *packed, const float *range, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!packed || !range) return fail(ctx, SAD_ERR_INVALID_ARG, "packed source or range is NULL");
    if (!aligned16(packed)) return fail(ctx, SAD_ERR_INVALID_ARG, "packed source is not 16-byte aligned");
    cudaStream_t st = cs(stream);
    float *dr = sad::pack_range_device(ctx->dev);
    cudaError_t e = cudaMemcpyAsync(dr, range, 6 * sizeof(float), cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = sad::launch_unpack(ctx->dev, packed, dr, st);
    if (e == cudaSuccess) e = sad::launch_records(ctx->dev, st);
    return cuda_status(ctx, e, "unpack sites");
}

int sad_set_candidate_grid(sad_ctx *ctx, int cell, sad_stream_t stream) {
    if (!ctx) return SAD_ERR_INVALID_ARG;
    const int m = ctx->H > ctx->W ? ctx->H : ctx->W;
    if (cell < 1 || cell > m) return fail(ctx, SAD_ERR_INVALID_ARG, "cell size %d outside [1, %d]", cell, m);
    ctx->cell = cell;
    ctx->GH = (ctx->H + cell - 1) / cell;
    ctx->GW = (ctx->W + cell - 1) / cell;
    ctx->PT = (long long)ctx->GH * ctx->GW;
    if (!ctx->bound) return SAD_OK;
    sad::Dev &d = ctx->dev;
    d.cell = ctx->cell;
    d.GH = ctx->GH;
    d.GW = ctx->GW;
    d.PT = ctx->PT;
    // the lists of the old grid mean nothing on the new one: start empty
    return cuda_status(ctx, sad::launch_clear_table(d, cs(stream)), "clear table");
}

int sad_get_table(sad_ctx *ctx, uint32_t *dst, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!dst) return fail(ctx, SAD_ERR_INVALID_ARG, "table destination is NULL");
    cudaStream_t st = cs(stream);
    sad::Counters c;
    r = read_counters(ctx, &c, st);
    if (r) return r;
    const uint32_t *plane0 = ctx->buf.table + (size_t)c.cur * ctx->PT * SAD_K;
    const uint32_t *plane1 = plane0 + (size_t)ctx->PT * 4;
    cudaError_t e = cudaMemcpy2DAsync(dst, 32, plane0, 16, 16, (size_t)ctx->PT, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = cudaMemcpy2DAsync(dst + 4, 32, plane1, 16, 16, (size_t)ctx->PT, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return cuda_status(ctx, e, "get table");
}

int sad_set_table(sad_ctx *ctx, const uint32_t *src, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!src) return fail(ctx, SAD_ERR_INVALID_ARG, "table source is NULL");
    cudaStream_t st = cs(stream);
    sad::Counters c;
    r = read_counters(ctx, &c, st);
    if (r) return r;
    uint32_t *plane0 = ctx->buf.table + (size_t)c.cur * ctx->PT * SAD_K;
    uint32_t *plane1 = plane0 + (size_t)ctx->PT * 4;
    cudaError_t e = cudaMemcpy2DAsync(plane0, 16, src, 32, 16, (size_t)ctx->PT, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = cudaMemcpy2DAsync(plane1, 16, src + 4, 32, 16, (size_t)ctx->PT, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return cuda_status(ctx, e, "set table");
}

int sad_get_stats(sad_ctx *ctx, sad_stats *out, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!out) return fail(ctx, SAD_ERR_INVALID_ARG, "stats destination is NULL");
    sad::Counters c;
    r = read_counters(ctx, &c, cs(stream));
    if (r) return r;
    out->hash_overflow = c.hash_overflow;
    out->nonfinite_pixels = c.nonfinite_pixels;
    out->empty_pixels = c.empty_pixels;
    out->dropped_ids = c.dropped_ids;
    out->pass_counter = c.pass_counter;
    out->adam_step = c.adam_step;
    out->current_table = c.cur;
    out->staging_fallbacks = c.staging_fallbacks;
    out->loss = c.loss;
    uint32_t hdr[4] = {0, 0, 0, 0};
    cudaError_t e = cudaMemcpy(hdr, reinterpret_cast<char *>(ctx->buf.workspace) + sad::densify_offset(ctx->H, ctx->W),
                               sizeof(hdr), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(ctx, e, "read densify header");
    out->n_split = hdr[0];
    out->n_pruned = hdr[1];
    out->n_active = hdr[2];
    out->check_failures = (uint32_t)(c.check_failures > 0xFFFFFFFFull ? 0xFFFFFFFFull : c.check_failures);
    return SAD_OK;
}

int sad_get_fit_state(sad_ctx *ctx, sad_fit_state *out, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!out) return fail(ctx, SAD_ERR_INVALID_ARG, "fit state destination is NULL");
    sad::Counters c;
    r = read_counters(ctx, &c, cs(stream));
    if (r) return r;
    out->pass_counter = c.pass_counter;
    out->adam_step = c.adam_step;
    out->seed = c.seed;
    out->reserved = 0;
    return SAD_OK;
}

int sad_set_fit_state(sad_ctx *ctx, const sad_fit_state *state, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!state) return fail(ctx, SAD_ERR_INVALID_ARG, "fit state is NULL");
    if (state->reserved != 0) return fail(ctx, SAD_ERR_INVALID_ARG, "fit state: reserved field must be 0");
    return cuda_status(ctx, sad::launch_set_fit_state(ctx->dev, state->pass_counter, state->adam_step, state->seed,
                                                      cs(stream)),
                       "set fit state");
}

int sad_get_loss(sad_ctx *ctx, double *loss, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!loss) return fail(ctx, SAD_ERR_INVALID_ARG, "loss destination is NULL");
    cudaStream_t st = cs(stream);
    cudaError_t e = cudaMemcpyAsync(loss, &reinterpret_cast<sad::Counters *>(ctx->buf.workspace)->loss,
                                    sizeof(double), cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return cuda_status(ctx, e, "get loss");
}

int sad_copy_loss(sad_ctx *ctx, double *dst, sad_stream_t stream) {
    int r = need_bound(ctx);
    if (r) return r;
    if (!dst) return fail(ctx, SAD_ERR_INVALID_ARG, "loss destination is NULL");
    cudaError_t e = cudaMemcpyAsync(dst, &reinterpret_cast<sad::Counters *>(ctx->buf.workspace)->loss,
                                    sizeof(double), cudaMemcpyDefault, cs(stream));
    return cuda_status(ctx, e, "copy loss");
}

const char *sad_last_error(const sad_ctx *ctx) { return ctx ? ctx->err : "context is NULL"; }

}  // extern "C"
