// sad_launch.h -- host-side launchers of the libsad kernels (internal).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace sad {

struct Dev {
    int H, W, N;
    long long P;
    int cell, GH, GW;  // candidate grid: ceil(H/cell) x ceil(W/cell) lists
    long long PT;      // GH * GW
    float *params, *grads, *adam_m, *adam_v;
    float4 *records;
    uint32_t *table;  // [2][2][PT][4]
    float *target, *image;
    float *stats;  // [6][N] budget-control statistics (optional)
    const uint8_t *frozen;  // [N] sites Adam leaves untouched (optional)
    uint4 *cand16;          // [N] packed candidate-site records (optional)
    bool f16;               // candidate updates rank on cand16
    bool tma_staging;       // propagating fit pass: persistent blocks, TMA-staged list blocks
    void *ws;
};

struct DensifyArgs {
    int grow;
    float prune_frac, alpha, eps, r_scale, log_tau_shift, offset_scale, fallback_offset;
};

struct AdamHyper {
    float lr[9];
    float beta1, beta2, eps;
};

size_t workspace_bytes(int H, int W, int N);
size_t densify_offset(int H, int W);

cudaError_t launch_init_counters(const Dev &d, uint32_t seed, cudaStream_t st);
cudaError_t launch_set_fit_state(const Dev &d, uint32_t pass_counter, uint32_t adam_step, uint32_t seed,
                                 cudaStream_t st);
cudaError_t launch_mark_inactive(const Dev &d, int from, cudaStream_t st);
cudaError_t launch_records(const Dev &d, cudaStream_t st);
cudaError_t launch_target_u8(const Dev &d, const uint8_t *src, cudaStream_t st);
cudaError_t launch_topk_exact(const Dev &d, const int64_t *pix, int64_t n, uint32_t *out, cudaStream_t st);
cudaError_t launch_seed(const Dev &d, cudaStream_t st);
cudaError_t launch_clear_table(const Dev &d, cudaStream_t st);
// score_cache (float32 ranking only): 0 = none, 1 = store the new lists'
// scores in the workspace, 2 = also take the own lists' scores from there
// (only between passes over unchanged records, i.e. within one refresh)
cudaError_t launch_propagate(const Dev &d, int jump, int G, cudaStream_t st, int score_cache = 0);
cudaError_t launch_pack_cand16(const Dev &d, cudaStream_t st);
cudaError_t launch_render(const Dev &d, float *image, cudaStream_t st);
cudaError_t launch_render_backward_det(const Dev &d, cudaStream_t st);
cudaError_t launch_densify(const Dev &d, const DensifyArgs &a, cudaStream_t st);
cudaError_t launch_tau_diffuse(const Dev &d, float lambda, cudaStream_t st);
cudaError_t launch_jfa3x3(const Dev &d, int jump, cudaStream_t st, int score_cache = 0);
cudaError_t launch_fit_tile_cached(const Dev &d, cudaStream_t st);
// a jump-1 or jump-2 propagation pass by the tile kernel (pixel grid,
// float32 ranking)
cudaError_t launch_propagate_tile(const Dev &d, int jump, int G, cudaStream_t st);
cudaError_t launch_fit_tile_cached_stats(const Dev &d, cudaStream_t st);
// the cached-list tile pass with order-independent sums into fixed ([NPARAM][N]
// 64-bit fixed point, 2^-40 units)
cudaError_t launch_fit_tile_cached_det(const Dev &d, unsigned long long *fixed, cudaStream_t st);
// finish_tiles > 0: block 0 also finishes the fitting pass that wrote that
// many tile partials (the propagating form), saving that pass its own launch
cudaError_t launch_adam(const Dev &d, const AdamHyper &h, cudaStream_t st, unsigned finish_tiles = 0);
// finish_tiles: where given, the pass's finishing step is left to the caller
cudaError_t launch_fit_tile(const Dev &d, int G, cudaStream_t st, unsigned *finish_tiles = nullptr);
cudaError_t prepare_fused();
float *pack_range_device(const Dev &d);
cudaError_t launch_pack(const Dev &d, uint32_t *packed, cudaStream_t st);
cudaError_t launch_unpack(const Dev &d, const uint32_t *packed, const float *range, cudaStream_t st);

}  // namespace sad
