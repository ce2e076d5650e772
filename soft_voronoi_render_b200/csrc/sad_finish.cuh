// sad_finish.cuh -- the end of a fitting pass (loss sum, table flip), shared
// by its own one-block launch and by the Adam launch that follows the pass in
// a fitting iteration.
#pragma once

#include "sad_device.cuh"

namespace sad {

// The end of a fitting pass, once every tile is done, run by one block of
// FINISH_THREADS threads: the loss from the tiles' partials (summed in
// double, always in the same order) and, for the propagating form, the other
// table made current and the pass counter advanced.
constexpr int FINISH_THREADS = 256;

__device__ __forceinline__ void finish_pass_block(void *ws, unsigned n_tiles, double P, int prop) {
    Counters *c = ws_counters(ws);
    const double *lp = ws_loss_partials(ws);
    // eight partials in flight per thread, added in index order
    double s = 0.0;
    unsigned q = threadIdx.x;
    for (; q + 7 * FINISH_THREADS < n_tiles; q += 8 * FINISH_THREADS) {
        double x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = lp[q + k * FINISH_THREADS];
#pragma unroll
        for (int k = 0; k < 8; ++k) s += x[k];
    }
    for (; q < n_tiles; q += FINISH_THREADS) s += lp[q];
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    __shared__ double red[FINISH_THREADS / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        s = threadIdx.x < FINISH_THREADS / 32 ? red[threadIdx.x] : 0.0;
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (threadIdx.x == 0) {
            if (n_tiles) c->loss = s / P;  // a pass without render leaves the loss alone
            c->tile_ticket = 0u;
            if (prop) {
                c->cur ^= 1u;
                c->pass_counter += 1u;
            }
        }
    }
}

}  // namespace sad
