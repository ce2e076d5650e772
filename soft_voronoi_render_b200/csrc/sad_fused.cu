// sad_fused.cu -- host launchers of the fused fitting pass (the kernel and
// its tile state are in sad_fused_kernel.cuh): the one-block finishing
// kernel, shared-memory opt-in, the persistent grid of the TMA-staged form,
// the list block's tensor map.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdlib>
#include <cstring>

#include "sad_finish.cuh"
#include "sad_fused_kernel.cuh"
#include "sad_launch.h"

namespace sad {

namespace {

// The end of a fitting pass as a launch of its own (sad_fit_iteration folds
// it into the Adam launch instead): no tile waits on a global round trip.
__global__ void __launch_bounds__(FINISH_THREADS) finish_pass_kernel(void *ws, unsigned n_tiles, double P, int prop) {
    finish_pass_block(ws, n_tiles, P, prop);
}

// the tile state exceeds the 48 KB default: opt in once per device (done
// when buffers are bound, so that a stream capture sees launches only); the
// persistent form also records how many blocks fill the device.  Threads
// that bind at the same time on one device compute and store the same
// values, so relaxed atomics suffice.
constexpr int MAX_DEV = 64;

template <int FY, bool PROP, bool STATS, bool TMA, bool BWD = true, int JK = 1, bool DET = false>
cudaError_t ensure_smem_attr(int *grid_blocks = nullptr) {
    static std::atomic<int> blocks[MAX_DEV];  // 0: not yet set up on that device; -1: no block fits
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool known = dev >= 0 && dev < MAX_DEV;
    int b = known ? blocks[dev].load(std::memory_order_relaxed) : 0;
    if (b == 0) {
        const int bytes = (int)sizeof(FusedSmem<FY, STATS, TMA, JK>);
        e = cudaFuncSetAttribute(fit_tile_kernel<FY, PROP, STATS, TMA, BWD, JK, DET>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        int per_sm = 0, sms = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &per_sm, fit_tile_kernel<FY, PROP, STATS, TMA, BWD, JK, DET>, FX * FY, (size_t)bytes);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        b = per_sm * sms > 0 ? per_sm * sms : -1;
        if (known) blocks[dev].store(b, std::memory_order_relaxed);
    }
    if (grid_blocks) *grid_blocks = b > 0 ? b : 0;
    return cudaSuccess;
}

// cuTensorMapEncodeTiled, looked up through the runtime (no link against the
// driver library); null where the driver does not offer it
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// The pixel-grid table as a 3-D array of 32-bit words for the staging copy:
// x = the 4 W words of an image row of one plane, y = the H rows, z = table
// * 2 + plane (plane stride P * 16 bytes).  The box is one tile's list block
// with its halo: 4 (FX + 2) words x (FY + 2) rows x both planes; positions
// outside the image read as zero, which the kernel masks by coordinates.
bool encode_list_map(const Dev &d, int FY, CUtensorMap *map) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode || (reinterpret_cast<uintptr_t>(d.table) & 15u) || d.cell != 1) return false;
    const cuuint64_t dims[3] = {4ull * (cuuint64_t)d.W, (cuuint64_t)d.H, 4ull};
    const cuuint64_t strides[2] = {16ull * (cuuint64_t)d.W, 16ull * (cuuint64_t)d.P};
    const cuuint32_t box[3] = {4u * HX, (cuuint32_t)FY + 2u, 2u};
    const cuuint32_t elem[3] = {1u, 1u, 1u};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, d.table, dims, strides, box, elem,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The bounds-checked build reads SAD_TEST_WITHHOLD_STAGING=1 from the
// environment and then withholds the first staging copy of every persistent
// block, so that a test can run the bounded wait's fallback to plain loads.
// The normal build never withholds a copy.
static uint32_t staging_test_flags() {
#ifdef SAD_CHECKS
    const char *v = std::getenv("SAD_TEST_WITHHOLD_STAGING");
    return (v && v[0] == '1') ? 1u : 0u;
#else
    return 0u;
#endif
}

// finish_tiles: where given, the finishing step is left to the caller (it
// gets the number of tile partials to sum); otherwise it is launched here
template <int FY, bool PROP, bool STATS>
cudaError_t launch_fit_tile_h(const Dev &d, int G, cudaStream_t st, unsigned *finish_tiles = nullptr) {
    // the propagating form works on the pixel grid only
    if (PROP && d.cell != 1) return cudaErrorInvalidValue;
    const TableGrid lists{d.cell, d.GW, (size_t)d.PT};
    const dim3 grid((d.W + FX - 1) / FX, (d.H + FY - 1) / FY);
    const uint32_t n_tiles = grid.x * grid.y;
    CUtensorMap map;
    std::memset(&map, 0, sizeof(map));
    cudaError_t e;
    bool staged = false;
    if constexpr (PROP && !STATS && FY == 16) {
        if (d.tma_staging && encode_list_map(d, FY, &map)) {
            // persistent blocks with the list block staged by TMA
            int blocks = 0;
            e = ensure_smem_attr<FY, true, false, true>(&blocks);
            if (e != cudaSuccess) return e;
            if (blocks < 1) return cudaErrorInvalidConfiguration;
            const unsigned nb = n_tiles < (uint32_t)blocks ? n_tiles : (unsigned)blocks;
            fit_tile_kernel<FY, true, false, true><<<nb, dim3(FX, FY), sizeof(FusedSmem<FY, false, true>), st>>>(
                d.records, d.table, d.target, d.H, d.W, d.N, G, d.image, d.grads, d.stats, d.ws, lists, map,
                (int)grid.x, n_tiles, nullptr, staging_test_flags());
            staged = true;
        }
    }
    if (!staged) {
        e = ensure_smem_attr<FY, PROP, STATS, false>();
        if (e != cudaSuccess) return e;
        fit_tile_kernel<FY, PROP, STATS, false><<<grid, dim3(FX, FY), sizeof(FusedSmem<FY, STATS>), st>>>(
            d.records, d.table, d.target, d.H, d.W, d.N, G, d.image, d.grads, d.stats, d.ws, lists, map,
            (int)grid.x, n_tiles);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (finish_tiles) {
        *finish_tiles = n_tiles;
        return cudaSuccess;
    }
    finish_pass_kernel<<<1, FINISH_THREADS, 0, st>>>(d.ws, n_tiles, (double)d.P, PROP ? 1 : 0);
    return cudaGetLastError();
}

// a jump-JK propagation pass (JK = 1, 2) by the tile kernel without its
// render and backward: the table flips and the pass counter advances, the
// loss stays
template <int FY, int JK>
cudaError_t launch_propagate_tile_h(const Dev &d, int G, cudaStream_t st) {
    const TableGrid lists{1, d.W, (size_t)d.P};
    cudaError_t e = ensure_smem_attr<FY, true, false, false, false, JK>();
    if (e != cudaSuccess) return e;
    const dim3 grid((d.W + FX - 1) / FX, (d.H + FY - 1) / FY);
    CUtensorMap map;
    std::memset(&map, 0, sizeof(map));
    fit_tile_kernel<FY, true, false, false, false, JK>
        <<<grid, dim3(FX, FY), sizeof(FusedSmem<FY, false, false, JK>), st>>>(
        d.records, d.table, d.target, d.H, d.W, d.N, G, nullptr, nullptr, nullptr, d.ws, lists, map, (int)grid.x,
        grid.x * grid.y);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    finish_pass_kernel<<<1, FINISH_THREADS, 0, st>>>(d.ws, 0u, (double)d.P, 1);
    return cudaGetLastError();
}

// the order-independent backward: the tile pass on the cached lists with
// its sums in 64-bit fixed point (added to grads by the caller's next step)
template <int FY>
cudaError_t launch_fit_tile_cached_det_h(const Dev &d, unsigned long long *fixed, cudaStream_t st) {
    const TableGrid lists{d.cell, d.GW, (size_t)d.PT};
    cudaError_t e = ensure_smem_attr<FY, false, false, false, true, 1, true>();
    if (e != cudaSuccess) return e;
    const dim3 grid((d.W + FX - 1) / FX, (d.H + FY - 1) / FY);
    CUtensorMap map;
    std::memset(&map, 0, sizeof(map));
    fit_tile_kernel<FY, false, false, false, true, 1, true><<<grid, dim3(FX, FY), sizeof(FusedSmem<FY, false>), st>>>(
        d.records, d.table, d.target, d.H, d.W, d.N, 0, d.image, d.grads, d.stats, d.ws, lists, map, (int)grid.x,
        grid.x * grid.y, fixed);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    finish_pass_kernel<<<1, FINISH_THREADS, 0, st>>>(d.ws, grid.x * grid.y, (double)d.P, 0);
    return cudaGetLastError();
}

// taller tiles amortise the halo and the per-tile work, but hold more
// distinct sites: use them unless sites are dense (< 4 pixels per site),
// where tiles would often exceed the 128-site index
bool tall_tiles(const Dev &d) { return (long long)d.H * d.W >= 4ll * d.N; }

}  // namespace

cudaError_t prepare_fused() {
    cudaError_t e = ensure_smem_attr<8, true, false, false>();
    if (e == cudaSuccess) e = ensure_smem_attr<16, true, false, false>();
    if (e == cudaSuccess) e = ensure_smem_attr<16, true, false, true>();
    if (e == cudaSuccess) e = ensure_smem_attr<8, false, false, false>();
    if (e == cudaSuccess) e = ensure_smem_attr<16, false, false, false>();
    if (e == cudaSuccess) e = ensure_smem_attr<8, false, true, false>();
    if (e == cudaSuccess) e = ensure_smem_attr<16, false, true, false>();
    if (e == cudaSuccess) e = ensure_smem_attr<8, true, false, false, false, 1>();
    if (e == cudaSuccess) e = ensure_smem_attr<16, true, false, false, false, 1>();
    if (e == cudaSuccess) e = ensure_smem_attr<8, true, false, false, false, 2>();
    if (e == cudaSuccess) e = ensure_smem_attr<16, true, false, false, false, 2>();
    if (e == cudaSuccess) e = ensure_smem_attr<8, false, false, false, true, 1, true>();
    if (e == cudaSuccess) e = ensure_smem_attr<16, false, false, false, true, 1, true>();
    return e;
}

cudaError_t launch_fit_tile_cached_det(const Dev &d, unsigned long long *fixed, cudaStream_t st) {
    return tall_tiles(d) ? launch_fit_tile_cached_det_h<16>(d, fixed, st)
                         : launch_fit_tile_cached_det_h<8>(d, fixed, st);
}

cudaError_t launch_propagate_tile(const Dev &d, int jump, int G, cudaStream_t st) {
    if (d.cell != 1 || d.f16 || (jump != 1 && jump != 2)) return cudaErrorInvalidValue;
    if (jump == 2)
        return tall_tiles(d) ? launch_propagate_tile_h<16, 2>(d, G, st) : launch_propagate_tile_h<8, 2>(d, G, st);
    return tall_tiles(d) ? launch_propagate_tile_h<16, 1>(d, G, st) : launch_propagate_tile_h<8, 1>(d, G, st);
}

cudaError_t launch_fit_tile(const Dev &d, int G, cudaStream_t st, unsigned *finish_tiles) {
    return tall_tiles(d) ? launch_fit_tile_h<16, true, false>(d, G, st, finish_tiles)
                         : launch_fit_tile_h<8, true, false>(d, G, st, finish_tiles);
}

cudaError_t launch_fit_tile_cached(const Dev &d, cudaStream_t st) {
    return tall_tiles(d) ? launch_fit_tile_h<16, false, false>(d, 0, st) : launch_fit_tile_h<8, false, false>(d, 0, st);
}

cudaError_t launch_fit_tile_cached_stats(const Dev &d, cudaStream_t st) {
    return tall_tiles(d) ? launch_fit_tile_h<16, false, true>(d, 0, st) : launch_fit_tile_h<8, false, true>(d, 0, st);
}

}  // namespace sad
