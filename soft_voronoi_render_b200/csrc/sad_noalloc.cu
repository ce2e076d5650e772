// sad_noalloc.cu -- render + loss + backward for callers that cannot allocate.
//
// Every other entry point runs on caller-bound buffers, including a
// caller-provided workspace.  Some callers cannot provide one: code that runs
// inside another framework's fixed memory budget, plugin interfaces that hand
// over only input and output pointers, or latency-critical paths that must
// not call cudaMalloc (it can synchronise the device).  For them this file
// keeps the backward pass's scratch (a 256-byte counter block and one double
// per tile of at least 32 x 8 pixels for the loss partials) in a file-scope device array that the
// library owns for the life of the process, on every GPU that loads it.
#include <atomic>
#include <cstdint>

#include "sad.h"
#include "sad_device.cuh"
#include "sad_launch.h"

namespace {

constexpr size_t kScratchBytes = SAD_NOALLOC_SCRATCH_BYTES;
constexpr int kTileX = 32, kTileY = 8;  // the smallest tile of the render + backward kernel
constexpr int kMaxDevices = 64;
constexpr int kMaxGridY = 65535;  // launch limit on the tile rows (gridDim.y)

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of g_noalloc_scratch per device ordinal, filled on the first
// call on that device.  Threads that make a first call at the same time look
// the address up each and store the same value, so a relaxed atomic suffices.
// The address belongs to the device's primary context: after a
// cudaDeviceReset it is stale and the process must not call this entry point
// again on that device.
std::atomic<void *> g_scratch_addr[kMaxDevices];

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int sad_backward_noalloc(int H, int W, int N_cap, const float *records, const uint32_t *table,
                                    const float *target, float *image, float *grads, double *loss,
                                    sad_stream_t stream) {
    if (H < 1 || W < 1 || N_cap < 1 || (long long)H * W >= (1ll << 31)) return SAD_ERR_INVALID_ARG;
    if (!records || !table || !target || !grads || !loss) return SAD_ERR_INVALID_ARG;
    if (!aligned(records, 32) || !aligned(table, 16) || !aligned(target, 16) || !aligned(grads, 16) ||
        (image && !aligned(image, 16)) || !aligned(loss, 8))
        return SAD_ERR_INVALID_ARG;
    const size_t tiles = (size_t)((W + kTileX - 1) / kTileX) * (size_t)((H + kTileY - 1) / kTileY);
    if (sad::COUNTERS_BYTES + tiles * sizeof(double) > kScratchBytes) return SAD_ERR_CAPACITY;
    if ((H + kTileY - 1) / kTileY > kMaxGridY) return SAD_ERR_CAPACITY;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SAD_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SAD_ERR_UNSUPPORTED;
    void *scratch = g_scratch_addr[dev].load(std::memory_order_relaxed);
    if (!scratch) {
        // host code only sees a stand-in for the array: ask for its address on
        // this device (a one-time set-up; do it before any stream capture)
        if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || !scratch) return SAD_ERR_CUDA;
        g_scratch_addr[dev].store(scratch, std::memory_order_relaxed);
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // a launch error read below must be this call's own, not one left pending
    // by earlier work of the caller
    (void)cudaGetLastError();

    // the array keeps the previous call's contents: the counters (current
    // table 0, last-tile ticket, statistics) must start at zero
    if (cudaMemsetAsync(scratch, 0, sad::COUNTERS_BYTES, st) != cudaSuccess) return SAD_ERR_CUDA;

    sad::Dev d{};
    d.H = H;
    d.W = W;
    d.N = N_cap;
    d.P = (long long)H * W;
    d.cell = 1;  // lists on the pixel grid
    d.GH = H;
    d.GW = W;
    d.PT = d.P;
    d.records = reinterpret_cast<float4 *>(const_cast<float *>(records));
    d.table = const_cast<uint32_t *>(table);
    d.target = const_cast<float *>(target);
    d.image = image;
    d.grads = grads;
    d.ws = scratch;
    if (sad::launch_fit_tile_cached(d, st) != cudaSuccess) return SAD_ERR_CUDA;
    const double *src = &reinterpret_cast<const sad::Counters *>(scratch)->loss;
    if (cudaMemcpyAsync(loss, src, sizeof(double), cudaMemcpyDeviceToDevice, st) != cudaSuccess) return SAD_ERR_CUDA;
    return SAD_OK;
}
