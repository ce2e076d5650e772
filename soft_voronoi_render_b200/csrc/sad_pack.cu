// sad_pack.cu -- the 16-byte evaluation record of a site ("Soft Anisotropic
// Diagrams for Differentiable Image Representation", summary B.2 "Packed
// storage for evaluation": the semantic values of a site quantised into four
// 32-bit words, with per-image min/scale values for ln tau and the radius).
//
// Field string (little-endian, 128 bits; bit offset and width):
//   x 0 (18)  y 18 (18)  cr 36 (10)  cg 46 (10)  cb 56 (10)
//   ln tau 66 (16)  r 82 (14)  theta 96 (14)  a 110 (14)  active 127 (1)
// Positions are 2^18 cells across the image, decoded at the cell centre;
// colours are clamped to [0, 1] in 1023 steps; ln tau, r and a map the
// per-image [lo, hi] of the active sites onto 2^b - 1 steps; theta is the
// axis angle (theta mod pi, which is all G depends on) in 2^14 steps.  All
// quantisation arithmetic is double with explicit round-to-nearest
// operations, rounded half up; decoded values are rounded once to float32.
// An inactive site packs to four zero words and decodes to x = -1.
#include <cstddef>

#include "sad_device.cuh"
#include "sad_launch.h"

namespace sad {

namespace {

constexpr int PACK_THREADS = 256;
constexpr double PI_D = 3.14159265358979323846;
constexpr double XY_CELLS = 262144.0;   // 2^18
constexpr double COLOUR_TOP = 1023.0;   // 2^10 - 1
constexpr double THETA_STEPS = 16384.0; // 2^14

struct Field {
    int off, bits;
};
constexpr Field F_X{0, 18}, F_Y{18, 18}, F_CR{36, 10}, F_CG{46, 10}, F_CB{56, 10}, F_LT{66, 16}, F_R{82, 14},
    F_TH{96, 14}, F_A{110, 14}, F_ACTIVE{127, 1};

// order-preserving map of a float onto uint32 (for atomicMin/atomicMax)
__device__ __forceinline__ uint32_t float_order(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_float(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

struct Bits128 {
    unsigned long long lo, hi;
    __device__ __forceinline__ void put(Field f, uint32_t v) {
        const unsigned long long x = (unsigned long long)v;
        if (f.off + f.bits <= 64) {
            lo |= x << f.off;
        } else if (f.off >= 64) {
            hi |= x << (f.off - 64);
        } else {
            lo |= x << f.off;
            hi |= x >> (64 - f.off);
        }
    }
    __device__ __forceinline__ uint32_t get(Field f) const {
        const unsigned long long mask = (1ull << f.bits) - 1ull;
        unsigned long long x;
        if (f.off + f.bits <= 64) {
            x = lo >> f.off;
        } else if (f.off >= 64) {
            x = hi >> (f.off - 64);
        } else {
            x = (lo >> f.off) | (hi << (64 - f.off));
        }
        return (uint32_t)(x & mask);
    }
};

// floor(t + 1/2) clamped to [0, top]; NaN -> 0
__device__ __forceinline__ uint32_t round_clamp(double t, double top) {
    if (t != t) return 0u;
    t = floor(__dadd_rn(t, 0.5));
    t = t < 0.0 ? 0.0 : (t > top ? top : t);
    return (uint32_t)t;
}

__device__ __forceinline__ uint32_t cell_clamp(double t, double cells) {
    if (t != t) return 0u;
    t = floor(t);
    t = t < 0.0 ? 0.0 : (t > cells - 1.0 ? cells - 1.0 : t);
    return (uint32_t)t;
}

__device__ __forceinline__ uint32_t range_q(float v, float lo, float hi, int bits) {
    const double top = (double)((1u << bits) - 1u);
    if (!((double)hi > (double)lo)) return 0u;
    const double t = __dmul_rn(__ddiv_rn(__dsub_rn((double)v, (double)lo), __dsub_rn((double)hi, (double)lo)), top);
    return round_clamp(t, top);
}

__device__ __forceinline__ float range_v(uint32_t q, float lo, float hi, int bits) {
    const double top = (double)((1u << bits) - 1u);
    return (float)__dadd_rn((double)lo, __dmul_rn((double)q, __ddiv_rn(__dsub_rn((double)hi, (double)lo), top)));
}

__global__ void pack_range_init_kernel(Counters *c) {
    if (threadIdx.x < 3) {
        c->pack_ord[threadIdx.x] = 0xFFFFFFFFu;     // running minimum
        c->pack_ord[3 + threadIdx.x] = 0u;          // running maximum
    }
}

// per-image lo/hi of ln tau, r and a over the active sites
__global__ void __launch_bounds__(PACK_THREADS) pack_range_kernel(const float *__restrict__ prm, int N,
                                                                  Counters *c) {
    const int i = blockIdx.x * PACK_THREADS + threadIdx.x;
    const size_t n = (size_t)N;
    uint32_t lo[3] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu}, hi[3] = {0u, 0u, 0u};
    if (i < N && prm[PX * n + i] >= 0.0f) {
        const int planes[3] = {PLT, PR, PA};
#pragma unroll
        for (int f = 0; f < 3; ++f) {
            const float v = __fadd_rn(prm[planes[f] * n + i], 0.0f);  // -0 -> +0
            if (v == v) {
                lo[f] = float_order(v);
                hi[f] = float_order(v);
            }
        }
    }
#pragma unroll
    for (int f = 0; f < 3; ++f) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo[f] = min(lo[f], __shfl_xor_sync(0xffffffffu, lo[f], o));
            hi[f] = max(hi[f], __shfl_xor_sync(0xffffffffu, hi[f], o));
        }
    }
    if ((threadIdx.x & 31) == 0) {
#pragma unroll
        for (int f = 0; f < 3; ++f) {
            if (lo[f] != 0xFFFFFFFFu) atomicMin(&c->pack_ord[f], lo[f]);
            if (hi[f] != 0u) atomicMax(&c->pack_ord[3 + f], hi[f]);
        }
    }
}

__global__ void pack_range_final_kernel(Counters *c) {
    if (threadIdx.x < 3) {
        const uint32_t lo = c->pack_ord[threadIdx.x], hi = c->pack_ord[3 + threadIdx.x];
        const bool any = lo != 0xFFFFFFFFu;  // no active site: the range is (0, 0)
        c->pack_range[threadIdx.x] = any ? order_float(lo) : 0.0f;
        c->pack_range[3 + threadIdx.x] = any ? order_float(hi) : 0.0f;
    }
}

__global__ void __launch_bounds__(PACK_THREADS) pack_kernel(const float *__restrict__ prm, int N, int H, int W,
                                                            const float *__restrict__ range,
                                                            uint4 *__restrict__ out) {
    const int i = blockIdx.x * PACK_THREADS + threadIdx.x;
    if (i >= N) return;
    const size_t n = (size_t)N;
    Bits128 b{0ull, 0ull};
    const float x = prm[PX * n + i];
    if (x >= 0.0f) {
        const float y = prm[PY * n + i];
        b.put(F_X, cell_clamp(__dmul_rn(__ddiv_rn((double)x, (double)W), XY_CELLS), XY_CELLS));
        b.put(F_Y, cell_clamp(__dmul_rn(__ddiv_rn((double)y, (double)H), XY_CELLS), XY_CELLS));
        const Field cf[3] = {F_CR, F_CG, F_CB};
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            double v = (double)prm[(PCR + q) * n + i];
            v = v < 0.0 ? 0.0 : (v > 1.0 ? 1.0 : v);
            b.put(cf[q], round_clamp(__dmul_rn(v, COLOUR_TOP), COLOUR_TOP));
        }
        b.put(F_LT, range_q(__fadd_rn(prm[PLT * n + i], 0.0f), range[0], range[3], F_LT.bits));
        b.put(F_R, range_q(__fadd_rn(prm[PR * n + i], 0.0f), range[1], range[4], F_R.bits));
        b.put(F_A, range_q(__fadd_rn(prm[PA * n + i], 0.0f), range[2], range[5], F_A.bits));
        double th = fmod((double)prm[PTH * n + i], PI_D);
        if (th < 0.0) th = __dadd_rn(th, PI_D);
        const uint32_t qt =
            th == th ? (uint32_t)floor(__dadd_rn(__dmul_rn(__ddiv_rn(th, PI_D), THETA_STEPS), 0.5)) : 0u;
        b.put(F_TH, qt & ((1u << F_TH.bits) - 1u));
        b.put(F_ACTIVE, 1u);
    }
    out[i] = make_uint4((uint32_t)b.lo, (uint32_t)(b.lo >> 32), (uint32_t)b.hi, (uint32_t)(b.hi >> 32));
}

__global__ void __launch_bounds__(PACK_THREADS) unpack_kernel(const uint4 *__restrict__ in, int N, int H, int W,
                                                              const float *__restrict__ range,
                                                              float *__restrict__ prm) {
    const int i = blockIdx.x * PACK_THREADS + threadIdx.x;
    if (i >= N) return;
    const size_t n = (size_t)N;
    const uint4 w = in[i];
    const Bits128 b{(unsigned long long)w.x | ((unsigned long long)w.y << 32),
                    (unsigned long long)w.z | ((unsigned long long)w.w << 32)};
    float v[NPARAM];
#pragma unroll
    for (int k = 0; k < NPARAM; ++k) v[k] = 0.0f;
    if (!b.get(F_ACTIVE)) {
        v[PX] = -1.0f;
    } else {
        v[PX] = (float)__ddiv_rn(__dmul_rn(__dadd_rn((double)b.get(F_X), 0.5), (double)W), XY_CELLS);
        v[PY] = (float)__ddiv_rn(__dmul_rn(__dadd_rn((double)b.get(F_Y), 0.5), (double)H), XY_CELLS);
        v[PCR] = (float)__ddiv_rn((double)b.get(F_CR), COLOUR_TOP);
        v[PCG] = (float)__ddiv_rn((double)b.get(F_CG), COLOUR_TOP);
        v[PCB] = (float)__ddiv_rn((double)b.get(F_CB), COLOUR_TOP);
        v[PLT] = range_v(b.get(F_LT), range[0], range[3], F_LT.bits);
        v[PR] = range_v(b.get(F_R), range[1], range[4], F_R.bits);
        v[PA] = range_v(b.get(F_A), range[2], range[5], F_A.bits);
        v[PTH] = (float)__dmul_rn((double)b.get(F_TH), __ddiv_rn(PI_D, THETA_STEPS));
    }
#pragma unroll
    for (int k = 0; k < NPARAM; ++k) prm[k * n + i] = v[k];
}

inline unsigned blocks(long long n) { return (unsigned)((n + PACK_THREADS - 1) / PACK_THREADS); }

}  // namespace

float *pack_range_device(const Dev &d) {
    return reinterpret_cast<float *>(reinterpret_cast<char *>(d.ws) + offsetof(Counters, pack_range));
}

cudaError_t launch_pack(const Dev &d, uint32_t *packed, cudaStream_t st) {
    Counters *c = reinterpret_cast<Counters *>(d.ws);
    pack_range_init_kernel<<<1, 32, 0, st>>>(c);
    pack_range_kernel<<<blocks(d.N), PACK_THREADS, 0, st>>>(d.params, d.N, c);
    pack_range_final_kernel<<<1, 32, 0, st>>>(c);
    pack_kernel<<<blocks(d.N), PACK_THREADS, 0, st>>>(d.params, d.N, d.H, d.W, pack_range_device(d),
                                                     reinterpret_cast<uint4 *>(packed));
    return cudaGetLastError();
}

cudaError_t launch_unpack(const Dev &d, const uint32_t *packed, const float *range, cudaStream_t st) {
    unpack_kernel<<<blocks(d.N), PACK_THREADS, 0, st>>>(reinterpret_cast<const uint4 *>(packed), d.N, d.H, d.W, range,
                                                       d.params);
    return cudaGetLastError();
}

}  // namespace sad
