// sad_device.cuh -- device-side definitions shared by the libsad kernels.
//
// Soft Anisotropic Diagrams ("Soft Anisotropic Diagrams for Differentiable
// Image Representation"): logit of site i at pixel centre x
//     l_i(x) = -tau_i (s ||x - p_i||_{G_i} - s r_i),   G_i = e^a u u^T + e^-a v v^T
// (reading notes, key designs 1-2).  The kernels evaluate it from a per-site
// record holding k = tau s, (A, B, C) = k^2 (G11, G12, G22) and b = k r as
//     l = b - sqrt(dx (A dx + B dy) + dy (C dy + B dx)),
// which is the same quantity; the top-K decisions use exactly the IEEE
// operation sequence of sad_logit() below.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace sad {

constexpr int K = 8;
constexpr uint32_t EMPTY = 0xFFFFFFFFu;
constexpr int NPARAM = 9;
constexpr int NSTAT = 6;  // budget-control statistics per site
constexpr int REC_F4 = 4;  // a record is 4 float4 = 64 bytes

// parameter planes
enum : int { PX = 0, PY, PLT, PR, PCR, PCG, PCB, PTH, PA };

// Workspace layout: counters and statistics at offset 0, loss partials after.
struct Counters {
    uint32_t pass_counter;   // propagation passes run so far
    uint32_t adam_step;      // Adam steps taken so far
    uint32_t cur;            // index (0/1) of the current candidate table
    uint32_t seed;           // injection seed
    uint32_t ticket_prop;    // last-block tickets (reset by the last block)
    uint32_t ticket_bwd;
    uint32_t ticket_adam;
    uint32_t staging_fallbacks;  // list-staging copies that did not arrive in time (tiles read from global)
    unsigned long long hash_overflow;
    unsigned long long nonfinite_pixels;
    unsigned long long empty_pixels;
    unsigned long long dropped_ids;
    double loss;
    unsigned long long check_failures;  // SAD_CHECKS builds: accesses refused by a bounds check
    uint32_t tile_ticket;    // persistent fit pass: tiles handed out beyond the first wave (reset by its finish)
    uint32_t pad2;
    double pad1[5];
    uint32_t pack_ord[6];    // order-preserving encodings of the pack ranges
    float pack_range[6];     // lo ln tau, lo r, lo a, hi ln tau, hi r, hi a
};
static_assert(sizeof(Counters) <= 256, "counter block exceeds its 256-byte slot");
constexpr size_t COUNTERS_BYTES = 256;

// Where a pixel's candidate list lives: the list of its cell on a grid of
// cell x cell pixel cells (summary B.3, "Candidate field"; cell = 1 is the
// pixel grid).  PT is the number of lists, the stride of a table plane.
struct TableGrid {
    int cell, GW;
    size_t PT;
    __device__ __forceinline__ size_t cell_of(int i, int j, size_t p) const {
        return cell == 1 ? p : (size_t)(j / cell) * GW + (size_t)(i / cell);
    }
};

// The ranking fields of site x's record -- x, y, A, B, C, b, the first 24 of
// its 64 bytes -- in one 256-bit load (the last two words of the 32 are not
// kept).  The records buffer is 32-byte aligned (sad_bind and the
// allocation-free entry point refuse one that is not).
__device__ __forceinline__ void load_rank_fields(const float4 *__restrict__ rec, uint32_t x, float &px, float &py,
                                                 float &A, float &B, float &C, float &b) {
    asm("ld.global.nc.v8.f32 {%0, %1, %2, %3, %4, %5, _, _}, [%6];"
        : "=f"(px), "=f"(py), "=f"(A), "=f"(B), "=f"(C), "=f"(b)
        : "l"(rec + (size_t)x * REC_F4));
}

// ---------------------------------------------------------------------------
// ranking: (logit desc, id asc)
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool ranks_above(float la, uint32_t ia, float lb, uint32_t ib) {
    return la > lb || (la == lb && ia < ib);
}

// Fixed-order float32 logit; returns NaN for NaN inputs.  Every operation is
// an explicit round-to-nearest intrinsic so that no contraction or reordering
// can change the bits that decide the top-K.
__device__ __forceinline__ float sad_logit(float px, float py, float A, float B, float C, float b,
                                           float fx, float fy) {
    const float dx = __fsub_rn(fx, px);
    const float dy = __fsub_rn(fy, py);
    const float bdy = __fmul_rn(B, dy);
    const float bdx = __fmul_rn(B, dx);
    const float u1 = __fmaf_rn(A, dx, bdy);
    const float u2 = __fmaf_rn(C, dy, bdx);
    float q = __fmaf_rn(dx, u1, __fmul_rn(dy, u2));
    q = (q < 0.0f) ? 0.0f : q;
    return __fsub_rn(b, __fsqrt_rn(q));
}

// Same logit, also returning the pieces the backward pass needs:
// (u1, u2) = G' delta and m = sqrt(delta^T G' delta) = k n.
__device__ __forceinline__ float sad_logit_parts(float px, float py, float A, float B, float C, float b,
                                                 float fx, float fy, float &dx, float &dy, float &u1,
                                                 float &u2, float &m) {
    dx = __fsub_rn(fx, px);
    dy = __fsub_rn(fy, py);
    const float bdy = __fmul_rn(B, dy);
    const float bdx = __fmul_rn(B, dx);
    u1 = __fmaf_rn(A, dx, bdy);
    u2 = __fmaf_rn(C, dy, bdx);
    float q = __fmaf_rn(dx, u1, __fmul_rn(dy, u2));
    q = (q < 0.0f) ? 0.0f : q;
    m = __fsqrt_rn(q);
    return __fsub_rn(b, m);
}

// ---------------------------------------------------------------------------
// injection randomness (an xorshift generator seeded per pass and pixel)
// ---------------------------------------------------------------------------
// MurmurHash3 32-bit finaliser (Austin Appleby, public domain).
__device__ __forceinline__ uint32_t fmix32(uint32_t h) {
    h ^= h >> 16;
    h *= 0x85ebca6bu;
    h ^= h >> 13;
    h *= 0xc2b2ae35u;
    h ^= h >> 16;
    return h;
}

// Marsaglia's xorshift32 with shifts (13, 17, 5).
__device__ __forceinline__ uint32_t xorshift32(uint32_t x) {
    x ^= x << 13;
    x ^= x >> 17;
    x ^= x << 5;
    return x;
}

__device__ __forceinline__ uint32_t inject_state(uint32_t seed, uint32_t pass, uint32_t pixel) {
    uint32_t h = fmix32(pixel ^ fmix32(seed ^ (pass * 0x9E3779B9u)));
    return h ? h : 1u;
}

// ---------------------------------------------------------------------------
// per-thread top-8 list kept in registers
// ---------------------------------------------------------------------------
template <int KN>
struct TopN {
    float l[KN];
    uint32_t id[KN];

    __device__ __forceinline__ void clear() {
#pragma unroll
        for (int q = 0; q < KN; ++q) {
            l[q] = -__int_as_float(0x7f800000);  // -inf
            id[q] = EMPTY;
        }
    }
    __device__ __forceinline__ bool has(uint32_t x) const {
        bool h = false;
#pragma unroll
        for (int q = 0; q < KN; ++q) h |= (id[q] == x);
        return h;
    }
    // insert a candidate known not to be in the list (bubble network)
    __device__ __forceinline__ void insert(float lv, uint32_t iv) {
#pragma unroll
        for (int q = 0; q < KN; ++q) {
            const bool a = ranks_above(lv, iv, l[q], id[q]);
            const float tl = a ? l[q] : lv;
            const uint32_t ti = a ? id[q] : iv;
            l[q] = a ? lv : l[q];
            id[q] = a ? iv : id[q];
            lv = tl;
            iv = ti;
        }
    }
    __device__ __forceinline__ bool beats_last(float lv, uint32_t iv) const {
        return ranks_above(lv, iv, l[KN - 1], id[KN - 1]);
    }
};
using Top8 = TopN<K>;

// Sum v[0..NV-1] over each maximal run of lanes holding the same key (runs in
// lane order; a warp covers 32 consecutive pixels of a row, and neighbouring
// pixels usually hold the same site in the same slot).  Afterwards the last
// lane of every run holds the run's total.  Returns true on those lanes.
template <int NV, typename T>
__device__ __forceinline__ bool warp_run_reduce(uint32_t key, T (&v)[NV], int lane) {
    constexpr unsigned FULL = 0xffffffffu;
    const uint32_t key_next = __shfl_down_sync(FULL, key, 1);
    const bool tail = lane == 31 || key_next != key;
    const uint32_t tails = __ballot_sync(FULL, tail);
    const uint32_t cont = ~tails;  // bit L: lanes L and L+1 share a run
    if (cont) {
        const uint32_t prev = tails & ((1u << lane) - 1u);
        const int start = prev ? 32 - __clz(prev) : 0;
        // doubling steps needed for the longest run (warp-uniform)
        int levels = 1;
        uint32_t r = cont & (cont >> 1);
        if (r) {
            levels = 2;
            r &= r >> 2;
            if (r) {
                levels = 3;
                r &= r >> 4;
                if (r) {
                    levels = 4;
                    r &= r >> 8;
                    if (r) levels = 5;
                }
            }
        }
#pragma unroll
        for (int L = 0; L < 5; ++L) {
            if (L < levels) {  // warp-uniform
                const int off = 1 << L;
                const bool take = lane - off >= start;
#pragma unroll
                for (int k = 0; k < NV; ++k) {
                    const T x = __shfl_up_sync(FULL, v[k], off);
                    if (take) v[k] += x;
                }
            }
        }
    }
    return tail;
}


// workspace views
__device__ __forceinline__ Counters *ws_counters(void *ws);

// Order-independent gradients: every contribution is rounded to a multiple
// of 2^-40 and summed in 64-bit fixed point (integer sums are exact, so
// their order does not matter); magnitudes up to 2^23 per sum.
constexpr float FIXED_SCALE = 1099511627776.0f;  // 2^40

// Bounds checks of the debug build (compiled with -DSAD_CHECKS): a failed
// check is counted in the statistics block and the guarded access is
// skipped; nothing traps.  In the normal build the checks compile away.
#ifdef SAD_CHECKS
__device__ __forceinline__ bool sad_check(bool ok, void *ws) {
    if (!ok) atomicAdd(&ws_counters(ws)->check_failures, 1ull);
    return ok;
}
#define SAD_CHECK(cond, ws) (::sad::sad_check((cond), (ws)))
#else
#define SAD_CHECK(cond, ws) (true)
#endif


__device__ __forceinline__ Counters *ws_counters(void *ws) { return reinterpret_cast<Counters *>(ws); }
__device__ __forceinline__ double *ws_loss_partials(void *ws) {
    return reinterpret_cast<double *>(reinterpret_cast<char *>(ws) + COUNTERS_BYTES);
}

}  // namespace sad
