// sad_kernels.cu -- sm_100a kernels of one Soft Anisotropic Diagrams fitting
// iteration ("Soft Anisotropic Diagrams for Differentiable Image
// Representation"; reading notes key designs 1-4; summary sections 4, 5 and
// B.2-B.5).
//
//   records_kernel      a1  per-site score record (fp64 math, fp32 fields)
//   topk_exact_kernel   a8  brute-force top-8 per pixel
//   seed_*_kernel       a9  seed pass of a refresh
//   propagate_kernel    a2/a3  one Jacobi candidate pass (+ injection)
//   render_kernel       a4  softmax blend of the current candidates
//   fixed_to_grads_kernel  adds the order-independent backward's 64-bit
//                       fixed-point sums (the tile pass, sad_fused.cu) to
//                       the gradients
//   adam_kernel         a7  Adam step + a1 for the updated sites
//   jfa3x3_kernel       optional 3x3 flood prepass (summary B.3)
//   tau_diffuse_kernel  Jacobi step on the ln tau gradients (summary B.6)
//   target_u8_kernel    8-bit RGB -> planar float32 target
// The fused steady-state pass (also the float backward) is in sad_fused_kernel.cuh with its
// launchers in sad_fused.cu, budget control in sad_densify.cu, the 16-byte site record in
// sad_pack.cu.
#include <cuda_fp16.h>

#include "sad_device.cuh"
#include "sad_finish.cuh"
#include "sad_launch.h"

namespace sad {

namespace {

constexpr int TILE_X = 32;  // image-space blocks: one warp per 32-pixel row segment
constexpr int TILE_Y = 8;
constexpr int TILE_THREADS = TILE_X * TILE_Y;
constexpr int SITE_THREADS = 256;
static_assert(SITE_THREADS == FINISH_THREADS, "Adam's first block runs a pass's finishing step");



// ---------------------------------------------------------------------------
// a1: per-site record, evaluated in double with the operation order of the
// definition, each field rounded once to float32.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void write_record(float4 *__restrict__ rec, int i, float px, float py, float lt,
                                             float r, float cr, float cg, float cb, float th, float a,
                                             double s) {
    float4 r0, r1, r2, r3;
    if (px >= 0.0f) {
        const double tau = exp((double)lt);
        const double k = __dmul_rn(tau, s);
        const double ep = exp((double)a), em = exp(-(double)a);
        double sn, c;
        sincos((double)th, &sn, &c);
        const double g11 = __dadd_rn(__dmul_rn(__dmul_rn(ep, c), c), __dmul_rn(__dmul_rn(em, sn), sn));
        const double g12 = __dmul_rn(__dmul_rn(__dsub_rn(ep, em), c), sn);
        const double g22 = __dadd_rn(__dmul_rn(__dmul_rn(ep, sn), sn), __dmul_rn(__dmul_rn(em, c), c));
        const double kk = __dmul_rn(k, k);
        r0 = make_float4(px, py, (float)__dmul_rn(kk, g11), (float)__dmul_rn(kk, g12));
        r1 = make_float4((float)__dmul_rn(kk, g22), (float)__dmul_rn(k, (double)r), (float)k, 0.0f);
        r2 = make_float4(cr, cg, cb, (float)c);
        r3 = make_float4((float)sn, (float)__dmul_rn(kk, ep), (float)__dmul_rn(kk, em), 0.0f);
    } else {
        r0 = make_float4(-1.0f, 0.0f, 0.0f, 0.0f);
        r1 = r2 = r3 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
    float4 *o = rec + (size_t)i * REC_F4;
    o[0] = r0;
    o[1] = r1;
    o[2] = r2;
    o[3] = r3;
}

__global__ void __launch_bounds__(SITE_THREADS) records_kernel(const float *__restrict__ prm, int N, double s,
                                                               float4 *__restrict__ rec) {
    const int i = blockIdx.x * SITE_THREADS + threadIdx.x;
    if (i >= N) return;
    const size_t n = (size_t)N;
    write_record(rec, i, prm[PX * n + i], prm[PY * n + i], prm[PLT * n + i], prm[PR * n + i],
                 prm[PCR * n + i], prm[PCG * n + i], prm[PCB * n + i], prm[PTH * n + i],
                 prm[PA * n + i], s);
}

__global__ void init_counters_kernel(Counters *c, uint32_t seed) {
    c->pass_counter = 0;
    c->adam_step = 0;
    c->cur = 0;
    c->seed = seed;
    c->ticket_prop = c->ticket_bwd = c->ticket_adam = 0;
    c->hash_overflow = c->nonfinite_pixels = c->empty_pixels = c->dropped_ids = 0;
    c->check_failures = 0;
    c->staging_fallbacks = 0;
    c->tile_ticket = 0;
    c->loss = 0.0;
}

__global__ void set_fit_state_kernel(Counters *c, uint32_t pass_counter, uint32_t adam_step, uint32_t seed) {
    c->pass_counter = pass_counter;
    c->adam_step = adam_step;
    c->seed = seed;
}

__global__ void mark_inactive_kernel(float *prm, int N, int from) {
    const int i = from + blockIdx.x * SITE_THREADS + threadIdx.x;
    if (i < N) prm[i] = -1.0f;  // x plane
}

// ---------------------------------------------------------------------------
// a8: exact top-8 by brute force; records staged through shared memory.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(SITE_THREADS) topk_exact_kernel(const float4 *__restrict__ rec, int N, int H,
                                                                  int W, float cs, const int64_t *__restrict__ pix,
                                                                  int64_t n_pix, uint32_t *__restrict__ out) {
    __shared__ float sx[SITE_THREADS], sy[SITE_THREADS], sA[SITE_THREADS], sB[SITE_THREADS],
        sC[SITE_THREADS], sb[SITE_THREADS];
    const int64_t q = (int64_t)blockIdx.x * SITE_THREADS + threadIdx.x;
    const int64_t P = (int64_t)H * W;
    int64_t p = -1;
    if (q < n_pix) p = pix ? pix[q] : q;
    const bool live = p >= 0 && p < P;
    const float fx = live ? ((float)(int)(p % W) + 0.5f) * cs : 0.0f;
    const float fy = live ? ((float)(int)(p / W) + 0.5f) * cs : 0.0f;
    Top8 t;
    t.clear();
    for (int base = 0; base < N; base += SITE_THREADS) {
        const int i = base + threadIdx.x;
        if (i < N) {
            const float4 r0 = __ldg(rec + (size_t)i * REC_F4);
            const float4 r1 = __ldg(rec + (size_t)i * REC_F4 + 1);
            sx[threadIdx.x] = r0.x;
            sy[threadIdx.x] = r0.y;
            sA[threadIdx.x] = r0.z;
            sB[threadIdx.x] = r0.w;
            sC[threadIdx.x] = r1.x;
            sb[threadIdx.x] = r1.y;
        } else {
            sx[threadIdx.x] = -1.0f;
        }
        __syncthreads();
        const int cnt = min(SITE_THREADS, N - base);
        if (live) {
            for (int j = 0; j < cnt; ++j) {
                if (!(sx[j] >= 0.0f)) continue;
                const float l = sad_logit(sx[j], sy[j], sA[j], sB[j], sC[j], sb[j], fx, fy);
                if (l != l) continue;
                const uint32_t id = (uint32_t)(base + j);
                if (t.beats_last(l, id)) t.insert(l, id);
            }
        }
        __syncthreads();
    }
    if (q < n_pix) {
        uint4 *o = reinterpret_cast<uint4 *>(out + q * K);
        o[0] = make_uint4(t.id[0], t.id[1], t.id[2], t.id[3]);
        o[1] = make_uint4(t.id[4], t.id[5], t.id[6], t.id[7]);
    }
}

// ---------------------------------------------------------------------------
// a9 seed pass: clear the current table, scatter each active site's id into
// slot 0 of the pixel (candidate-grid cell) containing it (atomicMin:
// smallest id wins).
// ---------------------------------------------------------------------------
__global__ void seed_clear_kernel(uint32_t *__restrict__ table, long long P, const Counters *__restrict__ c) {
    uint4 *t = reinterpret_cast<uint4 *>(table + (size_t)c->cur * (size_t)P * K);
    const long long n = 2 * P;
    const uint4 e = make_uint4(EMPTY, EMPTY, EMPTY, EMPTY);
    for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < n; q += (long long)gridDim.x * blockDim.x)
        t[q] = e;
}

__global__ void seed_scatter_kernel(const float *__restrict__ prm, int N, int H, int W, int cell, int GW,
                                    long long PT, uint32_t *__restrict__ table, const Counters *__restrict__ c) {
    const int i = blockIdx.x * SITE_THREADS + threadIdx.x;
    if (i >= N) return;
    const float px = prm[PX * (size_t)N + i], py = prm[PY * (size_t)N + i];
    if (!(px >= 0.0f) || !(py >= 0.0f)) return;
    const float fi = floorf(px), fj = floorf(py);
    if (fi >= (float)W || fj >= (float)H) return;
    const long long p = (long long)((int)fj / cell) * GW + (long long)((int)fi / cell);
    uint32_t *plane0 = table + (size_t)c->cur * (size_t)PT * K;
    atomicMin(plane0 + (size_t)p * 4, (uint32_t)i);
}

// ---------------------------------------------------------------------------
// a2/a3: one Jacobi propagation pass.
// ---------------------------------------------------------------------------
// A pass offers every pixel the 8 ids of each neighbour list (and the
// injections).  In a refresh most of them are new to the pixel and about 6
// of its 8 entries are replaced per pass, so the candidates are merged a
// batch of 8 at a time without branches: the batch is scored, ids the pixel
// already holds (or that repeat within the batch) are dropped, the batch is
// sorted by Batcher's odd-even merge network and merged into the running
// top-8 by a bitonic merge.  The top-8 of a set under the strict order
// (logit desc, id asc) does not depend on how the set is assembled, so this
// equals offering the ids one by one.

// compare-exchange: afterwards (la, ia) ranks above (lb, ib)
__device__ __forceinline__ void cx(float &la, uint32_t &ia, float &lb, uint32_t &ib) {
    const bool s = ranks_above(lb, ib, la, ia);
    const float tl = la;
    const uint32_t ti = ia;
    la = s ? lb : la;
    ia = s ? ib : ia;
    lb = s ? tl : lb;
    ib = s ? ti : ib;
}

// sort 8 entries best first: Batcher's odd-even merge sort (19 comparators)
__device__ __forceinline__ void sort8(float (&l)[K], uint32_t (&id)[K]) {
    cx(l[0], id[0], l[1], id[1]); cx(l[2], id[2], l[3], id[3]); cx(l[4], id[4], l[5], id[5]); cx(l[6], id[6], l[7], id[7]);
    cx(l[0], id[0], l[2], id[2]); cx(l[1], id[1], l[3], id[3]); cx(l[4], id[4], l[6], id[6]); cx(l[5], id[5], l[7], id[7]);
    cx(l[1], id[1], l[2], id[2]); cx(l[5], id[5], l[6], id[6]);
    cx(l[0], id[0], l[4], id[4]); cx(l[1], id[1], l[5], id[5]); cx(l[2], id[2], l[6], id[6]); cx(l[3], id[3], l[7], id[7]);
    cx(l[2], id[2], l[4], id[4]); cx(l[3], id[3], l[5], id[5]);
    cx(l[1], id[1], l[2], id[2]); cx(l[3], id[3], l[4], id[4]); cx(l[5], id[5], l[6], id[6]);
}

// the same network carrying a payload with each entry
__device__ __forceinline__ void cxp(float &la, uint32_t &ia, float &pa, float &lb, uint32_t &ib, float &pb) {
    const bool s = ranks_above(lb, ib, la, ia);
    const float tl = la, tp = pa;
    const uint32_t ti = ia;
    la = s ? lb : la;
    ia = s ? ib : ia;
    pa = s ? pb : pa;
    lb = s ? tl : lb;
    ib = s ? ti : ib;
    pb = s ? tp : pb;
}
__device__ __forceinline__ void sort8p(float (&l)[K], uint32_t (&id)[K], float (&p)[K]) {
#define SAD_CXP(a, b) cxp(l[a], id[a], p[a], l[b], id[b], p[b])
    SAD_CXP(0, 1); SAD_CXP(2, 3); SAD_CXP(4, 5); SAD_CXP(6, 7);
    SAD_CXP(0, 2); SAD_CXP(1, 3); SAD_CXP(4, 6); SAD_CXP(5, 7);
    SAD_CXP(1, 2); SAD_CXP(5, 6);
    SAD_CXP(0, 4); SAD_CXP(1, 5); SAD_CXP(2, 6); SAD_CXP(3, 7);
    SAD_CXP(2, 4); SAD_CXP(3, 5);
    SAD_CXP(1, 2); SAD_CXP(3, 4); SAD_CXP(5, 6);
#undef SAD_CXP
}

// keep the best 8 of the running list and a sorted batch: the better of
// t[i] and batch[7 - i] for every i are the 8 best, as a bitonic sequence,
// which half-cleaners at distances 4, 2 and 1 put in order
__device__ __forceinline__ void merge8(Top8 &t, const float (&l)[K], const uint32_t (&id)[K]) {
#pragma unroll
    for (int q = 0; q < K; ++q) {
        const bool b = ranks_above(l[K - 1 - q], id[K - 1 - q], t.l[q], t.id[q]);
        t.l[q] = b ? l[K - 1 - q] : t.l[q];
        t.id[q] = b ? id[K - 1 - q] : t.id[q];
    }
#pragma unroll
    for (int d = 4; d >= 1; d >>= 1)
#pragma unroll
        for (int q = 0; q < K; ++q)
            if ((q & d) == 0) cx(t.l[q], t.id[q], t.l[q + d], t.id[q + d]);
}

// Logit of site x at (fx, fy) for ranking candidates: from the float32 score
// record, or (F16) from the packed candidate-site record -- x, y as float32,
// (A, B) and (C, b) as binary16 pairs -- with the same operation order.
template <bool F16>
__device__ __forceinline__ float cand_logit(const float4 *__restrict__ rec, const uint4 *__restrict__ c16,
                                            uint32_t x, float fx, float fy, bool &active) {
    if constexpr (F16) {
        const uint4 v = __ldg(c16 + x);
        const float px = __uint_as_float(v.x), py = __uint_as_float(v.y);
        const float2 ab = __half22float2(*reinterpret_cast<const __half2 *>(&v.z));
        const float2 cb = __half22float2(*reinterpret_cast<const __half2 *>(&v.w));
        active = px >= 0.0f;
        return sad_logit(px, py, ab.x, ab.y, cb.x, cb.y, fx, fy);
    } else {
        float px, py, A, B, C, b;
        load_rank_fields(rec, x, px, py, A, B, C, b);
        active = px >= 0.0f;
        return sad_logit(px, py, A, B, C, b, fx, fy);
    }
}

// Offer up to 8 candidate ids as one batch.  Their records are fetched
// together (independent loads in flight).  With merge, invalid entries (id
// >= N, inactive site, NaN logit, an id already held or repeated earlier in
// the batch) become (-inf, EMPTY), which ranks below every candidate, and the
// batch is sorted and merged; the network is skipped when no active lane has
// a candidate that beats its last entry.  Without merge the candidates that
// beat the last entry are inserted one by one: the JFA prepass keeps 4
// entries (KN = 4) and takes few new ones per pass; without the network its
// kernel runs at 32 registers, 8 blocks per SM (a few bytes spill; measured
// faster than 40 registers at 6 blocks and 47 at 5).  DISTINCT: the batch
// is known to hold no id twice (a list this library wrote), so the merge
// skips the check of each id against the batch's earlier ones.
template <int NB, bool F16, bool MERGE, int KN = K, bool DISTINCT = false>
__device__ __forceinline__ void offer_batch(TopN<KN> &t, const uint32_t (&ids)[NB], const float4 *__restrict__ rec,
                                            const uint4 *__restrict__ c16, uint32_t N, float fx, float fy) {
    if constexpr (!MERGE) {
        float li[NB];
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            li[q] = __int_as_float(0x7fc00000);  // NaN: not a candidate
            const uint32_t x = ids[q];
            if (x < N && !t.has(x)) {
                // the score only for an active site (keeps fewer values live)
                if constexpr (F16) {
                    const uint4 v = __ldg(c16 + x);
                    if (__uint_as_float(v.x) >= 0.0f) {
                        const float2 ab = __half22float2(*reinterpret_cast<const __half2 *>(&v.z));
                        const float2 cb = __half22float2(*reinterpret_cast<const __half2 *>(&v.w));
                        li[q] = sad_logit(__uint_as_float(v.x), __uint_as_float(v.y), ab.x, ab.y, cb.x, cb.y, fx, fy);
                    }
                } else {
                    float px, py, A, B, C, b;
                    load_rank_fields(rec, x, px, py, A, B, C, b);
                    if (px >= 0.0f) li[q] = sad_logit(px, py, A, B, C, b, fx, fy);
                }
            }
        }
#pragma unroll
        for (int q = 0; q < NB; ++q)
            if (li[q] == li[q] && t.beats_last(li[q], ids[q]) && !t.has(ids[q])) t.insert(li[q], ids[q]);
        return;
    } else {
    float l[K];
    uint32_t id[K];
    bool enters = false;
#pragma unroll
    for (int q = 0; q < K; ++q) {
        l[q] = -__int_as_float(0x7f800000);
        id[q] = EMPTY;
        if (q < NB) {
            const uint32_t x = ids[q];
            bool fresh = x < N && !t.has(x);
            if constexpr (!DISTINCT) {
#pragma unroll
                for (int r = 0; r < q; ++r) fresh &= x != ids[r];
            }
            if (fresh) {
                bool active;
                const float lv = cand_logit<F16>(rec, c16, x, fx, fy, active);
                if (active && lv == lv) {
                    l[q] = lv;
                    id[q] = x;
                    enters |= t.beats_last(lv, x);
                }
            }
        }
    }
    if (__any_sync(__activemask(), enters)) {
        sort8(l, id);
        merge8(t, l, id);
    }
    }
}

// The pixel's own list as the first candidates of a pass into an empty list:
// re-scored in its previous order it is usually still sorted and free of
// repeats (the records do not change between refresh passes), and then it is
// the top-8 of its own candidates as it stands; otherwise its repeats are
// dropped and it is sorted.  Same result either way.  CACHED: the scores are
// the ones the previous pass of the same refresh stored beside the list (the
// same records, the same pixel: the same bits), so no record is fetched.
template <bool F16, bool MERGE, bool CACHED = false>
__device__ __forceinline__ void take_own_list(Top8 &t, const uint4 a, const uint4 b, const float4 *__restrict__ rec,
                                              const uint4 *__restrict__ c16, uint32_t N, float fx, float fy,
                                              const float4 *__restrict__ lc = nullptr) {
    const uint32_t ids[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    if constexpr (CACHED) {
        const float4 l0 = lc[0], l1 = lc[1];
        const float ls[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            // an empty slot was stored as -inf
            const bool v = ids[q] < N && ls[q] == ls[q] && ls[q] != -__int_as_float(0x7f800000);
            t.l[q] = v ? ls[q] : -__int_as_float(0x7f800000);
            t.id[q] = v ? ids[q] : EMPTY;
        }
        // float32 ranking: the previous pass wrote this list, sorted and
        // repeat-free, with these very scores (its empty slots, stored as
        // -inf, at the end).  F16 stored it in float32 order beside the
        // packed-record scores it ranks by, so it goes on to the check.
        if constexpr (!F16) return;
    } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            t.l[q] = -__int_as_float(0x7f800000);
            t.id[q] = EMPTY;
            if (ids[q] < N) {
                bool active;
                const float lv = cand_logit<F16>(rec, c16, ids[q], fx, fy, active);
                if (active && lv == lv) {
                    t.l[q] = lv;
                    t.id[q] = ids[q];
                }
            }
        }
    }
    bool clean = true;
#pragma unroll
    for (int q = 1; q < 8; ++q) {
        clean &= !ranks_above(t.l[q], t.id[q], t.l[q - 1], t.id[q - 1]);
#pragma unroll
        for (int r = 0; r < q; ++r) clean &= (t.id[q] == EMPTY) || (t.id[q] != t.id[r]);
    }
    if constexpr (MERGE) {
        if (__any_sync(__activemask(), !clean)) {
#pragma unroll
            for (int q = 1; q < 8; ++q)
#pragma unroll
                for (int r = 0; r < q; ++r)
                    if (t.id[q] != EMPTY && t.id[q] == t.id[r]) {
                        t.l[q] = -__int_as_float(0x7f800000);
                        t.id[q] = EMPTY;
                    }
            sort8(t.l, t.id);
        }
    } else if (!clean) {
        // the ids one by one into an empty list
        t.clear();
        offer_batch<8, F16, false>(t, ids, rec, c16, N, fx, fy);
    }
}

// H x W is the candidate grid; a cell is scored at its centre, (i + 0.5) cs
// (cs = 1: the pixel grid).  F16: candidates are ranked on the packed
// records c16 and the kept 8 re-scored with the float32 records.
// LC (score cache): 1 = store each list's ranking scores in lcache (two
// float4 per list, -inf for an empty slot; with F16 the packed-record scores,
// carried through the final float32 re-sort), 2 = also take the own list's
// scores from there; valid while the records stay unchanged, which holds
// between the passes of one refresh.
template <bool F16, bool MERGE, int LC = 0>
__global__ void __launch_bounds__(TILE_THREADS) propagate_kernel(const float4 *__restrict__ rec,
                                                                 const uint4 *__restrict__ c16, uint32_t *table,
                                                                 int H, int W, float cs, int N, int jump, int G,
                                                                 Counters *c, float4 *__restrict__ lcache) {
    const uint32_t cur = c->cur, pass = c->pass_counter, seed = c->seed;
    const size_t P = (size_t)H * W;
    const uint4 *in0 = reinterpret_cast<const uint4 *>(table + cur * P * K);
    const uint4 *in1 = in0 + P;
    uint4 *out0 = reinterpret_cast<uint4 *>(table + (cur ^ 1u) * P * K);
    uint4 *out1 = out0 + P;
    const int i = blockIdx.x * TILE_X + threadIdx.x;
    const int j = blockIdx.y * TILE_Y + threadIdx.y;
    if (i < W && j < H) {
        const size_t p = (size_t)j * W + i;
        const float fx = ((float)i + 0.5f) * cs, fy = ((float)j + 0.5f) * cs;
        Top8 t;
        take_own_list<F16, MERGE, LC == 2>(t, in0[p], in1[p], rec, c16, (uint32_t)N, fx, fy,
                                           LC == 2 ? lcache + 2 * p : nullptr);
        // the neighbours at (-k, 0), (+k, 0), (0, -k), (0, +k); one outside
        // the image offers nothing
#pragma unroll 1
        for (int d = 1; d < 5; ++d) {
            const int ni = i + (d == 1 ? -jump : (d == 2 ? jump : 0));
            const int nj = j + (d == 3 ? -jump : (d == 4 ? jump : 0));
            uint4 a = make_uint4(EMPTY, EMPTY, EMPTY, EMPTY), b = a;
            if (ni >= 0 && ni < W && nj >= 0 && nj < H) {
                const size_t pn = (size_t)nj * W + ni;
                a = in0[pn];
                b = in1[pn];
            }
            const uint32_t ids[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            // in a refresh (LC > 0) every list was written by the seed pass
            // or by a pass of this kernel, so it holds no id twice
            offer_batch<8, F16, MERGE, K, (LC > 0)>(t, ids, rec, c16, (uint32_t)N, fx, fy);
        }
        if (G > 0 && G <= 4) {
            // up to four injections: a half batch (no empty slots to check)
            uint32_t h = inject_state(seed, pass, (uint32_t)p);
            uint32_t ids[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (q < G) {
                    h = xorshift32(h);
                    ids[q] = __umulhi(h, (uint32_t)N);
                } else {
                    ids[q] = EMPTY;
                }
            }
            offer_batch<4, F16, MERGE>(t, ids, rec, c16, (uint32_t)N, fx, fy);
        } else if (G > 0) {
            uint32_t h = inject_state(seed, pass, (uint32_t)p);
#pragma unroll 1
            for (int g0 = 0; g0 < G; g0 += 8) {
                uint32_t ids[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    if (g0 + q < G) {
                        h = xorshift32(h);
                        ids[q] = __umulhi(h, (uint32_t)N);
                    } else {
                        ids[q] = EMPTY;
                    }
                }
                offer_batch<8, F16, MERGE>(t, ids, rec, c16, (uint32_t)N, fx, fy);
            }
        }
        float lrank[K];  // F16 with LC: each kept entry's packed-record score
        if constexpr (F16) {
            // the kept 8 in float32 logit order
#pragma unroll
            for (int q = 0; q < K; ++q) {
                lrank[q] = t.l[q];
                if (t.id[q] == EMPTY) continue;
                bool active;
                t.l[q] = cand_logit<false>(rec, nullptr, t.id[q], fx, fy, active);
            }
            if constexpr (LC > 0)
                sort8p(t.l, t.id, lrank);
            else
                sort8(t.l, t.id);
        }
        out0[p] = make_uint4(t.id[0], t.id[1], t.id[2], t.id[3]);
        out1[p] = make_uint4(t.id[4], t.id[5], t.id[6], t.id[7]);
        if constexpr (LC > 0) {
            const float *ls = F16 ? lrank : t.l;
            lcache[2 * p] = make_float4(ls[0], ls[1], ls[2], ls[3]);
            lcache[2 * p + 1] = make_float4(ls[4], ls[5], ls[6], ls[7]);
        }
    }
    // the last block to finish flips the double buffer and advances the pass
    // counter; every block has read both before taking its ticket
    __syncthreads();
    if (threadIdx.x == 0 && threadIdx.y == 0) {
        __threadfence();
        const unsigned total = gridDim.x * gridDim.y;
        if (atomicAdd(&c->ticket_prop, 1u) == total - 1) {
            c->cur = cur ^ 1u;
            c->pass_counter = pass + 1u;
            c->ticket_prop = 0;
            __threadfence();
        }
    }
}

// Packed candidate-site record of every site (summary B.2): x and y as
// float32, then (A, B) and (C, b) rounded to binary16 pairs (round to
// nearest even, overflow to infinity).
__global__ void __launch_bounds__(SITE_THREADS) pack_cand16_kernel(const float4 *__restrict__ rec, int N,
                                                                   uint4 *__restrict__ c16) {
    const int i = blockIdx.x * SITE_THREADS + threadIdx.x;
    if (i >= N) return;
    const float4 r0 = rec[(size_t)i * REC_F4];
    const float4 r1 = rec[(size_t)i * REC_F4 + 1];
    const __half2 ab = __floats2half2_rn(r0.z, r0.w);
    const __half2 cb = __floats2half2_rn(r1.x, r1.y);
    c16[i] = make_uint4(__float_as_uint(r0.x), __float_as_uint(r0.y), *reinterpret_cast<const uint32_t *>(&ab),
                        *reinterpret_cast<const uint32_t *>(&cb));
}

// One 3x3 flood pass of the optional JFA prepass (summary B.3): the 4 best
// distinct candidates of the lists at (i + a k, j + b k), a, b in {-1, 0, 1},
// go to slots 0-3; slots 4-7 are emptied.  The prepass starts from the seed
// pass, which leaves slots 1-7 empty, and every flood pass empties slots 4-7,
// so a pass reads only the first plane (slots 0-3) of each list and keeps a
// running top 4.  LC as in propagate_kernel: 1 = store the new lists' scores
// in lcache, 2 = also start from the own list's stored scores (its 4
// entries, in order) and offer only the 8 neighbours.
template <int LC = 0>
__global__ void __launch_bounds__(TILE_THREADS, 8) jfa3x3_kernel(const float4 *__restrict__ rec, uint32_t *table,
                                                              int H, int W, float cs, int N, int jump, Counters *c,
                                                              float4 *__restrict__ lcache) {
    const uint32_t cur = c->cur, pass = c->pass_counter;
    const size_t P = (size_t)H * W;
    const uint4 *in0 = reinterpret_cast<const uint4 *>(table + cur * P * K);
    uint4 *out0 = reinterpret_cast<uint4 *>(table + (cur ^ 1u) * P * K);
    uint4 *out1 = out0 + P;
    const int i = blockIdx.x * TILE_X + threadIdx.x;
    const int j = blockIdx.y * TILE_Y + threadIdx.y;
    if (i < W && j < H) {
        const size_t p = (size_t)j * W + i;
        const float fx = ((float)i + 0.5f) * cs, fy = ((float)j + 0.5f) * cs;
        TopN<4> t;
        t.clear();
        if constexpr (LC == 2) {
            // the own list is the previous pass's top 4, sorted and distinct
            const uint4 a = in0[p];
            const float4 l0 = lcache[2 * p];
            const uint32_t ids[4] = {a.x, a.y, a.z, a.w};
            const float ls[4] = {l0.x, l0.y, l0.z, l0.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const bool v = ids[q] < (uint32_t)N && ls[q] == ls[q] && ls[q] != -__int_as_float(0x7f800000);
                t.l[q] = v ? ls[q] : -__int_as_float(0x7f800000);
                t.id[q] = v ? ids[q] : EMPTY;
            }
        }
#pragma unroll 1
        for (int d = 0; d < 9; ++d) {
            if (LC == 2 && d == 4) continue;
            const int ni = i + (d % 3 - 1) * jump, nj = j + (d / 3 - 1) * jump;
            if (ni < 0 || ni >= W || nj < 0 || nj >= H) continue;
            const size_t pn = (size_t)nj * W + ni;
            const uint4 a = in0[pn];
            const uint32_t ids[4] = {a.x, a.y, a.z, a.w};
            offer_batch<4, false, false, 4>(t, ids, rec, nullptr, (uint32_t)N, fx, fy);
        }
        out0[p] = make_uint4(t.id[0], t.id[1], t.id[2], t.id[3]);
        out1[p] = make_uint4(EMPTY, EMPTY, EMPTY, EMPTY);
        if constexpr (LC > 0) lcache[2 * p] = make_float4(t.l[0], t.l[1], t.l[2], t.l[3]);
    }
    __syncthreads();
    if (threadIdx.x == 0 && threadIdx.y == 0) {
        __threadfence();
        const unsigned total = gridDim.x * gridDim.y;
        if (atomicAdd(&c->ticket_prop, 1u) == total - 1) {
            c->cur = cur ^ 1u;
            c->pass_counter = pass + 1u;
            c->ticket_prop = 0;
            __threadfence();
        }
    }
}

// ---------------------------------------------------------------------------
// a4: render
// ---------------------------------------------------------------------------
struct PixelSoftmax {
    float l[K];      // logits, then unnormalised weights e_q
    uint32_t id[K];
    unsigned valid;  // bit q set when slot q contributes
    float Z, cr, cg, cb;
};

// softmax over the valid slots of one pixel (max-subtracted); returns the
// number of valid slots
__device__ __forceinline__ int pixel_softmax(const uint4 a, const uint4 b, const float4 *__restrict__ rec,
                                             uint32_t N, float fx, float fy, PixelSoftmax &s,
                                             unsigned &dropped) {
    s.id[0] = a.x; s.id[1] = a.y; s.id[2] = a.z; s.id[3] = a.w;
    s.id[4] = b.x; s.id[5] = b.y; s.id[6] = b.z; s.id[7] = b.w;
    s.valid = 0;
    float M = -__int_as_float(0x7f800000);
#pragma unroll
    for (int q = 0; q < K; ++q) {
        s.l[q] = 0.0f;
        const uint32_t id = s.id[q];
        if (id >= N) {
            dropped += (id != EMPTY);
            continue;
        }
        // two loads, the second only for an active site: one 32-byte load
        // per slot raised this kernel from 40 to 63 registers and slowed it
        const float4 r0 = __ldg(rec + (size_t)id * REC_F4);
        if (!(r0.x >= 0.0f)) continue;
        const float2 r1 = __ldg(reinterpret_cast<const float2 *>(rec + (size_t)id * REC_F4 + 1));
        const float l = sad_logit(r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, fx, fy);
        if (!isfinite(l)) continue;
        s.l[q] = l;
        s.valid |= 1u << q;
        M = fmaxf(M, l);
    }
    s.Z = 0.0f;
    s.cr = s.cg = s.cb = 0.0f;
    if (!s.valid) return 0;
#pragma unroll
    for (int q = 0; q < K; ++q) {
        if (!(s.valid >> q & 1u)) continue;
        const float e = __expf(s.l[q] - M);
        const float4 r2 = __ldg(rec + (size_t)s.id[q] * REC_F4 + 2);
        s.l[q] = e;
        s.Z += e;
        s.cr = fmaf(e, r2.x, s.cr);
        s.cg = fmaf(e, r2.y, s.cg);
        s.cb = fmaf(e, r2.z, s.cb);
    }
    const float iz = 1.0f / s.Z;
    s.cr *= iz;
    s.cg *= iz;
    s.cb *= iz;
    return __popc(s.valid);
}

__global__ void __launch_bounds__(TILE_THREADS) render_kernel(const float4 *__restrict__ rec,
                                                              const uint32_t *__restrict__ table, int H, int W,
                                                              TableGrid tg, int N, float *__restrict__ image,
                                                              Counters *c) {
    const size_t P = (size_t)H * W;
    const uint4 *in0 = reinterpret_cast<const uint4 *>(table + (size_t)c->cur * tg.PT * K);
    const uint4 *in1 = in0 + tg.PT;
    const int i = blockIdx.x * TILE_X + threadIdx.x;
    const int j = blockIdx.y * TILE_Y + threadIdx.y;
    unsigned dropped = 0;
    bool empty = false;
    if (i < W && j < H) {
        const size_t p = (size_t)j * W + i;
        const size_t pt = tg.cell_of(i, j, p);
        PixelSoftmax s;
        const int nv = pixel_softmax(in0[pt], in1[pt], rec, (uint32_t)N, (float)i + 0.5f, (float)j + 0.5f, s,
                                     dropped);
        empty = nv == 0;
        image[p] = s.cr;
        image[P + p] = s.cg;
        image[2 * P + p] = s.cb;
    }
    const int ne = __syncthreads_count(empty);
    const int nd = __syncthreads_count(dropped != 0);
    if (threadIdx.x == 0 && threadIdx.y == 0) {
        if (ne) atomicAdd(&c->empty_pixels, (unsigned long long)ne);
        if (nd) atomicAdd(&c->dropped_ids, (unsigned long long)nd);
    }
}

// the deterministic backward's fixed-point sums, added to the gradients and
// cleared for the next call
__global__ void __launch_bounds__(SITE_THREADS) fixed_to_grads_kernel(unsigned long long *__restrict__ fixed,
                                                                      float *__restrict__ grads, long long n) {
    const long long q = (long long)blockIdx.x * SITE_THREADS + threadIdx.x;
    if (q >= n) return;
    const long long v = (long long)fixed[q];
    if (v) {
        grads[q] += (float)((double)v * 0x1p-40);
        fixed[q] = 0ull;
    }
}

// ---------------------------------------------------------------------------
// a7: Adam + a1 for every site; zeroes the gradients.
// ---------------------------------------------------------------------------
struct AdamArgs {
    float lr[NPARAM];
    float beta1, beta2, eps;
};

// beta^t for an integer t by repeated squaring in double (at most 2 log2 t
// roundings of relative size 2^-53: far below the float32 it is used in)
__device__ __forceinline__ double pow_uint(double b, uint32_t t) {
    double r = 1.0;
#pragma unroll 1
    while (t) {
        if (t & 1u) r *= b;
        b *= b;
        t >>= 1;
    }
    return r;
}

// 4 blocks/SM (64 registers): the kernel is latency-bound, more warps hide it
__global__ void __launch_bounds__(SITE_THREADS, 4) adam_kernel(float *__restrict__ prm, float *__restrict__ grads,
                                                            float *__restrict__ m1, float *__restrict__ m2,
                                                            float4 *__restrict__ rec, int N, int maxHW,
                                                            float xmax, float ymax, AdamArgs a,
                                                            const uint8_t *__restrict__ frozen, Counters *c,
                                                            unsigned finish_tiles, double P) {
    // the preceding propagating fit pass's finishing step (its own launch
    // otherwise): block 0 first
    if (finish_tiles && blockIdx.x == 0) finish_pass_block(c, finish_tiles, P, 1);
    const uint32_t t = c->adam_step + 1u;
    const int i = blockIdx.x * SITE_THREADS + threadIdx.x;
    if (i < N) {
        const size_t n = (size_t)N;
        // every load issued before the first use: one memory round trip
        float v[NPARAM], gk[NPARAM], m1k[NPARAM], m2k[NPARAM];
#pragma unroll
        for (int k = 0; k < NPARAM; ++k) {
            v[k] = prm[k * n + i];
            gk[k] = grads[k * n + i];
            m1k[k] = m1[k * n + i];
            m2k[k] = m2[k * n + i];
        }
        // frozen sites keep their parameters (summary section 7)
        if (v[PX] >= 0.0f && !(frozen && frozen[i])) {
            // bias corrections 1 - beta^t, every thread its own (no barrier),
            // applied as multiplications by their reciprocals
            const float ibc1 = (float)(1.0 / (1.0 - pow_uint((double)a.beta1, t)));
            const float ibc2 = (float)(1.0 / (1.0 - pow_uint((double)a.beta2, t)));
            const float sig_pos = (float)maxHW;
#pragma unroll
            for (int k = 0; k < NPARAM; ++k) {
                const float sig = (k == PX || k == PY || k == PR) ? sig_pos : 1.0f;
                const float gh = gk[k] * sig;
                const float mk = a.beta1 * m1k[k] + (1.0f - a.beta1) * gh;
                const float vk = a.beta2 * m2k[k] + (1.0f - a.beta2) * gh * gh;
                m1[k * n + i] = mk;
                m2[k * n + i] = vk;
                const float mh = mk * ibc1, vh = vk * ibc2;
                v[k] -= a.lr[k] * sig * mh / (sqrtf(vh) + a.eps);
            }
            // the step keeps the position inside the image (x < 0 marks a pruned site)
            v[PX] = fminf(fmaxf(v[PX], 0.0f), xmax);
            v[PY] = fminf(fmaxf(v[PY], 0.0f), ymax);
#pragma unroll
            for (int k = 0; k < NPARAM; ++k) prm[k * n + i] = v[k];
        }
#pragma unroll
        for (int k = 0; k < NPARAM; ++k) grads[k * n + i] = 0.0f;
        write_record(rec, i, v[PX], v[PY], v[PLT], v[PR], v[PCR], v[PCG], v[PCB], v[PTH], v[PA],
                     1.0 / (double)maxHW);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&c->ticket_adam, 1u) == gridDim.x - 1) {
            c->adam_step = t;
            c->ticket_adam = 0;
            __threadfence();
        }
    }
}

// ---------------------------------------------------------------------------
// tau diffusion (summary B.6): one Jacobi step on the ln tau gradients, the
// neighbourhood being the candidate list at the site's own pixel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(SITE_THREADS) tau_diffuse_kernel(const float *__restrict__ prm,
                                                                   const uint32_t *__restrict__ table,
                                                                   const float *__restrict__ grads, int H, int W,
                                                                   TableGrid tg, int N, float lambda,
                                                                   float *__restrict__ out,
                                                                   const Counters *__restrict__ c) {
    const int i = blockIdx.x * SITE_THREADS + threadIdx.x;
    if (i >= N) return;
    const size_t n = (size_t)N;
    const float *g = grads + PLT * n;
    const float gi = g[i];
    float res = gi;
    const float px = prm[PX * n + i], py = prm[PY * n + i];
    if (px >= 0.0f && py >= 0.0f) {
        const float fi = floorf(px), fj = floorf(py);
        if (fi < (float)W && fj < (float)H) {
            const size_t p = tg.cell_of((int)fi, (int)fj, (size_t)fj * W + (size_t)fi);
            const uint4 *t0 = reinterpret_cast<const uint4 *>(table + (size_t)c->cur * tg.PT * K);
            const uint4 a = t0[p], b = t0[tg.PT + p];
            const uint32_t ids[K] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            double sum = 0.0;
            int cnt = 0;
#pragma unroll
            for (int q = 0; q < K; ++q) {
                const uint32_t id = ids[q];
                if (id >= (uint32_t)N || id == (uint32_t)i) continue;
                if (!(prm[PX * n + id] >= 0.0f)) continue;
                sum += (double)g[id];
                ++cnt;
            }
            if (cnt > 0) res = (float)((1.0 - (double)lambda) * (double)gi + (double)lambda * (sum / cnt));
        }
    }
    out[i] = res;
}

// 8-bit interleaved RGB -> planar float32 target, one pixel per thread
__global__ void __launch_bounds__(SITE_THREADS) target_u8_kernel(const uint8_t *__restrict__ src, long long P,
                                                                 float *__restrict__ target) {
    const long long p = (long long)blockIdx.x * SITE_THREADS + threadIdx.x;
    if (p >= P) return;
    const uint8_t *px = src + 3 * p;
    target[p] = __fdiv_rn((float)px[0], 255.0f);
    target[P + p] = __fdiv_rn((float)px[1], 255.0f);
    target[2 * P + p] = __fdiv_rn((float)px[2], 255.0f);
}

inline dim3 tile_grid(int H, int W) { return dim3((W + TILE_X - 1) / TILE_X, (H + TILE_Y - 1) / TILE_Y); }
inline unsigned site_blocks(long long n) { return (unsigned)((n + SITE_THREADS - 1) / SITE_THREADS); }
inline Counters *host_counters(const Dev &d) { return reinterpret_cast<Counters *>(d.ws); }
inline TableGrid grid_of(const Dev &d) { return TableGrid{d.cell, d.GW, (size_t)d.PT}; }

}  // namespace

size_t densify_offset(int H, int W) {
    // loss partials sized for 8 x 8 tiles, the smallest tile any kernel uses
    const size_t tiles = (size_t)((W + 7) / 8) * (size_t)((H + 7) / 8);
    return (COUNTERS_BYTES + tiles * sizeof(double) + 255) / 256 * 256;
}

size_t fixed_offset(int H, int W, int N) {
    return (densify_offset(H, W) + 256 + 3 * sizeof(uint32_t) * (size_t)N + 255) / 256 * 256;
}

// the refresh's score cache: 8 float32 scores per list (32 bytes a pixel)
size_t lcache_offset(int H, int W, int N) {
    return (fixed_offset(H, W, N) + NPARAM * sizeof(unsigned long long) * (size_t)N + 255) / 256 * 256;
}

size_t workspace_bytes(int H, int W, int N) {
    // densify scratch: a 256-byte header, then the parent and free-slot lists;
    // then one float per site for tau diffusion; then the deterministic
    // backward's 64-bit sums, one per (parameter, site); then the refresh's
    // score cache
    return lcache_offset(H, W, N) + 8 * sizeof(float) * (size_t)H * (size_t)W;
}

cudaError_t launch_tau_diffuse(const Dev &d, float lambda, cudaStream_t st) {
    float *scratch = reinterpret_cast<float *>(reinterpret_cast<char *>(d.ws) + densify_offset(d.H, d.W) + 256 +
                                               2 * sizeof(uint32_t) * (size_t)d.N);
    tau_diffuse_kernel<<<site_blocks(d.N), SITE_THREADS, 0, st>>>(d.params, d.table, d.grads, d.H, d.W, grid_of(d),
                                                                  d.N, lambda, scratch, host_counters(d));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return cudaMemcpyAsync(d.grads + (size_t)PLT * d.N, scratch, sizeof(float) * (size_t)d.N,
                           cudaMemcpyDeviceToDevice, st);
}

cudaError_t launch_init_counters(const Dev &d, uint32_t seed, cudaStream_t st) {
    init_counters_kernel<<<1, 1, 0, st>>>(host_counters(d), seed);
    return cudaGetLastError();
}

cudaError_t launch_set_fit_state(const Dev &d, uint32_t pass_counter, uint32_t adam_step, uint32_t seed,
                                 cudaStream_t st) {
    set_fit_state_kernel<<<1, 1, 0, st>>>(host_counters(d), pass_counter, adam_step, seed);
    return cudaGetLastError();
}

cudaError_t launch_mark_inactive(const Dev &d, int from, cudaStream_t st) {
    if (from >= d.N) return cudaSuccess;
    mark_inactive_kernel<<<site_blocks(d.N - from), SITE_THREADS, 0, st>>>(d.params, d.N, from);
    return cudaGetLastError();
}

cudaError_t launch_target_u8(const Dev &d, const uint8_t *src, cudaStream_t st) {
    target_u8_kernel<<<site_blocks(d.P), SITE_THREADS, 0, st>>>(src, d.P, d.target);
    return cudaGetLastError();
}

cudaError_t launch_records(const Dev &d, cudaStream_t st) {
    records_kernel<<<site_blocks(d.N), SITE_THREADS, 0, st>>>(d.params, d.N, 1.0 / (double)(d.H > d.W ? d.H : d.W),
                                                            d.records);
    return cudaGetLastError();
}

cudaError_t launch_topk_exact(const Dev &d, const int64_t *pix, int64_t n, uint32_t *out, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    topk_exact_kernel<<<site_blocks(n), SITE_THREADS, 0, st>>>(d.records, d.N, d.GH, d.GW, (float)d.cell, pix, n,
                                                              out);
    return cudaGetLastError();
}

cudaError_t launch_clear_table(const Dev &d, cudaStream_t st) {
    seed_clear_kernel<<<148 * 8, 256, 0, st>>>(d.table, d.PT, host_counters(d));
    return cudaGetLastError();
}

cudaError_t launch_seed(const Dev &d, cudaStream_t st) {
    seed_clear_kernel<<<148 * 8, 256, 0, st>>>(d.table, d.PT, host_counters(d));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    seed_scatter_kernel<<<site_blocks(d.N), SITE_THREADS, 0, st>>>(d.params, d.N, d.H, d.W, d.cell, d.GW, d.PT,
                                                                 d.table, host_counters(d));
    return cudaGetLastError();
}

// propagation passes merge their candidates as batches (measured faster than
// one-by-one insertion at every jump of the refresh, and within 15 % of it
// for a lone jump-1 pass); the JFA prepass inserts
template <bool F16>
void launch_propagate_f(const Dev &d, int jump, int G, cudaStream_t st) {
    const uint4 *c16 = F16 ? d.cand16 : nullptr;
    propagate_kernel<F16, true><<<tile_grid(d.GH, d.GW), dim3(TILE_X, TILE_Y), 0, st>>>(
        d.records, c16, d.table, d.GH, d.GW, (float)d.cell, d.N, jump, G, host_counters(d), nullptr);
}

cudaError_t launch_propagate(const Dev &d, int jump, int G, cudaStream_t st, int score_cache) {
    // jumps 1 and 2 on the pixel grid: the tile kernel, whose tile index
    // scores every distinct candidate of a tile once from shared memory (a
    // refresh's passes after jump 4 read no score cache)
    if ((jump == 1 || jump == 2) && d.cell == 1 && !d.f16) return launch_propagate_tile(d, jump, G, st);
    if (score_cache == 0) {
        if (d.f16)
            launch_propagate_f<true>(d, jump, G, st);
        else
            launch_propagate_f<false>(d, jump, G, st);
        return cudaGetLastError();
    }
    float4 *lc = reinterpret_cast<float4 *>(reinterpret_cast<char *>(d.ws) + lcache_offset(d.H, d.W, d.N));
    const dim3 grid = tile_grid(d.GH, d.GW), block(TILE_X, TILE_Y);
    if (d.f16 && score_cache == 1)
        propagate_kernel<true, true, 1><<<grid, block, 0, st>>>(d.records, d.cand16, d.table, d.GH, d.GW,
                                                                (float)d.cell, d.N, jump, G, host_counters(d), lc);
    else if (d.f16)
        propagate_kernel<true, true, 2><<<grid, block, 0, st>>>(d.records, d.cand16, d.table, d.GH, d.GW,
                                                                (float)d.cell, d.N, jump, G, host_counters(d), lc);
    else if (score_cache == 1)
        propagate_kernel<false, true, 1><<<grid, block, 0, st>>>(d.records, nullptr, d.table, d.GH, d.GW,
                                                                 (float)d.cell, d.N, jump, G, host_counters(d), lc);
    else
        propagate_kernel<false, true, 2><<<grid, block, 0, st>>>(d.records, nullptr, d.table, d.GH, d.GW,
                                                                 (float)d.cell, d.N, jump, G, host_counters(d), lc);
    return cudaGetLastError();
}

cudaError_t launch_pack_cand16(const Dev &d, cudaStream_t st) {
    pack_cand16_kernel<<<site_blocks(d.N), SITE_THREADS, 0, st>>>(d.records, d.N, d.cand16);
    return cudaGetLastError();
}

cudaError_t launch_jfa3x3(const Dev &d, int jump, cudaStream_t st, int score_cache) {
    float4 *lc = reinterpret_cast<float4 *>(reinterpret_cast<char *>(d.ws) + lcache_offset(d.H, d.W, d.N));
    if (score_cache == 1)
        jfa3x3_kernel<1><<<tile_grid(d.GH, d.GW), dim3(TILE_X, TILE_Y), 0, st>>>(
            d.records, d.table, d.GH, d.GW, (float)d.cell, d.N, jump, host_counters(d), lc);
    else if (score_cache == 2)
        jfa3x3_kernel<2><<<tile_grid(d.GH, d.GW), dim3(TILE_X, TILE_Y), 0, st>>>(
            d.records, d.table, d.GH, d.GW, (float)d.cell, d.N, jump, host_counters(d), lc);
    else
        jfa3x3_kernel<0><<<tile_grid(d.GH, d.GW), dim3(TILE_X, TILE_Y), 0, st>>>(
            d.records, d.table, d.GH, d.GW, (float)d.cell, d.N, jump, host_counters(d), nullptr);
    return cudaGetLastError();
}

cudaError_t launch_render(const Dev &d, float *image, cudaStream_t st) {
    render_kernel<<<tile_grid(d.H, d.W), dim3(TILE_X, TILE_Y), 0, st>>>(d.records, d.table, d.H, d.W, grid_of(d),
                                                                        d.N, image, host_counters(d));
    return cudaGetLastError();
}

cudaError_t launch_render_backward_det(const Dev &d, cudaStream_t st) {
    unsigned long long *fixed =
        reinterpret_cast<unsigned long long *>(reinterpret_cast<char *>(d.ws) + fixed_offset(d.H, d.W, d.N));
    cudaError_t e = launch_fit_tile_cached_det(d, fixed, st);
    if (e != cudaSuccess) return e;
    const long long n = (long long)NPARAM * d.N;
    fixed_to_grads_kernel<<<site_blocks(n), SITE_THREADS, 0, st>>>(fixed, d.grads, n);
    return cudaGetLastError();
}

cudaError_t launch_adam(const Dev &d, const AdamHyper &h, cudaStream_t st, unsigned finish_tiles) {
    AdamArgs a;
    for (int k = 0; k < NPARAM; ++k) a.lr[k] = h.lr[k];
    a.beta1 = h.beta1;
    a.beta2 = h.beta2;
    a.eps = h.eps;
    adam_kernel<<<site_blocks(d.N), SITE_THREADS, 0, st>>>(d.params, d.grads, d.adam_m, d.adam_v, d.records, d.N,
                                                          d.H > d.W ? d.H : d.W, nextafterf((float)d.W, 0.0f),
                                                          nextafterf((float)d.H, 0.0f), a, d.frozen, host_counters(d),
                                                          finish_tiles, (double)d.P);
    return cudaGetLastError();
}

}  // namespace sad
