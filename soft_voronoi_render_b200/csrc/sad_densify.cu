// sad_densify.cu -- GPU-resident budget control: prune and densify
// ("Soft Anisotropic Diagrams for Differentiable Image Representation",
// summary B.5: sites are split by the score energy / mass^alpha along a
// covariance-estimated axis, children take target colours, reduced ln tau and
// r and fresh Adam state; the lowest removal scores are deactivated with
// x = -1; reading notes, key design 4: the error-density heuristic).
//
// densify_plan_kernel (one block) counts the active sites, selects the sites
// to prune (smallest removal delta) and to split (largest score) with an
// exact radix select on 64-bit keys (value, then smaller id first), applies
// the prune and lists the parents and the free slots in ascending id.
// densify_split_kernel then writes the two children of every parent.  The
// site count never leaves the device.
#include <cfloat>

#include "sad_device.cuh"
#include "sad_launch.h"

namespace sad {

namespace {

constexpr int PLAN_THREADS = 1024;
constexpr int SPLIT_THREADS = 256;

struct DensifyHeader {
    uint32_t n_split, n_prune, n_active, n_free;
};

// order-preserving map of a float (no NaN) onto uint32
__device__ __forceinline__ uint32_t ord_f32(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// the float32 split score E / max(m, eps)^alpha, IEEE division and square root
__device__ __forceinline__ float split_score(float m, float E, float alpha, float eps) {
    const float mm = m > eps ? m : eps;
    return alpha == 0.5f ? __fdiv_rn(E, __fsqrt_rn(mm)) : __fdiv_rn(E, powf(mm, alpha));
}

// selection keys: larger = chosen first; ties go to the smaller id; 0 = not eligible
__device__ __forceinline__ unsigned long long prune_key(const float *prm, const float *stats, int N, int i) {
    const float x = prm[PX * (size_t)N + i];
    const float d = stats[5 * (size_t)N + i];
    if (!(x >= 0.0f) || d != d) return 0ull;
    return ((unsigned long long)(~ord_f32(d)) << 32) | (unsigned long long)(~(uint32_t)i);
}

__device__ __forceinline__ unsigned long long split_key(const float *prm, const float *stats, int N, int i,
                                                        float alpha, float eps) {
    const float x = prm[PX * (size_t)N + i];
    if (!(x >= 0.0f)) return 0ull;
    const float sc = split_score(stats[i], stats[(size_t)N + i], alpha, eps);
    if (sc != sc) return 0ull;
    return ((unsigned long long)ord_f32(sc) << 32) | (unsigned long long)(~(uint32_t)i);
}

struct PlanSmem {
    uint32_t hist[256];
    uint32_t warp_tot[PLAN_THREADS / 32];
    unsigned long long prefix;
    uint32_t remaining, total;
};

__device__ uint32_t block_sum(PlanSmem &sm, uint32_t v) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) sm.warp_tot[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x < 32) {
        uint32_t t = sm.warp_tot[threadIdx.x];
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (threadIdx.x == 0) sm.total = t;
    }
    __syncthreads();
    return sm.total;
}

// The n-th largest non-zero key (n >= 1, at most the number of non-zero
// keys): eight rounds of an 8-bit MSB radix select over all sites.
template <typename KeyFn>
__device__ unsigned long long block_select(PlanSmem &sm, int N, uint32_t n, KeyFn key_of) {
    unsigned long long prefix = 0ull, mask = 0ull;
    uint32_t remaining = n;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int b = threadIdx.x; b < 256; b += PLAN_THREADS) sm.hist[b] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < N; i += PLAN_THREADS) {
            const unsigned long long k = key_of(i);
            if (k != 0ull && (k & mask) == prefix) atomicAdd(&sm.hist[(k >> shift) & 0xFFull], 1u);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t rem = remaining;
            int b = 255;
            for (; b > 0; --b) {
                if (sm.hist[b] >= rem) break;
                rem -= sm.hist[b];
            }
            sm.prefix = prefix | ((unsigned long long)b << shift);
            sm.remaining = rem;
        }
        __syncthreads();
        prefix = sm.prefix;
        remaining = sm.remaining;
        mask |= 0xFFull << shift;
        __syncthreads();
    }
    return prefix;
}

// write the ids i (ascending) with pred(i) into out[0 .. limit)
template <typename Pred>
__device__ void block_compact(PlanSmem &sm, int N, uint32_t limit, uint32_t *out, Pred pred) {
    uint32_t base = 0;
    for (int c0 = 0; c0 < N; c0 += PLAN_THREADS) {
        const int i = c0 + threadIdx.x;
        const bool f = i < N && pred(i);
        const uint32_t bal = __ballot_sync(0xffffffffu, f);
        const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
        if (lane == 0) sm.warp_tot[wid] = __popc(bal);
        __syncthreads();
        if (threadIdx.x < 32) {
            const uint32_t t = sm.warp_tot[threadIdx.x];
            uint32_t incl = t;
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
                if (threadIdx.x >= o) incl += x;
            }
            sm.warp_tot[threadIdx.x] = incl - t;  // exclusive prefix of warp totals
            if (threadIdx.x == 31) sm.total = incl;
        }
        __syncthreads();
        if (f) {
            const uint32_t pos = base + sm.warp_tot[wid] + __popc(bal & ((1u << lane) - 1u));
            if (pos < limit) out[pos] = (uint32_t)i;
        }
        base += sm.total;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(PLAN_THREADS) densify_plan_kernel(float *prm, const float *__restrict__ stats,
                                                                    int N, DensifyArgs a, uint32_t *parents,
                                                                    uint32_t *freel, DensifyHeader *hdr) {
    __shared__ PlanSmem sm;
    uint32_t act = 0, pe = 0;
    for (int i = threadIdx.x; i < N; i += PLAN_THREADS) {
        act += prm[PX * (size_t)N + i] >= 0.0f;
        pe += prune_key(prm, stats, N, i) != 0ull;
    }
    const uint32_t n_active = block_sum(sm, act);
    const uint32_t n_pe = block_sum(sm, pe);
    uint32_t n_prune = (uint32_t)((double)a.prune_frac * (double)n_active);
    if (n_prune > n_pe) n_prune = n_pe;
    if (n_prune > 0) {
        const unsigned long long T =
            block_select(sm, N, n_prune, [&](int i) { return prune_key(prm, stats, N, i); });
        for (int i = threadIdx.x; i < N; i += PLAN_THREADS) {
            const unsigned long long k = prune_key(prm, stats, N, i);
            if (k != 0ull && k >= T) prm[PX * (size_t)N + i] = -1.0f;
        }
    }
    __syncthreads();
    uint32_t fr = 0, se = 0;
    for (int i = threadIdx.x; i < N; i += PLAN_THREADS) {
        fr += !(prm[PX * (size_t)N + i] >= 0.0f);
        se += split_key(prm, stats, N, i, a.alpha, a.eps) != 0ull;
    }
    const uint32_t n_free = block_sum(sm, fr);
    const uint32_t n_se = block_sum(sm, se);
    long long want = (long long)n_prune + (long long)a.grow;
    if (want > (long long)n_free) want = n_free;
    if (want > (long long)n_se) want = n_se;
    const uint32_t n_split = want > 0 ? (uint32_t)want : 0u;
    if (n_split > 0) {
        const unsigned long long T =
            block_select(sm, N, n_split, [&](int i) { return split_key(prm, stats, N, i, a.alpha, a.eps); });
        block_compact(sm, N, n_split, parents, [&](int i) {
            const unsigned long long k = split_key(prm, stats, N, i, a.alpha, a.eps);
            return k != 0ull && k >= T;
        });
        block_compact(sm, N, n_split, freel, [&](int i) { return !(prm[PX * (size_t)N + i] >= 0.0f); });
    }
    if (threadIdx.x == 0) {
        hdr->n_split = n_split;
        hdr->n_prune = n_prune;
        hdr->n_active = n_active;
        hdr->n_free = n_free;
    }
}

__global__ void __launch_bounds__(SPLIT_THREADS) densify_split_kernel(float *prm, float *m1, float *m2,
                                                                      const float *__restrict__ stats,
                                                                      const float *__restrict__ target, int H,
                                                                      int W, int N, DensifyArgs a,
                                                                      const uint32_t *__restrict__ parents,
                                                                      const uint32_t *__restrict__ freel,
                                                                      const DensifyHeader *__restrict__ hdr) {
    const uint32_t r = blockIdx.x * SPLIT_THREADS + threadIdx.x;
    if (r >= hdr->n_split) return;
    const size_t n = (size_t)N;
    const uint32_t a_id = parents[r], b_id = freel[r];
    float pv[NPARAM];
#pragma unroll
    for (int j = 0; j < NPARAM; ++j) pv[j] = prm[j * n + a_id];
    // split axis: major eigenvector of the error-weighted second moment
    const double E = stats[n + a_id];
    double dx = 0.0, dy = 0.0;
    bool ok = false;
    if (E > 0.0) {
        const double cxx = (double)stats[2 * n + a_id] / E, cxy = (double)stats[3 * n + a_id] / E,
                     cyy = (double)stats[4 * n + a_id] / E;
        const double hm = 0.5 * (cxx - cyy);
        const double lam = 0.5 * (cxx + cyy) + sqrt(hm * hm + cxy * cxy);
        if (lam > 0.0) {
            double ex, ey;
            if (cxy != 0.0) {
                ex = lam - cyy;
                ey = cxy;
            } else if (cxx >= cyy) {
                ex = 1.0;
                ey = 0.0;
            } else {
                ex = 0.0;
                ey = 1.0;
            }
            const double nrm = sqrt(ex * ex + ey * ey);
            ex /= nrm;
            ey /= nrm;
            if (ex < 0.0 || (ex == 0.0 && ey < 0.0)) {
                ex = -ex;
                ey = -ey;
            }
            const double off = (double)a.offset_scale * sqrt(lam);
            dx = off * ex;
            dy = off * ey;
            ok = true;
        }
    }
    if (!ok) {
        // no usable statistics: the metric's long axis (v when a > 0, else u)
        const double th = pv[PTH], c = cos(th), s = sin(th), f = (double)a.fallback_offset;
        if (pv[PA] > 0.0f) {
            dx = -s * f;
            dy = c * f;
        } else {
            dx = c * f;
            dy = s * f;
        }
    }
    const double maxx = nextafter((double)(float)W, 0.0), maxy = nextafter((double)(float)H, 0.0);
    const size_t P = (size_t)H * W;
#pragma unroll
    for (int side = 0; side < 2; ++side) {
        const uint32_t dst = side == 0 ? a_id : b_id;
        const double sg = side == 0 ? 1.0 : -1.0;
        double x = (double)pv[PX] + sg * dx, y = (double)pv[PY] + sg * dy;
        x = x < 0.0 ? 0.0 : (x > maxx ? maxx : x);
        y = y < 0.0 ? 0.0 : (y > maxy ? maxy : y);
        float fxv = __double2float_rn(x), fyv = __double2float_rn(y);
        if (fxv >= (float)W) fxv = nextafterf((float)W, 0.0f);
        if (fyv >= (float)H) fyv = nextafterf((float)H, 0.0f);
        const size_t pix = (size_t)floorf(fyv) * W + (size_t)floorf(fxv);
        prm[PX * n + dst] = fxv;
        prm[PY * n + dst] = fyv;
        prm[PLT * n + dst] = pv[PLT] - a.log_tau_shift;
        prm[PR * n + dst] = pv[PR] * a.r_scale;
        prm[PCR * n + dst] = target[pix];
        prm[PCG * n + dst] = target[P + pix];
        prm[PCB * n + dst] = target[2 * P + pix];
        prm[PTH * n + dst] = pv[PTH];
        prm[PA * n + dst] = pv[PA];
#pragma unroll
        for (int j = 0; j < NPARAM; ++j) {
            m1[j * n + dst] = 0.0f;
            m2[j * n + dst] = 0.0f;
        }
    }
}

}  // namespace

cudaError_t launch_densify(const Dev &d, const DensifyArgs &a, cudaStream_t st) {
    char *base = reinterpret_cast<char *>(d.ws) + densify_offset(d.H, d.W);
    DensifyHeader *hdr = reinterpret_cast<DensifyHeader *>(base);
    uint32_t *parents = reinterpret_cast<uint32_t *>(base + 256);
    uint32_t *freel = parents + d.N;
    densify_plan_kernel<<<1, PLAN_THREADS, 0, st>>>(d.params, d.stats, d.N, a, parents, freel, hdr);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const unsigned blocks = (unsigned)((d.N + SPLIT_THREADS - 1) / SPLIT_THREADS);
    densify_split_kernel<<<blocks, SPLIT_THREADS, 0, st>>>(d.params, d.adam_m, d.adam_v, d.stats, d.target, d.H,
                                                          d.W, d.N, a, parents, freel, hdr);
    return cudaGetLastError();
}

}  // namespace sad
