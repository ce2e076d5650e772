// sad_fused_kernel.cuh -- device code of the fused fitting pass: the tile
// state and the kernel (host launchers and the one-block finishing kernel in
// sad_fused.cu, the only file that includes this one).
//
// One steady-state fitting pass over the image in a single kernel: the
// jump-1 candidate propagation (reading notes, key design 3;
// summary section 4 "Candidate maintenance") fused with the soft Apollonius
// render, the MSE loss and the analytic backward (summary B.4).
//
// A block owns a 32 x FY pixel tile (FY = 16 where there are at least 4
// pixels per site, else 8; one warp per row).  It first gathers the distinct
// site ids that appear in the candidate lists of the tile and of its
// one-pixel halo (the only lists a jump-1 pass can read) into a tile-local
// dense index of at most 128 sites, stages those sites' records in shared
// memory and gives each pixel a 128-bit membership mask.  The candidate union of a pixel is then the
// OR of five masks, so every distinct candidate is scored exactly once.  The
// same dense index is the per-tile gradient accumulator: the role the pages
// give to a hashed shared-memory table (summary section 5 and B.4), here
// built once per tile from the lists instead of by probing per contribution.
// A tile whose lists hold more than 128 distinct sites takes a generic path
// (per-candidate de-duplication against the running top-8, global atomics).
//
// The same kernel without the propagation (PROP = false) renders and
// differentiates the cached lists as they stand, for the iterations between
// candidate updates (summary B.3): no halo, no new lists, the pass counter
// and the current table are left alone.  Without the render and backward
// (BWD = false) it is a propagation pass on its own, at jump JK = 1 or 2
// (with a halo of width JK; at jump 2 the tile and its halo still hold at
// most about 120 distinct sites during a refresh, within the index).
#pragma once

#include <cuda.h>

#include "sad_device.cuh"

namespace sad {

namespace {

constexpr int FX = 32;                                 // tile width: one warp per row
constexpr int HX = FX + 2;                             // halo row length (halo width 1)
constexpr int UCAP = 128;                              // tile-local site capacity
constexpr int UW = UCAP / 32;                          // mask words
constexpr int UHASH_BITS = 9;
constexpr int UHASH = 1 << UHASH_BITS;
constexpr int UPROBES = 8;
constexpr uint32_t NOLOC = 0xFFFFFFFFu;
constexpr uint32_t NOSLOT = 0xFFFFu;
constexpr unsigned FULL = 0xffffffffu;

// top-8 list carrying each entry's tile-local index
struct Top8L {
    float l[K];
    uint32_t id[K];
    uint32_t lx[K];

    __device__ __forceinline__ void clear() {
#pragma unroll
        for (int q = 0; q < K; ++q) {
            l[q] = -__int_as_float(0x7f800000);
            id[q] = EMPTY;
            lx[q] = NOLOC;
        }
    }
    __device__ __forceinline__ bool has(uint32_t x) const {
        bool h = false;
#pragma unroll
        for (int q = 0; q < K; ++q) h |= (id[q] == x);
        return h;
    }
    __device__ __forceinline__ bool beats_last(float lv, uint32_t iv) const {
        return ranks_above(lv, iv, l[K - 1], id[K - 1]);
    }
    __device__ __forceinline__ void insert(float lv, uint32_t iv, uint32_t xv) {
#pragma unroll
        for (int q = 0; q < K; ++q) {
            const bool a = ranks_above(lv, iv, l[q], id[q]);
            const float tl = a ? l[q] : lv;
            const uint32_t ti = a ? id[q] : iv;
            const uint32_t tx = a ? lx[q] : xv;
            l[q] = a ? lv : l[q];
            id[q] = a ? iv : id[q];
            lx[q] = a ? xv : lx[q];
            lv = tl;
            iv = ti;
            xv = tx;
        }
    }
    // compare-exchange: entry i must rank above entry j
    __device__ __forceinline__ void cx(int i, int j) {
        const bool s = ranks_above(l[j], id[j], l[i], id[i]);
        const float a = l[i];
        const uint32_t b = id[i], c = lx[i];
        l[i] = s ? l[j] : l[i];
        id[i] = s ? id[j] : id[i];
        lx[i] = s ? lx[j] : lx[i];
        l[j] = s ? a : l[j];
        id[j] = s ? b : id[j];
        lx[j] = s ? c : lx[j];
    }
    __device__ __forceinline__ bool in_order() const {
        bool o = true;
#pragma unroll
        for (int q = 0; q + 1 < K; ++q) o &= !ranks_above(l[q + 1], id[q + 1], l[q], id[q]);
        return o;
    }
};

__device__ __forceinline__ uint32_t uhash(uint32_t id) { return (id * 2654435761u) >> (32 - UHASH_BITS); }

// insert a site id into the tile's key table (linear probing, compare-and-swap)
// and return the slot that holds it, or NOSLOT when the probes run out.  The
// lane that adds a new key also gives it the next dense tile-local index
// (lid, and ulist for the first UCAP of them).
__device__ __forceinline__ uint32_t ukey_insert(uint32_t *keys, uint32_t *lid, uint32_t *ulist, uint32_t *ucount,
                                                uint32_t id) {
    uint32_t s = uhash(id);
#pragma unroll 1
    for (int q = 0; q < UPROBES; ++q) {
        const uint32_t k = *reinterpret_cast<volatile uint32_t *>(keys + s);
        if (k == id) return s;
        if (k == EMPTY) {
            const uint32_t old = atomicCAS(keys + s, EMPTY, id);
            if (old == EMPTY) {
                const uint32_t u = atomicAdd(ucount, 1u);
                lid[s] = u;
                if (u < UCAP) ulist[u] = id;
                return s;
            }
            if (old == id) return s;
        }
        s = (s + 1) & (UHASH - 1);
    }
    return NOSLOT;
}

// insert once per run of equal ids on consecutive lanes: the first lane of
// the run inserts, the others take its slot (neighbouring pixels mostly hold
// the same id in the same slot, which would otherwise contend for one key).
// An id >= N inserts nothing and gets NOSLOT.
__device__ __forceinline__ uint32_t warp_insert(uint32_t *keys, uint32_t *lid, uint32_t *ulist, uint32_t *ucount,
                                                uint32_t id, uint32_t N, int lane) {
    const uint32_t prev = __shfl_up_sync(FULL, id, 1);
    const bool head = lane == 0 || prev != id;
    const uint32_t heads = __ballot_sync(FULL, head);
    const int start = 31 - __clz(heads & (0xFFFFFFFFu >> (31 - lane)));
    uint32_t s = NOSLOT;
    if (head && id < N) s = ukey_insert(keys, lid, ulist, ucount, id);
    return __shfl_sync(FULL, s, start);
}

__device__ __forceinline__ uint32_t ukey_lookup(const uint32_t *keys, const uint32_t *lid, uint32_t id) {
    uint32_t s = uhash(id);
#pragma unroll 1
    for (int q = 0; q < UPROBES; ++q) {
        const uint32_t k = keys[s];
        if (k == id) return lid[s];
        if (k == EMPTY) return NOLOC;
        s = (s + 1) & (UHASH - 1);
    }
    return NOLOC;
}

// four local indices (< 256) as the bytes of one word, and back
__device__ __forceinline__ uint32_t pack_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}
__device__ __forceinline__ uint32_t byte_of(uint32_t w, int q) { return __byte_perm(w, 0, 0x4440 | (q & 3)); }

// ---- TMA staging of the list block (shared-memory barrier + bulk tensor copy)
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// one arrival that also announces the bytes the copy will deliver
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// wait until the barrier's phase with the given parity has completed, giving
// up after a bounded number of polls (false: the copy did not arrive)
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, int polls) {
    const uint32_t a = smem_u32(bar);
#pragma unroll 1
    for (int n = 0; n < polls; ++n) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// 3-D tile copy global -> shared (no multicast), completion counted in bytes
// on the barrier.  x (words) must be a multiple of 4: 16-byte boundaries.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// JK: the jump of the propagation and the width of the halo (1, or 2 for
// the propagation alone)
template <int FY, bool STATS, bool TMA = false, int JK = 1>
struct FusedSmem {
    static constexpr int HXJ = FX + 2 * JK;  // halo row length
    static constexpr int FT = FX * FY, HN = HXJ * (FY + 2 * JK), RING = HN - FT;
    // TMA form: a tile's two list planes with the one-pixel halo, as the copy
    // lands them: [plane][halo row][4 words per halo column]
    static constexpr int LBZ = TMA ? 2 : 1, LBY = TMA ? FY + 2 : 1, LBX = TMA ? 4 * HX : 4;
    static constexpr uint32_t LBYTES = LBZ * LBY * LBX * 4;
    // The tile's (pixel, slot) entries grouped by site, each site's run padded
    // to a multiple of the group size gs (8, or 9 where that makes the groups
    // fit one per thread) so that every group belongs to one site: at most
    // FT + 7 UCAP / 8 groups.  Entry e of group g is stored at [e][g]; the
    // plane strides are 4 words modulo 32 so that the scatter's consecutive
    // entries (consecutive e) fall in distinct banks.
    static constexpr int GMAX = FY == 16 ? 9 : 8;
    static constexpr int NG = FT + 7 * UCAP / 8;
    static constexpr int NGS = (NG + 15) / 16 * 16 + 2;    // float2 planes
    static constexpr int NGS16 = (NG + 63) / 64 * 64 + 8;  // uint16 planes
    alignas(128) uint32_t lbuf[LBZ][LBY][LBX];
    uint64_t bar;                   // completion of the staging copy
    uint32_t keys[UHASH];
    uint32_t lid[UHASH];
    uint32_t ulist[UCAP];
    float4 urec[REC_F4][UCAP + 1];  // field-major; entry UCAP is all zero
    uint4 masks[HN];                // 128-bit membership of every tile + halo pixel
    uint32_t cnt[UCAP];             // (pixel, slot) entries per local site
    uint32_t cursor[UCAP];          // where each site's entries start
    float4 pixg[FT];                // per pixel: dL/dchat (3), chat . dL/dchat
    float2 ent_wl[GMAX][NGS];       // softmax weight, logit
    uint16_t ent_pu[GMAX][NGS16];   // pixel (low 9 bits), local site (high 7 bits)
    float ent_rd[STATS ? GMAX : 1][STATS ? NGS : 1];  // removal delta (budget statistics)
    float warp_loss[FY];
    uint32_t warp_cnt[3][FY];       // per warp: empty pixels, global-atomic pixels, dropped ids
    uint32_t n_groups;
    uint32_t next_tile;             // persistent form: the tile after this one
    uint32_t gs;                    // entries per group
    uint32_t ucount;
    int overflow;
};

// halo ring pixel r -> halo coordinates for a halo of width JK: the JK top
// rows, the JK bottom rows, then the JK left and JK right columns of each of
// the FY inner rows
template <int FY, int JK = 1>
__device__ __forceinline__ void ring_coords(int r, int &hx, int &hy) {
    constexpr int HXJ = FX + 2 * JK, HY = FY + 2 * JK;
    if (r < JK * HXJ) {
        hy = r / HXJ;
        hx = r - hy * HXJ;
    } else if (r < 2 * JK * HXJ) {
        const int q = r - JK * HXJ;
        hy = HY - JK + q / HXJ;
        hx = q - (q / HXJ) * HXJ;
    } else {
        const int q = r - 2 * JK * HXJ;
        const int c = q % (2 * JK);
        hy = JK + q / (2 * JK);
        hx = c < JK ? c : FX + c;
    }
}

// bounds of the run of equal keys (in lane order) that holds this lane
__device__ __forceinline__ void run_bounds(uint32_t key, int lane, int &start, int &tail_lane) {
    const uint32_t key_next = __shfl_down_sync(FULL, key, 1);
    const bool tail = lane == 31 || key_next != key;
    const uint32_t tails = __ballot_sync(FULL, tail);
    const uint32_t prev = tails & ((1u << lane) - 1u);
    start = prev ? 32 - __clz(prev) : 0;
    tail_lane = __ffs(tails & (0xFFFFFFFFu << lane)) - 1;
}

// gradient contributions of one (pixel, slot) with softmax weight w and logit
// l (both 0 for an unused slot, which then contributes exact zeros):
//   gamma = w (c . g - chat . g),  dL/dc = w g,  dL/dln tau = gamma l,
//   dL/dr = gamma k,  dL/dp = gamma G'delta / m,
//   dL/da = -gamma (k^2 e^a alpha^2 - k^2 e^-a beta^2) / (2 m),
//   dL/dtheta = -gamma alpha beta (k^2 e^a - k^2 e^-a) / m
// with m = sqrt(delta^T G' delta) = k n (0 where m = 0).
template <int NV>
__device__ __forceinline__ void slot_grad(const float4 r0, const float4 r1, const float4 r2, const float4 r3,
                                          float fx, float fy, float l, float w, float gr, float gg, float gb,
                                          float cdg, float (&v)[NV], float &dx, float &dy) {
    dx = fx - r0.x;
    dy = fy - r0.y;
    const float u1 = fmaf(r0.z, dx, r0.w * dy);
    const float u2 = fmaf(r1.x, dy, r0.w * dx);
    const float qf = fmaf(dx, u1, dy * u2);
    const float im = qf > 0.0f ? rsqrtf(qf) : 0.0f;
    const float gamma = w * (fmaf(r2.x, gr, fmaf(r2.y, gg, r2.z * gb)) - cdg);
    const float gi = gamma * im;
    const float al = r2.w * dx + r3.x * dy;   // u . delta
    const float be = -r3.x * dx + r2.w * dy;  // v . delta
    v[PX] = gi * u1;
    v[PY] = gi * u2;
    v[PLT] = gamma * l;
    v[PR] = gamma * r1.z;
    v[PCR] = w * gr;
    v[PCG] = w * gg;
    v[PCB] = w * gb;
    v[PTH] = -gi * al * be * (r3.y - r3.z);
    v[PA] = -0.5f * gi * (r3.y * al * al - r3.z * be * be);
}

// The same contributions added into the sums a of one site, with the factors
// that are the site's own left for the end (group_finish): a[PR] collects
// gamma (times k), a[PTH] gi al be (times -(k^2 e^a - k^2 e^-a)) and a[PA]
// gi (k^2 e^a al^2 - k^2 e^-a be^2) (times -1/2), where gi = gamma / m.
template <int NV>
__device__ __forceinline__ void slot_accumulate(const float4 r0, const float4 r1, const float4 r2, const float4 r3,
                                                float fx, float fy, float l, float w, float gr, float gg, float gb,
                                                float cdg, float (&a)[NV], float &dx, float &dy) {
    dx = fx - r0.x;
    dy = fy - r0.y;
    const float u1 = fmaf(r0.z, dx, r0.w * dy);
    const float u2 = fmaf(r1.x, dy, r0.w * dx);
    const float qf = fmaf(dx, u1, dy * u2);
    const float im = qf > 0.0f ? rsqrtf(qf) : 0.0f;
    const float gamma = w * (fmaf(r2.x, gr, fmaf(r2.y, gg, r2.z * gb)) - cdg);
    const float gi = gamma * im;
    const float al = fmaf(r2.w, dx, r3.x * dy);   // u . delta
    const float be = fmaf(r2.w, dy, -r3.x * dx);  // v . delta
    a[PX] = fmaf(gi, u1, a[PX]);
    a[PY] = fmaf(gi, u2, a[PY]);
    a[PLT] = fmaf(gamma, l, a[PLT]);
    a[PR] += gamma;
    a[PCR] = fmaf(w, gr, a[PCR]);
    a[PCG] = fmaf(w, gg, a[PCG]);
    a[PCB] = fmaf(w, gb, a[PCB]);
    const float gal = gi * al, gbe = gi * be;
    a[PTH] = fmaf(gal, be, a[PTH]);
    a[PA] = fmaf(gal, r3.y * al, a[PA]);
    a[PA] = fmaf(-gbe, r3.z * be, a[PA]);
}

template <int NV>
__device__ __forceinline__ void group_finish(const float4 r1, const float4 r3, float (&a)[NV]) {
    a[PR] *= r1.z;
    a[PTH] *= -(r3.y - r3.z);
    a[PA] *= -0.5f;
}

// budget-control statistics of one (pixel, slot) (summary B.4-B.5): mass w,
// energy w e, error-weighted second moments w e (dx^2, dx dy, dy^2) and the
// removal delta rd, with e = |chat - t|^2 = (P / 2)^2 |g|^2
template <int NV>
__device__ __forceinline__ void slot_stats(float w, float ex, float dx, float dy, float rd, float (&v)[NV]) {
    const float we = w * ex;
    v[NPARAM + 0] = w;
    v[NPARAM + 1] = we;
    v[NPARAM + 2] = we * dx * dx;
    v[NPARAM + 3] = we * dx * dy;
    v[NPARAM + 4] = we * dy * dy;
    v[NPARAM + 5] = rd;
}

// Removal delta of one slot: |(chat - w c) / (1 - w) - t|^2 - |chat - t|^2,
// evaluated as (a - b) . (a + b) with b = chat - t (er, eg, eb) and
// a - b = w (c_rest - c), c_rest the blend of the other slots.  Their
// unnormalised sums are Z - e_q and Z chat - e_q c, except for the dominant
// slot, whose are summed directly (zmm, cm*), so that removing a site that
// holds almost all the weight subtracts no two nearly equal numbers.  Where
// the other slots hold less than 1e-6 of the weight, 1 - w is clamped to
// 1e-6.
__device__ __forceinline__ float removal_delta(float eq, float4 c, bool dominant, float Z, float iz, float chr,
                                               float chg, float chb, float zmm, float cmr, float cmg, float cmb,
                                               float er, float eg, float eb) {
    const float w = eq * iz;
    const float oz = dominant ? zmm : Z - eq;
    const float ocr = dominant ? cmr : fmaf(-eq, c.x, chr * Z);
    const float ocg = dominant ? cmg : fmaf(-eq, c.y, chg * Z);
    const float ocb = dominant ? cmb : fmaf(-eq, c.z, chb * Z);
    float dr, dg, db;
    if (oz * iz >= 1e-6f) {
        const float ioz = 1.0f / oz;
        dr = w * (ocr * ioz - c.x);
        dg = w * (ocg * ioz - c.y);
        db = w * (ocb * ioz - c.z);
    } else {
        dr = ocr * iz * 1e6f - chr;
        dg = ocg * iz * 1e6f - chg;
        db = ocb * iz * 1e6f - chb;
    }
    return dr * (2.0f * er + dr) + dg * (2.0f * eg + dg) + db * (2.0f * eb + db);
}

// generic candidate offer (no tile index): dedup against the running list
__device__ __forceinline__ void offer_global(Top8L &t, uint32_t id, const float4 *__restrict__ rec, uint32_t N,
                                             float fx, float fy) {
    if (id >= N) return;
    if (t.has(id)) return;
    float px, py, A, B, C, b;
    load_rank_fields(rec, id, px, py, A, B, C, b);
    if (!(px >= 0.0f)) return;
    const float l = sad_logit(px, py, A, B, C, b, fx, fy);
    if (l != l) return;
    if (t.beats_last(l, id)) t.insert(l, id, NOLOC);
}

__device__ __forceinline__ void generic_pass(Top8L &t, const uint4 *__restrict__ in0, const uint4 *__restrict__ in1,
                                             const float4 *__restrict__ rec, uint32_t N, int H, int W, int i, int j,
                                             float fx, float fy, int jump) {
    // own list, then the neighbours at (-k, 0), (+k, 0), (0, -k), (0, +k)
#pragma unroll 1
    for (int d = 0; d < 5; ++d) {
        const int ni = i + (d == 1 ? -jump : (d == 2 ? jump : 0));
        const int nj = j + (d == 3 ? -jump : (d == 4 ? jump : 0));
        if (ni < 0 || ni >= W || nj < 0 || nj >= H) continue;
        const size_t pn = (size_t)nj * W + ni;
        const uint4 a = in0[pn], b = in1[pn];
        offer_global(t, a.x, rec, N, fx, fy);
        offer_global(t, a.y, rec, N, fx, fy);
        offer_global(t, a.z, rec, N, fx, fy);
        offer_global(t, a.w, rec, N, fx, fy);
        offer_global(t, b.x, rec, N, fx, fy);
        offer_global(t, b.y, rec, N, fx, fy);
        offer_global(t, b.z, rec, N, fx, fy);
        offer_global(t, b.w, rec, N, fx, fy);
    }
}

template <int FY, bool PROP, bool STATS, bool TMA, bool BWD = true, int JK = 1, bool DET = false>
__global__ void __launch_bounds__(FX * FY, 1024 / (FX * FY))
    fit_tile_kernel(const float4 *__restrict__ rec, uint32_t *table, const float *__restrict__ target, int H, int W,
                    int N, int G, float *__restrict__ image, float *__restrict__ grads, float *__restrict__ stats,
                    void *ws, TableGrid lists, const __grid_constant__ CUtensorMap lmap, int tiles_x,
                    uint32_t n_tiles, unsigned long long *__restrict__ fixed = nullptr,
                    uint32_t test_flags = 0) {
    static_assert(!(PROP && STATS), "the statistics come with the cached-list form");
    static_assert(!TMA || (PROP && !STATS), "list staging serves the propagating form");
    static_assert(BWD || (PROP && !STATS && !TMA), "the propagation alone is a form of the propagating pass");
    static_assert(JK == 1 || !BWD, "a wider halo serves the propagation alone");
    static_assert(JK == 1 || !TMA, "the staged list block has a one-pixel halo");
    static_assert(!DET || (!PROP && !STATS && BWD), "the order-independent sums serve the cached-list backward");
    using Smem = FusedSmem<FY, STATS, TMA, JK>;
    constexpr int HXJ = Smem::HXJ;
    constexpr int NV = STATS ? NPARAM + NSTAT : NPARAM;
    constexpr int FT = Smem::FT, HN = Smem::HN, RING = Smem::RING;
    constexpr int NRE = (RING * K + FT - 1) / FT;  // halo (pixel, slot) entries per thread
    extern __shared__ __align__(128) unsigned char fused_smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(fused_smem_raw);
    Counters *c = ws_counters(ws);
    const uint32_t cur = c->cur, pass = c->pass_counter, seed = c->seed;
    const int lane = threadIdx.x, ty = threadIdx.y;
    const int tid = ty * FX + lane;
    const size_t P = (size_t)H * W;
    // the cached-list form also reads lists kept per cell of a coarser grid
    const size_t PT = PROP ? P : lists.PT;
    const uint4 *in0 = reinterpret_cast<const uint4 *>(table + cur * PT * K);
    const uint4 *in1 = in0 + PT;
    uint4 *out0 = reinterpret_cast<uint4 *>(table + (cur ^ 1u) * P * K);
    uint4 *out1 = out0 + P;
    const uint32_t Nu = (uint32_t)N;

    // TMA form: a persistent block starts on tile blockIdx.x and takes its
    // next tile from a ticket as soon as it starts the current one, so that
    // the next tile's list block (tile + halo, both planes) is copied into
    // shared memory while it works on the current one.  A copy that does
    // not arrive within the wait's bound switches the block to global loads
    // (block-uniform, counted in staging_fallbacks).
    uint32_t tile = TMA ? blockIdx.x : blockIdx.y * gridDim.x + blockIdx.x;
    // test_flags bit 0 (set only by the bounds-checked build's tests): the
    // first staging copy is withheld, so the first wait runs out (after a
    // short bound) and the block falls back to plain loads
    const bool withhold = (test_flags & 1u) != 0;
    const int polls = withhold ? 1024 : (1 << 22);
    uint32_t phase = 0, lost_phase = 0;
    bool staged = TMA, lost = false;
    if constexpr (TMA) {
        staged = (smem_u32(&sm.lbuf[0][0][0]) & 127u) == 0u;
        if (tid == 0 && staged) {
            mbar_init(&sm.bar, 1u);
            if (tile < n_tiles && !withhold) {
                mbar_arrive_expect_tx(&sm.bar, Smem::LBYTES);
                tma_load_3d(&sm.lbuf[0][0][0], &lmap, &sm.bar, 4 * ((int)(tile % (uint32_t)tiles_x) * FX - 1),
                            (int)(tile / (uint32_t)tiles_x) * FY - 1, 2 * (int)cur);
            }
        }
        if (tid == 0 && !staged) atomicAdd(&c->staging_fallbacks, 1u);
        __syncthreads();
    }
#pragma unroll 1
    for (;;) {
    if (TMA && tile >= n_tiles) break;
    const int bx = TMA ? (int)(tile % (uint32_t)tiles_x) : (int)blockIdx.x;
    const int by = TMA ? (int)(tile / (uint32_t)tiles_x) : (int)blockIdx.y;
    const int i0 = bx * FX, j0 = by * FY;
    const int i = i0 + lane, j = j0 + ty;
    const bool inside = i < W && j < H;

    // ---- the lists first (staged copy, else global loads), then the target
    // halo entry e = tid + x FT is ring pixel e % RING, slot e / RING; rv[x]
    // holds its id, then its hash slot | mask cell << 16 (NOLOC: none)
    uint32_t own[K];
    uint32_t rv[NRE], rcell[NRE];
    bool got = false;
    if constexpr (TMA) {
        if (staged) got = mbar_wait_bounded(&sm.bar, phase, polls);
        if (got) {
            // halo row hy, halo column hx of plane z is lbuf[z][hy][4 hx ...]
            uint4 a = make_uint4(EMPTY, EMPTY, EMPTY, EMPTY), b = a;
            if (inside) {
                a = *reinterpret_cast<const uint4 *>(&sm.lbuf[0][ty + 1][4 * (lane + 1)]);
                b = *reinterpret_cast<const uint4 *>(&sm.lbuf[1][ty + 1][4 * (lane + 1)]);
            }
            own[0] = a.x; own[1] = a.y; own[2] = a.z; own[3] = a.w;
            own[4] = b.x; own[5] = b.y; own[6] = b.z; own[7] = b.w;
#pragma unroll
            for (int x = 0; x < NRE; ++x) {
                const int e = tid + x * FT;
                uint32_t id = EMPTY, cell = 0;
                if (e < RING * K) {
                    const int r = e % RING, q = e / RING;
                    int hx, hy;
                    ring_coords<FY, JK>(r, hx, hy);
                    cell = (uint32_t)(hy * HXJ + hx);
                    const int gi = i0 - JK + hx, gj = j0 - JK + hy;
                    if (gi >= 0 && gi < W && gj >= 0 && gj < H) id = sm.lbuf[q >> 2][hy][4 * hx + (q & 3)];
                }
                rv[x] = id;
                rcell[x] = cell;
            }
        }
    }
    if (!got) {
        uint4 a = make_uint4(EMPTY, EMPTY, EMPTY, EMPTY), b = a;
        if (inside) {
            const size_t p = (size_t)j * W + i;
            const size_t pt = PROP ? p : lists.cell_of(i, j, p);
            a = in0[pt];
            b = in1[pt];
        }
        own[0] = a.x; own[1] = a.y; own[2] = a.z; own[3] = a.w;
        own[4] = b.x; own[5] = b.y; own[6] = b.z; own[7] = b.w;
        if (PROP) {
#pragma unroll
            for (int x = 0; x < NRE; ++x) {
                const int e = tid + x * FT;
                uint32_t id = EMPTY, cell = 0;
                if (e < RING * K) {
                    const int r = e % RING, q = e / RING;
                    int hx, hy;
                    ring_coords<FY, JK>(r, hx, hy);
                    cell = (uint32_t)(hy * HXJ + hx);
                    const int gi = i0 - JK + hx, gj = j0 - JK + hy;
                    if (gi >= 0 && gi < W && gj >= 0 && gj < H)
                        id = table[cur * P * K + (size_t)(q >> 2) * P * 4 + ((size_t)gj * W + gi) * 4 + (q & 3)];
                }
                rv[x] = id;
                rcell[x] = cell;
            }
        }
    }
    // the target is read last: bring its lines into L2 now, registers later
    if (BWD && inside && lane == 0) {
        const size_t p = (size_t)j * W + i;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(target + p));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(target + P + p));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(target + 2 * P + p));
    }

    for (int q = tid; q < UHASH; q += FT) sm.keys[q] = EMPTY;
    if (PROP)
        for (int q = tid; q < HN; q += FT) sm.masks[q] = make_uint4(0, 0, 0, 0);
    if (tid < UCAP) sm.cnt[tid] = 0;
    if (tid < REC_F4) sm.urec[tid][UCAP] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tid == 0) {
        sm.ucount = 0;
        sm.overflow = 0;
    }
    if constexpr (TMA) {
        // every thread is done with the staging buffer: refill it with the
        // next tile's lists, unless a copy failed to arrive
        const bool all_got = __syncthreads_and(got || !staged) != 0;
        if (staged && !all_got) {
            staged = false;
            lost = true;
            lost_phase = phase;
            if (tid == 0) atomicAdd(&c->staging_fallbacks, 1u);
        }
        if (tid == 0) {
            const uint32_t next = gridDim.x + atomicAdd(&c->tile_ticket, 1u);
            sm.next_tile = next;
            if (staged && next < n_tiles) {
                mbar_arrive_expect_tx(&sm.bar, Smem::LBYTES);
                tma_load_3d(&sm.lbuf[0][0][0], &lmap, &sm.bar, 4 * ((int)(next % (uint32_t)tiles_x) * FX - 1),
                            (int)(next / (uint32_t)tiles_x) * FY - 1, 2 * (int)cur);
            }
        }
        phase ^= 1u;
    } else {
        __syncthreads();
    }

    // ---- A1: the distinct ids of the tile and halo lists -------------------
    uint32_t slot[K];  // hash slot of each own entry
    bool ok = true;
#pragma unroll
    for (int q = 0; q < K; ++q) {
        slot[q] = warp_insert(sm.keys, sm.lid, sm.ulist, &sm.ucount, own[q], Nu, lane);
        ok &= own[q] >= Nu || slot[q] != NOSLOT;
    }
    if (PROP) {
#pragma unroll
        for (int x = 0; x < NRE; ++x) {
            const uint32_t s = warp_insert(sm.keys, sm.lid, sm.ulist, &sm.ucount, rv[x], Nu, lane);
            ok &= rv[x] >= Nu || s != NOSLOT;
            rv[x] = s != NOSLOT ? (s | (rcell[x] << 16)) : NOLOC;
        }
    }
    if (!ok) sm.overflow = 1;
    __syncthreads();
    const bool fast = !sm.overflow && sm.ucount <= UCAP;  // block-uniform
    const uint32_t ucount = fast ? sm.ucount : 0u;

    // slot q's local index in byte q & 3 of own_lx[q >> 2] (0xFF: none)
    uint32_t own_lx_lo = 0xFFFFFFFFu, own_lx_hi = 0xFFFFFFFFu;
    if (fast) {
        // ---- A3: site records (loads in flight first), local indices, masks
        for (uint32_t u = tid; u < ucount; u += FT) {
            if (!SAD_CHECK(sm.ulist[u] < Nu, ws)) continue;
            const float4 *R = rec + (size_t)sm.ulist[u] * REC_F4;
            sm.urec[0][u] = __ldg(R);
            sm.urec[1][u] = __ldg(R + 1);
            sm.urec[2][u] = __ldg(R + 2);
            sm.urec[3][u] = __ldg(R + 3);
        }
        uint32_t ux[K];
#pragma unroll
        for (int q = 0; q < K; ++q)
            ux[q] = (slot[q] != NOSLOT && SAD_CHECK(slot[q] < UHASH && sm.lid[slot[q]] < UCAP, ws)) ? sm.lid[slot[q]]
                                                                                                   : 0xFFu;
        own_lx_lo = pack_bytes(ux[0], ux[1], ux[2], ux[3]);
        own_lx_hi = pack_bytes(ux[4], ux[5], ux[6], ux[7]);
        if (PROP) {
            uint32_t *m = reinterpret_cast<uint32_t *>(&sm.masks[(ty + JK) * HXJ + lane + JK]);
#pragma unroll
            for (int q = 0; q < K; ++q)
                if (ux[q] != 0xFFu) atomicOr(m + (ux[q] >> 5), 1u << (ux[q] & 31u));
#pragma unroll
            for (int x = 0; x < NRE; ++x) {
                if (rv[x] != NOLOC && SAD_CHECK((rv[x] & 0xFFFFu) < UHASH && (rv[x] >> 16) < (uint32_t)HN, ws)) {
                    const uint32_t u = sm.lid[rv[x] & 0xFFFFu];
                    if (SAD_CHECK(u < UCAP, ws))
                        atomicOr(reinterpret_cast<uint32_t *>(&sm.masks[rv[x] >> 16]) + (u >> 5), 1u << (u & 31u));
                }
            }
        }
    }
    __syncthreads();

    // ---- C: jump-1 propagation -------------------------------------------
    const float fx = (float)i + 0.5f, fy = (float)j + 0.5f;
    Top8L t;
    t.clear();
    unsigned dropped = 0;
    if (inside && !PROP) {
        // cached lists: every slot as it stands, like the standalone backward
        // (a repeated id counts twice, an id >= N is reported as dropped)
#pragma unroll
        for (int q = 0; q < K; ++q) {
            const uint32_t id = own[q];
            dropped += (id >= Nu && id != EMPTY);
            if (id >= Nu) continue;
            uint32_t u = byte_of(q < 4 ? own_lx_lo : own_lx_hi, q);
            float4 r0;
            float2 r1;
            if (u < UCAP) {
                r0 = sm.urec[0][u];
                r1 = make_float2(sm.urec[1][u].x, sm.urec[1][u].y);
            } else {
                u = NOLOC;
                load_rank_fields(rec, id, r0.x, r0.y, r0.z, r0.w, r1.x, r1.y);
            }
            if (!(r0.x >= 0.0f)) continue;
            t.l[q] = sad_logit(r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, fx, fy);
            t.id[q] = id;
            t.lx[q] = u;
        }
    }
    uint32_t nw[UW] = {0u, 0u, 0u, 0u};  // candidates the neighbours add (tile-local bits)
    float l8 = -__int_as_float(0x7f800000);
    if (inside && PROP) {
        if (fast) {
            // the pixel's own list re-scored in its previous order, which the
            // new scores rarely change
            int nslots = 0;
#pragma unroll
            for (int q = 0; q < K; ++q) {
                const uint32_t u = byte_of(q < 4 ? own_lx_lo : own_lx_hi, q);
                float l = -__int_as_float(0x7f800000);
                bool v = false;
                uint32_t gid = EMPTY;
                if (u != 0xFFu) {
                    ++nslots;
                    const float4 r0 = sm.urec[0][u];
                    const float4 r1 = sm.urec[1][u];
                    if (r0.x >= 0.0f) {
                        l = sad_logit(r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, fx, fy);
                        v = l == l;
                        gid = sm.ulist[u];
                    }
                }
                t.l[q] = v ? l : -__int_as_float(0x7f800000);
                t.id[q] = v ? gid : EMPTY;
                t.lx[q] = v ? u : NOLOC;
            }
            const int hc = (ty + JK) * HXJ + lane + JK;
            const uint4 own_mask = sm.masks[hc];
            // a list holding one id twice keeps it once (the pass works on sets)
            if (nslots != __popc(own_mask.x) + __popc(own_mask.y) + __popc(own_mask.z) + __popc(own_mask.w)) {
#pragma unroll
                for (int q = 1; q < K; ++q)
#pragma unroll
                    for (int r = 0; r < q; ++r)
                        if (t.id[q] != EMPTY && t.id[q] == t.id[r]) {
                            t.l[q] = -__int_as_float(0x7f800000);
                            t.id[q] = EMPTY;
                            t.lx[q] = NOLOC;
                        }
            }
            // the list is nearly sorted: odd-even transposition rounds until it
            // is in order (4 rounds = 8 passes always sort 8 entries)
#pragma unroll 1
            for (int round = 0; round < 4 && !t.in_order(); ++round) {
                t.cx(0, 1); t.cx(2, 3); t.cx(4, 5); t.cx(6, 7);
                t.cx(1, 2); t.cx(3, 4); t.cx(5, 6);
            }
            // the candidates the four neighbours add
            const uint4 mL = sm.masks[hc - JK], mR = sm.masks[hc + JK], mU = sm.masks[hc - JK * HXJ],
                        mD = sm.masks[hc + JK * HXJ];
            nw[0] = (mL.x | mR.x | mU.x | mD.x) & ~own_mask.x;
            nw[1] = (mL.y | mR.y | mU.y | mD.y) & ~own_mask.y;
            nw[2] = (mL.z | mR.z | mU.z | mD.z) & ~own_mask.z;
            nw[3] = (mL.w | mR.w | mU.w | mD.w) & ~own_mask.w;
            l8 = t.l[K - 1];
        }
    }
    // A neighbour's candidate can only enter if it scores at least the
    // pixel's current 8th, which insertions only raise: every candidate is
    // scored once against it, then the few that pass are inserted (in the
    // same order as scoring them one by one, so the same result).
    uint32_t pass_bits[UW] = {0u, 0u, 0u, 0u};
    if (inside && PROP && fast) {
#pragma unroll
        for (int w = 0; w < UW; ++w) {
            uint32_t bits = nw[w];
            while (bits) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1u;
                const uint32_t u = (uint32_t)(w * 32 + b);
                if (!SAD_CHECK(u < ucount, ws)) continue;
                const float4 r0 = sm.urec[0][u];
                const float2 r1 = *reinterpret_cast<const float2 *>(&sm.urec[1][u]);
                const float l = sad_logit(r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, fx, fy);
                // NaN (inactive site or NaN parameters) fails the test
                if (r0.x >= 0.0f && l >= l8) pass_bits[w] |= 1u << b;
            }
        }
    }
    if (inside && PROP) {
        if (fast) {
#pragma unroll
            for (int w = 0; w < UW; ++w) {
                uint32_t bits = pass_bits[w];
                while (bits) {
                    const uint32_t u = (uint32_t)(w * 32 + __ffs(bits) - 1);
                    bits &= bits - 1u;
                    if (!SAD_CHECK(u < ucount, ws)) continue;
                    const float4 r0 = sm.urec[0][u];
                    const float2 r1 = *reinterpret_cast<const float2 *>(&sm.urec[1][u]);
                    const float l = sad_logit(r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, fx, fy);
                    const uint32_t gid = sm.ulist[u];
                    if (t.beats_last(l, gid)) t.insert(l, gid, u);
                }
            }
        } else {
            generic_pass(t, in0, in1, rec, Nu, H, W, i, j, fx, fy, JK);
        }
        if (G > 0) {
            // two injections per round: both records in flight together
            uint32_t h = inject_state(seed, pass, (uint32_t)((size_t)j * W + i));
#pragma unroll 1
            for (int g = 0; g < G; g += 2) {
                uint32_t id[2];
                float px[2], py[2], A[2], B[2], C[2], b[2];
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    if (g + x < G) h = xorshift32(h);
                    id[x] = g + x < G ? __umulhi(h, Nu) : EMPTY;  // < N when drawn
                    load_rank_fields(rec, id[x] < Nu ? id[x] : 0u, px[x], py[x], A[x], B[x], C[x], b[x]);
                }
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const float l = sad_logit(px[x], py[x], A[x], B[x], C[x], b[x], fx, fy);
                    if (id[x] < Nu && px[x] >= 0.0f && l == l && t.beats_last(l, id[x]) && !t.has(id[x])) {
                        // a winner the tile index holds keeps its local index
                        const uint32_t u = fast ? ukey_lookup(sm.keys, sm.lid, id[x]) : NOLOC;
                        t.insert(l, id[x], u < ucount ? u : NOLOC);
                    }
                }
            }
        }
        const size_t p = (size_t)j * W + i;
        out0[p] = make_uint4(t.id[0], t.id[1], t.id[2], t.id[3]);
        out1[p] = make_uint4(t.id[4], t.id[5], t.id[6], t.id[7]);
    }
    // !BWD: a jump-1 propagation pass on its own (the whole block leaves here)
    if constexpr (!BWD) return;

    // ---- D: render, loss and backward on the new lists ---------------------
    // A slot is valid iff its logit is finite: every list form above leaves
    // -inf in the slots it does not fill.
    unsigned vmask = 0;
    float M = -__int_as_float(0x7f800000);
#pragma unroll
    for (int q = 0; q < K; ++q) {
        const bool v = inside && isfinite(t.l[q]);
        vmask |= (unsigned)v << q;
        M = v ? fmaxf(M, t.l[q]) : M;
    }
    const float Mf = vmask ? M : 0.0f;
    float Z = 0.0f, cr = 0.0f, cg = 0.0f, cb = 0.0f;
    bool far_slot = false;  // a slot whose site has no tile-local index
#pragma unroll
    for (int q = 0; q < K; ++q) {
        const bool v = vmask >> q & 1u;
        const float e = v ? __expf(t.l[q] - Mf) : 0.0f;
        Z += e;
        const float4 r2 = sm.urec[2][t.lx[q] < UCAP ? t.lx[q] : UCAP];  // NOLOC: the zero entry
        cr = fmaf(e, r2.x, cr);
        cg = fmaf(e, r2.y, cg);
        cb = fmaf(e, r2.z, cb);
        far_slot |= v && t.lx[q] == NOLOC;
    }
    if (__any_sync(FULL, far_slot)) {
#pragma unroll
        for (int q = 0; q < K; ++q) {
            if ((vmask >> q & 1u) && t.lx[q] == NOLOC) {
                const float e = __expf(t.l[q] - Mf);
                const float4 r2 = __ldg(rec + (size_t)t.id[q] * REC_F4 + 2);
                cr = fmaf(e, r2.x, cr);
                cg = fmaf(e, r2.y, cg);
                cb = fmaf(e, r2.z, cb);
            }
        }
    }
    const float iz = vmask ? __frcp_rn(Z) : 0.0f;
    cr *= iz;
    cg *= iz;
    cb *= iz;
    float lsum = 0.0f, gr = 0.0f, gg = 0.0f, gb = 0.0f;
    float er = 0.0f, eg = 0.0f, eb = 0.0f;
    if (inside) {
        const size_t p = (size_t)j * W + i;
        const float tr = __ldg(target + p), tg = __ldg(target + P + p), tb = __ldg(target + 2 * P + p);
        const float two_over_P = 2.0f / (float)P;
        er = cr - tr;
        eg = cg - tg;
        eb = cb - tb;
        lsum = er * er + eg * eg + eb * eb;
        gr = er * two_over_P;
        gg = eg * two_over_P;
        gb = eb * two_over_P;
        if (image) {
            image[p] = cr;
            image[P + p] = cg;
            image[2 * P + p] = cb;
        }
    }
    // STATS: the dominant slot (largest weight, first in slot order) and the
    // weight and colour sums of the other slots
    int qstar = -1;
    float zmm = 0.0f, cmr = 0.0f, cmg = 0.0f, cmb = 0.0f;
    if constexpr (STATS) {
        float emax = -1.0f;
#pragma unroll
        for (int q = 0; q < K; ++q) {
            const float e = (vmask >> q & 1u) ? __expf(t.l[q] - Mf) : -1.0f;
            if (e > emax) {
                emax = e;
                qstar = q;
            }
        }
#pragma unroll
        for (int q = 0; q < K; ++q) {
            if (!(vmask >> q & 1u) || q == qstar) continue;
            const float e = __expf(t.l[q] - Mf);
            const float4 c2 = t.lx[q] != NOLOC ? sm.urec[2][t.lx[q]] : __ldg(rec + (size_t)t.id[q] * REC_F4 + 2);
            zmm += e;
            cmr = fmaf(e, c2.x, cmr);
            cmg = fmaf(e, c2.y, cmg);
            cmb = fmaf(e, c2.z, cmb);
        }
    }
    // ---- D2: group the tile's (pixel, slot) entries by site ----------------
    // Entries whose site has a tile-local index are counted here and summed
    // site by site below; the rare rest (injected winners from outside the
    // tile index, crowded tiles) go straight to global atomics.
    unsigned global_adds = 0;
    const float cdg = fmaf(cr, gr, fmaf(cg, gg, cb * gb));
    sm.pixg[tid] = make_float4(gr, gg, gb, cdg);
    // slot q's place among its site's entries (16 bits, two slots a word):
    // the count's atomic returns where the run starts
    uint32_t offw[K / 2];
#pragma unroll
    for (int q = 0; q < K; ++q) {
        const bool vq = vmask >> q & 1u;
        // one counter update per run of equal sites in this slot
        const uint32_t key = (vq && t.lx[q] != NOLOC) ? t.lx[q] : EMPTY;
        int start, tail_lane;
        run_bounds(key, lane, start, tail_lane);
        uint32_t first = 0;
        if (lane == tail_lane && key != EMPTY && SAD_CHECK(key < UCAP, ws))
            first = atomicAdd(&sm.cnt[key], (uint32_t)(tail_lane - start + 1));
        first = __shfl_sync(FULL, first, tail_lane);
        const uint32_t off = (first + (uint32_t)(lane - start)) & 0xFFFFu;
        offw[q >> 1] = (q & 1) ? (offw[q >> 1] | off << 16) : off;
        if (vq && t.lx[q] == NOLOC) {
            const float4 *R = rec + (size_t)t.id[q] * REC_F4;
            const float4 r2 = __ldg(R + 2);
            const float eq = __expf(t.l[q] - Mf);
            float v[NV], dx, dy;
            slot_grad(__ldg(R), __ldg(R + 1), r2, __ldg(R + 3), fx, fy, t.l[q], eq * iz, gr, gg, gb, cdg, v, dx, dy);
            if constexpr (STATS)
                slot_stats(eq * iz, er * er + eg * eg + eb * eb, dx, dy,
                           removal_delta(eq, r2, q == qstar, Z, iz, cr, cg, cb, zmm, cmr, cmg, cmb, er, eg, eb), v);
            ++global_adds;
            if constexpr (DET) {
#pragma unroll
                for (int k = 0; k < NPARAM; ++k)
                    atomicAdd(fixed + (size_t)k * N + t.id[q], (unsigned long long)__float2ll_rn(v[k] * FIXED_SCALE));
            } else {
#pragma unroll
                for (int k = 0; k < NPARAM; ++k) atomicAdd(grads + (size_t)k * N + t.id[q], v[k]);
            }
            if constexpr (STATS) {
#pragma unroll
                for (int k = 0; k < NSTAT; ++k) atomicAdd(stats + (size_t)k * N + t.id[q], v[NPARAM + k]);
            }
        }
    }
    __syncthreads();
    if (ty == 0) {
        // exclusive scan of the 128 counts, each rounded up to a multiple of
        // the group size, by one warp (4 per lane).  Groups of 9 where they
        // then fit one per thread (the padding of groups of 8 pushes a full
        // tile just past one group per thread).
        uint32_t c4[4], run = 0, n9 = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            c4[e] = sm.cnt[lane * 4 + e];
            n9 += (c4[e] + 8u) / 9u;
        }
        n9 = __reduce_add_sync(FULL, n9);
        const uint32_t gs = (Smem::GMAX == 9 && n9 <= (uint32_t)FT) ? 9u : 8u;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            c4[e] = gs == 9u ? (c4[e] + 8u) / 9u * 9u : (c4[e] + 7u) & ~7u;
            run += c4[e];
        }
        uint32_t incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(FULL, incl, o);
            if (lane >= o) incl += x;
        }
        uint32_t base = incl - run;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sm.cursor[lane * 4 + e] = base;  // where the site's entries start
            base += c4[e];
        }
        if (lane == 31) {
            sm.n_groups = incl / gs;
            sm.gs = gs;
        }
    }
    __syncthreads();
    const uint32_t gs = sm.gs;
#pragma unroll
    for (int q = 0; q < K; ++q) {
        const bool vq = (vmask >> q & 1u) && t.lx[q] != NOLOC && SAD_CHECK(t.lx[q] < UCAP, ws);
        const uint32_t key = vq ? t.lx[q] : 0u;
        const uint32_t pos = sm.cursor[key] + (offw[q >> 1] >> ((q & 1) * 16) & 0xFFFFu);
        const uint32_t g = gs == 9u ? __umulhi(pos, 477218590u) : pos >> 3;  // pos / 9 exactly for pos < 2^16
        const uint32_t e = pos - g * gs;
        if (vq && SAD_CHECK(g < (uint32_t)Smem::NG && e < (uint32_t)Smem::GMAX, ws)) {
            const float eq = __expf(t.l[q] - Mf);
            sm.ent_wl[e][g] = make_float2(eq * iz, t.l[q]);
            sm.ent_pu[e][g] = (uint16_t)(tid | (key << 9));
            if constexpr (STATS)
                sm.ent_rd[e][g] = removal_delta(eq, sm.urec[2][key], q == qstar, Z, iz, cr, cg, cb, zmm, cmr, cmg,
                                                cmb, er, eg, eb);
        }
    }
    __syncthreads();
    // ---- D3: every thread sums one group of entries of one site ------------
    if constexpr (DET) {
        // order-independent: each entry's full contribution in fixed point,
        // the group and run sums in 64-bit integers
        const uint32_t ng = sm.n_groups;
        const float fx0 = (float)i0 + 0.5f, fy0 = (float)j0 + 0.5f;
#pragma unroll 1
        for (uint32_t g0 = 0; g0 < ng; g0 += FT) {
            if (g0 + (uint32_t)ty * 32u >= ng) break;  // warp-uniform
            const uint32_t g = g0 + (uint32_t)tid;
            uint32_t u = EMPTY;
            long long a[NPARAM];
#pragma unroll
            for (int k = 0; k < NPARAM; ++k) a[k] = 0;
            if (g < ng && SAD_CHECK(g < (uint32_t)Smem::NG && (sm.ent_pu[0][g] >> 9) < ucount, ws)) {
                u = sm.ent_pu[0][g] >> 9;
                const uint32_t rem = min(sm.cursor[u] + sm.cnt[u] - gs * g, gs);
                const float4 r0 = sm.urec[0][u], r1 = sm.urec[1][u], r2 = sm.urec[2][u], r3 = sm.urec[3][u];
#pragma unroll 1
                for (int e = 0; e < Smem::GMAX; ++e) {
                    if ((uint32_t)e >= rem) break;
                    if (!SAD_CHECK((sm.ent_pu[e][g] & 0x1FFu) < (uint32_t)FT, ws)) continue;
                    const uint32_t px = sm.ent_pu[e][g] & 0x1FFu;
                    const float2 wl = sm.ent_wl[e][g];
                    const float4 pa = sm.pixg[px];
                    float v[NPARAM], dx, dy;
                    slot_grad(r0, r1, r2, r3, fx0 + (float)(px & (FX - 1)), fy0 + (float)(px / FX), wl.y, wl.x, pa.x,
                              pa.y, pa.z, pa.w, v, dx, dy);
#pragma unroll
                    for (int k = 0; k < NPARAM; ++k) a[k] += __float2ll_rn(v[k] * FIXED_SCALE);
                }
            }
            const bool tail = warp_run_reduce(u, a, lane);
            if (tail && u != EMPTY) {
                const uint32_t gid = sm.ulist[u];
#pragma unroll
                for (int k = 0; k < NPARAM; ++k)
                    if (a[k]) atomicAdd(fixed + (size_t)k * N + gid, (unsigned long long)a[k]);
            }
        }
    } else {
        const uint32_t ng = sm.n_groups;
        const float fx0 = (float)i0 + 0.5f, fy0 = (float)j0 + 0.5f;
        const float half_P = 0.5f * (float)P, ex_scale = half_P * half_P;  // |chat - t|^2 = ex_scale |g|^2
#pragma unroll 1
        for (uint32_t g0 = 0; g0 < ng; g0 += FT) {
            if (g0 + (uint32_t)ty * 32u >= ng) break;  // warp-uniform
            const uint32_t g = g0 + (uint32_t)tid;
            uint32_t u = EMPTY;
            float a[NV];
#pragma unroll
            for (int k = 0; k < NV; ++k) a[k] = 0.0f;
            if (g < ng && SAD_CHECK(g < (uint32_t)Smem::NG && (sm.ent_pu[0][g] >> 9) < ucount, ws)) {
                u = sm.ent_pu[0][g] >> 9;
                const uint32_t rem = min(sm.cursor[u] + sm.cnt[u] - gs * g, gs);  // entries of the group (>= 1)
                const float4 r0 = sm.urec[0][u], r1 = sm.urec[1][u], r2 = sm.urec[2][u], r3 = sm.urec[3][u];
#pragma unroll
                for (int e = 0; e < Smem::GMAX; ++e) {
                    const bool ve = (uint32_t)e < rem && SAD_CHECK((sm.ent_pu[e][g] & 0x1FFu) < (uint32_t)FT, ws);
                    const uint32_t px = ve ? (uint32_t)(sm.ent_pu[e][g] & 0x1FFu) : 0u;
                    const float2 wl = sm.ent_wl[e][g];
                    const float4 pa = sm.pixg[px];
                    if (ve) {
                        float dx, dy;
                        slot_accumulate(r0, r1, r2, r3, fx0 + (float)(px & (FX - 1)), fy0 + (float)(px / FX), wl.y,
                                        wl.x, pa.x, pa.y, pa.z, pa.w, a, dx, dy);
                        if constexpr (STATS) {
                            float v[NV];
                            slot_stats(wl.x, ex_scale * (pa.x * pa.x + pa.y * pa.y + pa.z * pa.z), dx, dy,
                                       sm.ent_rd[e][g], v);
#pragma unroll
                            for (int k = NPARAM; k < NV; ++k) a[k] += v[k];
                        }
                    }
                }
                group_finish(r1, r3, a);
            }
            // groups of one site sit on consecutive lanes: sum each run across
            // lanes, then one global update per run
            const bool tail = warp_run_reduce(u, a, lane);
            if (tail && u != EMPTY) {
                const uint32_t gid = sm.ulist[u];
#pragma unroll
                for (int k = 0; k < NPARAM; ++k) atomicAdd(grads + (size_t)k * N + gid, a[k]);
                if constexpr (STATS) {
#pragma unroll
                    for (int k = 0; k < NSTAT; ++k) atomicAdd(stats + (size_t)k * N + gid, a[NPARAM + k]);
                }
            }
        }
    }

    // ---- E: loss partial, statistics, last-block epilogue ------------------
    for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(FULL, lsum, o);
    const unsigned b_empty = __ballot_sync(FULL, inside && !vmask);
    const unsigned b_global = __ballot_sync(FULL, global_adds != 0);
    const unsigned b_drop = __ballot_sync(FULL, dropped != 0);
    if (lane == 0) {
        sm.warp_loss[ty] = lsum;
        sm.warp_cnt[0][ty] = __popc(b_empty);
        sm.warp_cnt[1][ty] = __popc(b_global);
        sm.warp_cnt[2][ty] = __popc(b_drop);
    }
    __syncthreads();
    if (tid == 0) {
        float tl = 0.0f;
        unsigned n_empty = 0, n_global = 0, n_dropped = 0;
        for (int q = 0; q < FY; ++q) {
            tl += sm.warp_loss[q];
            n_empty += sm.warp_cnt[0][q];
            n_global += sm.warp_cnt[1][q];
            n_dropped += sm.warp_cnt[2][q];
        }
        // finish_pass_kernel, launched next, sums the partials
        ws_loss_partials(ws)[tile] = (double)tl;
        if (n_empty) atomicAdd(&c->empty_pixels, (unsigned long long)n_empty);
        if (n_global) atomicAdd(&c->hash_overflow, (unsigned long long)n_global);
        if (n_dropped) atomicAdd(&c->dropped_ids, (unsigned long long)n_dropped);
    }
    if (!TMA) break;
    tile = sm.next_tile;  // written before this tile's later barriers, rewritten after the next tile's first
    }
    // a copy that timed out may still land: let it finish (bounded) before
    // the block's shared memory is released
    if (TMA && lost && tid == 0) (void)mbar_wait_bounded(&sm.bar, lost_phase, polls);
}


}  // namespace

}  // namespace sad
