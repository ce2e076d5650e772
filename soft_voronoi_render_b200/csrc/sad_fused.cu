// sad_fused.cu -- one steady-state fitting pass over the image in a single
// kernel: the jump-1 candidate propagation (reading notes, key design 3;
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
// and the current table are left alone.
#include "sad_device.cuh"
#include "sad_launch.h"

namespace sad {

namespace {

constexpr int FX = 32;                                 // tile width: one warp per row
constexpr int HX = FX + 2;                             // halo row length
constexpr int UCAP = 128;                              // tile-local site capacity
constexpr int UW = UCAP / 32;                          // mask words
constexpr int UHASH_BITS = 9;
constexpr int UHASH = 1 << UHASH_BITS;
constexpr int UPROBES = 8;
constexpr uint32_t NOLOC = 0xFFFFFFFFu;
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

// storage slot of sorted entry idx: the low three bits are XORed with bits of
// the owning thread (idx >> 3), so that the 32 lanes reading entry 8 t + e
// of their own runs hit distinct banks
__device__ __forceinline__ uint32_t ent_slot(uint32_t idx) {
    const uint32_t t = idx >> 3;
    return idx ^ ((((t >> 3) & 3u) << 1) | ((t >> 1) & 1u));
}

__device__ __forceinline__ uint32_t uhash(uint32_t id) { return (id * 2654435761u) >> (32 - UHASH_BITS); }

// insert a site id into the tile's key table (linear probing, compare-and-swap)
__device__ __forceinline__ bool ukey_insert(uint32_t *keys, uint32_t id) {
    uint32_t s = uhash(id);
#pragma unroll 1
    for (int q = 0; q < UPROBES; ++q) {
        const uint32_t k = *reinterpret_cast<volatile uint32_t *>(keys + s);
        if (k == id) return true;
        if (k == EMPTY) {
            const uint32_t old = atomicCAS(keys + s, EMPTY, id);
            if (old == EMPTY || old == id) return true;
        }
        s = (s + 1) & (UHASH - 1);
    }
    return false;
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

template <int FY>
struct FusedSmem {
    static constexpr int FT = FX * FY, HN = HX * (FY + 2);
    uint32_t keys[UHASH];
    uint32_t lid[UHASH];
    uint32_t ulist[UCAP];
    float4 urec[REC_F4][UCAP];   // field-major: conflict-free for distinct sites
    uint4 masks[HN];             // 128-bit membership of every tile + halo pixel
    float acc[NPARAM][UCAP];      // the tile's gradient sums per local site
    uint32_t cnt[UCAP];           // (pixel, slot) entries per local site
    uint32_t cursor[UCAP];        // scatter cursor of the counting sort
    float4 pixg[FT];              // per pixel: dL/dchat (3), chat . dL/dchat
    float2 ent_wl[FT * K];        // entries grouped by site: softmax weight, logit
    uint16_t ent_pu[FT * K];      //   pixel (low 9 bits) and local site (high 7 bits)
    uint32_t ring_id[(HN - FT) * K];  // the halo lists, read once from the table
    float warp_loss[FY];
    uint32_t n_ent;
    uint32_t ucount;
    int overflow;
    int last;
};

// halo ring pixel r -> halo coordinates: top row, bottom row, then the left
// and right columns of the FY inner rows
template <int FY>
__device__ __forceinline__ void ring_coords(int r, int &hx, int &hy) {
    constexpr int HY = FY + 2;
    if (r < HX) {
        hx = r;
        hy = 0;
    } else if (r < 2 * HX) {
        hx = r - HX;
        hy = HY - 1;
    } else {
        const int q = r - 2 * HX;
        hy = 1 + (q >> 1);
        hx = (q & 1) ? HX - 1 : 0;
    }
}

__device__ __forceinline__ void set_bit(uint4 &m, uint32_t u) {
    const uint32_t b = 1u << (u & 31u);
    const uint32_t w = u >> 5;
    m.x |= (w == 0) ? b : 0u;
    m.y |= (w == 1) ? b : 0u;
    m.z |= (w == 2) ? b : 0u;
    m.w |= (w == 3) ? b : 0u;
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
__device__ __forceinline__ void slot_grad(const float4 r0, const float4 r1, const float4 r2, const float4 r3,
                                          float fx, float fy, float l, float w, float gr, float gg, float gb,
                                          float cdg, float (&v)[NPARAM]) {
    const float dx = fx - r0.x, dy = fy - r0.y;
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

// generic candidate offer (no tile index): dedup against the running list
__device__ __forceinline__ void offer_global(Top8L &t, uint32_t id, const float4 *__restrict__ rec, uint32_t N,
                                             float fx, float fy) {
    if (id >= N) return;
    if (t.has(id)) return;
    const float4 r0 = __ldg(rec + (size_t)id * REC_F4);
    if (!(r0.x >= 0.0f)) return;
    const float2 r1 = __ldg(reinterpret_cast<const float2 *>(rec + (size_t)id * REC_F4 + 1));
    const float l = sad_logit(r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, fx, fy);
    if (l != l) return;
    if (t.beats_last(l, id)) t.insert(l, id, NOLOC);
}

__device__ __forceinline__ void generic_pass(Top8L &t, const uint4 *__restrict__ in0, const uint4 *__restrict__ in1,
                                             const float4 *__restrict__ rec, uint32_t N, int H, int W, int i, int j,
                                             float fx, float fy) {
    // own list, then the neighbours at (-1, 0), (+1, 0), (0, -1), (0, +1)
#pragma unroll 1
    for (int d = 0; d < 5; ++d) {
        const int ni = i + (d == 1 ? -1 : (d == 2 ? 1 : 0));
        const int nj = j + (d == 3 ? -1 : (d == 4 ? 1 : 0));
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

template <int FY, bool PROP>
__global__ void __launch_bounds__(FX * FY, 1024 / (FX * FY)) fit_tile_kernel(const float4 *__restrict__ rec,
                                                                            uint32_t *table,
                                                         const float *__restrict__ target, int H, int W, int N,
                                                         int G, float *__restrict__ image,
                                                         float *__restrict__ grads, void *ws, TableGrid lists) {
    constexpr int FT = FX * FY, HY = FY + 2, HN = HX * HY, RING = HN - FT;
    extern __shared__ __align__(16) unsigned char fused_smem_raw[];
    FusedSmem<FY> &sm = *reinterpret_cast<FusedSmem<FY> *>(fused_smem_raw);
    Counters *c = ws_counters(ws);
    const uint32_t cur = c->cur, pass = c->pass_counter, seed = c->seed;
    const int lane = threadIdx.x, ty = threadIdx.y;
    const int tid = ty * FX + lane;
    const int i0 = blockIdx.x * FX, j0 = blockIdx.y * FY;
    const int i = i0 + lane, j = j0 + ty;
    const bool inside = i < W && j < H;
    const size_t P = (size_t)H * W;
    // the cached-list form also reads lists kept per cell of a coarser grid
    const size_t PT = PROP ? P : lists.PT;
    const uint4 *in0 = reinterpret_cast<const uint4 *>(table + cur * PT * K);
    const uint4 *in1 = in0 + PT;
    uint4 *out0 = reinterpret_cast<uint4 *>(table + (cur ^ 1u) * P * K);
    uint4 *out1 = out0 + P;
    const uint32_t Nu = (uint32_t)N;

    for (int q = tid; q < UHASH; q += FT) sm.keys[q] = EMPTY;
    if (PROP)
    for (int r = tid; r < RING; r += FT) {
        int hx, hy;
        ring_coords<FY>(r, hx, hy);
        sm.masks[hy * HX + hx] = make_uint4(0, 0, 0, 0);
    }
    for (int q = tid; q < NPARAM * UCAP; q += FT) (&sm.acc[0][0])[q] = 0.0f;
    if (tid < UCAP) sm.cnt[tid] = 0;
    if (tid == 0) {
        sm.ucount = 0;
        sm.overflow = 0;
    }
    __syncthreads();

    // the target is needed last; start its loads first
    float tr = 0.0f, tg = 0.0f, tb = 0.0f;
    if (inside) {
        const size_t p = (size_t)j * W + i;
        tr = __ldg(target + p);
        tg = __ldg(target + P + p);
        tb = __ldg(target + 2 * P + p);
    }
    // ---- A1: collect the distinct ids of the tile and halo lists ----------
    uint32_t own[K];
    {
        uint4 a = make_uint4(EMPTY, EMPTY, EMPTY, EMPTY), b = a;
        if (inside) {
            const size_t p = (size_t)j * W + i;
            const size_t pt = PROP ? p : lists.cell_of(i, j, p);
            a = in0[pt];
            b = in1[pt];
        }
        own[0] = a.x; own[1] = a.y; own[2] = a.z; own[3] = a.w;
        own[4] = b.x; own[5] = b.y; own[6] = b.z; own[7] = b.w;
    }
    bool ok = true;
#pragma unroll
    for (int q = 0; q < K; ++q) {
        // neighbouring pixels mostly hold the same id in the same slot
        const uint32_t id = own[q];
        const uint32_t prev = __shfl_up_sync(FULL, id, 1);
        if (id < Nu && !(lane > 0 && prev == id)) ok &= ukey_insert(sm.keys, id);
    }
    // the halo pixels x 8 slots, spread over all threads: entry e is halo
    // pixel e % RING, slot e / RING
    if (PROP)
    for (int e = tid; e < RING * K; e += FT) {
        const int r = e % RING, q = e / RING;
        int hx, hy;
        ring_coords<FY>(r, hx, hy);
        const int gi = i0 - 1 + hx, gj = j0 - 1 + hy;
        uint32_t id = EMPTY;
        if (gi >= 0 && gi < W && gj >= 0 && gj < H)
            id = table[cur * P * K + (size_t)(q >> 2) * P * 4 + ((size_t)gj * W + gi) * 4 + (q & 3)];
        sm.ring_id[e] = id;
        if (id < Nu) ok &= ukey_insert(sm.keys, id);
    }
    if (!ok) sm.overflow = 1;
    __syncthreads();

    // ---- A2: dense tile-local indices ------------------------------------
    for (int s = tid; s < UHASH; s += FT) {
        const uint32_t k = sm.keys[s];
        if (k != EMPTY) {
            const uint32_t u = atomicAdd(&sm.ucount, 1u);
            sm.lid[s] = u;
            if (u < UCAP) sm.ulist[u] = k;
        }
    }
    __syncthreads();
    const bool fast = !sm.overflow && sm.ucount <= UCAP;  // block-uniform
    const uint32_t ucount = fast ? sm.ucount : 0u;

    uint4 own_mask = make_uint4(0, 0, 0, 0);
    uint32_t own_lx_lo = 0xFFFFFFFFu, own_lx_hi = 0xFFFFFFFFu;  // slot q's local index in byte q (0xFF: none)
    if (fast) {
        // ---- A3: per-pixel local indices and membership masks --------------
#pragma unroll
        for (int q = 0; q < K; ++q) {
            const uint32_t u = own[q] < Nu ? ukey_lookup(sm.keys, sm.lid, own[q]) : NOLOC;
            if (u != NOLOC) set_bit(own_mask, u);
            const uint32_t b = (u == NOLOC ? 0xFFu : u) << ((q & 3) * 8);
            const uint32_t m = ~(0xFFu << ((q & 3) * 8));
            if (q < 4) own_lx_lo = (own_lx_lo & m) | b;
            else own_lx_hi = (own_lx_hi & m) | b;
        }
        if (PROP) sm.masks[(ty + 1) * HX + lane + 1] = own_mask;
        if (PROP)
        for (int e = tid; e < RING * K; e += FT) {
            const int r = e % RING;
            const uint32_t id = sm.ring_id[e];
            if (id >= Nu) continue;  // also the halo pixels outside the image
            int hx, hy;
            ring_coords<FY>(r, hx, hy);
            const uint32_t u = ukey_lookup(sm.keys, sm.lid, id);
            if (u != NOLOC) atomicOr(reinterpret_cast<uint32_t *>(&sm.masks[hy * HX + hx]) + (u >> 5), 1u << (u & 31u));
        }
        // ---- B: stage the tile's site records --------------------------------
        for (uint32_t u = tid; u < ucount; u += FT) {
            const float4 *R = rec + (size_t)sm.ulist[u] * REC_F4;
            sm.urec[0][u] = __ldg(R);
            sm.urec[1][u] = __ldg(R + 1);
            sm.urec[2][u] = __ldg(R + 2);
            sm.urec[3][u] = __ldg(R + 3);
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
            uint32_t u = NOLOC;
            float4 r0;
            float2 r1;
            if (fast) u = ((q < 4 ? own_lx_lo : own_lx_hi) >> ((q & 3) * 8)) & 0xFFu;
            if (u < UCAP) {
                r0 = sm.urec[0][u];
                r1 = make_float2(sm.urec[1][u].x, sm.urec[1][u].y);
            } else {
                u = NOLOC;
                r0 = __ldg(rec + (size_t)id * REC_F4);
                r1 = __ldg(reinterpret_cast<const float2 *>(rec + (size_t)id * REC_F4 + 1));
            }
            if (!(r0.x >= 0.0f)) continue;
            t.l[q] = sad_logit(r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, fx, fy);
            t.id[q] = id;
            t.lx[q] = u;
        }
    }
    if (inside && PROP) {
        if (fast) {
            // the pixel's own list re-scored in its previous order, which the
            // new scores rarely change
            int nslots = 0;
#pragma unroll
            for (int q = 0; q < K; ++q) {
                const uint32_t u = ((q < 4 ? own_lx_lo : own_lx_hi) >> ((q & 3) * 8)) & 0xFFu;
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
            // candidates the four neighbours add
            const int hc = (ty + 1) * HX + lane + 1;
            const uint4 mL = sm.masks[hc - 1], mR = sm.masks[hc + 1], mU = sm.masks[hc - HX],
                        mD = sm.masks[hc + HX];
            const uint32_t nw[UW] = {(mL.x | mR.x | mU.x | mD.x) & ~own_mask.x,
                                     (mL.y | mR.y | mU.y | mD.y) & ~own_mask.y,
                                     (mL.z | mR.z | mU.z | mD.z) & ~own_mask.z,
                                     (mL.w | mR.w | mU.w | mD.w) & ~own_mask.w};
#pragma unroll
            for (int w = 0; w < UW; ++w) {
                uint32_t bits = nw[w];
                while (bits) {
                    const uint32_t u = (uint32_t)(w * 32 + __ffs(bits) - 1);
                    bits &= bits - 1u;
                    const float4 r0 = sm.urec[0][u];
                    if (!(r0.x >= 0.0f)) continue;
                    const float4 r1 = sm.urec[1][u];
                    const float l = sad_logit(r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, fx, fy);
                    const uint32_t gid = sm.ulist[u];
                    if (l == l && t.beats_last(l, gid)) t.insert(l, gid, u);
                }
            }
        } else {
            generic_pass(t, in0, in1, rec, Nu, H, W, i, j, fx, fy);
        }
        if (G > 0) {
            uint32_t h = inject_state(seed, pass, (uint32_t)((size_t)j * W + i));
#pragma unroll 1
            for (int g = 0; g < G; ++g) {
                h = xorshift32(h);
                offer_global(t, __umulhi(h, Nu), rec, Nu, fx, fy);
            }
        }
        const size_t p = (size_t)j * W + i;
        out0[p] = make_uint4(t.id[0], t.id[1], t.id[2], t.id[3]);
        out1[p] = make_uint4(t.id[4], t.id[5], t.id[6], t.id[7]);
    }

    // ---- D: render, loss and backward on the new lists ---------------------
    unsigned vmask = 0;
    float M = -__int_as_float(0x7f800000);
#pragma unroll
    for (int q = 0; q < K; ++q) {
        if (inside && t.id[q] != EMPTY && isfinite(t.l[q])) {
            vmask |= 1u << q;
            M = fmaxf(M, t.l[q]);
        }
    }
    float Z = 0.0f, cr = 0.0f, cg = 0.0f, cb = 0.0f;
    bool far_slot = false;  // a slot whose site has no tile-local index
#pragma unroll
    for (int q = 0; q < K; ++q) {
        if (vmask >> q & 1u) {
            const float e = __expf(t.l[q] - M);
            Z += e;
            if (t.lx[q] != NOLOC) {
                const float4 r2 = sm.urec[2][t.lx[q]];
                cr = fmaf(e, r2.x, cr);
                cg = fmaf(e, r2.y, cg);
                cb = fmaf(e, r2.z, cb);
            } else {
                far_slot = true;
            }
        }
    }
    if (__any_sync(FULL, far_slot)) {
#pragma unroll
        for (int q = 0; q < K; ++q) {
            if ((vmask >> q & 1u) && t.lx[q] == NOLOC) {
                const float e = __expf(t.l[q] - M);
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
    if (inside) {
        const size_t p = (size_t)j * W + i;
        const float two_over_P = 2.0f / (float)P;
        const float er = cr - tr, eg = cg - tg, eb = cb - tb;
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
    // ---- D2: group the tile's (pixel, slot) entries by site ----------------
    // Entries whose site has a tile-local index are counted here and summed
    // site by site below; the rare rest (injected winners, crowded tiles) go
    // straight to global atomics.
    unsigned global_adds = 0;
    const float cdg = fmaf(cr, gr, fmaf(cg, gg, cb * gb));
    sm.pixg[tid] = make_float4(gr, gg, gb, cdg);
#pragma unroll
    for (int q = 0; q < K; ++q) {
        const bool vq = vmask >> q & 1u;
        // one counter update per run of equal sites in this slot
        const uint32_t key = (vq && t.lx[q] != NOLOC) ? t.lx[q] : EMPTY;
        int start, tail_lane;
        run_bounds(key, lane, start, tail_lane);
        if (lane == tail_lane && key != EMPTY) atomicAdd(&sm.cnt[key], (uint32_t)(tail_lane - start + 1));
        if (vq && t.lx[q] == NOLOC) {
            const float4 *R = rec + (size_t)t.id[q] * REC_F4;
            float v[NPARAM];
            slot_grad(__ldg(R), __ldg(R + 1), __ldg(R + 2), __ldg(R + 3), fx, fy, t.l[q], __expf(t.l[q] - M) * iz,
                      gr, gg, gb, cdg, v);
            ++global_adds;
#pragma unroll
            for (int k = 0; k < NPARAM; ++k) atomicAdd(grads + (size_t)k * N + t.id[q], v[k]);
        }
    }
    __syncthreads();
    if (ty == 0) {
        // exclusive scan of the 128 counts by one warp, 4 per lane
        uint32_t c4[4], run = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            c4[e] = sm.cnt[lane * 4 + e];
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
            sm.cursor[lane * 4 + e] = base;
            base += c4[e];
        }
        if (lane == 31) sm.n_ent = incl;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < K; ++q) {
        const bool vq = (vmask >> q & 1u) && t.lx[q] != NOLOC;
        const uint32_t key = vq ? t.lx[q] : EMPTY;
        int start, tail_lane;
        run_bounds(key, lane, start, tail_lane);
        uint32_t pos0 = 0;
        if (lane == tail_lane && key != EMPTY) pos0 = atomicAdd(&sm.cursor[key], (uint32_t)(tail_lane - start + 1));
        pos0 = __shfl_sync(FULL, pos0, tail_lane);
        if (vq) {
            const uint32_t pos = pos0 + (uint32_t)(lane - start);
            const uint32_t slot = ent_slot(pos);
            sm.ent_wl[slot] = make_float2(__expf(t.l[q] - M) * iz, t.l[q]);
            sm.ent_pu[slot] = (uint16_t)(tid | (key << 9));
        }
    }
    __syncthreads();
    // ---- D3: every thread sums a run of 8 consecutive entries -------------
    {
        const uint32_t n_ent = sm.n_ent;
        const float fx0 = (float)i0 + 0.5f, fy0 = (float)j0 + 0.5f;
        uint32_t cur = NOLOC;
        float4 r0 = make_float4(0.f, 0.f, 0.f, 0.f), r1 = r0, r2 = r0, r3 = r0;
        float a[NPARAM];
#pragma unroll
        for (int k = 0; k < NPARAM; ++k) a[k] = 0.0f;
        const uint32_t e0 = (uint32_t)tid * K;
#pragma unroll
        for (int e = 0; e < K; ++e) {
            const uint32_t idx = e0 + e;
            if (idx >= n_ent) break;
            const uint32_t pu = sm.ent_pu[ent_slot(idx)];
            const uint32_t u = pu >> 9, px = pu & 0x1FFu;
            if (u != cur) {
                if (cur != NOLOC) {
#pragma unroll
                    for (int k = 0; k < NPARAM; ++k) {
                        atomicAdd(&sm.acc[k][cur], a[k]);
                        a[k] = 0.0f;
                    }
                }
                cur = u;
                r0 = sm.urec[0][u];
                r1 = sm.urec[1][u];
                r2 = sm.urec[2][u];
                r3 = sm.urec[3][u];
            }
            const float2 wl = sm.ent_wl[ent_slot(idx)];
            const float4 pa = sm.pixg[px];
            float v[NPARAM];
            slot_grad(r0, r1, r2, r3, fx0 + (float)(px & (FX - 1)), fy0 + (float)(px / FX), wl.y, wl.x, pa.x,
                      pa.y, pa.z, pa.w, v);
#pragma unroll
            for (int k = 0; k < NPARAM; ++k) a[k] += v[k];
        }
        // the last sites of consecutive lanes repeat (entries are sorted):
        // sum each run across lanes first, then one update per run
        const uint32_t key = cur == NOLOC ? EMPTY : cur;
        const bool tail = warp_run_reduce(key, a, lane);
        if (tail && key != EMPTY) {
#pragma unroll
            for (int k = 0; k < NPARAM; ++k) atomicAdd(&sm.acc[k][key], a[k]);
        }
    }

    // ---- E: flush the tile accumulators, loss partial, last-block epilogue
    for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(FULL, lsum, o);
    if (lane == 0) sm.warp_loss[ty] = lsum;
    const int n_empty = __syncthreads_count(inside && !vmask);
    const int n_global = __syncthreads_count(global_adds != 0);
    const int n_dropped = PROP ? 0 : __syncthreads_count(dropped != 0);
    for (uint32_t e = tid; e < ucount * NPARAM; e += FT) {
        const uint32_t u = e % ucount, k = e / ucount;
        const float a = sm.acc[k][u];
        if (a != 0.0f) atomicAdd(grads + (size_t)k * N + sm.ulist[u], a);
    }
    if (tid == 0) {
        float tl = 0.0f;
        for (int q = 0; q < FY; ++q) tl += sm.warp_loss[q];
        ws_loss_partials(ws)[blockIdx.y * gridDim.x + blockIdx.x] = (double)tl;
        if (n_empty) atomicAdd(&c->empty_pixels, (unsigned long long)n_empty);
        if (n_global) atomicAdd(&c->hash_overflow, (unsigned long long)n_global);
        if (n_dropped) atomicAdd(&c->dropped_ids, (unsigned long long)n_dropped);
        __threadfence();
        sm.last = atomicAdd(&c->ticket_bwd, 1u) == gridDim.x * gridDim.y - 1;
    }
    __syncthreads();
    if (sm.last) {
        // every block has read cur/pass and written its partial: finish the pass
        const unsigned total = gridDim.x * gridDim.y;
        const volatile double *lp = ws_loss_partials(ws);
        double s = 0.0;
        for (unsigned q = tid; q < total; q += FT) s += lp[q];
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
        __shared__ double red[FT / 32];
        if (lane == 0) red[ty] = s;
        __syncthreads();
        if (tid == 0) {
            double tsum = 0.0;
            for (int q = 0; q < FY; ++q) tsum += red[q];
            c->loss = tsum / (double)P;
            if (PROP) {
                c->cur = cur ^ 1u;
                c->pass_counter = pass + 1u;
            }
            c->ticket_bwd = 0;
            __threadfence();
        }
    }
}

// the tile state exceeds the 48 KB default: opt in once per device (done
// when buffers are bound, so that a stream capture sees launches only)
template <int FY, bool PROP>
cudaError_t ensure_smem_attr() {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(fit_tile_kernel<FY, PROP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(FusedSmem<FY>));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    return cudaSuccess;
}

template <int FY, bool PROP>
cudaError_t launch_fit_tile_h(const Dev &d, int G, cudaStream_t st) {
    // the propagating form works on the pixel grid only
    if (PROP && d.cell != 1) return cudaErrorInvalidValue;
    const TableGrid lists{d.cell, d.GW, (size_t)d.PT};
    cudaError_t e = ensure_smem_attr<FY, PROP>();
    if (e != cudaSuccess) return e;
    const dim3 grid((d.W + FX - 1) / FX, (d.H + FY - 1) / FY);
    fit_tile_kernel<FY, PROP><<<grid, dim3(FX, FY), sizeof(FusedSmem<FY>), st>>>(d.records, d.table, d.target, d.H, d.W,
                                                                           d.N, G, d.image, d.grads, d.ws, lists);
    return cudaGetLastError();
}

}  // namespace

cudaError_t prepare_fused() {
    cudaError_t e = ensure_smem_attr<8, true>();
    if (e == cudaSuccess) e = ensure_smem_attr<16, true>();
    if (e == cudaSuccess) e = ensure_smem_attr<8, false>();
    if (e == cudaSuccess) e = ensure_smem_attr<16, false>();
    return e;
}

cudaError_t launch_fit_tile(const Dev &d, int G, cudaStream_t st) {
    // taller tiles amortise the halo and the per-tile work, but hold more
    // distinct sites: use them unless sites are dense (< 4 pixels per site),
    // where tiles would often exceed the 128-site index
    if ((long long)d.H * d.W >= 4ll * d.N) return launch_fit_tile_h<16, true>(d, G, st);
    return launch_fit_tile_h<8, true>(d, G, st);
}

cudaError_t launch_fit_tile_cached(const Dev &d, cudaStream_t st) {
    if ((long long)d.H * d.W >= 4ll * d.N) return launch_fit_tile_h<16, false>(d, 0, st);
    return launch_fit_tile_h<8, false>(d, 0, st);
}

}  // namespace sad
