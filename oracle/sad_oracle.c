/*
 * sad_oracle.c -- plain, slow CPU oracle for one Soft Anisotropic Diagrams
 * (SAD) fitting iteration.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA library, and the CUDA library never
 * calls it.
 *
 * Sources, by page title and section:
 *   [P1] "Soft Anisotropic Diagrams for Differentiable Image Representation"
 *        (paperlayer.ai summary of arXiv:2604.21984v2), sections 4, B.2-B.5.
 *   [P2] reading notes on the same paper (woaixuexisr.github.io), "key
 *        designs" 1-4: the metric G_i, d_mix, the softmax and the candidate
 *        update formula.
 *   [P4] "SAD: Soft Anisotropic Diagrams" project page, "Method".
 *
 * Conventions fixed here (the pages leave them open; see the readings list in
 * the design notes of this repository):
 *   - pixel (i, j) = (column, row) has centre x = (i + 0.5, j + 0.5) in pixels,
 *     pixel id = j * W + i; images are planar (3, H, W).
 *   - site parameters are 9 float32 planes of length N in the order
 *     x, y, ln tau, r, cr, cg, cb, theta, a.  A site is active iff x >= 0
 *     ([P1] B.2: inactive sites carry x < 0); a NaN x is inactive.
 *   - s = 1 / max(H, W); u = (cos theta, sin theta), v = (-sin theta, cos theta)
 *     and G = e^a u u^T + e^-a v v^T ([P2] key design 1, det G = 1).
 *   - logit l_i(x) = -tau_i (s ||x - p_i||_G - s r_i) ([P2] key design 2,
 *     [P4] Method); ranking key (l desc, site id asc); NaN logits drop out.
 *
 * Precision: render, loss, backward and Adam are evaluated in double from the
 * float32 parameters.  The top-K decisions (exact brute force and the
 * propagation pass) are taken in float32 -- the pages' training precision
 * ([P1] B.2: float32 site buffer) -- on a float32 per-site score record that
 * is itself computed in double and rounded once per field, with this fixed
 * operation order for the score of record R at pixel centre (fx, fy):
 *     dx = fx - R.x;  dy = fy - R.y
 *     u1 = fmaf(R.A, dx, R.B * dy);  u2 = fmaf(R.C, dy, R.B * dx)
 *     q  = fmaf(dx, u1, dy * u2);  q = (q < 0) ? 0 : q
 *     l  = R.b - sqrtf(q)
 * where k = tau s, (A, B, C) = k^2 (G11, G12, G22) and b = k r; this is the
 * same logit as above, rearranged as l = k r - sqrt(k^2 delta^T G delta).
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (oracle/build.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_SENTINEL 0xFFFFFFFFu
#define ORC_K 8
#define ORC_REC 16

enum { P_X = 0, P_Y, P_LT, P_R, P_CR, P_CG, P_CB, P_TH, P_A, P_COUNT };

static int omp_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static int omp_thread_id(void)
{
#ifdef _OPENMP
    return omp_get_thread_num();
#else
    return 0;
#endif
}

int orc_num_threads(void) { return omp_threads(); }

void orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------------ */
/* Per-site score records                                                    */
/* ------------------------------------------------------------------------ */

/*
 * Record of site i (16 values): x, y, A, B, C, b, k, 0, cr, cg, cb,
 * cos theta, sin theta, k^2 e^a, k^2 e^-a, 0 with k = tau s.  An inactive
 * site gets x = -1 and zeros elsewhere.  Every field is evaluated in double;
 * rec32 receives each field rounded once to float32, rec64 (optional) the
 * double values.  Metric from [P2] key design 1; fields follow the packed
 * candidate-site buffer of [P1] B.2 (position, (ln tau, r), direction, a).
 */
void orc_records(int H, int W, int N, const float *params, float *rec32, double *rec64)
{
    const double s = 1.0 / (double)(H > W ? H : W);
    for (int i = 0; i < N; ++i) {
        double f[ORC_REC];
        memset(f, 0, sizeof(f));
        const double px = params[P_X * N + i];
        if (px >= 0.0) {
            const double py = params[P_Y * N + i];
            const double tau = exp((double)params[P_LT * N + i]);
            const double r = params[P_R * N + i];
            const double th = params[P_TH * N + i];
            const double a = params[P_A * N + i];
            const double k = tau * s;
            const double ep = exp(a), em = exp(-a);
            const double c = cos(th), sn = sin(th);
            const double g11 = ep * c * c + em * sn * sn;
            const double g12 = (ep - em) * c * sn;
            const double g22 = ep * sn * sn + em * c * c;
            const double kk = k * k;
            f[0] = px;
            f[1] = py;
            f[2] = kk * g11;
            f[3] = kk * g12;
            f[4] = kk * g22;
            f[5] = k * r;
            f[6] = k;
            f[8] = params[P_CR * N + i];
            f[9] = params[P_CG * N + i];
            f[10] = params[P_CB * N + i];
            f[11] = c;
            f[12] = sn;
            f[13] = kk * ep;
            f[14] = kk * em;
        } else {
            f[0] = -1.0;
        }
        for (int q = 0; q < ORC_REC; ++q) {
            rec32[(size_t)i * ORC_REC + q] = (float)f[q];
            if (rec64) rec64[(size_t)i * ORC_REC + q] = f[q];
        }
    }
}

/* float32 logit of a record at a pixel centre, in the fixed order above */
static float score32(const float *R, float fx, float fy)
{
    const float dx = fx - R[0];
    const float dy = fy - R[1];
    const float bdy = R[3] * dy;
    const float bdx = R[3] * dx;
    const float u1 = fmaf(R[2], dx, bdy);
    const float u2 = fmaf(R[4], dy, bdx);
    const float dyu2 = dy * u2;
    float q = fmaf(dx, u1, dyu2);
    if (q < 0.0f) q = 0.0f;
    return R[5] - sqrtf(q);
}

float orc_score32(const float *rec32, int id, int i, int j)
{
    return score32(rec32 + (size_t)id * ORC_REC, (float)i + 0.5f, (float)j + 0.5f);
}

/* the same score at an arbitrary point (a candidate-grid cell centre) */
float orc_score32_at(const float *rec32, int id, float fx, float fy)
{
    return score32(rec32 + (size_t)id * ORC_REC, fx, fy);
}

/*
 * Candidate grid ([P1] B.3, "Candidate field"): the lists live on a grid of
 * ceil(W/cell) x ceil(H/cell) cells; cell (i, j) holds the pixels with
 * floor(x/cell) = i, floor(y/cell) = j and scores its candidates at its
 * centre ((i + 0.5) cell, (j + 0.5) cell).  cell = 1 is the pixel grid.
 * The functions below that take (GH, GW, cell) work on that grid.
 */
static float cell_centre(int i, int cell) { return ((float)i + 0.5f) * (float)cell; }

/* candidate a ranks above candidate b */
static int ranks_above(float la, uint32_t ia, float lb, uint32_t ib)
{
    return la > lb || (la == lb && ia < ib);
}

typedef struct {
    float l[ORC_K];
    uint32_t id[ORC_K];
    int n;
} topk_t;

static void topk_clear(topk_t *t) { t->n = 0; }

static int topk_has(const topk_t *t, uint32_t id)
{
    for (int q = 0; q < t->n; ++q)
        if (t->id[q] == id) return 1;
    return 0;
}

/* insert a candidate not present in t; keeps (l desc, id asc) order */
static void topk_insert(topk_t *t, float l, uint32_t id)
{
    if (t->n == ORC_K && !ranks_above(l, id, t->l[ORC_K - 1], t->id[ORC_K - 1])) return;
    int pos = t->n < ORC_K ? t->n : ORC_K - 1;
    while (pos > 0 && ranks_above(l, id, t->l[pos - 1], t->id[pos - 1])) {
        t->l[pos] = t->l[pos - 1];
        t->id[pos] = t->id[pos - 1];
        --pos;
    }
    t->l[pos] = l;
    t->id[pos] = id;
    if (t->n < ORC_K) t->n++;
}

static void topk_store(const topk_t *t, uint32_t *out)
{
    for (int q = 0; q < ORC_K; ++q) out[q] = q < t->n ? t->id[q] : ORC_SENTINEL;
}

/*
 * Exact top-K ([P1] abstract: the per-pixel list approximates the nearest
 * sites under the shading score; this is that quantity): every active site is
 * scored at every requested pixel.  pix == NULL means all pixels in order.
 * out: n_pix x 8 site ids, sentinel-padded.
 */
void orc_topk_exact_cell(int GH, int GW, int cell, int N, const float *rec32, const int64_t *pix, int64_t n_pix,
                         uint32_t *out)
{
    const int64_t P = (int64_t)GH * GW;
    if (!pix) n_pix = P;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t q = 0; q < n_pix; ++q) {
        const int64_t p = pix ? pix[q] : q;
        const float fx = cell_centre((int)(p % GW), cell), fy = cell_centre((int)(p / GW), cell);
        topk_t t;
        topk_clear(&t);
        for (int i = 0; i < N; ++i) {
            const float *R = rec32 + (size_t)i * ORC_REC;
            if (!(R[0] >= 0.0f)) continue;
            const float l = score32(R, fx, fy);
            if (l != l) continue;
            topk_insert(&t, l, (uint32_t)i);
        }
        topk_store(&t, out + q * ORC_K);
    }
}

/* ------------------------------------------------------------------------ */
/* Candidate propagation ([P2] key design 3, [P1] section 4 and B.3)          */
/* ------------------------------------------------------------------------ */

/* MurmurHash3 32-bit finaliser (Appleby, public domain) */
static uint32_t fmix32(uint32_t h)
{
    h ^= h >> 16;
    h *= 0x85ebca6bu;
    h ^= h >> 13;
    h *= 0xc2b2ae35u;
    h ^= h >> 16;
    return h;
}

/* Marsaglia, "Xorshift RNGs" (J. Stat. Soft. 2003), shift triple (13, 17, 5) */
static uint32_t xorshift32(uint32_t x)
{
    x ^= x << 13;
    x ^= x >> 17;
    x ^= x << 5;
    return x;
}

uint32_t orc_fmix32(uint32_t h) { return fmix32(h); }
uint32_t orc_xorshift32(uint32_t h) { return xorshift32(h); }

/*
 * The G injected site ids of pixel p in propagation pass number `pass`
 * ([P1] B.3: an xorshift generator seeded per pass and pixel).  State
 * h = fmix32(p ^ fmix32(seed ^ pass * 0x9E3779B9)), replaced by 1 if zero;
 * then h <- xorshift32(h) and id = floor(h * N / 2^32) (Lemire's
 * multiply-high range reduction) for each injection.
 */
void orc_inject_ids(uint32_t seed, uint32_t pass, uint32_t p, int N, int G, uint32_t *out)
{
    uint32_t h = fmix32(p ^ fmix32(seed ^ (pass * 0x9E3779B9u)));
    if (h == 0) h = 1;
    for (int g = 0; g < G; ++g) {
        h = xorshift32(h);
        out[g] = (uint32_t)(((uint64_t)h * (uint64_t)(uint32_t)N) >> 32);
    }
}

static void offer(topk_t *t, const float *rec32, int N, uint32_t id, float fx, float fy)
{
    if (id == ORC_SENTINEL || id >= (uint32_t)N) return;
    const float *R = rec32 + (size_t)id * ORC_REC;
    if (!(R[0] >= 0.0f)) return;
    if (topk_has(t, id)) return;
    const float l = score32(R, fx, fy);
    if (l != l) return;
    topk_insert(t, l, id);
}

/*
 * One Jacobi propagation pass at jump k:
 *   C_t(x) = topK( C_{t-1}(x) U C_{t-1}(x +- k e_x) U C_{t-1}(x +- k e_y) U G_t(x) )
 * (temporal reuse + self and 4-neighbour propagation + G stochastic
 * injections, all re-scored at x).  Out-of-image neighbours are skipped.
 * Here H x W is the candidate grid and x a cell centre (cell = 1: pixels);
 * injections are keyed on the cell index.  Tables are H W x 8 site ids.
 * 0 <= G <= 64.
 */
void orc_propagate_cell(int H, int W, int cell, int N, const float *rec32, const uint32_t *tin, uint32_t *tout,
                        int jump, int G, uint32_t seed, uint32_t pass)
{
    if (G > 64) G = 64;
    if (G < 0) G = 0;
#pragma omp parallel for schedule(dynamic, 4)
    for (int j = 0; j < H; ++j) {
        uint32_t inj[64];
        for (int i = 0; i < W; ++i) {
            const int64_t p = (int64_t)j * W + i;
            const float fx = cell_centre(i, cell), fy = cell_centre(j, cell);
            topk_t t;
            topk_clear(&t);
            for (int q = 0; q < ORC_K; ++q) offer(&t, rec32, N, tin[p * ORC_K + q], fx, fy);
            const int nx[4] = {i - jump, i + jump, i, i};
            const int ny[4] = {j, j, j - jump, j + jump};
            for (int d = 0; d < 4; ++d) {
                if (nx[d] < 0 || nx[d] >= W || ny[d] < 0 || ny[d] >= H) continue;
                const int64_t pn = (int64_t)ny[d] * W + nx[d];
                for (int q = 0; q < ORC_K; ++q) offer(&t, rec32, N, tin[pn * ORC_K + q], fx, fy);
            }
            if (G > 0) {
                orc_inject_ids(seed, pass, (uint32_t)p, N, G, inj);
                for (int q = 0; q < G; ++q) offer(&t, rec32, N, inj[q], fx, fy);
            }
            topk_store(&t, tout + p * ORC_K);
        }
    }
}

/*
 * Packed candidate sites ([P1] B.2: candidate-update kernels score from a
 * compact 16-byte per-site buffer of float16 pairs; the kept lists are then
 * used by the float32 renderer).  Reading of this build: the record keeps
 * the position in float32 (a binary16 position steps by 1-2 px between 2048
 * and 4096 px) and the score coefficients A, B, C and b as binary16 values;
 * the candidate update ranks candidates by the logit evaluated in the
 * float32 order above from those rounded coefficients, and the kept 8 are
 * re-scored with the float32 record and stored in (float32 logit desc, id
 * asc) order.
 */

/* x rounded to the nearest IEEE 754 binary16 value (ties to even; overflow
 * to infinity), returned as the float32 value it equals.  binary16 has an
 * 11-bit significand and exponents -14..15, with subnormals down to 2^-24:
 * the spacing of values near |x| is 2^(floor(log2 |x|) - 10), never below
 * 2^-24; the largest finite value is 65504 and |x| >= 65520 rounds to inf. */
static float to_binary16(float x)
{
    if (x != x) return x;
    const float ax = fabsf(x);
    if (ax >= 65520.0f) return copysignf(INFINITY, x);
    int e;
    frexpf(ax, &e); /* ax = m 2^e, 0.5 <= m < 1 */
    int qe = (e - 1) - 10;
    if (qe < -24) qe = -24;
    const float quantum = ldexpf(1.0f, qe);
    const float r = nearbyintf(ax / quantum) * quantum; /* default rounding: to nearest, ties to even */
    return copysignf(r, x);
}

float orc_to_binary16(float x) { return to_binary16(x); }

/* the selection record: rec32 with A, B, C and b rounded to binary16 */
void orc_cand16_record(int N, const float *rec32, float *rec_sel)
{
    for (int64_t i = 0; i < (int64_t)N * ORC_REC; ++i) rec_sel[i] = rec32[i];
    for (int i = 0; i < N; ++i)
        for (int f = 2; f <= 5; ++f) rec_sel[(size_t)i * ORC_REC + f] = to_binary16(rec32[(size_t)i * ORC_REC + f]);
}

/* re-score every kept list with the float32 record and store it in
 * (logit desc, id asc) order; sentinels stay last */
void orc_rescore_sort_cell(int GH, int GW, int cell, int N, const float *rec32, uint32_t *table)
{
    const int64_t P = (int64_t)GH * GW;
#pragma omp parallel for schedule(dynamic, 256)
    for (int64_t p = 0; p < P; ++p) {
        const float fx = cell_centre((int)(p % GW), cell), fy = cell_centre((int)(p / GW), cell);
        topk_t t;
        topk_clear(&t);
        for (int q = 0; q < ORC_K; ++q) {
            const uint32_t id = table[p * ORC_K + q];
            if (id == ORC_SENTINEL || id >= (uint32_t)N) continue;
            topk_insert(&t, score32(rec32 + (size_t)id * ORC_REC, fx, fy), id);
        }
        topk_store(&t, table + p * ORC_K);
    }
}

/*
 * Seed pass ([P1] B.3: the JFA prepass starts with a seed pass): clear the
 * table to the sentinel, then every active site whose position lies in the
 * image writes its id to slot 0 of the pixel containing it; the smallest id
 * wins where several sites share a pixel.
 */
void orc_seed_cell(int H, int W, int cell, int N, const float *params, uint32_t *table)
{
    const int GW = (W + cell - 1) / cell, GH = (H + cell - 1) / cell;
    const int64_t P = (int64_t)GH * GW;
    for (int64_t q = 0; q < P * ORC_K; ++q) table[q] = ORC_SENTINEL;
    for (int i = 0; i < N; ++i) {
        const float px = params[P_X * N + i], py = params[P_Y * N + i];
        if (!(px >= 0.0f) || !(py >= 0.0f)) continue;
        const int64_t ci = (int64_t)floorf(px), cj = (int64_t)floorf(py);
        if (ci >= W || cj >= H) continue;
        uint32_t *slot = table + ((cj / cell) * GW + ci / cell) * ORC_K;
        if ((uint32_t)i < slot[0]) slot[0] = (uint32_t)i;
    }
}

/* ------------------------------------------------------------------------ */
/* Render, loss and backward in double ([P2] key designs 1-2, [P1] B.4)       */
/* ------------------------------------------------------------------------ */

typedef struct {
    double px, py, tau, r, c[3], ep, em, ux, uy, vx, vy, g11, g12, g22;
    int active;
} site64_t;

static site64_t *sites64(int N, const float *params)
{
    site64_t *S = (site64_t *)calloc((size_t)(N > 0 ? N : 1), sizeof(site64_t));
    for (int i = 0; i < N; ++i) {
        site64_t *z = &S[i];
        z->px = params[P_X * N + i];
        z->active = z->px >= 0.0;
        z->py = params[P_Y * N + i];
        z->tau = exp((double)params[P_LT * N + i]);
        z->r = params[P_R * N + i];
        for (int ch = 0; ch < 3; ++ch) z->c[ch] = params[(P_CR + ch) * N + i];
        const double a = params[P_A * N + i], th = params[P_TH * N + i];
        z->ep = exp(a);
        z->em = exp(-a);
        z->ux = cos(th);
        z->uy = sin(th);
        z->vx = -z->uy;
        z->vy = z->ux;
        /* G = e^a u u^T + e^-a v v^T */
        z->g11 = z->ep * z->ux * z->ux + z->em * z->vx * z->vx;
        z->g12 = z->ep * z->ux * z->uy + z->em * z->vx * z->vy;
        z->g22 = z->ep * z->uy * z->uy + z->em * z->vy * z->vy;
    }
    return S;
}

typedef struct {
    int n;
    uint32_t id[ORC_K];
    double l[ORC_K], w[ORC_K], nrm[ORC_K], dx[ORC_K], dy[ORC_K];
    double chat[3];
} pixel64_t;

/*
 * Soft Apollonius render of one pixel from its candidate slots:
 * n_i = sqrt(delta^T G_i delta), d_i = s n_i - s r_i, l_i = -tau_i d_i,
 * w_i = exp(l_i - max l) / sum_j exp(l_j - max l), chat = sum_i w_i c_i.
 * Slots holding the sentinel, an out-of-range id, an inactive site or a
 * non-finite logit are skipped; no valid slot gives chat = 0 and n = 0.
 */
static void render_pixel(const site64_t *S, int N, double s, const uint32_t *slots, int64_t p, int W,
                         pixel64_t *o)
{
    const double x = (double)(p % W) + 0.5, y = (double)(p / W) + 0.5;
    o->n = 0;
    o->chat[0] = o->chat[1] = o->chat[2] = 0.0;
    for (int q = 0; q < ORC_K; ++q) {
        const uint32_t id = slots[q];
        if (id == ORC_SENTINEL || id >= (uint32_t)N || !S[id].active) continue;
        const site64_t *z = &S[id];
        const double dx = x - z->px, dy = y - z->py;
        double qq = z->g11 * dx * dx + 2.0 * z->g12 * dx * dy + z->g22 * dy * dy;
        if (qq < 0.0) qq = 0.0;
        const double n = sqrt(qq);
        const double l = -z->tau * (s * n - s * z->r);
        if (!isfinite(l)) continue;
        o->id[o->n] = id;
        o->l[o->n] = l;
        o->nrm[o->n] = n;
        o->dx[o->n] = dx;
        o->dy[o->n] = dy;
        o->n++;
    }
    if (o->n == 0) return;
    double M = o->l[0];
    for (int q = 1; q < o->n; ++q) M = o->l[q] > M ? o->l[q] : M;
    double Z = 0.0;
    for (int q = 0; q < o->n; ++q) {
        o->w[q] = exp(o->l[q] - M);
        Z += o->w[q];
    }
    for (int q = 0; q < o->n; ++q) {
        o->w[q] /= Z;
        for (int ch = 0; ch < 3; ++ch) o->chat[ch] += o->w[q] * S[o->id[q]].c[ch];
    }
}

/* image: 3 x P doubles */
void orc_render(int H, int W, int N, const float *params, const uint32_t *table, double *image)
{
    const int64_t P = (int64_t)H * W;
    const double s = 1.0 / (double)(H > W ? H : W);
    site64_t *S = sites64(N, params);
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < P; ++p) {
        pixel64_t o;
        render_pixel(S, N, s, table + p * ORC_K, p, W, &o);
        for (int ch = 0; ch < 3; ++ch) image[ch * P + p] = o.chat[ch];
    }
    free(S);
}

/* softmax weights of every pixel's slots (P x 8, zero for skipped slots) */
void orc_weights(int H, int W, int N, const float *params, const uint32_t *table, double *weights)
{
    const int64_t P = (int64_t)H * W;
    const double s = 1.0 / (double)(H > W ? H : W);
    site64_t *S = sites64(N, params);
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < P; ++p) {
        pixel64_t o;
        render_pixel(S, N, s, table + p * ORC_K, p, W, &o);
        for (int q = 0; q < ORC_K; ++q) weights[p * ORC_K + q] = 0.0;
        int u = 0;
        for (int q = 0; q < ORC_K && u < o.n; ++q)
            if (table[p * ORC_K + q] == o.id[u]) weights[p * ORC_K + q] = o.w[u++];
    }
    free(S);
}

/*
 * MSE loss L = (1/P) sum_x sum_ch (chat - t)^2 ([P2] key design 4: plain MSE;
 * [P1] B.4: normalised by pixel count) and its analytic gradient with
 * respect to the stored parameters ([P1] B.4: hand-derived top-K softmax
 * gradients), accumulated in double:
 *   g        = 2 (chat - t) / P
 *   dL/dc_i  = w_i g
 *   gamma_i  = dL/dl_i = w_i (c_i - chat) . g
 *   dL/dlntau_i = gamma_i l_i          (l is linear in tau)
 *   dL/dr_i  = gamma_i tau_i s
 *   dL/dn_i  = -gamma_i tau_i s, with, for alpha = u.delta, beta = v.delta,
 *     dn/dp     = -(e^a alpha u + e^-a beta v) / n
 *     dn/da     = (e^a alpha^2 - e^-a beta^2) / (2 n)
 *     dn/dtheta = alpha beta (e^a - e^-a) / n
 *   and all three taken as 0 where n = 0.
 * grads: 9 x N doubles in parameter-plane order (overwritten).  image
 * (optional): 3 x P doubles.  Returns L.
 */
double orc_loss_backward_stats(int H, int W, int N, const float *params, const uint32_t *table,
                               const float *target, double *grads, double *image, double *stats,
                               double *stats_abs);

double orc_loss_backward(int H, int W, int N, const float *params, const uint32_t *table,
                         const float *target, double *grads, double *image)
{
    return orc_loss_backward_stats(H, W, N, params, table, target, grads, image, NULL, NULL);
}

/*
 * As orc_loss_backward, and when stats is not NULL also the per-site
 * statistics of the budget control ([P1] B.4-B.5: mass, energy, weighted
 * second moments, removal delta), 6 x N doubles:
 *   m_i   = sum_x w_i
 *   E_i   = sum_x w_i e(x),                 e(x) = |chat - t|^2
 *   Sxx_i, Sxy_i, Syy_i = sum_x w_i e(x) (dx^2, dx dy, dy^2),  (dx, dy) = x - p_i
 *   D_i   = sum_x [ |(chat - w_i c_i) / max(1 - w_i, 1e-6) - t|^2 - e(x) ]
 * (D_i: the error after removing site i and renormalising the remaining
 * weights, minus the error with it).  stats_abs (optional, with stats)
 * receives the sums of the terms' absolute values, the scale against which
 * a float32 accumulation of the same sums is accurate.
 */
double orc_loss_backward_stats(int H, int W, int N, const float *params, const uint32_t *table,
                               const float *target, double *grads, double *image, double *stats,
                               double *stats_abs)
{
    const int64_t P = (int64_t)H * W;
    const double s = 1.0 / (double)(H > W ? H : W);
    site64_t *S = sites64(N, params);
    const int T = omp_threads();
    const int NA = P_COUNT + 12; /* gradients, statistics, their absolute sums */
    double *acc = (double *)calloc((size_t)T * NA * (size_t)(N > 0 ? N : 1), sizeof(double));
    double *lossp = (double *)calloc((size_t)T, sizeof(double));
#pragma omp parallel
    {
        const int tid = omp_thread_id();
        double *A = acc + (size_t)tid * NA * N;
        double *St = A + (size_t)P_COUNT * N;
        double lsum = 0.0;
#pragma omp for schedule(static)
        for (int64_t p = 0; p < P; ++p) {
            pixel64_t o;
            render_pixel(S, N, s, table + p * ORC_K, p, W, &o);
            double g[3], ex = 0.0;
            for (int ch = 0; ch < 3; ++ch) {
                const double e = o.chat[ch] - (double)target[ch * P + p];
                lsum += e * e;
                ex += e * e;
                g[ch] = 2.0 * e / (double)P;
                if (image) image[ch * P + p] = o.chat[ch];
            }
            if (stats) {
                for (int q = 0; q < o.n; ++q) {
                    const site64_t *z = &S[o.id[q]];
                    const int64_t i = o.id[q];
                    const double w = o.w[q];
                    double rem = 0.0;
                    const double den = (1.0 - w) > 1e-6 ? (1.0 - w) : 1e-6;
                    for (int ch = 0; ch < 3; ++ch) {
                        const double c2 = (o.chat[ch] - w * z->c[ch]) / den - (double)target[ch * P + p];
                        rem += c2 * c2;
                    }
                    const double t6[6] = {w, w * ex, w * ex * o.dx[q] * o.dx[q], w * ex * o.dx[q] * o.dy[q],
                                          w * ex * o.dy[q] * o.dy[q], rem - ex};
                    for (int r = 0; r < 6; ++r) {
                        St[r * (size_t)N + i] += t6[r];
                        St[(6 + r) * (size_t)N + i] += fabs(t6[r]);
                    }
                }
            }
            for (int q = 0; q < o.n; ++q) {
                const site64_t *z = &S[o.id[q]];
                const int64_t i = o.id[q];
                const double w = o.w[q];
                double gamma = 0.0;
                for (int ch = 0; ch < 3; ++ch) {
                    A[(P_CR + ch) * (size_t)N + i] += w * g[ch];
                    gamma += w * (z->c[ch] - o.chat[ch]) * g[ch];
                }
                A[P_LT * (size_t)N + i] += gamma * o.l[q];
                A[P_R * (size_t)N + i] += gamma * z->tau * s;
                const double dLdn = -gamma * z->tau * s;
                const double n = o.nrm[q];
                if (n > 0.0) {
                    const double al = z->ux * o.dx[q] + z->uy * o.dy[q];
                    const double be = z->vx * o.dx[q] + z->vy * o.dy[q];
                    const double dndx = -(z->ep * al * z->ux + z->em * be * z->vx) / n;
                    const double dndy = -(z->ep * al * z->uy + z->em * be * z->vy) / n;
                    const double dnda = (z->ep * al * al - z->em * be * be) / (2.0 * n);
                    const double dndt = al * be * (z->ep - z->em) / n;
                    A[P_X * (size_t)N + i] += dLdn * dndx;
                    A[P_Y * (size_t)N + i] += dLdn * dndy;
                    A[P_A * (size_t)N + i] += dLdn * dnda;
                    A[P_TH * (size_t)N + i] += dLdn * dndt;
                }
            }
        }
        lossp[tid] = lsum;
    }
    memset(grads, 0, sizeof(double) * P_COUNT * (size_t)N);
    if (stats) memset(stats, 0, sizeof(double) * 6 * (size_t)N);
    if (stats_abs) memset(stats_abs, 0, sizeof(double) * 6 * (size_t)N);
    double L = 0.0;
    for (int t = 0; t < T; ++t) {
        const double *A = acc + (size_t)t * NA * N;
        for (size_t q = 0; q < (size_t)P_COUNT * N; ++q) grads[q] += A[q];
        if (stats)
            for (size_t q = 0; q < (size_t)6 * N; ++q) stats[q] += A[(size_t)P_COUNT * N + q];
        if (stats_abs)
            for (size_t q = 0; q < (size_t)6 * N; ++q) stats_abs[q] += A[(size_t)(P_COUNT + 6) * N + q];
        L += lossp[t];
    }
    free(acc);
    free(lossp);
    free(S);
    return L / (double)P;
}

/*
 * Adam ([P2] key design 4: Adam on all site parameters; [P1] B.4: the
 * accumulated gradients are already normalised by the pixel count).  Position
 * and radius are optimised in the resolution-free units s x and s r, in which
 * the logit is written, so their gradient is scaled by 1/s and their step by
 * 1/s.  For every active site (x >= 0) and plane j:
 *   ghat = grad * sigma_j,  sigma_j = 1/s for x, y, r and 1 otherwise
 *   m <- b1 m + (1 - b1) ghat;   v <- b2 v + (1 - b2) ghat^2
 *   param <- param - lr_j sigma_j (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 * then the position is clamped into [0, W^-] x [0, H^-] (W^- the largest
 * float below W).  The clamp is a reading of this build, not a step of the
 * pages: they mark a pruned site with x < 0 ([P1] B.2, B.5), which an
 * optimiser step must not produce, and they say nothing about the upper
 * edges or y; clamping every coordinate into the image is the plainest way
 * to keep an active site active and inside the image it fits.  Inactive
 * sites are left untouched.  All arrays 9 x N doubles, in place.
 */
void orc_adam_frozen(int H, int W, int N, double *params, double *m, double *v, const double *grads,
                     const double *lr, double b1, double b2, double eps, int t, const uint8_t *frozen);

void orc_adam(int H, int W, int N, double *params, double *m, double *v, const double *grads,
              const double *lr, double b1, double b2, double eps, int t)
{
    orc_adam_frozen(H, W, N, params, m, v, grads, lr, b1, b2, eps, t, NULL);
}

/* As orc_adam; sites with frozen[i] != 0 are left untouched as well
 * ([P1] section 7: frozen sites are excluded from gradient updates). */
void orc_adam_frozen(int H, int W, int N, double *params, double *m, double *v, const double *grads,
                     const double *lr, double b1, double b2, double eps, int t, const uint8_t *frozen)
{
    const double s = 1.0 / (double)(H > W ? H : W);
    const double bc1 = 1.0 - pow(b1, (double)t);
    const double bc2 = 1.0 - pow(b2, (double)t);
    for (int i = 0; i < N; ++i) {
        if (!(params[P_X * (size_t)N + i] >= 0.0)) continue;
        if (frozen && frozen[i]) continue;
        for (int j = 0; j < P_COUNT; ++j) {
            const size_t q = (size_t)j * N + i;
            const double sig = (j == P_X || j == P_Y || j == P_R) ? 1.0 / s : 1.0;
            const double gh = grads[q] * sig;
            m[q] = b1 * m[q] + (1.0 - b1) * gh;
            v[q] = b2 * v[q] + (1.0 - b2) * gh * gh;
            const double mh = m[q] / bc1, vh = v[q] / bc2;
            params[q] -= lr[j] * sig * mh / (sqrt(vh) + eps);
        }
        /* the step keeps the position inside the image: x < 0 is the marker
           of a pruned site, not something an optimiser step may produce */
        const double xmax = (double)nextafterf((float)W, 0.0f), ymax = (double)nextafterf((float)H, 0.0f);
        double *x = &params[P_X * (size_t)N + i], *y = &params[P_Y * (size_t)N + i];
        *x = *x < 0.0 ? 0.0 : (*x > xmax ? xmax : *x);
        *y = *y < 0.0 ? 0.0 : (*y > ymax ? ymax : *y);
    }
}

/* ------------------------------------------------------------------------ */
/* Budget control: densify and prune ([P1] B.5, [P2] key design 4)            */
/* ------------------------------------------------------------------------ */

typedef struct {
    int grow;               /* net sites added per event */
    float prune_frac;       /* fraction of active sites pruned per event */
    float alpha;            /* score exponent */
    float eps;              /* mass floor */
    float r_scale;          /* child radius factor */
    float log_tau_shift;    /* subtracted from the children's ln tau */
    float offset_scale;     /* child offset = offset_scale * sqrt(lambda_max) */
    float fallback_offset;  /* child offset (px) when the second moment is degenerate */
} orc_densify_cfg;

typedef struct {
    float key;
    uint32_t id;
} keyed_t;

static int by_key_desc(const void *a, const void *b)
{
    const keyed_t *x = (const keyed_t *)a, *y = (const keyed_t *)b;
    if (x->key > y->key) return -1;
    if (x->key < y->key) return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id);
}

static int by_key_asc(const void *a, const void *b)
{
    const keyed_t *x = (const keyed_t *)a, *y = (const keyed_t *)b;
    if (x->key < y->key) return -1;
    if (x->key > y->key) return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id);
}

static int cmp_u32(const void *a, const void *b)
{
    const uint32_t x = *(const uint32_t *)a, y = *(const uint32_t *)b;
    return (x > y) - (x < y);
}

/* the float32 split score E / max(m, eps)^alpha (sqrt when alpha = 0.5) */
float orc_split_score(float m, float E, float alpha, float eps)
{
    const float mm = m > eps ? m : eps;
    return alpha == 0.5f ? E / sqrtf(mm) : E / powf(mm, alpha);
}

/*
 * One densify/prune event on float32 state.  stats: 6 x N float32 as
 * accumulated by the backward pass.  Decisions are taken on the float32
 * statistics:
 *   1. prune the floor(prune_frac * n_active) active sites with the smallest
 *      removal delta D (ties: smaller id first): x = -1.
 *   2. split the min(n_pruned + grow, free slots, remaining active) active
 *      sites with the largest score E / max(m, eps)^alpha (ties: smaller id);
 *      parents in ascending id take the free slots in ascending id.
 *   3. split geometry in double: C = S / E; major eigenvector e (sign: e.x > 0,
 *      or e.x == 0 and e.y > 0) with eigenvalue l; offset d = offset_scale *
 *      sqrt(l) * e; if E <= 0 or l <= 0, d = fallback_offset * (v if a > 0
 *      else u), the metric's long axis.  Child A (parent slot) at p + d,
 *      child B (free slot) at p - d, both clamped into the image; colour =
 *      target at the child's pixel; r *= r_scale; ln tau -= log_tau_shift;
 *      theta and a kept; Adam moments of both slots zeroed.
 * Returns the number of splits; *n_pruned receives the number pruned.
 */
int orc_densify_prune(int H, int W, int N, float *params, float *m1, float *m2, const float *stats,
                      const float *target, const orc_densify_cfg *cfg, int *n_pruned)
{
    const int64_t P = (int64_t)H * W;
    keyed_t *keys = (keyed_t *)malloc(sizeof(keyed_t) * (size_t)(N > 0 ? N : 1));
    uint32_t *freel = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)(N > 0 ? N : 1));
    uint32_t *parents = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)(N > 0 ? N : 1));
    int n_active = 0;
    for (int i = 0; i < N; ++i) n_active += params[P_X * N + i] >= 0.0f;
    int n_prune = (int)((double)cfg->prune_frac * (double)n_active);
    /* prune: smallest removal delta among active sites with a number */
    int nk = 0;
    for (int i = 0; i < N; ++i) {
        const float d = stats[5 * N + i];
        if (params[P_X * N + i] >= 0.0f && d == d) keys[nk++] = (keyed_t){d, (uint32_t)i};
    }
    if (n_prune > nk) n_prune = nk;
    qsort(keys, (size_t)nk, sizeof(keyed_t), by_key_asc);
    for (int q = 0; q < n_prune; ++q) params[P_X * N + keys[q].id] = -1.0f;
    /* split: largest score among the remaining active sites */
    nk = 0;
    for (int i = 0; i < N; ++i) {
        if (!(params[P_X * N + i] >= 0.0f)) continue;
        const float sc = orc_split_score(stats[0 * N + i], stats[1 * N + i], cfg->alpha, cfg->eps);
        if (sc == sc) keys[nk++] = (keyed_t){sc, (uint32_t)i};
    }
    int nf = 0;
    for (int i = 0; i < N; ++i)
        if (!(params[P_X * N + i] >= 0.0f)) freel[nf++] = (uint32_t)i;
    int n_split = n_prune + cfg->grow;
    if (n_split > nf) n_split = nf;
    if (n_split > nk) n_split = nk;
    if (n_split < 0) n_split = 0;
    qsort(keys, (size_t)nk, sizeof(keyed_t), by_key_desc);
    for (int q = 0; q < n_split; ++q) parents[q] = keys[q].id;
    qsort(parents, (size_t)n_split, sizeof(uint32_t), cmp_u32);
    const double maxx = nextafter((double)(float)W, 0.0), maxy = nextafter((double)(float)H, 0.0);
    for (int q = 0; q < n_split; ++q) {
        const uint32_t a_id = parents[q], b_id = freel[q];
        float pv[P_COUNT];
        for (int j = 0; j < P_COUNT; ++j) pv[j] = params[j * (size_t)N + a_id];
        const double E = stats[1 * N + a_id];
        double dx = 0.0, dy = 0.0;
        int ok = 0;
        if (E > 0.0) {
            const double cxx = stats[2 * N + a_id] / E, cxy = stats[3 * N + a_id] / E, cyy = stats[4 * N + a_id] / E;
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
                const double off = (double)cfg->offset_scale * sqrt(lam);
                dx = off * ex;
                dy = off * ey;
                ok = 1;
            }
        }
        if (!ok) {
            const double th = pv[P_TH], c = cos(th), sn = sin(th);
            const double f = (double)cfg->fallback_offset;
            if (pv[P_A] > 0.0f) {
                dx = -sn * f;
                dy = c * f;
            } else {
                dx = c * f;
                dy = sn * f;
            }
        }
        for (int side = 0; side < 2; ++side) {
            const uint32_t dst = side == 0 ? a_id : b_id;
            const double sg = side == 0 ? 1.0 : -1.0;
            double x = (double)pv[P_X] + sg * dx, y = (double)pv[P_Y] + sg * dy;
            x = x < 0.0 ? 0.0 : (x > maxx ? maxx : x);
            y = y < 0.0 ? 0.0 : (y > maxy ? maxy : y);
            float fxv = (float)x, fyv = (float)y;
            if (fxv >= (float)W) fxv = nextafterf((float)W, 0.0f);
            if (fyv >= (float)H) fyv = nextafterf((float)H, 0.0f);
            const int64_t pix = (int64_t)floorf(fyv) * W + (int64_t)floorf(fxv);
            params[P_X * (size_t)N + dst] = fxv;
            params[P_Y * (size_t)N + dst] = fyv;
            params[P_LT * (size_t)N + dst] = pv[P_LT] - cfg->log_tau_shift;
            params[P_R * (size_t)N + dst] = pv[P_R] * cfg->r_scale;
            for (int ch = 0; ch < 3; ++ch) params[(P_CR + ch) * (size_t)N + dst] = target[ch * P + pix];
            params[P_TH * (size_t)N + dst] = pv[P_TH];
            params[P_A * (size_t)N + dst] = pv[P_A];
            for (int j = 0; j < P_COUNT; ++j) {
                m1[j * (size_t)N + dst] = 0.0f;
                m2[j * (size_t)N + dst] = 0.0f;
            }
        }
    }
    free(keys);
    free(freel);
    free(parents);
    if (n_pruned) *n_pruned = n_prune;
    return n_split;
}

/* ------------------------------------------------------------------------ */
/* Tau diffusion ([P1] B.6)                                                   */
/* ------------------------------------------------------------------------ */

/*
 * One Jacobi step on the ln tau gradients: for every active site i whose
 * position lies in the image, with C = the valid active ids other than i in
 * the candidate list of the pixel containing p_i (the site's local candidate
 * neighbourhood), g_i <- (1 - lambda) g_i + lambda mean_{j in C} g_j, all
 * neighbours read before any write.  Sites with an empty C keep g_i.
 * grads: 9 x N doubles (plane ln tau updated in place); table: P x 8.
 */
void orc_tau_diffuse(int H, int W, int N, const float *params, const uint32_t *table, double *grads,
                     double lambda)
{
    double *g = grads + (size_t)P_LT * N;
    double *out = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    for (int i = 0; i < N; ++i) {
        out[i] = g[i];
        const float px = params[P_X * N + i], py = params[P_Y * N + i];
        if (!(px >= 0.0f) || !(py >= 0.0f)) continue;
        const int64_t ci = (int64_t)floorf(px), cj = (int64_t)floorf(py);
        if (ci >= W || cj >= H) continue;
        const uint32_t *slots = table + (cj * W + ci) * ORC_K;
        double sum = 0.0;
        int n = 0;
        for (int q = 0; q < ORC_K; ++q) {
            const uint32_t id = slots[q];
            if (id == ORC_SENTINEL || id >= (uint32_t)N || id == (uint32_t)i) continue;
            if (!(params[P_X * N + id] >= 0.0f)) continue;
            sum += g[id];
            ++n;
        }
        if (n > 0) out[i] = (1.0 - lambda) * g[i] + lambda * (sum / n);
    }
    memcpy(g, out, sizeof(double) * (size_t)N);
    free(out);
}

/* ------------------------------------------------------------------------ */
/* JFA prepass ([P1] B.3, optional prepass)                                   */
/* ------------------------------------------------------------------------ */

/*
 * One 3x3 flood pass at jump k: for each pixel, the distinct valid ids of the
 * lists at (i + a k, j + b k), a, b in {-1, 0, 1}, inside the image, re-scored
 * at the pixel; the 4 best by (logit desc, id asc) go to slots 0-3 and slots
 * 4-7 are emptied (the prepass fills only the first of the two four-id planes).
 */
void orc_jfa3x3_cell(int H, int W, int cell, int N, const float *rec32, const uint32_t *tin, uint32_t *tout,
                     int jump)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int j = 0; j < H; ++j) {
        for (int i = 0; i < W; ++i) {
            const int64_t p = (int64_t)j * W + i;
            const float fx = cell_centre(i, cell), fy = cell_centre(j, cell);
            topk_t t;
            topk_clear(&t);
            for (int b = -1; b <= 1; ++b)
                for (int a = -1; a <= 1; ++a) {
                    const int ni = i + a * jump, nj = j + b * jump;
                    if (ni < 0 || ni >= W || nj < 0 || nj >= H) continue;
                    const int64_t pn = (int64_t)nj * W + ni;
                    for (int q = 0; q < ORC_K; ++q) offer(&t, rec32, N, tin[pn * ORC_K + q], fx, fy);
                }
            for (int q = 0; q < ORC_K; ++q) tout[p * ORC_K + q] = (q < 4 && q < t.n) ? t.id[q] : ORC_SENTINEL;
        }
    }
}

/* pixel-grid (cell = 1) forms of the candidate-grid functions */
void orc_topk_exact(int H, int W, int N, const float *rec32, const int64_t *pix, int64_t n_pix, uint32_t *out)
{
    orc_topk_exact_cell(H, W, 1, N, rec32, pix, n_pix, out);
}

void orc_propagate(int H, int W, int N, const float *rec32, const uint32_t *tin, uint32_t *tout, int jump, int G,
                   uint32_t seed, uint32_t pass)
{
    orc_propagate_cell(H, W, 1, N, rec32, tin, tout, jump, G, seed, pass);
}

void orc_seed(int H, int W, int N, const float *params, uint32_t *table)
{
    orc_seed_cell(H, W, 1, N, params, table);
}

void orc_jfa3x3(int H, int W, int N, const float *rec32, const uint32_t *tin, uint32_t *tout, int jump)
{
    orc_jfa3x3_cell(H, W, 1, N, rec32, tin, tout, jump);
}

/* ------------------------------------------------------------------------ */
/* 16-byte evaluation record ([P1] B.2, "Packed storage for evaluation")     */
/* ------------------------------------------------------------------------ */

/*
 * Four 32-bit words per site, one little-endian 128-bit field string, bit
 * offset (width): x 0 (18), y 18 (18), cr 36 (10), cg 46 (10), cb 56 (10),
 * ln tau 66 (16), r 82 (14), theta 96 (14), a 110 (14), bits 124-126 zero,
 * bit 127 = active.  An inactive site packs to four zero words.
 *   x, y:   cell index floor(x / W 2^18) (clamped), decoded at the cell centre
 *           (q + 1/2) W / 2^18 (same with H for y);
 *   colour: round(clamp(c, 0, 1) 1023), decoded q / 1023;
 *   ln tau, r, a: round((v - lo) / (hi - lo) (2^b - 1)) with the per-image
 *           lo, hi of the active sites ([P1] B.2: per-image min/scale for
 *           ln tau and radius; the same for a), decoded lo + q (hi - lo) /
 *           (2^b - 1);
 *   theta:  the axis angle theta mod pi (G depends on the axis only),
 *           round(theta_m / pi 2^14) mod 2^14, decoded q pi / 2^14.
 * Rounding is floor(t + 1/2) in double; every decoded value is computed in
 * double and rounded once to float32.
 */
enum { PK_X = 0, PK_Y = 18, PK_CR = 36, PK_CG = 46, PK_CB = 56, PK_LT = 66, PK_R = 82, PK_TH = 96, PK_A = 110,
       PK_ACTIVE = 127 };
enum { PKW_XY = 18, PKW_C = 10, PKW_LT = 16, PKW_R = 14, PKW_TH = 14, PKW_A = 14 };

static void pk_put(uint32_t w[4], int off, int n, uint32_t v)
{
    for (int b = 0; b < n; ++b)
        if ((v >> b) & 1u) w[(off + b) >> 5] |= 1u << ((off + b) & 31);
}

static uint32_t pk_get(const uint32_t w[4], int off, int n)
{
    uint32_t v = 0;
    for (int b = 0; b < n; ++b) v |= ((w[(off + b) >> 5] >> ((off + b) & 31)) & 1u) << b;
    return v;
}

static uint32_t pk_round(double t, double top)
{
    if (t != t) return 0;
    t = floor(t + 0.5);
    if (t < 0.0) t = 0.0;
    if (t > top) t = top;
    return (uint32_t)t;
}

static const double PK_PI = 3.14159265358979323846;

/* cell index floor(t), clamped to [0, cells - 1] */
static uint32_t pk_cell(double t, double cells)
{
    if (t != t) return 0;
    t = floor(t);
    if (t < 0.0) t = 0.0;
    if (t > cells - 1.0) t = cells - 1.0;
    return (uint32_t)t;
}

static uint32_t pk_range_q(float v, float lo, float hi, int bits)
{
    const double top = (double)((1u << bits) - 1u);
    if (!((double)hi > (double)lo)) return 0;
    return pk_round(((double)v - (double)lo) / ((double)hi - (double)lo) * top, top);
}

static float pk_range_v(uint32_t q, float lo, float hi, int bits)
{
    const double top = (double)((1u << bits) - 1u);
    return (float)((double)lo + (double)q * (((double)hi - (double)lo) / top));
}

/* lohi = (lo ln tau, lo r, lo a, hi ln tau, hi r, hi a) over the active
 * sites (NaN values skipped, -0 taken as +0); all zero without any. */
void orc_pack_ranges(int N, const float *params, float *lohi)
{
    const int planes[3] = {P_LT, P_R, P_A};
    for (int f = 0; f < 3; ++f) {
        int any = 0;
        float lo = 0.0f, hi = 0.0f;
        for (int i = 0; i < N; ++i) {
            if (!(params[P_X * N + i] >= 0.0f)) continue;
            const float v = params[planes[f] * N + i] + 0.0f;
            if (v != v) continue;
            if (!any || v < lo) lo = v;
            if (!any || v > hi) hi = v;
            any = 1;
        }
        lohi[f] = lo;
        lohi[3 + f] = hi;
    }
}

void orc_pack_sites(int H, int W, int N, const float *params, const float *lohi, uint32_t *packed)
{
    const double cells = (double)(1u << PKW_XY), top_c = (double)((1u << PKW_C) - 1u);
    const double tq = (double)(1u << PKW_TH);
    for (int i = 0; i < N; ++i) {
        uint32_t *w = packed + (size_t)i * 4;
        w[0] = w[1] = w[2] = w[3] = 0;
        const float x = params[P_X * N + i], y = params[P_Y * N + i];
        if (!(x >= 0.0f)) continue;
        pk_put(w, PK_X, PKW_XY, pk_cell((double)x / (double)W * cells, cells));
        pk_put(w, PK_Y, PKW_XY, pk_cell((double)y / (double)H * cells, cells));
        const int cp[3] = {P_CR, P_CG, P_CB}, co[3] = {PK_CR, PK_CG, PK_CB};
        for (int c = 0; c < 3; ++c) {
            double v = (double)params[cp[c] * N + i];
            if (v < 0.0) v = 0.0;
            if (v > 1.0) v = 1.0;
            pk_put(w, co[c], PKW_C, pk_round(v * top_c, top_c));
        }
        pk_put(w, PK_LT, PKW_LT, pk_range_q(params[P_LT * N + i] + 0.0f, lohi[0], lohi[3], PKW_LT));
        pk_put(w, PK_R, PKW_R, pk_range_q(params[P_R * N + i] + 0.0f, lohi[1], lohi[4], PKW_R));
        pk_put(w, PK_A, PKW_A, pk_range_q(params[P_A * N + i] + 0.0f, lohi[2], lohi[5], PKW_A));
        double th = fmod((double)params[P_TH * N + i], PK_PI);
        if (th < 0.0) th += PK_PI;
        const uint32_t qt = th == th ? (uint32_t)floor(th / PK_PI * tq + 0.5) : 0u;
        pk_put(w, PK_TH, PKW_TH, qt & ((1u << PKW_TH) - 1u));
        pk_put(w, PK_ACTIVE, 1, 1u);
    }
}

void orc_unpack_sites(int H, int W, int N, const uint32_t *packed, const float *lohi, float *params)
{
    const double cells = (double)(1u << PKW_XY), top_c = (double)((1u << PKW_C) - 1u);
    const double tq = (double)(1u << PKW_TH);
    for (int i = 0; i < N; ++i) {
        const uint32_t *w = packed + (size_t)i * 4;
        for (int p = 0; p < P_COUNT; ++p) params[p * N + i] = 0.0f;
        if (!pk_get(w, PK_ACTIVE, 1)) {
            params[P_X * N + i] = -1.0f;
            continue;
        }
        params[P_X * N + i] = (float)(((double)pk_get(w, PK_X, PKW_XY) + 0.5) * (double)W / cells);
        params[P_Y * N + i] = (float)(((double)pk_get(w, PK_Y, PKW_XY) + 0.5) * (double)H / cells);
        params[P_CR * N + i] = (float)((double)pk_get(w, PK_CR, PKW_C) / top_c);
        params[P_CG * N + i] = (float)((double)pk_get(w, PK_CG, PKW_C) / top_c);
        params[P_CB * N + i] = (float)((double)pk_get(w, PK_CB, PKW_C) / top_c);
        params[P_LT * N + i] = pk_range_v(pk_get(w, PK_LT, PKW_LT), lohi[0], lohi[3], PKW_LT);
        params[P_R * N + i] = pk_range_v(pk_get(w, PK_R, PKW_R), lohi[1], lohi[4], PKW_R);
        params[P_A * N + i] = pk_range_v(pk_get(w, PK_A, PKW_A), lohi[2], lohi[5], PKW_A);
        params[P_TH * N + i] = (float)((double)pk_get(w, PK_TH, PKW_TH) * (PK_PI / tq));
    }
}
