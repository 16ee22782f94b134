/*
 * vq_oracle.c -- CPU oracle for the VQ-MoE expert path.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load or call this code. The
 * product path (the CUDA library) shares nothing with it: no headers, no
 * helpers, no tables.
 *
 * It is a plain, slow, obviously correct implementation of what the path
 * computes, in double precision, following the format the VQ model cards
 * describe:
 *
 *   - Qwen3.5-397B-A17B-VQ-2.6bpw card, "Methodology": each d-weight subvector
 *     of an expert weight row stores one log2(K)-bit index into a per-tensor
 *     codebook of K fp16 entries, with one fp16 scale per (row, 64 weights).
 *   - same card and the 2.4bpw card, "Methodology" / "Sub-byte bit-packing":
 *     the codes are packed into uint32 words, row-local, in 32-code blocks.
 *   - Qwen3.5-397B-A17B-VQ-2.4bpw card, "Changelog 2026-10-01 (vq-skipzero)":
 *     dead output rows have their codes and scales dropped and output exact
 *     zeros; the live rows are unchanged.
 *   - Qwen3.8-Flash-Next and gemma-4 cards: MoE experts selected top-k from
 *     router logits (10-of-512, 128 experts top-8).
 *
 * Readings where the pages are silent:
 *   R3  bit order: code j of a row occupies bits [j*b, j*b + b) of the row's
 *       bit string; bit i of that string is bit (i % 32) of word i / 32
 *       (least significant bit first). A 32-code block is then exactly b
 *       words, and each row starts at its own word 0 (row-local).
 *   R4  subvector direction: code j covers the d consecutive weights
 *       [j*d, j*d + d) of its row.
 *   R1  routing weights: softmax of the selected logits (renorm = 1), or the
 *       full softmax over all experts evaluated at the selected ones
 *       (renorm = 0).
 *   R2  top-k order: larger logit first; equal logits -> smaller expert index
 *       first; NaN ranks below every number.
 *   SwiGLU: h = silu(g) * u with silu(z) = z / (1 + exp(-z)).
 *
 * Dequantised weights: w = fp32(centroid) * fp32(scale). Both factors are
 * fp16, so the product has at most 22 significant bits and is exact in fp32;
 * computing it in double gives the identical value.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- numbers */

/* IEEE 754 binary16 -> double (exact). 1 sign bit, 5 exponent bits (bias 15),
 * 10 fraction bits. */
double vqo_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int ex = (h >> 10) & 0x1F;
    int fr = h & 0x3FF;
    double v;
    if (ex == 0)
        v = ldexp((double)fr, -24);                 /* subnormal: fr * 2^-24 */
    else if (ex == 31)
        v = fr ? NAN : INFINITY;
    else
        v = ldexp((double)(fr + 1024), ex - 25);    /* (1 + fr/2^10) * 2^(ex-15) */
    return sign ? -v : v;
}

/* bfloat16 -> double (exact). 1 sign bit, 8 exponent bits (bias 127),
 * 7 fraction bits. */
double vqo_bf16_to_f64(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int ex = (b >> 7) & 0xFF;
    int fr = b & 0x7F;
    double v;
    if (ex == 0)
        v = ldexp((double)fr, -133);                /* subnormal: fr * 2^(1-127-7) */
    else if (ex == 255)
        v = fr ? NAN : INFINITY;
    else
        v = ldexp((double)(fr + 128), ex - 134);    /* (1 + fr/2^7) * 2^(ex-127) */
    return sign ? -v : v;
}

/* double -> bfloat16 bits, round to nearest, ties to even (one rounding,
 * straight from the double value). */
uint16_t vqo_f64_to_bf16(double v)
{
    if (isnan(v))
        return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return sign | 0x7F80;
    int e2;
    frexp(a, &e2);                  /* a = m * 2^e2, m in [0.5, 1) */
    int E = e2 - 1;                 /* a in [2^E, 2^(E+1)) */
    int q = (E < -126) ? -133 : E - 7;   /* spacing of bf16 values near a */
    double n = ldexp(a, -q);        /* exact: scaling by a power of two */
    double fl = floor(n);
    double rem = n - fl;
    double r;
    if (rem > 0.5)
        r = fl + 1.0;
    else if (rem < 0.5)
        r = fl;
    else
        r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    double rv = ldexp(r, q);        /* rounded magnitude */
    if (rv >= ldexp(1.0, 128))
        return sign | 0x7F80;       /* overflow to infinity */
    if (rv < ldexp(1.0, -126))      /* subnormal (r <= 128 here; 128 is the smallest normal) */
        return sign | (uint16_t)r;
    int e3;
    double m = frexp(rv, &e3);      /* rv = m * 2^e3, m in [0.5, 1) */
    int ex = e3 - 1 + 127;
    int fr = (int)(ldexp(m, 8) - 128.0);   /* m*2^8 in [128, 256) */
    return sign | (uint16_t)(ex << 7) | (uint16_t)fr;
}

/* ---------------------------------------------------------------- packing */

/* Words per packed row: ncode codes of `bits` bits, ncode a multiple of 32,
 * so each 32-code block is exactly `bits` words. */
size_t vqo_row_words(int ncode, int bits)
{
    return (size_t)(ncode / 32) * (size_t)bits;
}

/* Pack one row, bit by bit, per reading R3. */
void vqo_pack_row(const uint16_t *codes, int ncode, int bits, uint32_t *out)
{
    size_t nw = vqo_row_words(ncode, bits);
    memset(out, 0, nw * sizeof(uint32_t));
    for (int j = 0; j < ncode; ++j) {
        for (int q = 0; q < bits; ++q) {
            uint32_t bit = ((uint32_t)codes[j] >> q) & 1u;
            size_t i = (size_t)j * bits + q;        /* position in the row's bit string */
            out[i / 32] |= bit << (i % 32);
        }
    }
}

/* Unpack one row per reading R3: code j = bits [j*b, j*b+b) of the row. */
void vqo_unpack_row(const uint32_t *words, int ncode, int bits, uint16_t *codes)
{
    size_t nw = vqo_row_words(ncode, bits);
    for (int j = 0; j < ncode; ++j) {
        size_t i0 = (size_t)j * bits;
        size_t w = i0 / 32;
        uint64_t window = words[w];
        if (w + 1 < nw)
            window |= (uint64_t)words[w + 1] << 32;
        codes[j] = (uint16_t)((window >> (i0 % 32)) & ((1u << bits) - 1u));
    }
}

/* Is row r of expert e live? A NULL bitmap means every row is live. */
static int is_live(const uint32_t *bitmap, int rows, int e, int r)
{
    if (!bitmap)
        return 1;
    int nw = (rows + 31) / 32;
    return (bitmap[(size_t)e * nw + r / 32] >> (r % 32)) & 1u;
}

/* Pack codes [E, rows, ncode] into live rows only, expert-major (skipzero:
 * dead rows are dropped, live rows keep their bytes). Returns the number of
 * packed (live) rows. */
long vqo_pack(const uint16_t *codes, int E, int rows, int ncode, int bits,
              const uint32_t *bitmap, uint32_t *out)
{
    size_t nw = vqo_row_words(ncode, bits);
    long n = 0;
    for (int e = 0; e < E; ++e)
        for (int r = 0; r < rows; ++r)
            if (is_live(bitmap, rows, e, r)) {
                vqo_pack_row(codes + ((size_t)e * rows + r) * ncode, ncode, bits, out + (size_t)n * nw);
                ++n;
            }
    return n;
}

/* Compact the live rows of a per-row array [E, rows, row_elems] of uint16. */
long vqo_compact_u16(const uint16_t *src, int E, int rows, int row_elems,
                     const uint32_t *bitmap, uint16_t *out)
{
    long n = 0;
    for (int e = 0; e < E; ++e)
        for (int r = 0; r < rows; ++r)
            if (is_live(bitmap, rows, e, r)) {
                memcpy(out + (size_t)n * row_elems, src + ((size_t)e * rows + r) * row_elems,
                       (size_t)row_elems * sizeof(uint16_t));
                ++n;
            }
    return n;
}

/* ---------------------------------------------------------------- modules */

typedef struct {
    int32_t E, rows, cols, d, bits;
    const uint32_t *words;     /* packed live rows, expert-major, vqo_row_words(cols/d, bits) per row */
    const uint16_t *scales;    /* fp16 [live rows, cols/64] */
    const uint16_t *codebook;  /* fp16 [2^bits, d] */
    const uint32_t *bitmap;    /* [E, ceil(rows/32)], bit set = live; NULL = all live */
    const uint16_t *biases;    /* fp16 [live rows, cols/64]: an affine offset per group; NULL = none */
} vqo_module;

/* Packed-row index of every row of expert e (-1 for dead rows). */
static void live_rows(const vqo_module *m, int e, long *idx)
{
    long base = 0;
    for (int e2 = 0; e2 < e; ++e2)
        for (int r = 0; r < m->rows; ++r)
            base += is_live(m->bitmap, m->rows, e2, r);
    for (int r = 0; r < m->rows; ++r)
        idx[r] = is_live(m->bitmap, m->rows, e, r) ? base++ : -1;
}

/* Dequantise expert e of a module: W[r, c] = C[code(r, c/d)][c % d] * s[r, c/64]
 * (+ b[r, c/64] for a module with biases); dead rows are all zero. The biases
 * carry a reading, not a formula from the pages: the Qwen3.5-397B-A17B-VQ-2.4bpw
 * card's "2026-09-20 correction" names a fallback format "affine 3-bit, group
 * 64" (three layers had fallen through to it before they were refitted as VQ)
 * and prints no formula; the reading is the group-wise affine form
 * w = s * q + b, an fp16 scale and an fp16 bias per (row, 64 weights), which
 * is d = 1 with the identity codebook C[q] = q plus the bias.
 * W is [rows, cols] row-major. */
void vqo_dequant(const vqo_module *m, int e, double *W)
{
    int ncode = m->cols / m->d;
    int ngroup = m->cols / 64;
    size_t nw = vqo_row_words(ncode, m->bits);
    long *idx = (long *)malloc(sizeof(long) * m->rows);
    live_rows(m, e, idx);
#pragma omp parallel for schedule(static)
    for (int r = 0; r < m->rows; ++r) {
        double *w = W + (size_t)r * m->cols;
        if (idx[r] < 0) {
            for (int c = 0; c < m->cols; ++c)
                w[c] = 0.0;
            continue;
        }
        uint16_t *codes = (uint16_t *)malloc(sizeof(uint16_t) * ncode);
        vqo_unpack_row(m->words + (size_t)idx[r] * nw, ncode, m->bits, codes);
        for (int c = 0; c < m->cols; ++c) {
            double centroid = vqo_f16_to_f64(m->codebook[(size_t)codes[c / m->d] * m->d + c % m->d]);
            double scale = vqo_f16_to_f64(m->scales[(size_t)idx[r] * ngroup + c / 64]);
            /* without biases the product alone (adding +0.0 would turn a -0.0 product into +0.0) */
            w[c] = m->biases ? centroid * scale + vqo_f16_to_f64(m->biases[(size_t)idx[r] * ngroup + c / 64])
                             : centroid * scale;
        }
        free(codes);
    }
    free(idx);
}

/* y[t, r] = sum_c W[r, c] * x[t, c] in double, for a dense W [rows, cols]. */
static void matvec(const double *W, int rows, int cols, const double *x, int T, double *y)
{
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r)
        for (int t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int c = 0; c < cols; ++c)
                acc += W[(size_t)r * cols + c] * x[(size_t)t * cols + c];
            y[(size_t)t * rows + r] = acc;
        }
}

/* Single-module GEMV: y[t, r] = sum_c W_e[r, c] * x[t, c], x bf16 [T, cols]. */
void vqo_gemv(const vqo_module *m, int e, const uint16_t *x_bf16, int T, double *y)
{
    double *W = (double *)malloc(sizeof(double) * (size_t)m->rows * m->cols);
    double *x = (double *)malloc(sizeof(double) * (size_t)T * m->cols + 1);
    vqo_dequant(m, e, W);
    for (size_t i = 0; i < (size_t)T * m->cols; ++i)
        x[i] = vqo_bf16_to_f64(x_bf16[i]);
    matvec(W, m->rows, m->cols, x, T, y);
    free(x);
    free(W);
}

/* ---------------------------------------------------------------- routing */

/* Does logit a (expert ia) rank before logit b (expert ib)? Reading R2. */
static int ranks_before(float a, int ia, float b, int ib)
{
    int na = isnan(a), nb = isnan(b);
    if (na || nb) {
        if (na && nb)
            return ia < ib;
        return nb;                   /* a number ranks before NaN */
    }
    if (a > b)
        return 1;
    if (a < b)
        return 0;
    return ia < ib;                  /* equal values (incl. -0 == +0) */
}

/* Top-k of one token's logits and its routing weights (reading R1). */
static void route_token(const float *l, int E, int k, int renorm, int32_t *ids, double *w)
{
    char *taken = (char *)calloc((size_t)E, 1);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || ranks_before(l[e], e, l[best], best)))
                best = e;
        taken[best] = 1;
        ids[j] = best;
    }
    double top = (double)l[ids[0]];
    double denom = 0.0;
    if (renorm) {
        for (int j = 0; j < k; ++j)
            denom += exp((double)l[ids[j]] - top);
    } else {
        for (int e = 0; e < E; ++e)
            denom += exp((double)l[e] - top);
    }
    for (int j = 0; j < k; ++j)
        w[j] = exp((double)l[ids[j]] - top) / denom;
    free(taken);
}

/* Route T tokens and bucket the T*k (token, slot) pairs by expert.
 * ids/w [T, k]; counts [E]; offsets [E+1] exclusive prefix sums of counts;
 * perm [T*k]: pair indices p = t*k + j grouped by expert, increasing p inside
 * each expert's bucket. Returns 0, or -1 when k is not in [1, E]. */
int vqo_route(const float *logits, int T, int E, int k, int renorm,
              int32_t *ids, double *w, int32_t *counts, int32_t *offsets, int32_t *perm)
{
    if (k < 1 || k > E)
        return -1;
    for (int t = 0; t < T; ++t)
        route_token(logits + (size_t)t * E, E, k, renorm, ids + (size_t)t * k, w + (size_t)t * k);
    for (int e = 0; e < E; ++e)
        counts[e] = 0;
    for (long p = 0; p < (long)T * k; ++p)
        counts[ids[p]] += 1;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    long pos = 0;
    for (int e = 0; e < E; ++e)
        for (long p = 0; p < (long)T * k; ++p)
            if (ids[p] == e)
                perm[pos++] = (int32_t)p;
    return 0;
}

/* ---------------------------------------------------------------- MoE layer */

static double silu(double z)
{
    return z / (1.0 + exp(-z));
}

/* MoE SwiGLU layer for a list of tokens:
 *   y[i] = sum_j w[t, j] * W_down,e_j ( silu(W_gate,e_j x[t]) * (W_up,e_j x[t]) ),
 * t = tok[i], (e_j, w[t, j]) its top-k experts and weights, j ascending.
 * gate/up: [inter, hidden]; down: [hidden, inter]. y is [ntok, hidden].
 * Each needed expert is dequantised once. Returns 0, or -1 on bad arguments. */
int vqo_moe(const vqo_module *gate, const vqo_module *up, const vqo_module *down,
            int hidden, int inter, const uint16_t *x_bf16, const float *logits, int E,
            int k, int renorm, const int32_t *tok, int ntok, double *y)
{
    if (k < 1 || k > E || gate->rows != inter || gate->cols != hidden || up->rows != inter ||
        up->cols != hidden || down->rows != hidden || down->cols != inter)
        return -1;
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)ntok * k);
    double *wts = (double *)malloc(sizeof(double) * (size_t)ntok * k);
    double *out = (double *)malloc(sizeof(double) * (size_t)ntok * k * hidden);  /* per-pair down outputs */
    for (int i = 0; i < ntok; ++i)
        route_token(logits + (size_t)tok[i] * E, E, k, renorm, ids + (size_t)i * k, wts + (size_t)i * k);

    double *Wg = (double *)malloc(sizeof(double) * (size_t)inter * hidden);
    double *Wu = (double *)malloc(sizeof(double) * (size_t)inter * hidden);
    double *Wd = (double *)malloc(sizeof(double) * (size_t)hidden * inter);
    double *x = (double *)malloc(sizeof(double) * hidden);
    double *g = (double *)malloc(sizeof(double) * inter);
    double *u = (double *)malloc(sizeof(double) * inter);
    double *h = (double *)malloc(sizeof(double) * inter);
    for (int e = 0; e < E; ++e) {
        int used = 0;
        for (long p = 0; p < (long)ntok * k; ++p)
            used |= (ids[p] == e);
        if (!used)
            continue;
        vqo_dequant(gate, e, Wg);
        vqo_dequant(up, e, Wu);
        vqo_dequant(down, e, Wd);
        for (long p = 0; p < (long)ntok * k; ++p) {
            if (ids[p] != e)
                continue;
            int t = tok[p / k];
            for (int c = 0; c < hidden; ++c)
                x[c] = vqo_bf16_to_f64(x_bf16[(size_t)t * hidden + c]);
            matvec(Wg, inter, hidden, x, 1, g);
            matvec(Wu, inter, hidden, x, 1, u);
            for (int c = 0; c < inter; ++c)
                h[c] = silu(g[c]) * u[c];
            matvec(Wd, hidden, inter, h, 1, out + (size_t)p * hidden);
        }
    }
    for (int i = 0; i < ntok; ++i)
        for (int r = 0; r < hidden; ++r) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += wts[(size_t)i * k + j] * out[((size_t)i * k + j) * hidden + r];
            y[(size_t)i * hidden + r] = acc;
        }
    free(h); free(u); free(g); free(x); free(Wd); free(Wu); free(Wg);
    free(out); free(wts); free(ids);
    return 0;
}

int vqo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sets the OpenMP threads of the oracle's loops (n >= 1); a timing knob for
 * the CPU baseline, which reports the oracle on one thread and on all. */
void vqo_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}
