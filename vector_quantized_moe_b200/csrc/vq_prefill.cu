// Prefill path of the VQ-MoE layer on sm_100a: per expert bucket a grouped
// GEMM on the 5th-generation tensor cores (tcgen05.mma, fp32 accumulators in
// tensor memory) with the weight tiles decoded on chip.
//
// Format (VQ model cards): Qwen3.5-397B-A17B-VQ-2.6bpw "Methodology" (one
// index per d-weight subvector into an fp16 codebook, fp16 scale per
// (row, 64 weights)); Qwen3.5-397B-A17B-VQ-2.4bpw "Methodology" (uint32
// words, row-local 32-code blocks) and "Changelog 2026-10-01" (skipzero).
// The gemma-4 card ("Faster prefill") describes its Apple-GPU prefill only as
// decoding weights in chunks before the matmul; this kernel is a new design.
//
// One CTA per SM, persistent over (expert, 128-row weight tile, token tile)
// work items. Warp roles:
//   warp 0     TMA: activation tiles (fp16, 128B-swizzled, one 64-column
//              k-step per stage) and packed-code tiles (a chunk of CH k-steps)
//   warp 1     owns the tensor memory; one thread issues tcgen05.mma
//   warps 2+   NWG warpgroups taking the k-steps in turn: thread i of a
//              warpgroup decodes row i of the weight tile (unpack, codebook
//              lookup, x fp16 scale) into registers, waits until the MMA that
//              last read the tensor-memory stage has finished, and stores the
//              row into lane i, where tcgen05.mma reads its A operand; all
//              then run the epilogue from tensor memory, on interleaved
//              32-column blocks
// D[row, token] = sum_k W[row, k] X[token, k]: the weight tile is the
// M=128 operand (in tensor memory), the tokens of the bucket the N operand
// (16..BN, shared memory), so small buckets waste no M rows. Tensor memory
// holds the accumulators (nmod x BN columns) and the A stages left beside
// them; the MMAs of a tile start once both warpgroups have read the previous
// tile's accumulators.
// Every mbarrier wait is bounded; on a timeout the CTA records an error word,
// stops, and frees its tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <utility>

#include "vq_device.cuh"
#include "vq_internal.h"
#include "vq_sm100.cuh"

namespace vq {
namespace {

constexpr int BM = 128;             // weight rows per tile = TMEM lanes
constexpr int NWG = 2;              // dequant/epilogue warpgroups (take k-steps in turn)
constexpr int NTHREADS = 64 + 128 * NWG;   // TMA warp, MMA warp, the warpgroups
constexpr int A_COLS = 32;          // tensor-memory columns of one 128 x 64 fp16 weight tile
constexpr int TMEM_COLS = 512;
// Tokens per tile. One M = 128, K = 16 instruction costs the same for any
// N <= 192, so gate/up takes 192-token tiles: its two fp32 accumulators
// (2 x 192 columns) leave 128 tensor-memory columns, two A stages of both
// modules' weight tiles. down (one module) takes 256-token tiles.
__host__ __device__ constexpr int bn_of(int nmod) { return nmod == 2 ? 192 : 256; }
// A stages (decoded weight tiles of the nmod modules) in tensor memory: what
// the accumulators leave, at most 4
__host__ __device__ constexpr int a_stages_of(int nmod)
{
    return (TMEM_COLS - nmod * bn_of(nmod)) / (nmod * A_COLS) < 4 ? (TMEM_COLS - nmod * bn_of(nmod)) / (nmod * A_COLS)
                                                                    : 4;
}
static_assert(a_stages_of(2) >= NWG && a_stages_of(1) >= NWG, "each warpgroup needs an A stage of its own");

// k-steps whose code bits fill whole 16-byte units (a TMA box of code words
// starts on a 16-byte boundary)
__host__ __device__ constexpr int chunk_steps_aligned(int kb)
{
    int ch = 1;
    while ((ch * kb) % 128)
        ++ch;
    return ch;
}

// Steps per code chunk. Where whole 16-byte units take 4 or more steps (e.g.
// d = 4 with an odd code width: 144, 176 or 208 bits a step), a chunk is half
// that: its bits are then an odd multiple of 64, and the odd chunks start 64
// bits into their box, which begins on the 16-byte boundary below them.
__host__ __device__ constexpr bool chunk_split(int kb) { return chunk_steps_aligned(kb) >= 4; }
__host__ __device__ constexpr int chunk_steps(int kb)
{
    return chunk_split(kb) ? chunk_steps_aligned(kb) / 2 : chunk_steps_aligned(kb);
}
// words per row of a chunk's box: its bits, plus the 64-bit lead of odd chunks
__host__ __device__ constexpr int chunk_words(int kb)
{
    return chunk_split(kb) ? (64 + chunk_steps(kb) * kb + 127) / 128 * 4 : chunk_steps(kb) * kb / 32;
}
// first word of chunk c's box (a multiple of 4)
__host__ __device__ constexpr int chunk_x(int kb, int c)
{
    return (c * chunk_steps(kb) * kb - (chunk_split(kb) && (c & 1) ? 64 : 0)) / 32;
}

__host__ __device__ constexpr int log2i(int v) { return v <= 1 ? 0 : 1 + log2i(v / 2); }

constexpr int B_STAGES = 4;           // at most this many activation tiles in shared memory
constexpr int CODE_STAGES = 2;
constexpr long SMEM_LIMIT = 227L * 1024;
// the codebook replica count is sized for this many activation stages, the
// alignment slack, barriers and a tile table of up to 1024 experts (more
// experts take activation stages instead)
__host__ __device__ constexpr int design_b_stages(int nmod) { return nmod == 2 ? 3 : 4; }
constexpr long SMEM_RESERVE = 1024 + 1024 + 4L * 1024;

// bytes of one code stage of one module: the chunk's packed codes of BM rows,
// then the scales of an 8-group block
__host__ __device__ constexpr long code_stage_bytes(int d, int bits)
{
    return (long)128 * chunk_words((64 / d) * bits) * 4 + 128 * 16;
}

// codebook replicas in shared memory (log2, at most 16 replicas): as many as
// fit next to the operand and code stages
__host__ __device__ constexpr int prefill_log_rep(int d, int bits, int nmod)
{
    const long left = SMEM_LIMIT - SMEM_RESERVE - (long)design_b_stages(nmod) * bn_of(nmod) * 128 -
                      (long)CODE_STAGES * nmod * code_stage_bytes(d, bits);
    int lr = 0;
    while (lr < 4 && (long)nmod * (1L << bits) * d * 2 * (2L << lr) <= left)
        ++lr;
    return lr;
}

template <int D, int BITS, int NMOD>
struct PG {
    static constexpr int KB = (64 / D) * BITS;       // code bits of one row per 64-column step
    static constexpr int CH = chunk_steps(KB);       // steps per code chunk
    static constexpr bool SPLIT = chunk_split(KB);   // odd chunks start 64 bits into their box
    static constexpr int CHW = chunk_words(KB);      // words per row of a chunk's box
    static constexpr uint32_t MASK = (1u << BITS) - 1u;
    static constexpr int LREP = prefill_log_rep(D, BITS, NMOD);
    static constexpr int L = LREP + 1 + log2i(D);    // code -> byte offset of its replica row
};

struct PrefillArgs {
    CUtensorMap tmap_b;       // activations fp16 [slots, K], box {64, BN}, 128B swizzle
    CUtensorMap tmap_c[2];    // packed codes u32 [live rows, row_words], box {CHW, BM}
    CUtensorMap tmap_s[2];    // scales fp16 [live rows, ngroups], box {8, BM}
    ModDev mod[2];
    int nmod;
    const int32_t *offsets;
    const int32_t *active;
    const int32_t *n_active;
    int K;                    // contraction length
    int rows;                 // weight rows (M)
    int sa, sc;               // operand stages, code stages
    uint32_t off_a, off_b, off_c, off_cb, off_tiles, off_bar;
    int scale_tma;            // scales staged by TMA with the code chunks (else read per thread)
    void *out;                // SwiGLU: fp16 [slots, rows]; else fp32 [slots, rows] (module 0)
    void *out2;               // not SwiGLU, two modules: module 1's fp32 [slots, rows]
    int swiglu;
    const float *sxinv;       // per slot, 2^-k of its activation row's scale (NULL: the caller applies it)
    int8_t *hexp;             // SwiGLU: per (slot, 32-row block), the exponent its fp16 h values carry
    int nblk32;               // SwiGLU: rows / 32
    int *err;
    uint32_t wait_limit;      // polls of a bounded wait before it gives up
};

// a * b + c on fp16 pairs, one rounding to nearest even: the weight pair
// C[q] * s + bias (bias 0 without the affine arm).
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c)
{
    __half2 r = __hfma2(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b),
                        *reinterpret_cast<__half2 *>(&c));
    return *reinterpret_cast<uint32_t *>(&r);
}

// ------------------------------------------------------------------ dequant

template <int BITS, int NW>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[NW], int pos)
{
    const int wi = pos >> 5, sh = pos & 31;
    if (sh + BITS <= 32)
        return (w[wi] >> sh) & ((1u << BITS) - 1u);
    return __funnelshift_r(w[wi], w[wi + 1], sh) & ((1u << BITS) - 1u);
}

// The 16-byte-aligned words of a chunk row that hold k-step JJ's code bits,
// the chunk's first code starting OFF bits into the row.
template <int D, int BITS, int JJ, int OFF>
struct Win {
    static constexpr int KB = (64 / D) * BITS;
    static constexpr int W0 = ((OFF + JJ * KB) / 32) & ~3;
    static constexpr int W1 = (((OFF + JJ * KB + KB + 31) / 32) + 3) & ~3;
    static constexpr int NV = (W1 - W0) / 4;
    static constexpr int BASE = OFF + JJ * KB - 32 * W0;
    static_assert(W1 <= chunk_words(KB), "the window stays inside the chunk's box");
};

// Byte offset of the lane's replica of the code at bit `pos` of the window:
// (code << L) | rep_off, formed with one shift and one mask-or.
template <int BITS, int L, int NW>
__device__ __forceinline__ uint32_t entry_off(const uint32_t (&w)[NW], int pos, uint32_t rep_off)
{
    const int wi = pos >> 5, sh = pos & 31;
    uint32_t v;
    int s;
    if (sh + BITS <= 32) {
        v = w[wi];
        s = sh;
    } else {
        v = __funnelshift_r(w[wi], w[wi + 1], sh);
        s = 0;
    }
    const uint32_t x = s >= L ? (v >> (s - L)) : (v << (L - s));
    return (x & (((1u << BITS) - 1u) << L)) | rep_off;
}

// One row of the 128 x 64 fp16 weight tile for k-step JJ of a code chunk:
// 64 weights = 64/D codes read from the chunk row `crow` in shared memory,
// each a codebook entry (the lane's replica) times the row's scale plus the
// row's bias (one fp16 fused multiply-add, rounded to nearest; the bias is 0
// without the affine arm), as 32 words o[c] = weights (2c, 2c+1), the layout
// of one tensor-memory lane of the MMA's A operand.
template <int D, int BITS, int L, int JJ, int OFF>
__device__ __forceinline__ void dequant_step(const uint8_t *crow, const char *cb, uint32_t rep_off, uint32_t s2,
                                             uint32_t b2, bool live, uint32_t (&o)[32])
{
    using W = Win<D, BITS, JJ, OFF>;
    constexpr int NC = 64 / D;
    uint32_t w[4 * W::NV];
#pragma unroll
    for (int v = 0; v < W::NV; ++v) {
        const uint4 q = reinterpret_cast<const uint4 *>(crow)[W::W0 / 4 + v];
        w[4 * v] = q.x;
        w[4 * v + 1] = q.y;
        w[4 * v + 2] = q.z;
        w[4 * v + 3] = q.w;
    }
    if constexpr (D == 1) {
#pragma unroll
        for (int c = 0; c < NC; c += 2) {
            const uint32_t v = (uint32_t)*reinterpret_cast<const uint16_t *>(
                                   cb + entry_off<BITS, L>(w, W::BASE + c * BITS, rep_off)) |
                               ((uint32_t)*reinterpret_cast<const uint16_t *>(
                                    cb + entry_off<BITS, L>(w, W::BASE + (c + 1) * BITS, rep_off))
                                << 16);
            o[c >> 1] = hfma2(v, s2, b2);
        }
    } else if constexpr (D == 2) {
#pragma unroll
        for (int c = 0; c < NC; ++c)
            o[c] = hfma2(*reinterpret_cast<const uint32_t *>(cb + entry_off<BITS, L>(w, W::BASE + c * BITS, rep_off)),
                         s2, b2);
    } else if constexpr (D == 4) {
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const uint2 v = *reinterpret_cast<const uint2 *>(cb + entry_off<BITS, L>(w, W::BASE + c * BITS, rep_off));
            o[2 * c] = hfma2(v.x, s2, b2);
            o[2 * c + 1] = hfma2(v.y, s2, b2);
        }
    } else {
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const uint4 v = *reinterpret_cast<const uint4 *>(cb + entry_off<BITS, L>(w, W::BASE + c * BITS, rep_off));
            o[4 * c] = hfma2(v.x, s2, b2);
            o[4 * c + 1] = hfma2(v.y, s2, b2);
            o[4 * c + 2] = hfma2(v.z, s2, b2);
            o[4 * c + 3] = hfma2(v.w, s2, b2);
        }
    }
    if (!live) {
#pragma unroll
        for (int q = 0; q < 32; ++q)
            o[q] = 0u;
    }
}

// ------------------------------------------------------------------ kernel

struct Item {
    int e, m0, q0, n;
};

template <int BN>
__device__ __forceinline__ Item item_of(long it, int MT, const int *tiles, int n_act, const int32_t *active,
                                        const int32_t *offsets)
{
    const int mt = (int)it % MT;   // item counts fit 32 bits (a host check)
    const int ntg = (int)it / MT;
    int lo = 0, hi = n_act;   // last ai with tiles[ai] <= ntg
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tiles[mid] <= ntg)
            lo = mid;
        else
            hi = mid;
    }
    Item r;
    r.e = active[lo];
    const int nt = ntg - tiles[lo];
    r.m0 = mt * BM;
    r.q0 = offsets[r.e] + nt * BN;
    r.n = min(BN, offsets[r.e + 1] - r.q0);
    return r;
}

// packed row of the first row of an m-tile (m0 is a multiple of 128)
__device__ __forceinline__ int tile_prow0(const ModDev &m, int e, int m0)
{
    if (!m.bitmap)
        return e * m.rows + m0;
    return (int)m.rank[(long)e * m.bm_words + (m0 >> 5)];
}

template <int D, int BITS, int NMOD>
__global__ void __launch_bounds__(NTHREADS, 1) vq_prefill_gemm_kernel(const __grid_constant__ PrefillArgs a)
{
    using P = PG<D, BITS, NMOD>;
    constexpr int BN = bn_of(NMOD);
    constexpr uint32_t B_TILE = BN * 128;
    // one code stage per module: the chunk's packed codes, then the scales of
    // the 8-group block holding its k-steps
    constexpr uint32_t CODE_STAGE = BM * P::CHW * 4 + BM * 16;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw;
    if (smem_u32(smem) & 1023u) {   // the 128-byte swizzle needs 1024-byte aligned tiles
        if (threadIdx.x == 0)
            atomicExch(a.err, 20);
        return;
    }
    uint8_t *sm_b = smem + a.off_b;
    uint8_t *sm_c = smem + a.off_c;
    char *sm_cb = reinterpret_cast<char *>(smem + a.off_cb);
    int *tiles = reinterpret_cast<int *>(smem + a.off_tiles);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + a.off_bar);
    constexpr int SAT = a_stages_of(NMOD);
    uint64_t *full_a = bars;                                      // A stages (tensor memory)
    uint64_t *full_b = bars + 2 * SAT, *empty_b = full_b + a.sa;  // activation stages
    uint64_t *full_c = empty_b + a.sa, *empty_c = full_c + a.sc;  // code stages
    // with as many A stages as activation stages, k-step k uses stage k % sa of both, and one
    // commit per k-step frees both
    const bool a_alias = SAT == a.sa;
    uint64_t *empty_a = a_alias ? empty_b : bars + SAT;
    uint64_t *acc_full = empty_c + a.sc, *acc_empty = acc_full + 1, *drain_bar = acc_empty + 1;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(drain_bar + 1);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain_bar + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int nmod = NMOD;
    // codebooks in shared memory: per module [K][R replicas][d] fp16, lane l
    // reading replica l % R spreads a warp's random lookups over more banks
    constexpr int log_rep = P::LREP;
    const int cb_bytes = ((1 << BITS) << log_rep) * D * 2;
    for (int i = threadIdx.x; i < nmod * (cb_bytes / 2); i += NTHREADS) {
        const int m = i / (cb_bytes / 2), h = i % (cb_bytes / 2);
        const int comp = h % D, slot = h / D;
        reinterpret_cast<uint16_t *>(sm_cb + m * cb_bytes)[h] =
            (m == 0 ? a.mod[0].codebook : a.mod[1].codebook)[(slot >> log_rep) * D + comp];
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < SAT; ++s) {
            mbar_init(&full_a[s], 128);
            mbar_init(&bars[SAT + s], 1);
        }
        for (int s = 0; s < a.sa; ++s) {
            mbar_init(&full_b[s], 1);
            mbar_init(&empty_b[s], 1);
        }
        for (int s = 0; s < a.sc; ++s) {
            mbar_init(&full_c[s], 1);
            mbar_init(&empty_c[s], 128 * NWG);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 128 * NWG);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // accumulators: nmod x BN columns; then SAT stages of nmod A tiles
    const uint32_t acc_cols = (uint32_t)nmod * BN;
    const uint32_t tmem_cols = TMEM_COLS;
    static_assert(NMOD * BN + SAT * NMOD * A_COLS <= TMEM_COLS, "tensor memory");
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(tmem_cols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    grid_dep_launch();   // the next kernel may start its prologue; it waits for this one's results
    grid_dep_wait();

    // tile prefix over the active experts: tiles[ai] = first global n-tile of expert active[ai]
    // (warp 2 scans 32 experts per step, so the loads of a step are in flight together)
    const int n_act = *a.n_active;
    if (warp == 2) {
        int run = 0;
        for (int a0 = 0; a0 < n_act; a0 += 32) {
            const int ai = a0 + lane;
            int nt = 0;
            if (ai < n_act) {
                const int e = a.active[ai];
                nt = (a.offsets[e + 1] - a.offsets[e] + BN - 1) / BN;
            }
            int incl = nt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o)
                    incl += v;
            }
            if (ai < n_act)
                tiles[ai] = run + incl - nt;
            run += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0)
            tiles[n_act] = run;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int MT = (a.rows + BM - 1) / BM;
    const long n_items = (long)tiles[n_act] * MT;
    const int ksteps = a.K / 64;
    const int nchunks = ksteps / P::CH;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        // Two independent streams in work-item order: code chunks (into sc stages) and activation
        // tiles (into sa stages). One thread tests both (without blocking) and issues whichever has
        // a free stage, so a code chunk never waits behind activation stages that only the MMAs
        // free. A wait gives up after wait_limit idle polls.
        if (lane == 0) {
            uint32_t ks = 0, st = 0, ph = 0, cks = 0, cst = 0, cph = 0;   // operand / code stage counters
            long itc = blockIdx.x, itb = blockIdx.x;   // the streams' current work items
            int c = 0, kb = 0;                         // next chunk / k-step within them
            int prow0[2] = {0, 0};
            int q0 = 0;
            if (itc < n_items) {
                const Item itm = item_of<BN>(itc, MT, tiles, n_act, a.active, a.offsets);
                for (int m = 0; m < nmod; ++m)
                    prow0[m] = tile_prow0(a.mod[m], itm.e, itm.m0);
                q0 = itm.q0;
            }
            bool ok = a.wait_limit != 0 || n_items <= blockIdx.x || mbar_give_up(abort_flag, a.err, 1);
            uint32_t idle = 0;   // polls since the last issue
            while (ok && (itc < n_items || itb < n_items)) {
                bool did = false;
                if (itc < n_items && mbar_test_wait(&empty_c[cst], cph ^ 1)) {
                    mbar_expect_tx(&full_c[cst], (uint32_t)(nmod * (a.scale_tma ? CODE_STAGE : BM * P::CHW * 4)));
                    for (int m = 0; m < nmod; ++m) {
                        uint8_t *stg = sm_c + ((size_t)cst * nmod + m) * CODE_STAGE;
                        tma_load_2d(stg, &a.tmap_c[m], chunk_x(P::KB, c), prow0[m], &full_c[cst]);
                        if (a.scale_tma)
                            tma_load_2d(stg + BM * P::CHW * 4, &a.tmap_s[m], (c * P::CH) & ~7, prow0[m],
                                        &full_c[cst]);
                    }
                    ++cks;
                    if (++cst == (uint32_t)a.sc) {
                        cst = 0;
                        cph ^= 1;
                    }
                    if (++c == nchunks) {
                        c = 0;
                        itc += gridDim.x;
                        if (itc < n_items) {
                            const Item itm = item_of<BN>(itc, MT, tiles, n_act, a.active, a.offsets);
                            for (int m = 0; m < nmod; ++m)
                                prow0[m] = tile_prow0(a.mod[m], itm.e, itm.m0);
                        }
                    }
                    did = true;
                }
                if (itb < n_items && mbar_test_wait(&empty_b[st], ph ^ 1)) {
                    if (kb == 0)
                        q0 = item_of<BN>(itb, MT, tiles, n_act, a.active, a.offsets).q0;
                    mbar_expect_tx(&full_b[st], (uint32_t)B_TILE);
                    tma_load_2d(sm_b + (size_t)st * B_TILE, &a.tmap_b, kb * 64, q0, &full_b[st]);
                    ++ks;
                    if (++st == (uint32_t)a.sa) {
                        st = 0;
                        ph ^= 1;
                    }
                    if (++kb == ksteps) {
                        kb = 0;
                        itb += gridDim.x;
                    }
                    did = true;
                }
                if (did) {
                    idle = 0;
                } else if (++idle >= a.wait_limit) {
                    ok = mbar_give_up(abort_flag, a.err, 2);
                } else {
                    if ((idle & 63) == 63 && *abort_flag)
                        ok = false;
                    __nanosleep(32);   // leave the issue slots to the dequant warps of this sub-partition
                }
            }
            // the loads issued have landed before the CTA leaves (the last use of each stage): after
            // a give-up the other warps may not have waited for them
            for (uint32_t s = 0; s < (uint32_t)a.sa && s < ks; ++s)
                mbar_drain(&full_b[(ks - 1 - s) % a.sa], ((ks - 1 - s) / a.sa) & 1);
            for (uint32_t s = 0; s < (uint32_t)a.sc && s < cks; ++s)
                mbar_drain(&full_c[(cks - 1 - s) % a.sc], ((cks - 1 - s) / a.sc) & 1);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t ast = 0, aph = 0, st = 0, ph = 0, nacc = 0;   // A stage / activation stage counters
            bool ok = true, issued = false;
            for (long it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                const Item itm = item_of<BN>(it, MT, tiles, n_act, a.active, a.offsets);
                const int n16 = (itm.n + 15) & ~15;
                const uint32_t idesc = idesc_f16(BM, n16);
                // both warpgroups' epilogues of the previous item have read the accumulators
                if (!(ok = mbar_wait(acc_empty, (nacc & 1) ^ 1, abort_flag, a.err, 9, a.wait_limit)))
                    break;
                ++nacc;
                tc_fence_after();
                for (int k = 0; k < ksteps; ++k) {
                    if (!(ok = mbar_wait(&full_a[ast], aph, abort_flag, a.err, 4, a.wait_limit)))
                        break;
                    if (!(ok = mbar_wait(&full_b[st], ph, abort_flag, a.err, 5, a.wait_limit)))
                        break;
                    tc_fence_after();
                    const uint64_t bdesc = sw128_desc(smem_u32(sm_b + (size_t)st * B_TILE));
                    // the two modules' MMAs alternate: consecutive MMAs into one
                    // accumulator depend on each other, the two accumulators do not
#pragma unroll
                    for (int k16 = 0; k16 < 4; ++k16)
                        for (int m = 0; m < nmod; ++m) {
                            const uint32_t a_tmem = tmem + acc_cols + (ast * nmod + m) * A_COLS;
                            umma_ts(tmem + m * BN, a_tmem + 8 * k16, bdesc + 2 * k16, idesc, (k | k16) != 0);
                        }
                    umma_commit(&empty_b[st]);
                    if (!a_alias)
                        umma_commit(&empty_a[ast]);
                    issued = true;
                    if (++st == (uint32_t)a.sa) {
                        st = 0;
                        ph ^= 1;
                    }
                    if (++ast == (uint32_t)SAT) {
                        ast = 0;
                        aph ^= 1;
                    }
                }
                if (ok)
                    umma_commit(acc_full);
            }
            if (issued) {
                // every MMA has completed before the tensor memory is freed (after a give-up
                // elsewhere in the CTA, the last ones may still run)
                umma_commit(drain_bar);
                mbar_drain(drain_bar, 0);
            }
        }
    } else {
        // ---------------------------------------------------------- dequant + epilogue
        const int wg = (warp - 2) >> 2;   // warpgroup: takes k-steps with k % NWG == wg
        const int rowi = 32 * (warp & 3) + lane;
        const uint32_t rep_off = (uint32_t)(lane & ((1 << log_rep) - 1)) * (2 * D);
        const uint32_t lane_addr = (uint32_t)(32 * (warp & 3)) << 16;
        uint32_t st = 0, ph = 0, cst = 0, cph = 0, nit = 0;
        bool ok = true;
        for (long it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            const Item itm = item_of<BN>(it, MT, tiles, n_act, a.active, a.offsets);
            const int r = itm.m0 + rowi;
            int lrow[2] = {-1, -1};
            long prow[2] = {-1, -1};
            for (int m = 0; m < nmod; ++m) {
                const ModDev &md = a.mod[m];
                prow[m] = r < a.rows ? live_row(md.bitmap, md.rank, md.bm_words, md.rows, itm.e, r) : -1;
                lrow[m] = prow[m] >= 0 ? (int)(prow[m] - tile_prow0(md, itm.e, itm.m0)) : -1;
            }
            for (int c = 0; c < nchunks && ok; ++c) {
                if (!(ok = mbar_wait(&full_c[cst], cph, abort_flag, a.err, 6, a.wait_limit)))
                    break;
                const uint8_t *crow[2];
                const uint16_t *srow[2];
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const uint8_t *stg = sm_c + ((size_t)cst * nmod + (m < nmod ? m : 0)) * CODE_STAGE;
                    const int lr = lrow[m] >= 0 ? lrow[m] : 0;
                    crow[m] = stg + (size_t)lr * P::CHW * 4;
                    srow[m] = reinterpret_cast<const uint16_t *>(stg + BM * P::CHW * 4) + lr * 8 + ((c * P::CH) & 7);
                }
                // the row's fp16 scale of k-step j, as a half2 pair
                auto sfetch = [&](int m, int j) {
                    uint32_t sc;
                    if (a.scale_tma)
                        sc = srow[m][j];
                    else
                        sc = prow[m] >= 0 ? ldg_u16(a.mod[m].scales + prow[m] * a.mod[m].ngroups + c * P::CH + j) : 0u;
                    return sc | (sc << 16);
                };
                // the row's fp16 bias of k-step j (the affine arm), as a half2 pair; 0 without
                auto bfetch = [&](int m, int j) {
                    const uint16_t *bi = a.mod[m].biases;
                    const uint32_t b = (bi && prow[m] >= 0) ? ldg_u16(bi + prow[m] * a.mod[m].ngroups + c * P::CH + j) : 0u;
                    return b | (b << 16);
                };
                // the chunk's steps, its first code OFF bits into the box row
                auto chunk = [&](auto off_c) {
                constexpr int OFF = decltype(off_c)::value;
                auto step = [&](auto jj_c) {
                    constexpr int JJ = decltype(jj_c)::value;
                    if (!ok)
                        return;
                    if ((c * P::CH + JJ) % NWG == wg) {
                        const uint32_t a_tmem = tmem + lane_addr + acc_cols + st * nmod * A_COLS;
                        // decode both modules first (their A tiles are adjacent columns of the
                        // stage, stored with one instruction); the wait for the stage's previous
                        // MMA overlaps the decode
                        uint32_t o[32 * NMOD];
                        dequant_step<D, BITS, P::L, JJ, OFF>(crow[0], sm_cb, rep_off, sfetch(0, JJ), bfetch(0, JJ),
                                                             lrow[0] >= 0, *reinterpret_cast<uint32_t(*)[32]>(o));
                        if constexpr (NMOD == 2)
                            dequant_step<D, BITS, P::L, JJ, OFF>(crow[1], sm_cb + cb_bytes, rep_off, sfetch(1, JJ),
                                                                 bfetch(1, JJ), lrow[1] >= 0,
                                                                 *reinterpret_cast<uint32_t(*)[32]>(o + 32));
                        if (!(ok = mbar_wait(&empty_a[st], ph ^ 1, abort_flag, a.err, 7, a.wait_limit)))
                            return;
                        tc_fence_after();   // the stage's previous MMA has read it
                        if constexpr (NMOD == 2)
                            tmem_st64(a_tmem, o);
                        else
                            tmem_st32(a_tmem, *reinterpret_cast<uint32_t(*)[32]>(o));
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&full_a[st]);
                    }
                    if (++st == (uint32_t)SAT) {
                        st = 0;
                        ph ^= 1;
                    }
                };
                [&]<int... J>(std::integer_sequence<int, J...>) {
                    (step(std::integral_constant<int, J>{}), ...);
                }(std::make_integer_sequence<int, P::CH>{});
                };
                if constexpr (P::SPLIT) {
                    if (c & 1)
                        chunk(std::integral_constant<int, 64>{});
                    else
                        chunk(std::integral_constant<int, 0>{});
                } else {
                    chunk(std::integral_constant<int, 0>{});
                }
                mbar_arrive(&empty_c[cst]);
                if (++cst == (uint32_t)a.sc) {
                    cst = 0;
                    cph ^= 1;
                }
            }
            if (!ok)
                break;
            // epilogue: accumulators of this tile are complete; the warpgroups
            // take alternate 32-column blocks
            if (!(ok = mbar_wait(acc_full, nit & 1, abort_flag, a.err, 8, a.wait_limit)))
                break;
            ++nit;
            tc_fence_after();
            for (int cb0 = 32 * wg; cb0 < itm.n; cb0 += 32 * NWG) {
                uint32_t g[32], u[32];
                tmem_ld32(tmem + lane_addr + cb0, g);
                if (nmod == 2)
                    tmem_ld32(tmem + lane_addr + BN + cb0, u);
                tmem_wait_ld();

                if (NMOD == 2 && a.swiglu) {
                    // the tile's 32 token columns j: the accumulators carry each token's activation
                    // scale 2^k, undone exactly; h = silu(g) u in fp32. The down GEMM reads h as fp16, so
                    // each (slot, 32-row block) is stored times 2^e, e putting the block's largest |h| in
                    // [2^14, 2^15), and e is recorded (the slot's blocks are brought to one exponent
                    // before the down GEMM). The warp's rows lie inside the module or outside it whole
                    // (rows is a multiple of 32).
                    const int wrow0 = itm.m0 + 32 * (warp & 3);
                    if (wrow0 < a.rows) {
                        // lane j holds the inverse activation scale of column j
                        const float fl = cb0 + lane < itm.n ? a.sxinv[itm.q0 + cb0 + lane] : 0.f;
                        // eight columns at a time, in three passes (h; the columns' largest |h|;
                        // scaled stores), so that each pass's eight operations are independent
                        int my_e = 0;   // lane j: the exponent of column j
#pragma unroll
                        for (int j0 = 0; j0 < 32; j0 += 8) {
                            float hv[8];
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const float f = __shfl_sync(0xFFFFFFFFu, fl, j0 + j);
                                const float gv = __uint_as_float(g[j0 + j]) * f, uv = __uint_as_float(u[j0 + j]) * f;
                                hv[j] = __fdividef(gv, 1.f + __expf(-gv)) * uv;
                            }
                            uint32_t mx[8];   // column j's largest |h| over the warp's 32 rows, in every lane
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                mx[j] = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(hv[j]) & 0x7FFFFFFFu);
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int n = cb0 + j0 + j;
                                const int e = scale_exp(mx[j]);
                                my_e = lane == j0 + j ? e : my_e;
                                if (n < itm.n)
                                    reinterpret_cast<__half *>(a.out)[(long)(itm.q0 + n) * a.rows + r] =
                                        __float2half_rn(hv[j] * pow2f_normal(e));
                            }
                        }
                        if (cb0 + lane < itm.n)
                            a.hexp[(long)(itm.q0 + cb0 + lane) * a.nblk32 + (wrow0 >> 5)] = (int8_t)my_e;
                    }
                } else if (r < a.rows) {
                    // fp32 accumulators of one module, or of both (then u holds module 1's), times the
                    // inverse activation scale when the kernel applies it
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int n = cb0 + j;
                        if (n >= itm.n)
                            break;
                        const long o = (long)(itm.q0 + n) * a.rows + r;
                        const float f = a.sxinv ? a.sxinv[itm.q0 + n] : 1.f;
                        reinterpret_cast<float *>(a.out)[o] = __uint_as_float(g[j]) * f;
                        if (nmod == 2)
                            reinterpret_cast<float *>(a.out2)[o] = __uint_as_float(u[j]) * f;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(acc_empty);   // the next item's MMAs may overwrite the accumulators
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols));
    }
}

// gathered activations: Xg[q, :] = x16[perm[q] / k, :] (the token's scaled fp16
// row) and sxinv[q] = xinv[perm[q] / k] (its inverse scale)
__global__ void vq_gather_kernel(const __half *__restrict__ x16, const float *__restrict__ xinv,
                                 const int32_t *__restrict__ perm, int k, long slots, int H, __half *__restrict__ xg,
                                 float *__restrict__ sxinv)
{
    grid_dep_launch();   // the next kernel may start its prologue; it waits for this one's results
    grid_dep_wait();
    const int per_row = H / 8;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < slots * per_row; i += (long)gridDim.x * blockDim.x) {
        const long q = i / per_row;
        const int c = (int)(i % per_row) * 8;
        const long t = perm[q] / k;
        *reinterpret_cast<uint4 *>(xg + q * H + c) = ldg_u128(x16 + t * H + c);
        if (c == 0)
            sxinv[q] = xinv[t];
    }
}

// The gate/up epilogue stored each (slot, 32-row block) of h with its own
// exponent e_b (hexp). Per slot q, every block is brought to the slot's
// exponent E = min_b e_b (the one of its largest |h|): hs *= 2^(E - e_b), a
// power of two <= 1, exact unless a value falls into fp16's subnormal range;
// and the slot's pair p = perm[q] gets wh[p] = w[p] * 2^-E, the routing weight
// that the combine applies to the down projection. One warp per slot; the
// lanes take consecutive 16-byte chunks of the row, so each load and store of
// the warp covers 512 contiguous bytes.
__global__ void vq_hnorm_kernel(__half *__restrict__ h, const int8_t *__restrict__ hexp, long slots, int nblk,
                                const int32_t *__restrict__ perm, const float *__restrict__ w, float *__restrict__ wh)
{
    grid_dep_launch();   // the next kernel may start its prologue; it waits for this one's results
    grid_dep_wait();
    const int lane = threadIdx.x & 31;
    const long nwarps = (long)gridDim.x * (blockDim.x >> 5);
    for (long q = blockIdx.x * (long)(blockDim.x >> 5) + (threadIdx.x >> 5); q < slots; q += nwarps) {
        const int8_t *eq = hexp + q * nblk;
        int E = 127;
        for (int b = lane; b < nblk; b += 32)
            E = min(E, (int)eq[b]);
        E = max(__reduce_min_sync(0xFFFFFFFFu, E), -126);
        if (lane == 0) {
            const int p = perm[q];
            wh[p] = w[p] * pow2f(-E);
        }
        uint4 *row = reinterpret_cast<uint4 *>(h + q * nblk * 32);
        for (int c = lane; c < nblk * 4; c += 32) {   // chunk c: 8 values of block c / 4
            const int d = max(E - (int)eq[c >> 2], -64);   // beyond 2^-64 every fp16 value becomes 0
            if (d >= 0)
                continue;
            const float sc = pow2f(d);
            uint4 x = row[c];
            __half2 *hw = reinterpret_cast<__half2 *>(&x);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __half22float2(hw[i]);   // exact; the product too, then one rounding
                hw[i] = __floats2half2_rn(f.x * sc, f.y * sc);
            }
            row[c] = x;
        }
    }
}

// ------------------------------------------------------------------ host side

int chw_of(int d, int bits);

// fp16 activations [rows, cols]: boxes of 64 columns x bn rows, 128-byte swizzle
bool map_act(CUtensorMap *map, const void *base, long rows, int cols, int bn)
{
    return tma_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, (uint64_t)cols, (uint64_t)rows, 64, (uint32_t)bn,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

// fp16 scales [live rows, ngroups]: boxes of 8 groups x BM rows
bool map_scales(CUtensorMap *map, const ModDev &m)
{
    return tma_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, m.scales, (uint64_t)m.ngroups, (uint64_t)m.live_rows, 8,
                      BM, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// packed codes [live rows, row_words]: boxes of one chunk x BM rows
bool map_codes(CUtensorMap *map, const ModDev &m)
{
    return tma_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, m.codes, (uint64_t)m.row_words, (uint64_t)m.live_rows,
                      (uint32_t)chw_of(m.d, m.bits), BM, CU_TENSOR_MAP_SWIZZLE_NONE);
}

int chw_of(int d, int bits) { return chunk_words((64 / d) * bits); }

// k-steps a module's columns must be a multiple of (whole 16-byte units; a
// split geometry then has an even number of chunks)
int ch_of(int d, int bits) { return chunk_steps_aligned((64 / d) * bits); }

struct SmemPlan {
    int sa, sc;
    uint32_t off_a, off_b, off_c, off_cb, off_tiles, off_bar, total;
};

SmemPlan smem_plan(int nmod, int d, int bits, int E)
{
    const uint32_t limit = 227 * 1024 - 1024;   // minus the alignment slack
    const uint32_t code_stage = (uint32_t)(nmod * code_stage_bytes(d, bits));
    const uint32_t cb =
        (uint32_t)align_up((size_t)nmod * ((size_t)1 << bits) * d * 2 << prefill_log_rep(d, bits, nmod), 128);
    const uint32_t tiles = (uint32_t)align_up((size_t)(E + 1) * 4, 128);
    SmemPlan p{};
    for (int sa = B_STAGES; sa >= 2; --sa) {
        p.sa = sa;
        p.sc = CODE_STAGES;
        p.off_a = 0;
        p.off_b = 0;
        p.off_c = p.off_b + (uint32_t)sa * bn_of(nmod) * 128;
        p.off_cb = p.off_c + p.sc * code_stage;
        p.off_tiles = p.off_cb + cb;
        p.off_bar = (uint32_t)align_up(p.off_tiles + tiles, 8);
        p.total = p.off_bar + (2 * sa + 2 * a_stages_of(nmod) + 2 * p.sc + 3) * 8 + 16 + 1024;
        if (p.total <= limit + 1024)
            return p;
    }
    p.total = 0;
    return p;
}

template <int D, int BITS, int NMOD>
cudaError_t launch_gemm(const PrefillArgs &a, int ctas, uint32_t smem, cudaStream_t s)
{
    auto k = vq_prefill_gemm_kernel<D, BITS, NMOD>;
    cudaError_t err = set_smem_limit_once((const void *)k, (int)smem);
    if (err != cudaSuccess)
        return err;
    // An ordinary launch, not a programmatic one: launched early, the persistent CTAs (a whole SM's
    // shared memory and a third of its registers each) crowd the memory-bound kernel before them
    // off the SMs and slow it more than their own prologue gains (the 4096-token Zipf layer's step
    // took 5.7 ms with a programmatic launch, 5.0 ms without).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ctas);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    return cudaLaunchKernelEx(&cfg, k, a);
}

cudaError_t dispatch_gemm(const PrefillArgs &a, int d, int bits, int ctas, uint32_t smem, cudaStream_t s)
{
#define VQ_PGEMM(D_, B_) \
    if (d == D_ && bits == B_) \
        return a.nmod == 2 ? launch_gemm<D_, B_, 2>(a, ctas, smem, s) : launch_gemm<D_, B_, 1>(a, ctas, smem, s);
    VQ_GEOMETRIES(VQ_PGEMM)
#undef VQ_PGEMM
    return cudaErrorInvalidValue;
}

struct PrefillPlan {
    RoutingLayout r;
    size_t x16, xinv, xg, sxinv, h, hexp, wh, dp, total;
};

PrefillPlan plan_prefill(const vq_moe_layer *L, int T, int k)
{
    PrefillPlan p{};
    size_t o = 0;
    p.r = plan_routing(o, T, k, L->gate.E);
    const size_t tk = (size_t)T * k;
    const size_t H = L->gate.cols, I = L->gate.rows;
    p.x16 = o; o = align_up(o + (size_t)T * H * 2, 256);     // scaled fp16 activations, per token
    p.xinv = o; o = align_up(o + (size_t)T * 4, 256);        // their inverse scales
    p.xg = o; o = align_up(o + tk * H * 2, 256);             // gathered by bucket slot
    p.sxinv = o; o = align_up(o + tk * 4, 256);
    p.h = o; o = align_up(o + tk * I * 2, 256);              // SwiGLU output, scaled fp16
    p.hexp = o; o = align_up(o + tk * (I / 32), 256);        // exponents of its 32-row blocks
    p.wh = o; o = align_up(o + tk * 4, 256);                 // routing weights times the h scales
    p.dp = o; o = align_up(o + tk * L->down.rows * 4, 256);  // per-slot down outputs
    p.total = o;
    return p;
}

// The tensor maps and shared-memory layout of one GEMM launch: nmod modules
// (same geometry and shape) against the fp16 activations act [slots, K].
vq_status setup_gemm(PrefillArgs &a, const vq_module *m0, const vq_module *m1, const void *act, long slots, int E,
                     SmemPlan &sp)
{
    a.mod[0] = make_moddev(*m0);
    a.mod[1] = make_moddev(m1 ? *m1 : *m0);
    a.nmod = m1 ? 2 : 1;
    sp = smem_plan(a.nmod, a.mod[0].d, a.mod[0].bits, E);
    if (sp.total == 0)
        return VQ_ERR_UNSUPPORTED;   // the geometry's stages and codebooks do not fit shared memory
    if (!map_act(&a.tmap_b, act, slots, a.mod[0].cols, bn_of(a.nmod)) || !map_codes(&a.tmap_c[0], a.mod[0]) ||
        !map_codes(&a.tmap_c[1], a.mod[1]))
        return VQ_ERR_CUDA;
    a.scale_tma = a.mod[0].ngroups % 8 == 0;
    if (a.scale_tma && (!map_scales(&a.tmap_s[0], a.mod[0]) || !map_scales(&a.tmap_s[1], a.mod[1])))
        return VQ_ERR_CUDA;
    a.K = a.mod[0].cols;
    a.rows = a.mod[0].rows;
    a.sa = sp.sa;
    a.sc = sp.sc;
    a.off_a = sp.off_a;
    a.off_b = sp.off_b;
    a.off_c = sp.off_c;
    a.off_cb = sp.off_cb;
    a.off_tiles = sp.off_tiles;
    a.off_bar = sp.off_bar;
    a.wait_limit = current_wait_limit();
    return VQ_OK;
}

bool module_prefill_ok(const vq_module &m)
{
    const int row_words = (m.cols / m.d / 32) * m.bits;
    return row_words % 4 == 0 && m.cols % (64 * ch_of(m.d, m.bits)) == 0;
}

}  // namespace

size_t prefill_workspace_size(const vq_moe_layer *L, int T, int k)
{
    return plan_prefill(L, T, k).total;
}

vq_status run_prefill(const vq_moe_layer *L, const uint16_t *x, int T, const float *logits, int k, int renorm, void *y,
                      int y_dtype, void *ws, size_t ws_bytes, cudaStream_t s)
{
    if (!module_prefill_ok(L->gate) || !module_prefill_ok(L->up) || !module_prefill_ok(L->down))
        return VQ_ERR_UNSUPPORTED;
    if (L->gate.d != L->up.d || L->gate.bits != L->up.bits)
        return VQ_ERR_UNSUPPORTED;   // gate and up share one fused tile
    if (smem_plan(2, L->gate.d, L->gate.bits, L->gate.E).total == 0 ||
        smem_plan(1, L->down.d, L->down.bits, L->gate.E).total == 0)
        return VQ_ERR_UNSUPPORTED;   // stages and codebooks do not fit shared memory (checked before any launch)
    if (!tma_available())
        return VQ_ERR_CUDA;
    const int E = L->gate.E, H = L->gate.cols, I = L->gate.rows;
    if (T == 0)
        return VQ_OK;
    const PrefillPlan p = plan_prefill(L, T, k);
    if (ws_bytes < p.total)
        return VQ_ERR_WORKSPACE;
    int32_t *ids = ws_at<int32_t>(ws, p.r.ids);
    float *w = ws_at<float>(ws, p.r.w);
    int32_t *offsets = ws_at<int32_t>(ws, p.r.offsets);
    int32_t *perm = ws_at<int32_t>(ws, p.r.perm);
    int32_t *pos = ws_at<int32_t>(ws, p.r.pos);
    int32_t *active = ws_at<int32_t>(ws, p.r.active);
    int32_t *nact = ws_at<int32_t>(ws, p.r.nact);
    int *err = ws_at<int>(ws, p.r.err);
    __half *x16 = ws_at<__half>(ws, p.x16);
    float *xinv = ws_at<float>(ws, p.xinv);
    __half *xg = ws_at<__half>(ws, p.xg);
    float *sxinv = ws_at<float>(ws, p.sxinv);
    __half *hh = ws_at<__half>(ws, p.h);
    int8_t *hexp = ws_at<int8_t>(ws, p.hexp);
    float *wh = ws_at<float>(ws, p.wh);
    float *dp = ws_at<float>(ws, p.dp);
    const long tk = (long)T * k;
    // the kernels count work items in 32 bits
    for (int m = 0; m < 2; ++m) {
        const long bn = bn_of(2 - m), rows = m ? H : I;
        if (((tk + bn - 1) / bn + E) * ((rows + BM - 1) / BM) >= INT_MAX)
            return VQ_ERR_UNSUPPORTED;
    }

    trace_point(0, s);
    cudaError_t e = launch_route(logits, T, E, k, renorm, ids, w, offsets, perm, pos, active, nact, nullptr, nullptr,
                                 x, x16, xinv, H, err, s, true);
    if (e != cudaSuccess)
        return VQ_ERR_CUDA;
    trace_point(1, s);
    {
        cudaLaunchConfig_t cfg = {};
        const long n = tk * (H / 8);
        cfg.gridDim = dim3((unsigned)std::min<long>((n + 255) / 256, 8192));
        cfg.blockDim = dim3(256);
        cfg.stream = s;
        e = cudaLaunchKernelEx(&cfg, vq_gather_kernel, (const __half *)x16, (const float *)xinv, (const int32_t *)perm,
                               k, tk, H, xg, sxinv);
        if (e != cudaSuccess)
            return VQ_ERR_CUDA;
    }
    trace_point(2, s);

    const int sms = num_sms();
    // gate/up with the SwiGLU epilogue -> h fp16 [slots, inter]
    {
        PrefillArgs a{};
        SmemPlan sp;
        if (const vq_status st = setup_gemm(a, &L->gate, &L->up, xg, tk, E, sp); st != VQ_OK)
            return st;
        a.offsets = offsets;
        a.active = active;
        a.n_active = nact;
        a.out = hh;
        a.swiglu = 1;
        a.sxinv = sxinv;
        a.hexp = hexp;
        a.nblk32 = I / 32;
        a.err = err;
        e = dispatch_gemm(a, a.mod[0].d, a.mod[0].bits, sms, sp.total, s);
        if (e != cudaSuccess)
            return VQ_ERR_CUDA;
    }
    trace_point(3, s);
    // the slots' h blocks to one exponent per slot
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)std::max<long>(1, std::min<long>((tk + 7) / 8, 4096)));
        cfg.blockDim = dim3(256);
        cfg.stream = s;
        e = cudaLaunchKernelEx(&cfg, vq_hnorm_kernel, hh, (const int8_t *)hexp, tk, I / 32, (const int32_t *)perm,
                               (const float *)w, wh);
        if (e != cudaSuccess)
            return VQ_ERR_CUDA;
    }
    // down -> fp32 per-slot outputs [slots, hidden], still times the slot's h scale (the combine undoes it)
    {
        PrefillArgs a{};
        SmemPlan sp;
        if (const vq_status st = setup_gemm(a, &L->down, nullptr, hh, tk, E, sp); st != VQ_OK)
            return st;
        a.offsets = offsets;
        a.active = active;
        a.n_active = nact;
        a.out = dp;
        a.swiglu = 0;
        a.err = err;
        e = dispatch_gemm(a, a.mod[0].d, a.mod[0].bits, sms, sp.total, s);
        if (e != cudaSuccess)
            return VQ_ERR_CUDA;
    }
    trace_point(4, s);
    e = launch_combine(dp, 1, 0, wh, pos, T, k, H, y, y_dtype, s, true);
    trace_point(5, s);
    return e == cudaSuccess ? VQ_OK : VQ_ERR_CUDA;
}

namespace {

__global__ void vq_gemm_tables_kernel(int E, int expert, int T, int32_t *offsets, int32_t *active, int32_t *nact,
                                      int *err)
{
    grid_dep_launch();
    grid_dep_wait();
    for (int i = threadIdx.x; i <= E; i += blockDim.x)
        offsets[i] = i <= expert ? 0 : T;
    if (threadIdx.x == 0) {
        active[0] = expert;
        *nact = 1;
        *err = 0;
    }
}

struct GemmPlan {
    size_t err, offsets, active, nact, x16, xinv, total;
};

GemmPlan plan_gemm(const vq_module *m, int T)
{
    GemmPlan p{};
    size_t o = 0;
    p.err = o; o = align_up(o + 4, 256);
    p.offsets = o; o = align_up(o + (size_t)(m->E + 1) * 4, 256);
    p.active = o; o = align_up(o + 4, 256);
    p.nact = o; o = align_up(o + 4, 256);
    p.x16 = o; o = align_up(o + (size_t)T * m->cols * 2, 256);
    p.xinv = o; o = align_up(o + (size_t)T * 4, 256);
    p.total = o;
    return p;
}

}  // namespace

size_t gemm_workspace_size(const vq_module *m, int T) { return plan_gemm(m, T).total; }

vq_status run_gemm(const vq_module *m0, const vq_module *m1, int expert, const uint16_t *x, int T, float *y0, float *y1,
                   void *ws, size_t ws_bytes, cudaStream_t s)
{
    if (!module_prefill_ok(*m0) || (m1 && !module_prefill_ok(*m1)) ||
        smem_plan(m1 ? 2 : 1, m0->d, m0->bits, m0->E).total == 0)
        return VQ_ERR_UNSUPPORTED;
    if (!tma_available())
        return VQ_ERR_CUDA;
    if (T == 0)
        return VQ_OK;
    const GemmPlan p = plan_gemm(m0, T);
    if (ws_bytes < p.total)
        return VQ_ERR_WORKSPACE;
    // the kernels count work items in 32 bits
    if (((long)(T + bn_of(m1 ? 2 : 1) - 1) / bn_of(m1 ? 2 : 1) + 1) * ((m0->rows + BM - 1) / BM) >= INT_MAX)
        return VQ_ERR_UNSUPPORTED;
    int32_t *offsets = ws_at<int32_t>(ws, p.offsets), *active = ws_at<int32_t>(ws, p.active);
    int32_t *nact = ws_at<int32_t>(ws, p.nact);
    int *err = ws_at<int>(ws, p.err);
    __half *x16 = ws_at<__half>(ws, p.x16);
    float *xinv = ws_at<float>(ws, p.xinv);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaError_t e = cudaLaunchKernelEx(&cfg, vq_gemm_tables_kernel, m0->E, expert, T, offsets, active, nact, err);
    if (e == cudaSuccess)
        e = launch_convert(x, x16, xinv, T, m0->cols, s, false);
    if (e != cudaSuccess)
        return VQ_ERR_CUDA;
    PrefillArgs a{};
    SmemPlan sp;
    if (const vq_status st = setup_gemm(a, m0, m1, x16, T, m0->E, sp); st != VQ_OK)
        return st;
    a.offsets = offsets;
    a.active = active;
    a.n_active = nact;
    a.out = y0;
    a.out2 = y1;
    a.swiglu = 0;
    a.sxinv = xinv;
    a.err = err;
    e = dispatch_gemm(a, a.mod[0].d, a.mod[0].bits, num_sms(), sp.total, s);
    return e == cudaSuccess ? VQ_OK : VQ_ERR_CUDA;
}

}  // namespace vq
