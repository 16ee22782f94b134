// Decode path of the VQ-MoE layer on sm_100a: a grouped GEMV that streams the
// packed codes and group scales of the experts that received tokens, decodes
// them in registers against a shared-memory codebook, and contracts them with
// the routed activations on the tensor cores (mma.sync m16n8k16, fp16 in,
// fp32 accumulate); plus the SwiGLU, combine and diagnostic kernels.
//
// Format (VQ model cards): Qwen3.5-397B-A17B-VQ-2.6bpw "Methodology" (index per
// d-weight subvector into an fp16 codebook, fp16 scale per (row, 64 weights));
// Qwen3.5-397B-A17B-VQ-2.4bpw "Methodology" (uint32 words, row-local 32-code
// blocks) and "Changelog 2026-10-01" (skipzero rows). The kernel design is
// this library's own: the cards only name their Apple-GPU kernels.
//
// Work decomposition of the grouped GEMV. A warp owns 32 weight rows (two
// m16 tiles) of one expert, one slice of the 64-column groups, and the
// expert's tokens eight at a time (the n8 dimension). Lane (g = lane/4,
// t = lane%4) of the warp holds rows g, g+8 of each tile and, in every
// 64-column group, the 16 columns [16t, 16t+16): the 16/d codes of those
// columns are one contiguous bit range of the row, so each lane loads and
// decodes its own codes. Inside a group the four k16 steps all lie in the
// group, so the tensor core sums exactly one scale group per step and the
// fp32 scale is applied once per group to the partial sums.
#include <algorithm>
#include <cmath>

#include "vq_device.cuh"
#include "vq_internal.h"
#include "vq_sm100.cuh"

namespace vq {
namespace {

// Words that hold QB bits starting at bit (j * QB) % 32 of a word, for the
// worst j (every lane quarter j of a row starts at bit j * QB).
__host__ __device__ constexpr int words_spanned(int qb)
{
    int w = 0;
    for (int j = 0; j < 32; ++j) {
        const int n = ((j * qb) % 32 + qb + 31) / 32;
        w = n > w ? n : w;
    }
    return w;
}

template <int D, int BITS>
struct Geo {
    static constexpr int CODES = 16 / D;               // codes of one lane in one group
    static constexpr int QB = CODES * BITS;            // their bits
    static constexpr bool ALIGNED = (QB % 32) == 0;    // their bit range starts on a word
    static constexpr int NW = (QB + 31) / 32;          // words once shifted down to bit 0
    static constexpr int LW = words_spanned(QB);       // words loaded from the row (at most NW + 1)
    static constexpr int EW = D <= 2 ? 1 : D / 2;      // shared-memory words per codebook entry
    static constexpr uint32_t MASK = (1u << BITS) - 1u;
    static constexpr int LOG_REP = codebook_log_rep(D, BITS);   // replicas per entry (log2)
    // code -> byte offset of its replica block: code << LSH (entries of 4 * EW bytes)
    static constexpr int LSH = LOG_REP + (EW == 1 ? 2 : EW == 2 ? 3 : 4);
};

// Load the words holding lane-quarter j (= 4*group + t) of a packed row.
template <int D, int BITS>
__device__ __forceinline__ void load_quarter(const uint32_t *row, long j, bool live,
                                             uint32_t (&w)[Geo<D, BITS>::LW], int &o)
{
    using G = Geo<D, BITS>;
    const long bit0 = j * G::QB;
    const uint32_t *p = row + (bit0 >> 5);
    o = (int)(bit0 & 31);
    if constexpr (G::ALIGNED && G::NW == 2) {
        uint2 v = make_uint2(0u, 0u);
        if (live)
            v = ldg_u64(p);
        w[0] = v.x;
        w[1] = v.y;
    } else if constexpr (G::ALIGNED) {
#pragma unroll
        for (int i = 0; i < G::LW; ++i)
            w[i] = live ? ldg_u32(p + i) : 0u;
    } else {
        const int need = (o + G::QB + 31) >> 5;
#pragma unroll
        for (int i = 0; i < G::LW; ++i)
            w[i] = (live && i < need) ? ldg_u32(p + i) : 0u;
    }
}

// The lane's CODES codes from the loaded words.
template <int D, int BITS>
__device__ __forceinline__ void extract_codes(const uint32_t (&w)[Geo<D, BITS>::LW], int o,
                                              uint32_t (&c)[Geo<D, BITS>::CODES])
{
    using G = Geo<D, BITS>;
    uint32_t n[G::NW];
#pragma unroll
    for (int i = 0; i < G::NW; ++i)
        n[i] = G::ALIGNED ? w[i] : __funnelshift_r(w[i], (!G::ALIGNED && i + 1 < G::LW) ? w[i + 1] : 0u, o);
#pragma unroll
    for (int k = 0; k < G::CODES; ++k) {
        const int p = k * BITS, wi = p >> 5, sh = p & 31;
        if (sh + BITS <= 32)
            c[k] = (n[wi] >> sh) & G::MASK;
        else
            c[k] = __funnelshift_r(n[wi], n[wi + 1], sh) & G::MASK;
    }
}

// The byte offsets (in the shared-memory codebook) of the lane's replica of
// each of its CODES codes: code k sits at bit o + k * BITS of the loaded
// words, and its offset (code << LSH) | rep_off takes one shift and one
// mask-or.
template <int D, int BITS>
__device__ __forceinline__ void code_offsets(const uint32_t (&w)[Geo<D, BITS>::LW], int o, uint32_t rep_off,
                                             uint32_t (&off)[Geo<D, BITS>::CODES])
{
    using G = Geo<D, BITS>;
    static_assert(BITS + G::LSH <= 32, "offsets fit 32 bits");
    uint32_t n[G::NW];
#pragma unroll
    for (int i = 0; i < G::NW; ++i)
        n[i] = G::ALIGNED ? w[i] : __funnelshift_r(w[i], (!G::ALIGNED && i + 1 < G::LW) ? w[i + 1] : 0u, o);
#pragma unroll
    for (int k = 0; k < G::CODES; ++k) {
        const int p = k * BITS, wi = p >> 5, sh = p & 31;
        uint32_t v;
        int at;   // bit of v where the code starts
        if (sh + BITS <= 32) {
            v = n[wi];
            at = sh;
        } else {
            v = __funnelshift_r(n[wi], n[wi + 1], sh);
            at = 0;
        }
        const uint32_t x = at >= G::LSH ? v >> (at - G::LSH) : v << (G::LSH - at);
        off[k] = (x & (G::MASK << G::LSH)) | rep_off;
    }
}

// a_words from byte offsets formed by code_offsets (d >= 2).
template <int D>
__device__ __forceinline__ void a_words_off(const char *cbb, const uint32_t *off, int s, uint32_t &lo, uint32_t &hi)
{
    if constexpr (D == 2) {
        lo = *reinterpret_cast<const uint32_t *>(cbb + off[2 * s]);
        hi = *reinterpret_cast<const uint32_t *>(cbb + off[2 * s + 1]);
    } else if constexpr (D == 4) {
        const uint2 v = *reinterpret_cast<const uint2 *>(cbb + off[s]);
        lo = v.x;
        hi = v.y;
    } else {
        const uint4 v = *reinterpret_cast<const uint4 *>(cbb + off[s >> 1]);
        lo = (s & 1) ? v.z : v.x;
        hi = (s & 1) ? v.w : v.y;
    }
}

// fp16x2 A-operand words of one row for k16 step s: lo covers k-slots
// (2t, 2t+1) = columns 16t+4s+{0,1} of the group, hi covers slots
// (2t+8, 2t+9) = columns 16t+4s+{2,3}.
template <int D>
__device__ __forceinline__ void a_words(const uint32_t *cbs, int log_rep, int rep, const uint32_t *c, int s,
                                        uint32_t &lo, uint32_t &hi)
{
    if constexpr (D == 1) {
        const uint32_t e0 = cbs[(c[4 * s + 0] << log_rep) | rep];
        const uint32_t e1 = cbs[(c[4 * s + 1] << log_rep) | rep];
        const uint32_t e2 = cbs[(c[4 * s + 2] << log_rep) | rep];
        const uint32_t e3 = cbs[(c[4 * s + 3] << log_rep) | rep];
        lo = (e0 & 0xFFFFu) | (e1 << 16);
        hi = (e2 & 0xFFFFu) | (e3 << 16);
    } else if constexpr (D == 2) {
        lo = cbs[(c[2 * s] << log_rep) | rep];
        hi = cbs[(c[2 * s + 1] << log_rep) | rep];
    } else if constexpr (D == 4) {
        const uint2 v = reinterpret_cast<const uint2 *>(cbs)[(c[s] << log_rep) | rep];
        lo = v.x;
        hi = v.y;
    } else {
        const uint4 v = reinterpret_cast<const uint4 *>(cbs)[(c[s >> 1] << log_rep) | rep];
        lo = (s & 1) ? v.z : v.x;
        hi = (s & 1) ? v.w : v.y;
    }
}

// Fill the shared-memory codebook: entry c replica r at slot (c << log_rep) | r.
// Lane l reads replica l & (rep-1), which spreads a warp's random lookups over
// distinct banks when rep is the full count (32 / 16 / 8 for 4 / 8 / 16-byte entries).
template <int D, int BITS>
__device__ __forceinline__ void fill_codebook(uint32_t *cbs, const uint16_t *codebook, int log_rep)
{
    const int n = (1 << BITS) << log_rep;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int c = i >> log_rep;
        if constexpr (D == 1)
            cbs[i] = codebook[c];
        else if constexpr (D == 2)
            cbs[i] = reinterpret_cast<const uint32_t *>(codebook)[c];
        else if constexpr (D == 4)
            reinterpret_cast<uint2 *>(cbs)[i] = reinterpret_cast<const uint2 *>(codebook)[c];
        else
            reinterpret_cast<uint4 *>(cbs)[i] = reinterpret_cast<const uint4 *>(codebook)[c];
    }
}

__device__ __forceinline__ void store_out(void *out, int dtype, long idx, float v)
{
    if (dtype == VQ_F32)
        reinterpret_cast<float *>(out)[idx] = v;
    else
        reinterpret_cast<uint16_t *>(out)[idx] = f32_to_bf16_bits(v);
}

// bf16 activations of one 64-column group, as lane (g, t) holds them: 16
// values of token g, columns [16t, 16t + 16) (the quad of lanes 4g..4g+3
// holds the token's group). They are converted to fp16 in place after a
// multiplication by 2^k, k putting the token's largest |x| in the group in
// [2^14, 2^15) (scale_exp), so every bf16 value keeps its precision and none
// overflows. f0 and f1 receive 2^-k of tokens 2t and 2t + 1, the columns of
// the lane's accumulator fragment, which undo the scale of the group's sums
// exactly. Every lane of the warp must call this.
__device__ __forceinline__ void scale_group_bf16(uint32_t (&bw)[8], float &f0, float &f1)
{
    uint32_t m = max(bf16x8_max_mag(make_uint4(bw[0], bw[1], bw[2], bw[3])),
                     bf16x8_max_mag(make_uint4(bw[4], bw[5], bw[6], bw[7])));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    const int k = scale_exp(m << 16);
    const float s = pow2f_normal(k);
#pragma unroll
    for (int i = 0; i < 8; ++i)
        bw[i] = bf16x2_to_f16x2_scaled(bw[i], s);
    const float inv = pow2f(-k);
    const int t = threadIdx.x & 3;
    f0 = __shfl_sync(0xFFFFFFFFu, inv, 8 * t);
    f1 = __shfl_sync(0xFFFFFFFFu, inv, 8 * t + 4);
}

constexpr int GEMV_THREADS = 256;
constexpr int GEMV_PD = 3;   // groups of loads in flight per warp

// d=2 with 8-bit codes: each codebook entry owns a 256-byte line holding 32
// per-lane replicas of module 0 (bytes 0..127) and of module 1 (128..255).
// A code byte then turns into its lane's smem address with one byte permute:
// offset = code * 256 + module * 128 + lane * 4, and a warp's 32 lookups hit
// 32 distinct banks.
template <int D, int BITS>
struct FastByteCodes {
    static constexpr bool value = (D == 2 && BITS == 8);
};

template <int D, int BITS>
__device__ __forceinline__ void fill_codebook_lines(uint32_t *cbs, const uint16_t *cb0, const uint16_t *cb1, int nmod)
{
    const int n = 256 * 64;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int c = i >> 6, m = (i >> 5) & 1;
        const uint16_t *cb = m ? cb1 : cb0;
        cbs[i] = (m < nmod) ? reinterpret_cast<const uint32_t *>(cb)[c] : 0u;
    }
}

// Loads of one 64-column group for one lane: the code words of its four rows
// and their fp16 scales (the activations, L1-resident, are read when used).
template <int D, int BITS>
struct GroupLoads {
    uint32_t cw[4][Geo<D, BITS>::LW];
    int co[4];
    uint16_t sv[4];
};

// fp16 1.0 in both halves: an A fragment of ones makes the MMA sum a group's activations.
constexpr uint32_t F16X2_ONES = 0x3C003C00u;

template <int D, int BITS, int PD>
__global__ void __launch_bounds__(GEMV_THREADS, 2) vq_grouped_gemv_kernel(const __grid_constant__ GemvArgs a)
{
    using G = Geo<D, BITS>;
    constexpr bool FAST = FastByteCodes<D, BITS>::value;
    extern __shared__ __align__(16) uint32_t cbs[];

    // modules per CTA: the fast layout holds both codebooks; otherwise blockIdx.y picks one
    const int cta_mods = FAST ? a.nmod : 1;
    if constexpr (FAST)
        fill_codebook_lines<D, BITS>(cbs, a.mod[0].codebook, a.mod[1].codebook, a.nmod);
    else
        fill_codebook<D, BITS>(cbs, (blockIdx.y == 0 ? a.mod[0] : a.mod[1]).codebook,
                               (blockIdx.y == 0 ? a.mod[0] : a.mod[1]).log_rep);
    __syncthreads();
    grid_dep_launch();   // the next kernel may start its prologue; it waits for this one's results
    grid_dep_wait();

    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int wpc = blockDim.x >> 5;
    const long gwarp = (long)blockIdx.x * wpc + (threadIdx.x >> 5);
    const long nwarps = (long)gridDim.x * wpc;

    const int n_act = a.offsets ? *a.n_active : 1;
    const ModDev m0 = FAST ? a.mod[0] : (blockIdx.y == 0 ? a.mod[0] : a.mod[1]);
    const int nblk = (m0.rows + 31) >> 5;
    const int S = a.slices;
    const long n_items = (long)n_act * nblk * S * cta_mods;

    for (long it = gwarp; it < n_items; it += nwarps) {
        long rest = it;
        const int slice = (int)(rest % S);
        rest /= S;
        const int blk = (int)(rest % nblk);
        rest /= nblk;
        const int mi = FAST ? (int)(rest % cta_mods) : (int)blockIdx.y;
        const int ai = FAST ? (int)(rest / cta_mods) : (int)rest;
        const ModDev &m = (mi == 0) ? a.mod[0] : a.mod[1];
        void *const out = (mi == 0) ? a.out[0] : a.out[1];
        const int rep = lane & (m.rep - 1);
        const uint32_t lane_sel = (uint32_t)(mi * 128 + lane * 4);

        const int e = a.offsets ? a.active[ai] : a.expert;
        const int q0 = a.offsets ? a.offsets[e] : 0;
        const int n = a.offsets ? a.offsets[e + 1] - q0 : a.T;

        // rows of this lane: i = 0,1 -> tile 0 rows g, g+8; i = 2,3 -> tile 1.
        // prow[i] = packed-row index, -1 for a dead row or a row past the end.
        int prow[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = blk * 32 + 8 * i + g;
            prow[i] = r < m.rows ? (int)live_row(m.bitmap, m.rank, m.bm_words, m.rows, e, r) : -1;
        }
        // slice s covers groups [s * ngroups / S, (s + 1) * ngroups / S) (possibly none)
        const int gbeg = (int)((long)slice * m.ngroups / S), gend = (int)((long)(slice + 1) * m.ngroups / S);

        for (int tok0 = 0; tok0 < n; tok0 += 8) {
            const bool has_tok = tok0 + g < n;
            const uint16_t *arow = nullptr;
            if (has_tok) {
                const int q = q0 + tok0 + g;
                const long ar = a.act_by_slot ? (long)q : (a.perm ? (long)(a.perm[q] / a.top_k) : (long)(tok0 + g));
                arow = reinterpret_cast<const uint16_t *>(a.act) + ar * (long)m.cols + 16 * t;
            }
            float acc[2][4];
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = 0.f;

            GroupLoads<D, BITS> st[PD];
            auto issue = [&](GroupLoads<D, BITS> &L, int grp) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const bool lv = prow[i] >= 0;
                    load_quarter<D, BITS>(m.codes + (long)prow[i] * m.row_words, 4L * grp + t, lv, L.cw[i], L.co[i]);
                    L.sv[i] = lv ? ldg_u16(m.scales + (long)prow[i] * m.ngroups + grp) : (uint16_t)0;
                }
            };
            auto compute = [&](const GroupLoads<D, BITS> &L, int grp) {
                uint4 av0 = make_uint4(0u, 0u, 0u, 0u), av1 = av0;
                if (has_tok) {
                    av0 = ldg_u128(arow + (long)grp * 64);
                    av1 = ldg_u128(arow + (long)grp * 64 + 8);
                }
                uint32_t bw[8] = {av0.x, av0.y, av0.z, av0.w, av1.x, av1.y, av1.z, av1.w};
                float f0 = 1.f, f1 = 1.f;   // inverse activation scales of the fragment's token columns
                if (a.act_bf16)
                    scale_group_bf16(bw, f0, f1);
                float tmp[2][4];
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tmp[i][j] = 0.f;
                if constexpr (FAST) {
                    const char *cbb = reinterpret_cast<const char *>(cbs);
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
#pragma unroll
                        for (int rt = 0; rt < 2; ++rt) {
                            uint32_t A[4];
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint32_t sel = 0x5504u | ((uint32_t)(2 * (s & 1) + h) << 4);
                                const uint32_t wlo = L.cw[2 * rt][s >> 1], whi = L.cw[2 * rt + 1][s >> 1];
                                A[2 * h] = *reinterpret_cast<const uint32_t *>(cbb + __byte_perm(wlo, lane_sel, sel));
                                A[2 * h + 1] = *reinterpret_cast<const uint32_t *>(cbb + __byte_perm(whi, lane_sel, sel));
                            }
                            mma_16816(tmp[rt], A, bw[2 * s], bw[2 * s + 1]);
                        }
                    }
                } else {
                    uint32_t c[4][G::CODES];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        extract_codes<D, BITS>(L.cw[i], L.co[i], c[i]);
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
#pragma unroll
                        for (int rt = 0; rt < 2; ++rt) {
                            uint32_t A[4];
                            a_words<D>(cbs, m.log_rep, rep, c[2 * rt], s, A[0], A[2]);
                            a_words<D>(cbs, m.log_rep, rep, c[2 * rt + 1], s, A[1], A[3]);
                            mma_16816(tmp[rt], A, bw[2 * s], bw[2 * s + 1]);
                        }
                    }
                }
                // affine arm: b * (the group's activation sum), the sum from one MMA against ones
                float xs[4] = {0.f, 0.f, 0.f, 0.f};
                if (m.biases) {
                    const uint32_t ones[4] = {F16X2_ONES, F16X2_ONES, F16X2_ONES, F16X2_ONES};
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_16816(xs, ones, bw[2 * s], bw[2 * s + 1]);
                    // (not prefetched with the codes: only biased modules pay for these loads)
                    float bv[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        bv[i] = prow[i] >= 0 ? f16_to_f32(ldg_u16(m.biases + (long)prow[i] * m.ngroups + grp)) : 0.f;
#pragma unroll
                    for (int rt = 0; rt < 2; ++rt) {
                        const float blo = bv[2 * rt], bhi = bv[2 * rt + 1];
                        acc[rt][0] = fmaf(blo * xs[0], f0, acc[rt][0]);
                        acc[rt][1] = fmaf(blo * xs[1], f1, acc[rt][1]);
                        acc[rt][2] = fmaf(bhi * xs[0], f0, acc[rt][2]);
                        acc[rt][3] = fmaf(bhi * xs[1], f1, acc[rt][3]);
                    }
                }
#pragma unroll
                for (int rt = 0; rt < 2; ++rt) {
                    const float slo = f16_to_f32(L.sv[2 * rt]);
                    const float shi = f16_to_f32(L.sv[2 * rt + 1]);
                    if (a.act_bf16) {   // (sum * scale) * 2^-k: the power of two is exact
                        acc[rt][0] = fmaf(tmp[rt][0] * slo, f0, acc[rt][0]);
                        acc[rt][1] = fmaf(tmp[rt][1] * slo, f1, acc[rt][1]);
                        acc[rt][2] = fmaf(tmp[rt][2] * shi, f0, acc[rt][2]);
                        acc[rt][3] = fmaf(tmp[rt][3] * shi, f1, acc[rt][3]);
                    } else {
                        acc[rt][0] = fmaf(tmp[rt][0], slo, acc[rt][0]);
                        acc[rt][1] = fmaf(tmp[rt][1], slo, acc[rt][1]);
                        acc[rt][2] = fmaf(tmp[rt][2], shi, acc[rt][2]);
                        acc[rt][3] = fmaf(tmp[rt][3], shi, acc[rt][3]);
                    }
                }
            };

            // ring of PD groups: loads of the next PD-1 groups are in flight
            // while one group is decoded and multiplied
#pragma unroll
            for (int s = 0; s < PD - 1; ++s)
                if (gbeg + s < gend)
                    issue(st[s], gbeg + s);
            for (int grp = gbeg; grp < gend; grp += PD) {
#pragma unroll
                for (int s = 0; s < PD; ++s) {
                    if (grp + s + PD - 1 < gend)
                        issue(st[(s + PD - 1) % PD], grp + s + PD - 1);
                    if (grp + s < gend)
                        compute(st[s], grp + s);
                }
            }

            // lane holds rows (g, g+8) of each tile for bucket tokens tok0 + 2t + {0, 1}
#pragma unroll
            for (int rt = 0; rt < 2; ++rt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int r = blk * 32 + 16 * rt + 8 * hf + g;
                    if (r >= m.rows)
                        continue;
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int tk = tok0 + 2 * t + cc;
                        if (tk >= n)
                            continue;
                        const float v = prow[2 * rt + hf] >= 0 ? acc[rt][2 * hf + cc] : 0.f;
                        store_out(out, a.out_dtype, (long)slice * a.out_slice_stride + (long)(q0 + tk) * m.rows + r, v);
                    }
                }
        }
    }
}

// ------------------------------------------------------------ TMA-fed grouped GEMV
//
// The same warp-level decomposition, with the packed codes, the group scales
// and the token tile's activations streamed by TMA through a ring of
// shared-memory stages of 256 weight rows x CG scale groups. A CTA has 16
// consumer warps in two halves and one producer warp whose lane 0 issues the
// stage's tensor loads. Consumer warp w takes rows [32 (w % 8), +32) of the
// stage (two m16 tiles, four rows per lane) and half w / 8 of its groups; the
// two halves' partial sums of a row tile meet in shared memory when a piece of
// work ends. (Measured: 8 warps of 64 rows are slower; 16 warps hide more
// latency at 96 registers per thread.) For d=2/8-bit codes a
// stage row is 128 bytes loaded with the 128-byte swizzle, and m16 row g of a
// warp is weight row sigma(g) (even rows in the first half-warp, odd rows in
// the second), so a warp's 8-byte code reads hit distinct banks. Each wait on
// a barrier is bounded.
//
// Work split. A work item is (token tile, module, 256-row block) and has
// spp = groups / CG stages. The stages of all items form one sequence that is
// cut into contiguous ranges of L stages, one per CTA, so every CTA streams
// about the same number of bytes whatever the number of items. An item cut
// between CTAs yields one partial sum per CTA (a piece), written to output
// slice (CTA - first CTA of the item); the CTA that holds the item's last
// stage writes zeros to the slices past its piece. L >= min_units bounds the
// pieces of an item by the slice count, and readers sum the slices in a fixed
// order, so results do not depend on timing.

constexpr int TG_HALVES = 2;                     // consumer warp sets splitting a stage's groups
constexpr int TG_RT = 2;                         // m16 row tiles per consumer warp
constexpr int TG_RL = 2 * TG_RT;                 // weight rows per lane
constexpr int TG_WROWS = 16 * TG_RT;             // weight rows per consumer warp
constexpr int TG_WPH = 8;                        // consumer warps per half
constexpr int TG_CONSUMERS = TG_HALVES * TG_WPH;
constexpr int TG_THREADS = 32 * (TG_CONSUMERS + 1);
constexpr int TG_ROWS = TG_WROWS * TG_WPH;
// per warp pair: 2 buffers of 4 * TG_RT floats per lane
constexpr int TG_XCHG_BYTES = TG_HALVES > 1 ? TG_WPH * 2 * (4 * TG_RT) * 32 * 4 : 0;
constexpr int TG_BAR_BYTES = 1024;

// Scale groups per stage: the codes of one row of a stage fill whole 16-byte
// units, and the count is even so the two halves get the same share.
__host__ __device__ constexpr int tg_stage_groups(int d, int bits)
{
    if (d == 2 && bits == 8)
        return 4;
    const int gb = (64 / d) * bits;   // bits of one row per group
    int cg = 1;
    while ((cg * gb) % 128)
        ++cg;
    return (cg % TG_HALVES) ? TG_HALVES * cg : cg;
}

template <int D, int BITS>
struct TGeo {
    static constexpr bool SWZ = (D == 2 && BITS == 8);
    static constexpr int CG = tg_stage_groups(D, BITS);
    static constexpr int HG = CG / TG_HALVES;       // groups of one half
    static constexpr int GB = (64 / D) * BITS;      // bits per row per group
    static constexpr int SRB = CG * GB / 8;         // bytes per row per stage
    static constexpr int ACOLS = CG * 64;           // activation columns per stage
    static constexpr int ACW = ACOLS < 256 ? ACOLS : 256;   // columns per activation box
    // a stage holds one 16-byte scale (and bias) box row per weight row: at most 8 groups
    static_assert(CG <= 8, "a stage's groups fit one 8-group scale box row");
    // the paired scale loads of a half read 2 * HG bytes at byte offsets that are multiples of their size
    static_assert(HG != 2 || CG % 2 == 0, "4-byte scale pairs stay aligned");
    static_assert(HG != 4 || CG % 8 == 0, "8-byte scale quads stay aligned");
};

struct GemvTmaArgs {
    CUtensorMap tmap[2];      // codes: u32 [live rows, row_words], box {SRB/4, 256}
    CUtensorMap tmap_sc[2];   // scales: fp16 [live rows, ngroups], box {8, 256}
    CUtensorMap tmap_bi[2];   // biases (affine arm), as the scales
    CUtensorMap tmap_act;     // activations: 16-bit [act rows, cols], box {ACW, 1}
    GemvArgs g;
    int ns;
    uint32_t stage_bytes, off_sc, off_bi, off_act;   // stage layout: codes | scales | [biases] | activations
    uint32_t off_stage, off_xchg, off_bar;
    int *err;
};

__device__ __forceinline__ int tg_sigma(int g) { return g < 4 ? 2 * g : 2 * (g - 4) + 1; }

__device__ __forceinline__ int tg_prow0(const ModDev &m, int e, int r0)
{
    if (!m.bitmap)
        return e * m.rows + r0;
    return (int)m.rank[(long)e * m.bm_words + (r0 >> 5)];
}

template <int D, int BITS>
__device__ __forceinline__ void tg_read_quarter(const uint8_t *row, int gq, int t, int br,
                                                uint32_t (&w)[Geo<D, BITS>::LW], int &o)
{
    using G = Geo<D, BITS>;
    using TG = TGeo<D, BITS>;
    if constexpr (TG::SWZ) {
        const int c = 2 * gq + (t >> 1);
        const uint2 v = *reinterpret_cast<const uint2 *>(row + (((c ^ (br & 7)) << 4) | ((t & 1) << 3)));
        w[0] = v.x;
        w[1] = v.y;
        o = 0;
    } else {
        const int off = (4 * gq + t) * G::QB;
        const uint32_t *p = reinterpret_cast<const uint32_t *>(row) + (off >> 5);
        o = off & 31;
        if constexpr (G::ALIGNED) {
#pragma unroll
            for (int i = 0; i < G::LW; ++i)
                w[i] = p[i];
        } else {
            const int need = (o + G::QB + 31) >> 5;
#pragma unroll
            for (int i = 0; i < G::LW; ++i)
                w[i] = i < need ? p[i] : 0u;
        }
    }
}

// One work item as both the producer and the consumers see it.
struct TgItem {
    int e;    // expert
    int q0;   // first output slot of the token tile (bucket slot, or token in single-expert mode)
    int n;    // tokens in the tile
    int mi;   // module
    int rb;   // 256-row block
};

// (32-bit index arithmetic: 64-bit division is a long instruction sequence)
__device__ __forceinline__ TgItem tg_item(const GemvArgs &a, long item, int nrb, int cta_mods, bool fast)
{
    TgItem r;
    const int it32 = (int)item;
    const int rest = it32 / nrb;
    r.rb = it32 - rest * nrb;
    r.mi = fast ? (cta_mods == 2 ? (rest & 1) : 0) : (int)blockIdx.y;
    const int tile = fast && cta_mods == 2 ? (rest >> 1) : rest;
    if (a.passes) {
        const int2 pt = a.passes[tile];
        r.e = pt.x & 0xFFFF;
        r.n = pt.x >> 16;
        r.q0 = pt.y;
    } else {
        r.e = a.expert;
        r.q0 = (int)tile * VQ_PASS_TOKENS;
        r.n = min(VQ_PASS_TOKENS, a.T - r.q0);
    }
    return r;
}

// ABF16: activations in bf16 (else fp16). DENSE: no module of the launch has a
// live bitmap. BIAS: the modules carry per-group biases (the affine arm): each
// group adds b * (its activation sum), the sum from one more MMA per k16 step
// against an A fragment of ones.
template <int D, int BITS, bool ABF16, bool DENSE, bool BIAS>
__global__ void __launch_bounds__(TG_THREADS, 1) vq_gemv_tma_kernel(const __grid_constant__ GemvTmaArgs A)
{
    using G = Geo<D, BITS>;
    using TG = TGeo<D, BITS>;
    constexpr bool FAST = FastByteCodes<D, BITS>::value;
    // groups decoded together by a warp: one when 16 consumer warps share the
    // register file (96 per thread), two with 8
    constexpr int GP = (TG_HALVES == 1 && TG::HG % 2 == 0) ? 2 : 1;
    const GemvArgs &a = A.g;
    extern __shared__ __align__(1024) uint8_t tg_smem_raw[];
    uint8_t *smem = tg_smem_raw;
    if (smem_u32(smem) & 1023u) {   // the 128-byte swizzle needs 1024-byte aligned stages
        if (threadIdx.x == 0 && A.err)
            atomicExch(A.err, 19);
        return;
    }
    uint32_t *cbs = reinterpret_cast<uint32_t *>(smem);
    uint8_t *stages = smem + A.off_stage;
    float *xchg = reinterpret_cast<float *>(smem + A.off_xchg);   // [pair][buffer][8][32]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + A.off_bar);
    uint64_t *empty = full + A.ns;
    uint64_t *xfull = empty + A.ns;          // [pair][buffer]: the second half's sums are in the buffer
    uint64_t *xempty = xfull + 2 * TG_WPH;   // [pair][buffer]: the first half has read the buffer
    volatile int *abort_flag = reinterpret_cast<volatile int *>(xempty + 2 * TG_WPH);

    const int cta_mods = FAST ? a.nmod : 1;
    if constexpr (FAST)
        fill_codebook_lines<D, BITS>(cbs, a.mod[0].codebook, a.mod[1].codebook, a.nmod);
    else
        fill_codebook<D, BITS>(cbs, (blockIdx.y == 0 ? a.mod[0] : a.mod[1]).codebook,
                               (blockIdx.y == 0 ? a.mod[0] : a.mod[1]).log_rep);
    if (threadIdx.x == 0) {
        for (int i = 0; i < A.ns; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], TG_CONSUMERS);
        }
        for (int i = 0; i < 2 * TG_WPH; ++i) {
            mbar_init(&xfull[i], 32);
            mbar_init(&xempty[i], 32);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    grid_dep_launch();   // the next kernel may start its prologue; it waits for this one's results
    grid_dep_wait();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const ModDev &m0 = FAST ? a.mod[0] : (blockIdx.y == 0 ? a.mod[0] : a.mod[1]);
    const int nrb = (m0.rows + TG_ROWS - 1) / TG_ROWS;
    const int spp = m0.ngroups / TG::CG;
    const long n_tiles = a.passes ? (long)*a.n_passes : (long)((a.T + VQ_PASS_TOKENS - 1) / VQ_PASS_TOKENS);
    const long U = n_tiles * cta_mods * nrb * spp;
    long L = (U + gridDim.x - 1) / gridDim.x;
    if (L < a.min_units)
        L = a.min_units;
    if (a.slices == 1)
        L = (L + spp - 1) / spp * spp;   // whole items only
    const long u0 = min(U, (long)blockIdx.x * L);
    const long u1 = min(U, u0 + L);
    const uint32_t stage_bytes_codes = (uint32_t)TG_ROWS * TG::SRB;

    if (warp == TG_CONSUMERS) {
        // ------------------------------------------------ producer: codes, scales and the
        // activation rows of the item's tokens for every stage, one barrier per stage
        if (lane == 0) {
            uint32_t k = 0, slot = 0, ph = 0;   // stages issued; ring slot and phase of stage k
            bool ok = true;
            TgItem it{};
            int prow0 = 0, mi = 0;
            int arow[VQ_PASS_TOKENS];
            uint32_t tx = 0;
            long item = u0 / spp;
            int j = (int)(u0 % spp);
            for (long u = u0; u < u1 && ok; ++u, j = (j + 1 == spp) ? 0 : j + 1, item += (j == 0)) {
                if (u == u0 || j == 0) {
                    it = tg_item(a, item, nrb, cta_mods, FAST);
                    mi = it.mi;
                    prow0 = tg_prow0(mi == 0 ? a.mod[0] : a.mod[1], it.e, it.rb * TG_ROWS);
                    for (int i = 0; i < it.n; ++i) {
                        const int q = it.q0 + i;
                        arow[i] = a.act_by_slot ? q : (a.perm ? a.perm[q] / a.top_k : q);
                    }
                    tx = stage_bytes_codes + (uint32_t)TG_ROWS * 16 * (BIAS ? 2 : 1) + (uint32_t)it.n * TG::ACOLS * 2;
                }
                if (!(ok = mbar_wait(&empty[slot], ph ^ 1, abort_flag, A.err, 11, a.wait_limit)))
                    break;
                uint8_t *sb = stages + (size_t)slot * A.stage_bytes;
                mbar_expect_tx(&full[slot], tx);
                const int g0 = j * TG::CG;
                tma_load_2d(sb, &A.tmap[mi], g0 * TG::GB / 32, prow0, &full[slot]);
                tma_load_2d(sb + A.off_sc, &A.tmap_sc[mi], g0 & ~7, prow0, &full[slot]);
                if constexpr (BIAS)
                    tma_load_2d(sb + A.off_bi, &A.tmap_bi[mi], g0 & ~7, prow0, &full[slot]);
                for (int i = 0; i < it.n; ++i)
                    for (int c = 0; c < TG::ACOLS; c += TG::ACW)
                        tma_load_2d(sb + A.off_act + (size_t)i * TG::ACOLS * 2 + c * 2, &A.tmap_act, g0 * 64 + c,
                                    arow[i], &full[slot]);
                ++k;
                if (++slot == (uint32_t)A.ns) {
                    slot = 0;
                    ph ^= 1;
                }
            }
            // after a give-up, the copies issued land before this thread leaves (the last use of each
            // slot). A normal end needs no wait: the consumers wait for every stage they read.
            if (!ok) {
                for (uint32_t s = 0; s < (uint32_t)A.ns && s < k; ++s) {
                    const uint32_t kk = k - 1 - s;
                    mbar_drain(&full[kk % A.ns], (kk / A.ns) & 1);
                }
            }
        }
        return;
    }

    // ---------------------------------------------------- consumers
    const int half = warp / TG_WPH, wr = warp % TG_WPH;
    const int g = lane >> 2, t = lane & 3;
    const int sg = tg_sigma(g);
    uint32_t slot = 0, ph = 0, xk = 0;   // stage ring; pieces exchanged by this warp pair
    bool ok = true;
    TgItem it{};
    int prow[TG_RL];
    // Row b of a stage holds the codes of packed row prow0 + b. Without a live
    // bitmap this lane's rows are b = 32 wr + 8 i + sigma(g), so one base and
    // immediates address all four; with one, each row has its own offsets
    // (a dead row reads row 0: its sums are never stored, so the inner loop
    // has no branches).
    const int bd = TG_WROWS * wr + sg;
    // 128-byte swizzled rows (d=2, 8-bit codes): 16-byte chunk c of row b sits at
    // chunk c ^ (b & 7); this lane reads chunk 2 gq + t/2, half t%2, and with the
    // group's bits kept apart that is koff ^ ((gq - first group of the half) << 5)
    const uint32_t koff = ((uint32_t)(((2 * half * TG::HG) | (t >> 1)) ^ sg) << 4) | ((uint32_t)(t & 1) << 3);
    uint32_t roff[TG_RL], soff[TG_RL];
    int swz[TG_RL];
#pragma unroll
    for (int i = 0; i < TG_RL; ++i) {
        roff[i] = (uint32_t)((bd + 8 * i) * TG::SRB);
        soff[i] = A.off_sc + (uint32_t)((bd + 8 * i) * 16);
        swz[i] = sg;
    }
    int rows = 0, rep = 0, log_rep = 0, r0 = 0;
    uint32_t lane_sel = 0, aoff = 0;
    // the lane's replica within an entry's block of replicas (d >= 2)
    const uint32_t rep_off = (uint32_t)(lane & ((1 << G::LOG_REP) - 1)) * (4 * G::EW);
    float acc[TG_RT][4];
    long item = u0 / spp;
    int j = (int)(u0 % spp);
    long u = u0;
    for (; u < u1 && ok; ++u, j = (j + 1 == spp) ? 0 : j + 1, item += (j == 0)) {
        if (u == u0 || j == 0) {
            it = tg_item(a, item, nrb, cta_mods, FAST);
            const ModDev &m = it.mi == 0 ? a.mod[0] : a.mod[1];
            rows = m.rows;
            rep = lane & (m.rep - 1);
            log_rep = m.log_rep;
            lane_sel = (uint32_t)(it.mi * 128 + lane * 4);
            r0 = it.rb * TG_ROWS;
            const int prow0 = tg_prow0(m, it.e, r0);
#pragma unroll
            for (int i = 0; i < TG_RL; ++i) {
                const int r = r0 + TG_WROWS * wr + 8 * i + sg;
                if constexpr (DENSE) {
                    prow[i] = r < rows ? 0 : -1;
                } else {
                    prow[i] = r < rows ? (int)live_row(m.bitmap, m.rank, m.bm_words, rows, it.e, r) : -1;
                    const int b = prow[i] >= 0 ? prow[i] - prow0 : 0;
                    roff[i] = (uint32_t)(b * TG::SRB);
                    soff[i] = A.off_sc + (uint32_t)(b * 16);
                    swz[i] = b & 7;
                }
            }
            // token g of the tile; lanes past the tile's count read token 0 (a broadcast,
            // no extra shared-memory traffic) and their output columns are never stored
            aoff = A.off_act + (uint32_t)((g < it.n ? g : 0) * TG::ACOLS * 2 + t * 32);
#pragma unroll
            for (int i = 0; i < TG_RT; ++i)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    acc[i][q] = 0.f;
        }

        if (!(ok = mbar_wait(&full[slot], ph, abort_flag, A.err, 13, a.wait_limit)))
            break;
        const uint8_t *sb = stages + (size_t)slot * A.stage_bytes;
        const uint8_t *ssc = sb + 2 * ((j * TG::CG) & 7);
        // with 2 or 4 groups per half, the fp16 scales of a row's groups in this half are adjacent:
        // one 4- or 8-byte load per row and stage (4- or 8-byte aligned: the scale box rows are 16 bytes
        // and a half starts at byte 2 * HG * half of the stage's groups)
        constexpr bool PAIR_SC = (TG::HG == 2 || TG::HG == 4) && GP == 1;
        uint2 sc2[TG_RL];
        if constexpr (PAIR_SC) {
#pragma unroll
            for (int i = 0; i < TG_RL; ++i) {
                const uint8_t *p = ssc + (DENSE ? soff[0] + i * 8 * 16 : soff[i]) + 2 * half * TG::HG;
                if constexpr (TG::HG == 2)
                    sc2[i] = make_uint2(*reinterpret_cast<const uint32_t *>(p), 0u);
                else
                    sc2[i] = *reinterpret_cast<const uint2 *>(p);
            }
        }
#pragma unroll
        for (int gh = 0; gh < TG::HG; gh += GP) {
            uint32_t cw[GP][TG_RL][G::LW];
            int co[GP];
            float sv[GP][TG_RL];
            uint32_t bw[GP][8];
            float fa[GP][2];   // bf16 activations: inverse scales of the fragment's token columns
            float bvv[BIAS ? TG_RL : 1];   // biases of the lane's rows (GP == 1 with them)
#pragma unroll
            for (int uu = 0; uu < GP; ++uu) {
                const int gq = half * TG::HG + gh + uu;   // group within the stage
                co[uu] = 0;
                if constexpr (TG::SWZ && DENSE) {
                    // rows bd + 8i share the swizzle key sigma(g): one offset, then immediates
                    const uint8_t *p = sb + roff[0] + (koff ^ (uint32_t)((gq - half * TG::HG) << 5));
#pragma unroll
                    for (int i = 0; i < TG_RL; ++i) {
                        const uint2 v = *reinterpret_cast<const uint2 *>(p + i * 8 * TG::SRB);
                        cw[uu][i][0] = v.x;
                        cw[uu][i][1] = v.y;
                    }
                } else if constexpr (TG::SWZ) {
                    const int c = 2 * gq + (t >> 1);
#pragma unroll
                    for (int i = 0; i < TG_RL; ++i) {
                        const uint2 v = *reinterpret_cast<const uint2 *>(
                            sb + roff[i] + ((uint32_t)((c ^ swz[i]) << 4) | ((uint32_t)(t & 1) << 3)));
                        cw[uu][i][0] = v.x;
                        cw[uu][i][1] = v.y;
                    }
                } else if constexpr (DENSE) {
                    const int bit = (4 * gq + t) * G::QB;
                    co[uu] = bit & 31;
                    const uint32_t *p = reinterpret_cast<const uint32_t *>(sb + roff[0]) + (bit >> 5);
#pragma unroll
                    for (int i = 0; i < TG_RL; ++i)
#pragma unroll
                        for (int q = 0; q < G::LW; ++q)
                            cw[uu][i][q] = p[i * 8 * TG::SRB / 4 + q];
                } else {
                    // the lane's bit range [bit, bit + QB) of the row; reading LW words may take
                    // one word past it (still inside the stage), whose bits are masked off
                    const int bit = (4 * gq + t) * G::QB;
                    co[uu] = bit & 31;
#pragma unroll
                    for (int i = 0; i < TG_RL; ++i) {
                        const uint32_t *p = reinterpret_cast<const uint32_t *>(sb + roff[i]) + (bit >> 5);
#pragma unroll
                        for (int q = 0; q < G::LW; ++q)
                            cw[uu][i][q] = p[q];
                    }
                }
                if constexpr (PAIR_SC) {
#pragma unroll
                    for (int i = 0; i < TG_RL; ++i) {
                        const uint32_t wv = gh < 2 ? sc2[i].x : sc2[i].y;
                        sv[uu][i] = f16_to_f32((uint16_t)((gh & 1) ? wv >> 16 : wv));
                    }
                } else if constexpr (DENSE) {
                    const uint8_t *p = ssc + soff[0] + 2 * gq;
#pragma unroll
                    for (int i = 0; i < TG_RL; ++i)
                        sv[uu][i] = f16_to_f32(*reinterpret_cast<const uint16_t *>(p + i * 8 * 16));
                } else {
#pragma unroll
                    for (int i = 0; i < TG_RL; ++i)
                        sv[uu][i] = f16_to_f32(*reinterpret_cast<const uint16_t *>(ssc + soff[i] + 2 * gq));
                }
                if constexpr (BIAS) {
                    const uint8_t *bb = sb + (A.off_bi - A.off_sc) + 2 * ((j * TG::CG) & 7) + 2 * gq;
#pragma unroll
                    for (int i = 0; i < TG_RL; ++i)
                        bvv[i] = f16_to_f32(*reinterpret_cast<const uint16_t *>(
                            bb + (DENSE ? soff[0] + i * 8 * 16 : soff[i])));
                }
                const uint4 v0 = *reinterpret_cast<const uint4 *>(sb + aoff + gq * 128);
                const uint4 v1 = *reinterpret_cast<const uint4 *>(sb + aoff + gq * 128 + 16);
                bw[uu][0] = v0.x; bw[uu][1] = v0.y; bw[uu][2] = v0.z; bw[uu][3] = v0.w;
                bw[uu][4] = v1.x; bw[uu][5] = v1.y; bw[uu][6] = v1.z; bw[uu][7] = v1.w;
                if constexpr (ABF16)
                    scale_group_bf16(bw[uu], fa[uu][0], fa[uu][1]);
            }
            if (gh + GP >= TG::HG) {   // every read of this stage by the warp is done
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[slot]);
            }
            // codes (d=1) or their codebook byte offsets (d >= 2)
            uint32_t c[GP][TG_RL][G::CODES];
            if constexpr (!FAST) {
#pragma unroll
                for (int uu = 0; uu < GP; ++uu)
#pragma unroll
                    for (int i = 0; i < TG_RL; ++i) {
                        if constexpr (D == 1)
                            extract_codes<D, BITS>(cw[uu][i], co[uu], c[uu][i]);
                        else
                            code_offsets<D, BITS>(cw[uu][i], co[uu], rep_off, c[uu][i]);
                    }
            }
            float tmp[GP][TG_RT][4];
#pragma unroll
            for (int uu = 0; uu < GP; ++uu)
#pragma unroll
                for (int i = 0; i < TG_RT; ++i)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        tmp[uu][i][q] = 0.f;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
#pragma unroll
                for (int uu = 0; uu < GP; ++uu) {
#pragma unroll
                    for (int rt = 0; rt < TG_RT; ++rt) {
                        uint32_t Aw[4];
                        if constexpr (FAST) {
                            const char *cbb = reinterpret_cast<const char *>(cbs);
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint32_t sel = 0x5504u | ((uint32_t)(2 * (s & 1) + h) << 4);
                                Aw[2 * h] = *reinterpret_cast<const uint32_t *>(
                                    cbb + __byte_perm(cw[uu][2 * rt][s >> 1], lane_sel, sel));
                                Aw[2 * h + 1] = *reinterpret_cast<const uint32_t *>(
                                    cbb + __byte_perm(cw[uu][2 * rt + 1][s >> 1], lane_sel, sel));
                            }
                        } else if constexpr (D == 1) {
                            a_words<D>(cbs, log_rep, rep, c[uu][2 * rt], s, Aw[0], Aw[2]);
                            a_words<D>(cbs, log_rep, rep, c[uu][2 * rt + 1], s, Aw[1], Aw[3]);
                        } else {
                            const char *cbb = reinterpret_cast<const char *>(cbs);
                            a_words_off<D>(cbb, c[uu][2 * rt], s, Aw[0], Aw[2]);
                            a_words_off<D>(cbb, c[uu][2 * rt + 1], s, Aw[1], Aw[3]);
                        }
                        mma_16816(tmp[uu][rt], Aw, bw[uu][2 * s], bw[uu][2 * s + 1]);
                    }
                }
            }
            if constexpr (BIAS) {
                // b * (the group's activation sum of tokens 2t, 2t + 1), the sums from an MMA against ones
                static_assert(GP == 1, "biases with one group per warp step");
                float xs[4] = {0.f, 0.f, 0.f, 0.f};
                const uint32_t ones[4] = {F16X2_ONES, F16X2_ONES, F16X2_ONES, F16X2_ONES};
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_16816(xs, ones, bw[0][2 * s], bw[0][2 * s + 1]);
                const float x0 = ABF16 ? xs[0] * fa[0][0] : xs[0], x1 = ABF16 ? xs[1] * fa[0][1] : xs[1];
#pragma unroll
                for (int rt = 0; rt < TG_RT; ++rt) {
                    acc[rt][0] = fmaf(bvv[2 * rt], x0, acc[rt][0]);
                    acc[rt][1] = fmaf(bvv[2 * rt], x1, acc[rt][1]);
                    acc[rt][2] = fmaf(bvv[2 * rt + 1], x0, acc[rt][2]);
                    acc[rt][3] = fmaf(bvv[2 * rt + 1], x1, acc[rt][3]);
                }
            }
#pragma unroll
            for (int uu = 0; uu < GP; ++uu)
#pragma unroll
                for (int rt = 0; rt < TG_RT; ++rt) {
                    const float slo = sv[uu][2 * rt], shi = sv[uu][2 * rt + 1];
                    if constexpr (ABF16) {   // (sum * scale) * 2^-k: the power of two is exact
                        acc[rt][0] = fmaf(tmp[uu][rt][0] * slo, fa[uu][0], acc[rt][0]);
                        acc[rt][1] = fmaf(tmp[uu][rt][1] * slo, fa[uu][1], acc[rt][1]);
                        acc[rt][2] = fmaf(tmp[uu][rt][2] * shi, fa[uu][0], acc[rt][2]);
                        acc[rt][3] = fmaf(tmp[uu][rt][3] * shi, fa[uu][1], acc[rt][3]);
                    } else {
                        acc[rt][0] = fmaf(tmp[uu][rt][0], slo, acc[rt][0]);
                        acc[rt][1] = fmaf(tmp[uu][rt][1], slo, acc[rt][1]);
                        acc[rt][2] = fmaf(tmp[uu][rt][2], shi, acc[rt][2]);
                        acc[rt][3] = fmaf(tmp[uu][rt][3], shi, acc[rt][3]);
                    }
                }
        }
        if (++slot == (uint32_t)A.ns) {
            slot = 0;
            ph ^= 1;
        }

        if (j != spp - 1 && u != u1 - 1)
            continue;
        // ------------------------------------------------ end of a piece: the second half hands its
        // sums to the first through a 2-buffer ring per warp pair; the first half adds them (always in
        // this order) and stores the piece
        const int xb = (int)(xk & 1);
        const uint32_t xph = (xk >> 1) & 1;
        ++xk;
        float *xs = xchg + (size_t)(wr * 2 + xb) * (4 * TG_RT) * 32;
        if (TG_HALVES == 1) {
            // one warp set: the sums are complete
        } else if (half == 1) {
            if (!(ok = mbar_wait(&xempty[wr * 2 + xb], xph ^ 1, abort_flag, A.err, 14, a.wait_limit)))
                break;
#pragma unroll
            for (int v = 0; v < 4 * TG_RT; ++v)
                xs[v * 32 + lane] = acc[v >> 2][v & 3];
            mbar_arrive(&xfull[wr * 2 + xb]);
            continue;
        } else {
            if (!(ok = mbar_wait(&xfull[wr * 2 + xb], xph, abort_flag, A.err, 15, a.wait_limit)))
                break;
#pragma unroll
            for (int v = 0; v < 4 * TG_RT; ++v)
                acc[v >> 2][v & 3] += xs[v * 32 + lane];
            mbar_arrive(&xempty[wr * 2 + xb]);
        }

        void *const out = it.mi == 0 ? a.out[0] : a.out[1];
        const int piece = (int)blockIdx.x - (int)item * spp / (int)L;
        // zeros past the item's last piece, unless the routing launch cleared those slices
        const int last = (j == spp - 1 && !a.slices_zeroed) ? a.slices : piece + 1;
        // lane holds rows r0 + 32 wr + 8 i + sigma(g) for tile tokens 2t + {0, 1}
#pragma unroll
        for (int rt = 0; rt < TG_RT; ++rt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int i = 2 * rt + hf;
                const int r = r0 + TG_WROWS * wr + 8 * i + tg_sigma(g);
                if (r >= rows)
                    continue;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int tk = 2 * t + cc;
                    if (tk >= it.n)
                        continue;
                    const float v = prow[i] >= 0 ? acc[rt][2 * hf + cc] : 0.f;
                    const long o = (long)(it.q0 + tk) * rows + r;
                    store_out(out, a.out_dtype, (long)piece * a.out_slice_stride + o, v);
                    for (int sl = piece + 1; sl < last; ++sl)
                        store_out(out, a.out_dtype, (long)sl * a.out_slice_stride + o, 0.f);
                }
            }
    }
    if (!ok) {
        // a give-up: the producer may have copied up to ns stages past the one this warp stopped at and
        // left already; they land before the CTA can exit. A stage never issued gives up after a short
        // bound (the producer, if still running, drains its own copies when it sees the abort).
        for (int s = 0; s < A.ns && u + s < u1; ++s) {
            const uint32_t sl = (slot + (uint32_t)s) % (uint32_t)A.ns;
            const uint32_t p = (slot + (uint32_t)s) >= (uint32_t)A.ns ? (ph ^ 1u) : ph;
            for (uint32_t i = 0; i < (1u << 14); ++i)
                if (mbar_try_wait(&full[sl], p))
                    break;
        }
    }
}

// ------------------------------------------------------------ SwiGLU and combine

// SwiGLU of bucket slot q. The GEMVs read the slot's token t = perm[q] / top_k
// scaled by 2^k_t, so g = xinv[t] * sum_s G[s, q, :] and u = xinv[t] *
// sum_s U[s, q, :] (xinv[t] = 2^-k_t, exact), with the slices summed in order;
// h = silu(g) * u in fp32. The down GEMV takes h as an fp16 operand, so the
// slot's row is stored as hs[q, :] = fp16(h * 2^e_q), e_q putting the slot's
// largest |h| in [2^14, 2^15) (scale_exp): no overflow for any finite h and
// fp16's full precision for the values that matter. The inverse scale goes
// into the routing weight of the slot's pair p = perm[q]: wh[p] = w[p] *
// 2^-e_q (exact), which the combine applies to the down projection. One block
// per slot (grid-stride); up to 8 elements per thread stay in registers
// between the row's maximum and the stores (longer rows are computed again,
// with the same arithmetic). S > 0: the slice count is a compile-time
// constant, so every load of an element is issued before the first add;
// S == 0: any count.
constexpr int SWIGLU_THREADS = 256;
constexpr int SWIGLU_KEEP = 8;

template <int S>
__global__ void __launch_bounds__(SWIGLU_THREADS) vq_swiglu_kernel(
    const float *__restrict__ G, const float *__restrict__ U, int slices, long slice_stride, int slots, int inter,
    const int32_t *__restrict__ perm, int top_k, const float *__restrict__ xinv, const float *__restrict__ w,
    __half *__restrict__ h, float *__restrict__ wh)
{
    __shared__ uint32_t red[SWIGLU_THREADS / 32];
    grid_dep_launch();   // the next kernel may start its prologue; it waits for this one's results
    grid_dep_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int q = blockIdx.x; q < slots; q += gridDim.x) {
        const int p = perm[q];
        const float f = xinv[p / top_k];
        const long row = (long)q * inter;
        auto h_at = [&](int c) {
            float gs = 0.f, us = 0.f;
            if constexpr (S > 0) {
                float gv[S], uv[S];
#pragma unroll
                for (int i = 0; i < S; ++i) {
                    gv[i] = G[i * slice_stride + row + c];
                    uv[i] = U[i * slice_stride + row + c];
                }
#pragma unroll
                for (int i = 0; i < S; ++i) {
                    gs += gv[i];
                    us += uv[i];
                }
            } else {
                for (int i = 0; i < slices; ++i) {
                    gs += G[i * slice_stride + row + c];
                    us += U[i * slice_stride + row + c];
                }
            }
            const float g = gs * f, u = us * f;
            return __fdividef(g, 1.f + __expf(-g)) * u;
        };
        float hv[SWIGLU_KEEP];
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < SWIGLU_KEEP; ++i) {
            const int c = threadIdx.x + i * SWIGLU_THREADS;
            hv[i] = c < inter ? h_at(c) : 0.f;
            m = max(m, __float_as_uint(hv[i]) & 0x7FFFFFFFu);
        }
        for (int c = threadIdx.x + SWIGLU_KEEP * SWIGLU_THREADS; c < inter; c += SWIGLU_THREADS)
            m = max(m, __float_as_uint(h_at(c)) & 0x7FFFFFFFu);
        m = __reduce_max_sync(0xFFFFFFFFu, m);
        if (lane == 0)
            red[warp] = m;
        __syncthreads();
        m = red[0];
#pragma unroll
        for (int i = 1; i < SWIGLU_THREADS / 32; ++i)
            m = max(m, red[i]);
        const int e = scale_exp(m);
        const float sc = pow2f_normal(e);
        if (threadIdx.x == 0)
            wh[p] = w[p] * pow2f(-e);
#pragma unroll
        for (int i = 0; i < SWIGLU_KEEP; ++i) {
            const int c = threadIdx.x + i * SWIGLU_THREADS;
            if (c < inter)
                h[row + c] = __float2half_rn(hv[i] * sc);
        }
        for (int c = threadIdx.x + SWIGLU_KEEP * SWIGLU_THREADS; c < inter; c += SWIGLU_THREADS)
            h[row + c] = __float2half_rn(h_at(c) * sc);
        __syncthreads();   // red is reused by the next slot
    }
}

// y[t, :] = sum_j w[t, j] * sum_s D[s, pos[t*k + j], :], slots in order j and
// slices in order s (w carries the inverse of the power-of-two scale of the
// pair's down-projection operand); a block per token (and column range), four
// columns per thread. The loads of 8 slots x S slices are issued before any
// is used.
template <int S>
__global__ void __launch_bounds__(256) vq_combine_kernel(const float *__restrict__ D, int slices, long slice_stride,
                                                         const float *__restrict__ w, const int32_t *__restrict__ pos,
                                                         int T, int k, int hidden, void *y, int y_dtype)
{
    __shared__ long q_s[32];
    __shared__ float w_s[32];
    grid_dep_launch();   // the next kernel may start its prologue; it waits for this one's results
    grid_dep_wait();
    const int h4 = hidden >> 2;
    for (int tok = blockIdx.x; tok < T; tok += gridDim.x) {
        __syncthreads();   // q_s / w_s of the previous token are no longer read
        if (threadIdx.x < k) {
            q_s[threadIdx.x] = (long)pos[(long)tok * k + threadIdx.x] * hidden;
            w_s[threadIdx.x] = w[(long)tok * k + threadIdx.x];
        }
        __syncthreads();
        for (int c4 = blockIdx.y * blockDim.x + threadIdx.x; c4 < h4; c4 += gridDim.y * blockDim.x) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if constexpr (S == 0) {   // any slice count
                for (int j = 0; j < k; ++j) {
                    float4 part = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int q = 0; q < slices; ++q) {
                        const float4 v = reinterpret_cast<const float4 *>(D + q * slice_stride + q_s[j])[c4];
                        part.x += v.x;
                        part.y += v.y;
                        part.z += v.z;
                        part.w += v.w;
                    }
                    const float wj = w_s[j];
                    acc.x = fmaf(wj, part.x, acc.x);
                    acc.y = fmaf(wj, part.y, acc.y);
                    acc.z = fmaf(wj, part.z, acc.z);
                    acc.w = fmaf(wj, part.w, acc.w);
                }
            }
            for (int j0 = 0; S > 0 && j0 < k; j0 += 8) {
                float4 v[8][S > 0 ? S : 1];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
#pragma unroll
                    for (int q = 0; q < S; ++q)
                        v[jj][q] = j0 + jj < k ? reinterpret_cast<const float4 *>(D + q * slice_stride + q_s[j0 + jj])[c4]
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    if (j0 + jj >= k)
                        break;
                    // 0 + v[0] as in the slice-loop form (turns a -0 sum into +0)
                    float4 part = make_float4(0.f + v[jj][0].x, 0.f + v[jj][0].y, 0.f + v[jj][0].z, 0.f + v[jj][0].w);
#pragma unroll
                    for (int q = 1; q < S; ++q) {
                        part.x += v[jj][q].x;
                        part.y += v[jj][q].y;
                        part.z += v[jj][q].z;
                        part.w += v[jj][q].w;
                    }
                    const float wj = w_s[j0 + jj];
                    acc.x = fmaf(wj, part.x, acc.x);
                    acc.y = fmaf(wj, part.y, acc.y);
                    acc.z = fmaf(wj, part.z, acc.z);
                    acc.w = fmaf(wj, part.w, acc.w);
                }
            }
            const long o = (long)tok * hidden + 4 * c4;
            if (y_dtype == VQ_F32) {
                *reinterpret_cast<float4 *>(reinterpret_cast<float *>(y) + o) = acc;
            } else {
                const uint2 b = make_uint2((uint32_t)f32_to_bf16_bits(acc.x) | ((uint32_t)f32_to_bf16_bits(acc.y) << 16),
                                           (uint32_t)f32_to_bf16_bits(acc.z) | ((uint32_t)f32_to_bf16_bits(acc.w) << 16));
                *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(y) + o) = b;
            }
        }
    }
}

// ------------------------------------------------------------ diagnostics

__global__ void vq_unpack_kernel(const ModDev m, int e, uint16_t *out)
{
    const int ncode = m.cols / m.d;
    const long n = (long)m.rows * ncode;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const int r = (int)(i / ncode), j = (int)(i % ncode);
        const long pr = live_row(m.bitmap, m.rank, m.bm_words, m.rows, e, r);
        if (pr < 0) {
            out[i] = 0xFFFF;
            continue;
        }
        const uint32_t *row = m.codes + pr * m.row_words;
        const long bit = (long)j * m.bits;
        const long wi = bit >> 5;
        const uint32_t lo = row[wi];
        const uint32_t hi = (wi + 1 < m.row_words) ? row[wi + 1] : 0u;
        out[i] = (uint16_t)(__funnelshift_r(lo, hi, (uint32_t)(bit & 31)) & ((1u << m.bits) - 1u));
    }
}

__global__ void vq_dequant_kernel(const ModDev m, int e, float *out)
{
    const long n = (long)m.rows * m.cols;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const int r = (int)(i / m.cols), c = (int)(i % m.cols);
        const long pr = live_row(m.bitmap, m.rank, m.bm_words, m.rows, e, r);
        if (pr < 0) {
            out[i] = 0.f;
            continue;
        }
        const uint32_t *row = m.codes + pr * m.row_words;
        const long bit = (long)(c / m.d) * m.bits;
        const long wi = bit >> 5;
        const uint32_t lo = row[wi];
        const uint32_t hi = (wi + 1 < m.row_words) ? row[wi + 1] : 0u;
        const uint32_t code = __funnelshift_r(lo, hi, (uint32_t)(bit & 31)) & ((1u << m.bits) - 1u);
        const float centroid = f16_to_f32(m.codebook[(long)code * m.d + c % m.d]);
        const float scale = f16_to_f32(m.scales[pr * m.ngroups + c / 64]);
        out[i] = centroid * scale;   // exact: two fp16 factors
    }
}

// ------------------------------------------------------------ launch helpers

template <typename K, typename... Args>
cudaError_t launch(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int D, int BITS>
cudaError_t gemv_dispatch(const GemvArgs &a, cudaStream_t s, bool pdl)
{
    auto k = vq_grouped_gemv_kernel<D, BITS, GEMV_PD>;
    cudaError_t err = set_smem_limit_once((const void *)k, 227 * 1024);
    if (err != cudaSuccess)
        return err;
    const size_t smem = gemv_smem_bytes(a.mod[0]);
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, GEMV_THREADS, smem) != cudaSuccess || occ < 1)
        occ = 1;
    const bool both = FastByteCodes<D, BITS>::value;
    const int gy = both ? 1 : a.nmod;
    const int ctas = std::max(1, num_sms() * occ / gy);
    return launch(k, dim3(ctas, gy), dim3(GEMV_THREADS), smem, s, pdl, a);
}

struct TgPlan {
    int ns;
    uint32_t stage, off_sc, off_bi, off_act, off_stage, off_xchg, off_bar, total;
};

// Shared-memory layout of the TMA kernel for a module's geometry (with the bias
// box in each stage when the module has biases).
TgPlan tg_plan(const ModDev &m)
{
    TgPlan p{};
    const uint32_t cb = (uint32_t)align_up(gemv_smem_bytes(m), 1024);
    const int cg = tg_stage_groups(m.d, m.bits);
    const uint32_t codes = (uint32_t)TG_ROWS * (uint32_t)(cg * (64 / m.d) * m.bits / 8);
    p.off_sc = codes;
    p.off_bi = codes + (uint32_t)TG_ROWS * 16;
    p.off_act = p.off_bi + (m.biases ? (uint32_t)TG_ROWS * 16 : 0u);
    p.stage = (uint32_t)align_up(p.off_act + (uint32_t)VQ_PASS_TOKENS * cg * 64 * 2, 1024);
    const uint32_t limit = 227 * 1024 - 1024;   // opt-in maximum less the alignment slack
    const uint32_t fixed = cb + TG_XCHG_BYTES + TG_BAR_BYTES;
    p.ns = limit > fixed ? (int)std::min<uint32_t>(8, (limit - fixed) / p.stage) : 0;
    p.off_stage = cb;
    p.off_xchg = cb + p.ns * p.stage;
    p.off_bar = p.off_xchg + TG_XCHG_BYTES;
    p.total = p.off_bar + TG_BAR_BYTES + 1024;
    return p;
}

// The TMA kernel takes the module: 16-byte packed rows, 8-group scale rows,
// whole stages per row and at least two stages in shared memory. d = 8
// modules run on the register-prefetch kernel: under a repeatability stress
// (the 2048-token skipzero layer's d = 8 down projection, decoded again and
// again) the TMA kernel returned, in about one call in eight, wrong sums for
// a few rows of its first warp pair; the cause is not found.
bool tg_ok(const ModDev &m)
{
    const int cg = tg_stage_groups(m.d, m.bits);
    return m.d != 8 && tma_available() && m.row_words % 4 == 0 && m.ngroups % 8 == 0 && m.ngroups % cg == 0 &&
           tg_plan(m).ns >= 2;
}

template <int D, int BITS>
cudaError_t gemv_tma_dispatch(const GemvArgs &a, cudaStream_t s, bool pdl)
{
    using TG = TGeo<D, BITS>;
    GemvTmaArgs A{};
    A.g = a;
    for (int i = 0; i < a.nmod; ++i) {
        const ModDev &m = a.mod[i];
        if (!tma_map_2d(&A.tmap[i], CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, m.codes, (uint64_t)m.row_words,
                        (uint64_t)m.live_rows, (uint32_t)(TG::SRB / 4), (uint32_t)TG_ROWS,
                        TG::SWZ ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    const bool bias = a.mod[0].biases != nullptr;   // the modules of a launch agree (plan_decode)
    for (int i = 0; i < a.nmod; ++i) {
        const ModDev &m = a.mod[i];
        if (!tma_map_2d(&A.tmap_sc[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, m.scales, (uint64_t)m.ngroups,
                        (uint64_t)m.live_rows, 8, (uint32_t)TG_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
        if (bias && !tma_map_2d(&A.tmap_bi[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, m.biases, (uint64_t)m.ngroups,
                                (uint64_t)m.live_rows, 8, (uint32_t)TG_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    if (!tma_map_2d(&A.tmap_act, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, a.act, (uint64_t)a.mod[0].cols,
                    (uint64_t)a.act_rows, (uint32_t)TG::ACW, 1, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (a.nmod == 1) {
        A.tmap[1] = A.tmap[0];
        A.tmap_sc[1] = A.tmap_sc[0];
        A.tmap_bi[1] = A.tmap_bi[0];
    }
    const TgPlan p = tg_plan(a.mod[0]);
    A.ns = p.ns;
    A.stage_bytes = p.stage;
    A.off_sc = p.off_sc;
    A.off_bi = p.off_bi;
    A.off_act = p.off_act;
    A.off_stage = p.off_stage;
    A.off_xchg = p.off_xchg;
    A.off_bar = p.off_bar;
    A.err = a.err;
    bool dense = true;
    for (int i = 0; i < a.nmod; ++i)
        dense = dense && !a.mod[i].bitmap;
    using KFn = void (*)(const GemvTmaArgs);
    const KFn kernels[2][2][2] = {
        {{vq_gemv_tma_kernel<D, BITS, false, false, false>, vq_gemv_tma_kernel<D, BITS, false, false, true>},
         {vq_gemv_tma_kernel<D, BITS, false, true, false>, vq_gemv_tma_kernel<D, BITS, false, true, true>}},
        {{vq_gemv_tma_kernel<D, BITS, true, false, false>, vq_gemv_tma_kernel<D, BITS, true, false, true>},
         {vq_gemv_tma_kernel<D, BITS, true, true, false>, vq_gemv_tma_kernel<D, BITS, true, true, true>}}};
    const KFn k = kernels[a.act_bf16 ? 1 : 0][dense ? 1 : 0][bias ? 1 : 0];
    // the layout of every module of a geometry is the same, so its size is fixed per kernel
    cudaError_t err = set_smem_limit_once((const void *)k, (int)p.total);
    if (err != cudaSuccess)
        return err;
    const bool both = FastByteCodes<D, BITS>::value;
    const int gy = both ? 1 : a.nmod;
    const int ctas = std::max(1, num_sms() / gy);
    return launch(k, dim3(ctas, gy), dim3(TG_THREADS), p.total, s, pdl, A);
}

bool tma_for(const ModDev *mods, int nmod)
{
    bool tma = true;
    for (int i = 0; i < nmod; ++i)
        tma = tma && tg_ok(mods[i]);
    return tma;
}

}  // namespace

size_t gemv_smem_bytes(const ModDev &m)
{
    if (m.d == 2 && m.bits == 8)
        return 256 * 256;   // 256-byte line per entry, both modules
    const int ew = m.d <= 2 ? 1 : m.d / 2;
    return ((size_t)1 << m.bits) * (size_t)m.rep * ew * 4;
}

GemvPlan gemv_plan(const ModDev *mods, int nmod, double n_tiles_expected, int slices)
{
    const ModDev &m = mods[0];
    GemvPlan p{1, 0};
    if (tma_for(mods, nmod)) {
        // stage ranges of about U / CTAs; an item of spp stages then spans at most
        // ceil((spp - 1) / L) + 1 CTAs, which sets the slice count (at most 4)
        const int cg = tg_stage_groups(m.d, m.bits);
        const long spp = m.ngroups / cg;
        const bool both = m.d == 2 && m.bits == 8;
        const int cta_mods = both ? nmod : 1;
        const int ctas = std::max(1, num_sms() / (both ? 1 : nmod));
        const long nrb = (m.rows + TG_ROWS - 1) / TG_ROWS;
        const double units = std::max(1.0, n_tiles_expected) * cta_mods * nrb * spp;
        const long L = std::max(1L, (long)std::ceil(units / ctas));
        const long pieces = spp > 1 ? (spp - 2) / L + 2 : 1;
        p.slices = slices > 0 ? slices : (int)std::min(4L, pieces);
        // L >= min_units keeps the pieces of an item within the slices
        p.min_units = p.slices > 1 ? (int)((spp - 1 + p.slices - 2) / (p.slices - 1)) : (int)spp;
        return p;
    }
    // register-prefetch kernel: split the 64-column groups into slices until
    // there are about 32 warp items per SM
    if (slices > 0) {
        p.slices = slices;
        return p;
    }
    const long per = (m.rows + 31) / 32;
    const long items1 = (long)std::ceil(std::max(1.0, n_tiles_expected)) * per * nmod;
    int s = 1;
    while (m.ngroups % (2 * s) == 0 && m.ngroups / (2 * s) >= 2 && items1 * s < 32L * num_sms())
        s *= 2;
    p.slices = s;
    return p;
}

cudaError_t launch_gemv(const GemvArgs &args, cudaStream_t s, bool pdl)
{
    GemvArgs a = args;
    a.wait_limit = current_wait_limit();
    const ModDev &m = a.mod[0];
    const bool tma = tma_for(a.mod, a.nmod);
#define VQ_GEMV(D_, B_)                                                        \
    if (m.d == D_ && m.bits == B_)                                             \
        return tma ? gemv_tma_dispatch<D_, B_>(a, s, pdl) : gemv_dispatch<D_, B_>(a, s, pdl);
    VQ_GEOMETRIES(VQ_GEMV)
#undef VQ_GEMV
    return cudaErrorInvalidValue;
}

cudaError_t launch_swiglu(const float *G, const float *U, int slices, long slice_stride, int slots, int inter,
                          const int32_t *perm, int top_k, const float *xinv, const float *w, __half *h, float *wh,
                          cudaStream_t s, bool pdl)
{
    const dim3 grid((unsigned)std::max(1, std::min(slots, 8192)));
#define VQ_SWIGLU(S_) launch(vq_swiglu_kernel<S_>, grid, dim3(SWIGLU_THREADS), 0, s, pdl, G, U, slices, slice_stride, \
                             slots, inter, perm, top_k, xinv, w, h, wh)
    switch (slices) {
    case 1: return VQ_SWIGLU(1);
    case 2: return VQ_SWIGLU(2);
    case 3: return VQ_SWIGLU(3);
    case 4: return VQ_SWIGLU(4);
    default: return VQ_SWIGLU(0);
    }
#undef VQ_SWIGLU
}

cudaError_t launch_combine(const float *D, int slices, long slice_stride, const float *w, const int32_t *pos, int T,
                           int k, int hidden, void *y, int y_dtype, cudaStream_t s, bool pdl)
{
    const int blocks = T < 8192 ? (T > 0 ? T : 1) : 8192;
    // few tokens: spread each token's columns over several blocks
    const int h4 = hidden / 4;
    int ysplit = 1;
    while (blocks * ysplit < 2 * num_sms() && ysplit * 256 < h4)
        ysplit *= 2;
    const dim3 grid(blocks, ysplit);
#define VQ_COMBINE(S_) launch(vq_combine_kernel<S_>, grid, dim3(256), 0, s, pdl, D, slices, slice_stride, w, pos, T, k, \
                              hidden, y, y_dtype)
    switch (slices) {
    case 1: return VQ_COMBINE(1);
    case 2: return VQ_COMBINE(2);
    case 3: return VQ_COMBINE(3);
    case 4: return VQ_COMBINE(4);
    default: return VQ_COMBINE(0);
    }
#undef VQ_COMBINE
}

cudaError_t launch_unpack(const ModDev &m, int expert, uint16_t *out, cudaStream_t s)
{
    const long n = (long)m.rows * (m.cols / m.d);
    const int blocks = (int)((n + 255) / 256 < 8192 ? (n + 255) / 256 : 8192);
    vq_unpack_kernel<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(m, expert, out);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const ModDev &m, int expert, float *out, cudaStream_t s)
{
    const long n = (long)m.rows * m.cols;
    const int blocks = (int)((n + 255) / 256 < 8192 ? (n + 255) / 256 : 8192);
    vq_dequant_kernel<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(m, expert, out);
    return cudaGetLastError();
}

}  // namespace vq
