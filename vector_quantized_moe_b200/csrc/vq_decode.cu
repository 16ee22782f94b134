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
#include "vq_device.cuh"
#include "vq_internal.h"

namespace vq {
namespace {

template <int D, int BITS>
struct Geo {
    static constexpr int CODES = 16 / D;               // codes of one lane in one group
    static constexpr int QB = CODES * BITS;            // their bits
    static constexpr bool ALIGNED = (QB % 32) == 0;    // their bit range starts on a word
    static constexpr int NW = (QB + 31) / 32;          // words once shifted down to bit 0
    static constexpr int LW = ALIGNED ? NW : NW + 1;   // words loaded from the row
    static constexpr int EW = D <= 2 ? 1 : D / 2;      // shared-memory words per codebook entry
    static constexpr uint32_t MASK = (1u << BITS) - 1u;
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
        n[i] = G::ALIGNED ? w[i] : __funnelshift_r(w[i], w[i + (G::ALIGNED ? 0 : 1)], o);
#pragma unroll
    for (int k = 0; k < G::CODES; ++k) {
        const int p = k * BITS, wi = p >> 5, sh = p & 31;
        if (sh + BITS <= 32)
            c[k] = (n[wi] >> sh) & G::MASK;
        else
            c[k] = __funnelshift_r(n[wi], n[wi + 1], sh) & G::MASK;
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
    const int gps = m0.ngroups / S;
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
        const int gbeg = slice * gps, gend = gbeg + gps;

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
                if (a.act_bf16) {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        bw[i] = bf16x2_to_f16x2(bw[i]);
                }
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
#pragma unroll
                for (int rt = 0; rt < 2; ++rt) {
                    const float slo = f16_to_f32(L.sv[2 * rt]);
                    const float shi = f16_to_f32(L.sv[2 * rt + 1]);
                    acc[rt][0] = fmaf(tmp[rt][0], slo, acc[rt][0]);
                    acc[rt][1] = fmaf(tmp[rt][1], slo, acc[rt][1]);
                    acc[rt][2] = fmaf(tmp[rt][2], shi, acc[rt][2]);
                    acc[rt][3] = fmaf(tmp[rt][3], shi, acc[rt][3]);
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

// ------------------------------------------------------------ SwiGLU and combine

__global__ void vq_swiglu_kernel(const float *__restrict__ G, const float *__restrict__ U, int slices, long slice_stride,
                                 long n, __half *__restrict__ h)
{
    grid_dep_wait();
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        float gs = 0.f, us = 0.f;
        for (int s = 0; s < slices; ++s) {
            gs += G[s * slice_stride + i];
            us += U[s * slice_stride + i];
        }
        const float silu = gs / (1.f + __expf(-gs));
        h[i] = __float2half_rn(silu * us);
    }
}

__global__ void vq_combine_kernel(const float *__restrict__ D, int slices, long slice_stride, const float *__restrict__ w,
                                  const int32_t *__restrict__ pos, int T, int k, int hidden, void *y, int y_dtype)
{
    grid_dep_wait();
    const long n = (long)T * hidden;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const int tok = (int)(i / hidden), r = (int)(i % hidden);
        float acc = 0.f;
        for (int j = 0; j < k; ++j) {
            const long q = pos[(long)tok * k + j];
            float part = 0.f;
            for (int s = 0; s < slices; ++s)
                part += D[s * slice_stride + q * hidden + r];
            acc = fmaf(w[(long)tok * k + j], part, acc);
        }
        store_out(y, y_dtype, i, acc);
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
cudaError_t gemv_dispatch(const GemvArgs &a, int ctas, size_t smem, cudaStream_t s, bool pdl)
{
    auto k = vq_grouped_gemv_kernel<D, BITS, GEMV_PD>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (err != cudaSuccess)
            return err;
        attr_set = true;
    }
    const int gy = FastByteCodes<D, BITS>::value ? 1 : a.nmod;
    return launch(k, dim3(ctas, gy), dim3(GEMV_THREADS), smem, s, pdl, a);
}

template <int D, int BITS>
int gemv_occupancy(size_t smem)
{
    auto k = vq_grouped_gemv_kernel<D, BITS, GEMV_PD>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, GEMV_THREADS, smem) != cudaSuccess)
        return 1;
    return n > 0 ? n : 1;
}

}  // namespace

size_t gemv_smem_bytes(const ModDev &m)
{
    if (m.d == 2 && m.bits == 8)
        return 256 * 256;   // 256-byte line per entry, both modules
    const int ew = m.d <= 2 ? 1 : m.d / 2;
    return ((size_t)1 << m.bits) * (size_t)m.rep * ew * 4;
}

bool gemv_both_modules_per_cta(int d, int bits) { return d == 2 && bits == 8; }

int gemv_ctas_per_sm(int d, int bits, size_t smem)
{
#define VQ_OCC(D_, B_) \
    if (d == D_ && bits == B_) return gemv_occupancy<D_, B_>(smem);
    VQ_GEOMETRIES(VQ_OCC)
#undef VQ_OCC
    return 1;
}

cudaError_t launch_gemv(const GemvArgs &a, int ctas_per_mod, cudaStream_t s, bool pdl)
{
    const ModDev &m = a.mod[0];
    const size_t smem = gemv_smem_bytes(m);
#define VQ_GEMV(D_, B_) \
    if (m.d == D_ && m.bits == B_) return gemv_dispatch<D_, B_>(a, ctas_per_mod, smem, s, pdl);
    VQ_GEOMETRIES(VQ_GEMV)
#undef VQ_GEMV
    return cudaErrorInvalidValue;
}

cudaError_t launch_swiglu(const float *G, const float *U, int slices, long slice_stride, int slots, int inter, __half *h,
                          cudaStream_t s, bool pdl)
{
    const long n = (long)slots * inter;
    const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    return launch(vq_swiglu_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, s, pdl, G, U, slices, slice_stride, n, h);
}

cudaError_t launch_combine(const float *D, int slices, long slice_stride, const float *w, const int32_t *pos, int T, int k,
                           int hidden, void *y, int y_dtype, cudaStream_t s, bool pdl)
{
    const long n = (long)T * hidden;
    const int blocks = (int)((n + 255) / 256 < 8192 ? (n + 255) / 256 : 8192);
    return launch(vq_combine_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, s, pdl, D, slices, slice_stride, w, pos,
                  T, k, hidden, y, y_dtype);
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
