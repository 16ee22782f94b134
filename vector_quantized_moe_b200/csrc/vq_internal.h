// Internal interface between the C ABI (vq_api.cpp) and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/vq_moe.h"

// The geometries (d, bits) the kernels are instantiated for.
#define VQ_GEOMETRIES(X) \
    X(1, 3) X(1, 4) X(2, 8) X(2, 10) X(2, 11) X(4, 8) X(4, 9) X(4, 11) X(4, 13) X(8, 12)

// Token tile of the decode GEMV: bucket slots contracted together per pass over a weight tile.
#define VQ_PASS_TOKENS 8

namespace vq {

constexpr size_t CODEBOOK_SMEM_BUDGET = 100 * 1024;   // replicated codebook per CTA (decode)

// Decode codebook replicas in shared memory (log2): the per-lane count that
// spreads a warp's lookups over all banks (128 bytes / entry; d=1 entries take
// a 32-bit word), halved until the module's replicated codebook fits the budget.
__host__ __device__ constexpr int codebook_log_rep(int d, int bits)
{
    const long entry = d <= 2 ? 4 : 2 * d;
    int lr = 0;
    while ((1L << (lr + 1)) <= 128 / entry)
        ++lr;
    while (lr > 0 && (1L << bits) * entry * (1L << lr) > (long)CODEBOOK_SMEM_BUDGET)
        --lr;
    return lr;
}

// A module as the kernels see it.
struct ModDev {
    const uint32_t *codes;
    const uint16_t *scales;
    const uint16_t *biases;   // NULL: none
    const uint16_t *codebook;
    const uint32_t *bitmap;
    const uint32_t *rank;
    int E, rows, cols, d, bits;
    int row_words;   // uint32 words per packed row
    int ngroups;     // cols / 64
    int bm_words;    // ceil(rows / 32)
    int64_t live_rows;  // packed rows in codes / scales
    int rep;         // codebook replicas in shared memory (power of two)
    int log_rep;
};

ModDev make_moddev(const vq_module &m);

// Grouped GEMV over the experts that received tokens (tensor-core m16n8k16).
// One launch covers nmod modules that share the same activation and geometry.
struct GemvArgs {
    ModDev mod[2];
    int nmod;
    const void *act;        // activation rows: fp16 (or bf16 when act_bf16) [tokens or slots, cols]
    int act_bf16;
    int act_by_slot;        // 1: activation row = bucket slot q; 0: token (perm[q] / top_k, or t)
    long act_rows;          // rows of the activation array
    const int32_t *offsets; // [E + 1] bucket offsets; NULL -> single expert over T tokens
    const int32_t *perm;    // [T*k] pair ids in bucket order (bf16 act: token = perm[q] / top_k)
    int top_k;
    const int32_t *active;  // experts with tokens, ascending
    const int32_t *n_active;
    const int2 *passes;     // token tiles of the buckets (route: passes / n_passes); NULL in single-expert mode
    const int32_t *n_passes;
    int expert;             // single-expert mode
    int T;                  // single-expert mode: tokens
    int slices;             // partial-sum slices of the output (the reader sums them in order)
    int min_units;          // TMA kernel: least weight stages per CTA (bounds the pieces of a work item)
    int slices_zeroed;      // slices beyond the first are zero on entry (cleared by the routing launch)
    void *out[2];           // per module: [slices][slots][rows]
    int out_dtype;          // VQ_F32 or VQ_BF16
    long out_slice_stride;  // elements between slices
    int *err;               // device error word for bounded waits (may be NULL)
    uint32_t wait_limit;    // polls of a bounded wait before it gives up (current_wait_limit())
};

// Launches the TMA-fed kernel when the modules allow it (16-byte packed rows,
// whole stages), else the register-prefetch kernel. a.slices and a.min_units
// must come from gemv_plan for the same modules.
cudaError_t launch_gemv(const GemvArgs &a, cudaStream_t s, bool pdl);
// Output slices and least stages per CTA for nmod modules sharing a launch,
// sized for the expected number of token tiles; slices > 0 fixes the slice
// count instead (any count >= 1 is valid for either kernel).
struct GemvPlan {
    int slices;
    int min_units;
};
GemvPlan gemv_plan(const ModDev *mods, int nmod, double n_tiles_expected, int slices = 0);
size_t gemv_smem_bytes(const ModDev &m);

// Routing + bucketing. pos = inverse of perm; active/n_active as above (may be NULL).
// When x is not NULL the same launch also writes, per token t, x16[t] =
// fp16(x[t] * 2^k_t) [T, H] and xinv[t] = 2^-k_t (k_t puts the token's largest
// |x| in [2^14, 2^15)); when err is not NULL it is cleared.
// Up to three device spans of 32-bit words that a routing launch clears (after
// its grid-dependency wait): the partial-sum slices beyond the first, which a
// GEMV launch with slices_zeroed set then leaves to the items that write them.
struct ZeroSpans {
    float *p[3];
    long n[3];   // words
};

// passes / n_passes (may be NULL): the token tiles of the buckets, see VQ_PASS_TOKENS.
cudaError_t launch_route(const float *logits, int T, int E, int k, int renorm, int32_t *ids, float *w,
                         int32_t *offsets, int32_t *perm, int32_t *pos, int32_t *active, int32_t *n_active,
                         int2 *passes, int32_t *n_passes, const uint16_t *x, __half *x16, float *xinv, int H,
                         int *err, cudaStream_t s, bool pdl, const ZeroSpans *zero = nullptr);

// x16[t] = fp16(x[t] * 2^k_t), xinv[t] = 2^-k_t for t < T (as the routing launch does).
cudaError_t launch_convert(const uint16_t *x, __half *x16, float *xinv, int T, int H, cudaStream_t s, bool pdl);

// Per bucket slot q (pair p = perm[q], token t = p / top_k): g = xinv[t] *
// sum_s G[s, q, :], u = xinv[t] * sum_s U[s, q, :], h = silu(g) * u;
// h16[q, :] = fp16(h * 2^e_q) and wh[p] = w[p] * 2^-e_q, e_q putting the
// slot's largest |h| in [2^14, 2^15).
cudaError_t launch_swiglu(const float *G, const float *U, int slices, long slice_stride, int slots, int inter,
                          const int32_t *perm, int top_k, const float *xinv, const float *w, __half *h, float *wh,
                          cudaStream_t s, bool pdl);

// y[t, r] = sum_j w[t*k + j] * sum_s D[s, pos[t*k + j], r]
cudaError_t launch_combine(const float *D, int slices, long slice_stride, const float *w, const int32_t *pos, int T,
                           int k, int hidden, void *y, int y_dtype, cudaStream_t s, bool pdl);

cudaError_t launch_unpack(const ModDev &m, int expert, uint16_t *out, cudaStream_t s);
cudaError_t launch_dequant(const ModDev &m, int expert, float *out, cudaStream_t s);

int num_sms();

// 2D tiled TMA tensor map over a row-major [outer, inner] array (vq_tma.cpp).
bool tma_available();
bool tma_map_2d(CUtensorMap *map, CUtensorMapDataType dtype, int elem_bytes, const void *base, uint64_t inner,
                uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Front of a MoE workspace (each section 256-byte aligned): the device error
// word at offset 0 (cleared by the routing kernel, set by a kernel whose
// bounded wait gave up), then the routing tables.
struct RoutingLayout {
    size_t err, ids, w, offsets, perm, pos, active, nact, npass, passes;
};
// Upper bound on the token tiles of T*k pairs over E experts.
inline size_t max_passes(int T, int k, int E)
{
    const size_t tk = (size_t)T * k;
    return tk / VQ_PASS_TOKENS + (tk < (size_t)E ? tk : (size_t)E) + 1;
}
inline RoutingLayout plan_routing(size_t &o, int T, int k, int E)
{
    RoutingLayout r;
    const size_t tk = (size_t)T * k;
    r.err = o;     o = align_up(o + 4, 256);
    r.ids = o;     o = align_up(o + tk * 4, 256);
    r.w = o;       o = align_up(o + tk * 4, 256);
    r.offsets = o; o = align_up(o + (size_t)(E + 1) * 4, 256);
    r.perm = o;    o = align_up(o + tk * 4, 256);
    r.pos = o;     o = align_up(o + tk * 4, 256);
    r.active = o;  o = align_up(o + (size_t)E * 4, 256);
    r.nact = o;    o = align_up(o + 4, 256);
    r.npass = o;   o = align_up(o + 4, 256);
    r.passes = o;  o = align_up(o + max_passes(T, k, E) * 8, 256);
    return r;
}

template <typename T>
T *ws_at(void *ws, size_t off) { return reinterpret_cast<T *>(reinterpret_cast<char *>(ws) + off); }

// Stage-boundary tracing (vq_set_trace_events): records event i on stream s if set.
void trace_point(int i, cudaStream_t s);

// Polls of a bounded barrier wait in the kernels launched by this thread
// (vq_set_wait_limit; 2^22 by default).
uint32_t current_wait_limit();

// Sets a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t set_smem_limit_once(const void *kernel, int bytes);

// Prefill path (vq_prefill.cu).
size_t prefill_workspace_size(const vq_moe_layer *L, int T, int k);
vq_status run_prefill(const vq_moe_layer *L, const uint16_t *x, int T, const float *logits, int k, int renorm,
                      void *y, int y_dtype, void *ws, size_t ws_bytes, cudaStream_t s);

// One expert's tcgen05 GEMM of one or two modules (vq_prefill.cu).
size_t gemm_workspace_size(const vq_module *m, int T);
vq_status run_gemm(const vq_module *m0, const vq_module *m1, int expert, const uint16_t *x, int T, float *y0,
                   float *y1, void *ws, size_t ws_bytes, cudaStream_t s);

// Data-free VQ fit (vq_fit.cu).
size_t fit_workspace_size(int K, int d);
vq_status run_fit(const uint16_t *w, int rows, int cols, int d, int K, const int32_t *sample, int n_sample,
                  const int32_t *init, int iters, uint16_t *scales, uint16_t *codebook, uint16_t *codes, void *ws,
                  size_t ws_bytes, cudaStream_t s);

}  // namespace vq
