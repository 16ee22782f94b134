// Top-k router and expert bucketing for the VQ-MoE layer (sm_100a).
//
// Routing follows the MoE layers of the VQ model cards (Qwen3.8-Flash-Next:
// 10-of-512 experts; gemma-4-26b-a4b: 128 experts, top-8). Order of the
// top-k: larger logit first, ties to the smaller expert index, NaN last.
// Weights: softmax of the selected logits (renorm) or the full softmax over
// all experts evaluated at the selected ones.
//
// Bucketing: counts per expert, exclusive prefix sums (offsets), and a stable
// permutation of the pairs p = t*k + j grouped by expert (increasing p inside
// a bucket), its inverse (pos), and the ascending list of experts with
// tokens. Every step is integer work or a fixed-order reduction, so the
// tables are bit-identical from run to run.
#include <algorithm>

#include "vq_device.cuh"
#include "vq_internal.h"

namespace vq {
namespace {

constexpr int ROUTE_THREADS = 512;    // routing CTAs: 128 registers per thread hold a lane's sorted keys
constexpr int BUCKET_THREADS = 1024;  // the bucketing CTA of large batches
constexpr int BUCKET_MAX_E_PARALLEL = 1024;   // per-warp histograms fit shared memory up to here

// Monotone map of a float to uint32: NaN -> 0 (lowest), -0 -> +0.
__device__ __forceinline__ uint32_t order_key(float v)
{
    if (v != v)
        return 0u;
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u)
        u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 64-bit key: value first, then the smaller index wins. Always >= 1.
__device__ __forceinline__ uint64_t expert_key(float v, int e)
{
    return ((uint64_t)order_key(v) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)e);
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1)
        v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Inverse of order_key (NaN comes back as a NaN, -0 as +0).
__device__ __forceinline__ float key_value(uint32_t key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// One warp routes one token. Lane j < k ends with the j-th selection.
// Round j takes the largest key below the previous round's winner: a scan of
// the lane's keys (held in registers for E <= 512, re-read otherwise), then
// two 32-bit max reductions over the warp (the value word, then the index
// word among the lanes that tie on it). The round loop is kept rolled: the
// kernel runs once per layer with a cold instruction cache, so short code
// matters more than unrolling.
template <int PER_LANE>
__device__ __forceinline__ void route_token(const float *l, int E, int k, int renorm, int lane,
                                            int32_t *ids, float *w)
{
    int my_id = 0;
    float my_l = 0.f, top = 0.f;
    uint64_t keys[PER_LANE > 0 ? PER_LANE : 1];
    if constexpr (PER_LANE > 0) {
        // all loads first (a clamped index keeps them unconditional and independent);
        // plain loads, since the warm-up pass reads its logits from shared memory
        float v[PER_LANE];
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i)
            v[i] = l[min(lane + 32 * i, E - 1)];
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) {
            const int e = lane + 32 * i;
            keys[i] = e < E ? expert_key(v[i], e) : 0ull;
        }
    }
    uint64_t prev = ~0ull;
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
        uint64_t best = 0ull;
        if constexpr (PER_LANE > 0) {
#pragma unroll
            for (int i = 0; i < PER_LANE; ++i)
                best = (keys[i] < prev && keys[i] > best) ? keys[i] : best;
        } else {
            for (int e = lane; e < E; e += 32) {
                const uint64_t key = expert_key(l[e], e);
                best = (key < prev && key > best) ? key : best;
            }
        }
        const uint32_t hi = (uint32_t)(best >> 32);
        const uint32_t H = __reduce_max_sync(0xFFFFFFFFu, hi);
        const uint32_t Lw = __reduce_max_sync(0xFFFFFFFFu, hi == H ? (uint32_t)best : 0u);
        prev = ((uint64_t)H << 32) | Lw;
        if (j == 0)
            top = key_value(H);
        if (lane == j) {
            my_id = (int)(0xFFFFFFFFu - Lw);
            my_l = key_value(H);
        }
    }
    const float num = lane < k ? expf(my_l - top) : 0.f;
    float den;
    if (renorm) {
        den = warp_sum(num);
    } else {
        float s = 0.f;
        for (int e = lane; e < E; e += 32)
            s += expf(l[e] - top);
        den = warp_sum(s);
    }
    if (lane < k) {
        ids[lane] = my_id;
        w[lane] = num / den;
    }
}

// Tokens [t_begin, t_end), one per warp, over warps [w0, w0 + nw) of the CTA.
template <int PER_LANE>
__device__ void route_tokens(const float *logits, int t_begin, int t_end, int E, int k, int renorm, int32_t *ids,
                             float *w, int w0, int nw)
{
    const int lane = threadIdx.x & 31;
    for (int t = t_begin + (threadIdx.x >> 5) - w0; t < t_end; t += nw)
        route_token<PER_LANE>(logits + (long)t * E, E, k, renorm, lane, ids + (long)t * k, w + (long)t * k);
}

// Called by the warps [w0, w0 + nw) of the CTA.
// Not inlined: the routing kernel's warm-up pass and its real pass run the same code.
__device__ __noinline__ void route_range(const float *logits, int t_begin, int t_end, int E, int k, int renorm,
                                        int32_t *ids,
                            float *w, int w0, int nw)
{
    if (E <= 128)
        route_tokens<4>(logits, t_begin, t_end, E, k, renorm, ids, w, w0, nw);
    else if (E <= 512)
        route_tokens<16>(logits, t_begin, t_end, E, k, renorm, ids, w, w0, nw);
    else
        route_tokens<0>(logits, t_begin, t_end, E, k, renorm, ids, w, w0, nw);
}

// Bucketing by one CTA (pos, active, n_active, passes and n_passes may be NULL). passes[i] describes the i-th tile
// of VQ_PASS_TOKENS consecutive bucket slots, experts ascending: x = expert | (slots in the tile << 16), y = first
// slot; n_passes receives their number. Warp c of `chunks` handles pairs [c*P, (c+1)*P) with
// its own histogram row, so the stable scatter runs in parallel. `ids` may point to global or shared memory; every
// intermediate table lives in shared memory: hist [chunks][E] and base [E + 1] int32.
__device__ __noinline__ void bucket(const int32_t *ids, int npairs, int E, int32_t *offsets, int32_t *perm,
                                    int32_t *pos,
                       int32_t *active, int32_t *n_active, int2 *passes, int32_t *n_passes, int32_t *hist,
                       int32_t *base, int chunks)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < chunks * E; i += blockDim.x)
        hist[i] = 0;
    __syncthreads();
    const int per = (npairs + chunks - 1) / chunks;
    if (warp < chunks) {
        const int p0 = warp * per, p1 = min(npairs, p0 + per);
        for (int p = p0 + lane; p < p1; p += 32)
            atomicAdd(&hist[warp * E + ids[p]], 1);
    }
    __syncthreads();
    // per expert: totals and per-chunk exclusive bases (relative to the bucket)
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int c = 0; c < chunks; ++c) {
            const int v = hist[c * E + e];
            hist[c * E + e] = run;
            run += v;
        }
        base[e] = run;   // count for now
    }
    __syncthreads();
    // exclusive scans over the experts of (pairs, active experts, token tiles): thread i owns the
    // experts [i*EPT, (i+1)*EPT); a warp scan, a scan of the warp totals, then each thread writes
    // its experts' offsets, active-list entries and token tiles
    {
        __shared__ int wtot[32][3];
        const int EPT = (E + blockDim.x - 1) / blockDim.x;
        const int e0 = threadIdx.x * EPT;
        int v[3] = {0, 0, 0};
        for (int i = 0; i < EPT; ++i) {
            const int e = e0 + i;
            const int c = e < E ? base[e] : 0;
            v[0] += c;
            v[1] += c > 0;
            v[2] += (c + VQ_PASS_TOKENS - 1) / VQ_PASS_TOKENS;
        }
        int inc[3] = {v[0], v[1], v[2]};
#pragma unroll
        for (int o = 1; o < 32; o <<= 1)
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const int x = __shfl_up_sync(0xFFFFFFFFu, inc[q], o);
                if (lane >= o)
                    inc[q] += x;
            }
        if (lane == 31)
            for (int q = 0; q < 3; ++q)
                wtot[warp][q] = inc[q];
        __syncthreads();
        const int nw = blockDim.x >> 5;
        if (warp == 0) {
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                int t = lane < nw ? wtot[lane][q] : 0;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int x = __shfl_up_sync(0xFFFFFFFFu, t, o);
                    if (lane >= o)
                        t += x;
                }
                if (lane < nw)
                    wtot[lane][q] = t;   // inclusive over warps
            }
        }
        __syncthreads();
        int run[3];
#pragma unroll
        for (int q = 0; q < 3; ++q)
            run[q] = (warp > 0 ? wtot[warp - 1][q] : 0) + inc[q] - v[q];
        for (int i = 0; i < EPT; ++i) {
            const int e = e0 + i;
            if (e >= E)
                break;
            const int c = base[e];
            base[e] = run[0];
            offsets[e] = run[0];
            if (c > 0) {
                if (active)
                    active[run[1]] = e;
                if (passes) {
                    // tiles of VQ_PASS_TOKENS slots of this expert's bucket, in bucket order
                    const int np = (c + VQ_PASS_TOKENS - 1) / VQ_PASS_TOKENS;
                    for (int t = 0; t < np; ++t)
                        passes[run[2] + t] = make_int2(e | (min(VQ_PASS_TOKENS, c - VQ_PASS_TOKENS * t) << 16),
                                                       run[0] + VQ_PASS_TOKENS * t);
                }
            }
            run[0] += c;
            run[1] += c > 0;
            run[2] += (c + VQ_PASS_TOKENS - 1) / VQ_PASS_TOKENS;
        }
        if (threadIdx.x == 0) {
            base[E] = wtot[nw - 1][0];
            offsets[E] = wtot[nw - 1][0];
            if (n_active)
                *n_active = wtot[nw - 1][1];
            if (n_passes)
                *n_passes = wtot[nw - 1][2];
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < chunks * E; i += blockDim.x)
        hist[i] += base[i % E];
    __syncthreads();
    if (warp < chunks) {
        int32_t *cur = hist + warp * E;
        const int p0 = warp * per, p1 = min(npairs, p0 + per);
        const unsigned lt = (1u << lane) - 1u;
        for (int b = p0; b < p1; b += 32) {
            const int p = b + lane;
            const bool v = p < p1;
            const int e = v ? ids[p] : -1;
            const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
            if (v) {
                const int slot = cur[e] + __popc(peers & lt);
                perm[slot] = p;
                if (pos)
                    pos[p] = slot;
            }
            __syncwarp();
            if (v && (31 - __clz(peers)) == lane)
                cur[e] += __popc(peers);
            __syncwarp();
        }
    }
}

// x16[t, :] = fp16(x[t, :] * 2^k_t) and xinv[t] = 2^-k_t for the tokens
// [t0, t1), one token per warp over the warps [w0, w0 + nw) of the CTA. k_t
// brings the token's largest |x| into [2^14, 2^15) (scale_exp), so every bf16
// value keeps its full precision in fp16 (down to 2^-28 of the largest) and no
// value overflows; the consumers undo the scale exactly in fp32. Rows of
// H % 8 == 0 elements are 16-byte aligned; the row is read twice (the second
// time from L1).
__device__ void convert_rows(const uint16_t *x, __half *x16, float *xinv, int t0, int t1, int H, int w0, int nw)
{
    if (!x)
        return;
    const int lane = threadIdx.x & 31;
    const int n8 = H / 8;
    for (int t = t0 + (int)(threadIdx.x >> 5) - w0; t < t1; t += nw) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (long)t * H);
        uint4 *dst = reinterpret_cast<uint4 *>(x16 + (long)t * H);
        uint32_t m = 0;
        for (int i0 = lane; i0 < n8; i0 += 8 * 32) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = i0 + 32 * u < n8 ? ldg_u128(src + i0 + 32 * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                m = max(m, bf16x8_max_mag(v[u]));
        }
        m = __reduce_max_sync(0xFFFFFFFFu, m);
        const int k = scale_exp(m << 16);
        const float s = pow2f_normal(k);
        if (lane == 0 && xinv)
            xinv[t] = pow2f(-k);
        for (int i0 = lane; i0 < n8; i0 += 8 * 32) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + 32 * u < n8)
                    v[u] = ldg_u128(src + i0 + 32 * u);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + 32 * u < n8) {
                    uint4 o;
                    o.x = bf16x2_to_f16x2_scaled(v[u].x, s);
                    o.y = bf16x2_to_f16x2_scaled(v[u].y, s);
                    o.z = bf16x2_to_f16x2_scaled(v[u].z, s);
                    o.w = bf16x2_to_f16x2_scaled(v[u].w, s);
                    dst[i0 + 32 * u] = o;
                }
        }
    }
}

// Warps that scatter in parallel: one per 256 pairs (at most one per warp of the CTA).
__host__ __device__ __forceinline__ int bucket_chunks(int E, int npairs, int threads)
{
    if (E > BUCKET_MAX_E_PARALLEL)
        return 1;
    const int c = (npairs + 255) / 256;
    return c < 1 ? 1 : (c > threads / 32 ? threads / 32 : c);
}

// Outputs of the fused kernel's warm-up pass (one token): ids and weights of k
// slots, offsets [E + 1], perm and pos [k], active [E], counts, token tiles.
__host__ __device__ __forceinline__ size_t warmup_smem_ints(int E, int k) { return 2 * (size_t)E + 8 * (size_t)k + 8; }

// Shared memory of a bucketing CTA: hist, base and (fused kernel) the pair ids
// and the warm-up scratch.
__host__ __device__ __forceinline__ size_t bucket_smem_ints(int E, int npairs, bool fused, int threads, int k = 0)
{
    return (size_t)bucket_chunks(E, npairs, threads) * E + (size_t)E + 1 +
           (fused ? (size_t)npairs + warmup_smem_ints(E, k) : 0);
}

// Clears this CTA's share of the spans (32-bit words, coalesced).
__device__ void zero_spans(const ZeroSpans &z, int cta, int nctas)
{
    const long stride = (long)nctas * blockDim.x;
    for (int q = 0; q < 3; ++q)
        for (long i = (long)cta * blockDim.x + threadIdx.x; i < z.n[q]; i += stride)
            z.p[q][i] = 0.f;
}

// Small T: CTA 0 routes every token and buckets the pairs; CTAs 1.. clear the
// zero spans.
__global__ void __launch_bounds__(ROUTE_THREADS) vq_route_fused_kernel(const float *logits, int T, int E, int k,
                                                                      int renorm, int32_t *ids, float *w,
                                                                      int32_t *offsets, int32_t *perm, int32_t *pos,
                                                                      int32_t *active, int32_t *n_active,
                                                                      int2 *passes, int32_t *n_passes,
                                                                      const uint16_t *x, __half *x16, float *xinv, int H,
                                                                      int *err, const ZeroSpans zero)
{
    if (blockIdx.x > 0) {
        grid_dep_launch();
        grid_dep_wait();   // the previous call's readers of these slices have finished
        zero_spans(zero, blockIdx.x - 1, gridDim.x - 1);
        return;
    }
    extern __shared__ int32_t sm[];
    const int npairs = T * k, chunks = bucket_chunks(E, npairs, ROUTE_THREADS);
    int32_t *hist = sm, *base = sm + (size_t)chunks * E, *s_ids = base + E + 1;
    grid_dep_launch();   // the next kernel may start its prologue; it waits for this one's results

    // Warm-up while the previous kernel on the stream finishes: one token of
    // zero logits through the same routing and bucketing code, with every
    // output in shared memory, so the real pass finds its instructions cached;
    // and the logits prefetched into L2. Nothing global is read or written
    // here except the prefetch hints.
    {
        int32_t *wu = s_ids + npairs;
        int32_t *w_ids = wu, *w_off = w_ids + 2 * k, *w_perm = w_off + E + 1, *w_pos = w_perm + k;
        int32_t *w_act = w_pos + k, *w_cnt = w_act + E;
        int2 *w_tiles = reinterpret_cast<int2 *>(w_cnt + 2 + ((reinterpret_cast<uintptr_t>(w_cnt + 2) & 4) ? 1 : 0));
        float *zeros = reinterpret_cast<float *>(hist);   // E zero logits in the histogram area
        for (int e = threadIdx.x; e < E; e += blockDim.x)
            zeros[e] = 0.f;
        const long lbytes = (long)T * E * 4;
        for (long o = (long)threadIdx.x * 128; o < lbytes; o += (long)blockDim.x * 128)
            asm volatile("prefetch.L2 [%0];" ::"l"(reinterpret_cast<const char *>(logits) + o));   // generic address
        __syncthreads();
        if (threadIdx.x < 32)
            route_range(zeros, 0, 1, E, k, renorm, w_ids, reinterpret_cast<float *>(w_ids + k), 0, 1);
        __syncthreads();
        bucket(w_ids, k, E, w_off, w_perm, w_pos, w_act, w_cnt, w_tiles, w_cnt + 1, hist, base,
               bucket_chunks(E, k, ROUTE_THREADS));
        __syncthreads();
    }
    grid_dep_wait();
    if (err && threadIdx.x == 0)
        *err = 0;
    const int nw = blockDim.x >> 5, warp = threadIdx.x >> 5;
    if (T < nw) {
        // warps [0, T) route one token each while the others convert the activations
        if (warp < T)
            route_range(logits, 0, T, E, k, renorm, ids, w, 0, T);
        else
            convert_rows(x, x16, xinv, 0, T, H, T, nw - T);
    } else {
        route_range(logits, 0, T, E, k, renorm, ids, w, 0, nw);
        convert_rows(x, x16, xinv, 0, T, H, 0, nw);
    }
    __syncthreads();
    for (int p = threadIdx.x; p < npairs; p += blockDim.x)
        s_ids[p] = ids[p];   // written by this CTA above; read back once
    __syncthreads();
    bucket(s_ids, npairs, E, offsets, perm, pos, active, n_active, passes, n_passes, hist, base, chunks);
}

// Large T: many CTAs route, then one CTA buckets.
constexpr int ROUTE_TOKENS_PER_CTA = 256;     // up to this many tokens: the fused one-CTA routing
constexpr int TOPK_TOKENS_PER_CTA = 32;       // more: top-k CTAs of this many tokens (2 per warp), then bucketing

__global__ void __launch_bounds__(ROUTE_THREADS) vq_route_topk_kernel(const float *logits, int T, int E, int k,
                                                                     int renorm, int32_t *ids, float *w,
                                                                     const uint16_t *x, __half *x16, float *xinv, int H,
                                                                     int *err, const ZeroSpans zero)
{
    grid_dep_launch();   // the next kernel may start its prologue; it waits for this one's results
    grid_dep_wait();
    if (err && blockIdx.x == 0 && threadIdx.x == 0)
        *err = 0;
    zero_spans(zero, blockIdx.x, gridDim.x);
    const int t0 = blockIdx.x * TOPK_TOKENS_PER_CTA;
    convert_rows(x, x16, xinv, t0, min(T, t0 + TOPK_TOKENS_PER_CTA), H, 0, blockDim.x >> 5);
    route_range(logits, t0, min(T, t0 + TOPK_TOKENS_PER_CTA), E, k, renorm, ids, w, 0, blockDim.x >> 5);
}

__global__ void __launch_bounds__(BUCKET_THREADS) vq_bucket_kernel(const int32_t *ids, int npairs, int E,
                                                                 int32_t *offsets, int32_t *perm, int32_t *pos,
                                                                 int32_t *active, int32_t *n_active, int2 *passes,
                                                                 int32_t *n_passes)
{
    extern __shared__ int32_t sm[];
    const int chunks = bucket_chunks(E, npairs, BUCKET_THREADS);
    grid_dep_launch();   // the next kernel may start its prologue; it waits for this one's results
    grid_dep_wait();
    bucket(ids, npairs, E, offsets, perm, pos, active, n_active, passes, n_passes, sm, sm + (size_t)chunks * E,
           chunks);
}

// The activation conversion alone: warps over the tokens.
__global__ void __launch_bounds__(256) vq_convert_kernel(const uint16_t *x, __half *x16, float *xinv, int T, int H)
{
    grid_dep_launch();   // the next kernel may start its prologue; it waits for this one's results
    grid_dep_wait();
    const int wpc = blockDim.x >> 5;
    convert_rows(x, x16, xinv, blockIdx.x * wpc, T, H, 0, gridDim.x * wpc);
}

template <typename K, typename... Args>
cudaError_t launch_ex(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, Args... args)
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

}  // namespace

cudaError_t launch_route(const float *logits, int T, int E, int k, int renorm, int32_t *ids, float *w,
                         int32_t *offsets, int32_t *perm, int32_t *pos, int32_t *active, int32_t *n_active,
                         int2 *passes, int32_t *n_passes, const uint16_t *x, __half *x16, float *xinv, int H,
                         int *errw, cudaStream_t s, bool pdl, const ZeroSpans *zero)
{
    ZeroSpans z{};
    if (zero)
        z = *zero;
    const long zwords = z.n[0] + z.n[1] + z.n[2];
    // clearing CTAs for the fused launch: about 16 words per thread
    const int zctas = zwords > 0 ? (int)std::min<long>(64, (zwords + 16L * ROUTE_THREADS - 1) / (16L * ROUTE_THREADS)) : 0;
    // dynamic shared memory of a bucketing CTA: at most 32 x 1024 histogram rows
    // + bases (the 1024-thread bucketing CTA, 135 KB), or 16 x 1024 rows + bases
    // + 8192 pair ids + the warm-up scratch (the fused CTA, 112 KB); the kernels'
    // static tables come on top
    constexpr size_t ROUTE_SMEM_MAX = 170 * 1024;
    {
        cudaError_t err = set_smem_limit_once((const void *)vq_route_fused_kernel, (int)ROUTE_SMEM_MAX);
        if (err == cudaSuccess)
            err = set_smem_limit_once((const void *)vq_bucket_kernel, (int)ROUTE_SMEM_MAX);
        if (err != cudaSuccess)
            return err;
    }
    const bool fused = T <= ROUTE_TOKENS_PER_CTA;
    const size_t smem = bucket_smem_ints(E, T * k, fused, fused ? ROUTE_THREADS : BUCKET_THREADS, k) * sizeof(int32_t);
    if (smem > ROUTE_SMEM_MAX)
        return cudaErrorInvalidValue;
    if (fused)
        return launch_ex(vq_route_fused_kernel, dim3(1 + zctas), dim3(ROUTE_THREADS), smem, s, pdl, logits, T, E, k,
                         renorm, ids, w, offsets, perm, pos, active, n_active, passes, n_passes, x, x16, xinv, H, errw, z);
    const int ctas = (T + TOPK_TOKENS_PER_CTA - 1) / TOPK_TOKENS_PER_CTA;
    // many tokens: the activations are converted by a launch of their own, over the whole GPU
    cudaError_t err = launch_ex(vq_route_topk_kernel, dim3(ctas), dim3(ROUTE_THREADS), 0, s, pdl, logits, T, E, k,
                                renorm, ids, w, (const uint16_t *)nullptr, (__half *)nullptr, (float *)nullptr, H, errw,
                                z);
    if (err == cudaSuccess && x)
        err = launch_ex(vq_convert_kernel, dim3(std::max(1, std::min((T + 7) / 8, 4096))), dim3(256), 0, s, pdl, x,
                        x16, xinv, T, H);
    if (err != cudaSuccess)
        return err;
    return launch_ex(vq_bucket_kernel, dim3(1), dim3(BUCKET_THREADS), smem, s, pdl, (const int32_t *)ids, T * k, E,
                     offsets, perm, pos, active, n_active, passes, n_passes);
}

}  // namespace vq

namespace vq {

cudaError_t launch_convert(const uint16_t *x, __half *x16, float *xinv, int T, int H, cudaStream_t s, bool pdl)
{
    const int blocks = std::max(1, std::min((T + 7) / 8, 2048));
    return launch_ex(vq_convert_kernel, dim3(blocks), dim3(256), 0, s, pdl, x, x16, xinv, T, H);
}

}  // namespace vq
