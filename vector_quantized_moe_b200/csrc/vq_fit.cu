// Data-free VQ fit of one weight tensor on sm_100a: the codebook, codes and
// scales the expert path consumes, fit in pure weight space by k-means /
// Lloyd over the weight subvectors of a drawn subsample (VQ model cards,
// "Methodology": Qwen3.5-397B-A17B-VQ-2.6bpw, Qwen3.8-Flash-Next-VQ-4.4bpw,
// GLM-5.3-Flash-VQ-2.7bpw). The cards give the scale's shape (fp16 per row and 64
// weights), not its derivation; here it is the group's largest |w|.
//
// Kernels (one launch each, stream-ordered):
//   scales   one thread per (row, 64-weight group): the largest |w|, fp16
//   init     centroid k = the normalised subvector init[k]
//   assign   one thread per subvector, the centroids (fp32) in shared memory,
//            read by all threads of a block in step (broadcasts): the nearest
//            one by fp32 squared distance, components summed in order with
//            no fused multiply-add, ties to the lower index. On the sample it
//            adds the point to its centroid's exact fixed-point sums (64-bit
//            integer atomics: order-free, so deterministic); on the whole
//            tensor it writes the code.
//   update   centroid = exact mean of its points rounded to fp32 (kept when
//            it has none); clears the sums
//   round    the codebook to fp16; the fp32 centroids become those values
// Distance work is plain fp32 ALU on the CUDA cores: a d-wide difference is
// far too small a contraction for the tensor cores.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "vq_device.cuh"
#include "vq_internal.h"

namespace vq {
namespace {

constexpr int FIT_THREADS = 256;
constexpr int FIT_MAX_CENTROID_FLOATS = 32768;   // K * d: 128 KB of shared memory
constexpr float FIX_SCALE = 1099511627776.0f;    // 2^40: fixed-point fraction of the sums

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__global__ void vq_fit_scales_kernel(const uint16_t *__restrict__ w, int rows, int cols, uint16_t *__restrict__ scales)
{
    const int ng = cols / 64;
    const long n = (long)rows * ng;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const long r = i / ng;
        const int q = (int)(i % ng);
        const uint4 *p = reinterpret_cast<const uint4 *>(w + r * cols + (long)q * 64);
        uint32_t m = 0;   // largest |w| as bf16 magnitude bits (ordered like the values)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint4 v = p[j];
            const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                m = max(m, x[h] & 0x7FFFu);
                m = max(m, (x[h] >> 16) & 0x7FFFu);
            }
        }
        scales[i] = __half_as_ushort(__float2half_rn(__uint_as_float(m << 16)));
    }
}

// The normalised subvector `sub` (row sub / (cols/D), weights D * (sub % (cols/D)) ..).
template <int D>
__device__ __forceinline__ void load_subvector(const uint16_t *w, const uint16_t *scales, int cols, long sub,
                                               float (&v)[D])
{
    const int per_row = cols / D;
    const long r = sub / per_row;
    const int c0 = (int)(sub % per_row) * D;
    const float s = __half2float(__ushort_as_half(scales[r * (cols / 64) + c0 / 64]));
#pragma unroll
    for (int t = 0; t < D; ++t) {
        const float x = bf16_bits_to_f32(w[r * cols + c0 + t]);
        v[t] = s != 0.f ? __fdiv_rn(x, s) : 0.f;
    }
}

template <int D>
__global__ void vq_fit_init_kernel(const uint16_t *__restrict__ w, const uint16_t *__restrict__ scales, int cols,
                                   long n_sub, const int32_t *__restrict__ init, int K, float *__restrict__ cent,
                                   int *err)
{
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K)
        return;
    const long sub = init[k];
    float v[D];
    if (sub < 0 || sub >= n_sub) {
        atomicExch(err, 1);
        for (int t = 0; t < D; ++t)
            v[t] = 0.f;
    } else {
        load_subvector<D>(w, scales, cols, sub, v);
    }
#pragma unroll
    for (int t = 0; t < D; ++t)
        cent[(long)k * D + t] = v[t];
}

template <int D>
struct Vec;
template <>
struct Vec<1> {
    __device__ static void get(const float *p, float (&c)[1]) { c[0] = p[0]; }
};
template <>
struct Vec<2> {
    __device__ static void get(const float *p, float (&c)[2])
    {
        const float2 a = *reinterpret_cast<const float2 *>(p);
        c[0] = a.x;
        c[1] = a.y;
    }
};
template <>
struct Vec<4> {
    __device__ static void get(const float *p, float (&c)[4])
    {
        const float4 a = *reinterpret_cast<const float4 *>(p);
        c[0] = a.x;
        c[1] = a.y;
        c[2] = a.z;
        c[3] = a.w;
    }
};
template <>
struct Vec<8> {
    __device__ static void get(const float *p, float (&c)[8])
    {
        const float4 a = *reinterpret_cast<const float4 *>(p);
        const float4 b = *reinterpret_cast<const float4 *>(p + 4);
        c[0] = a.x;
        c[1] = a.y;
        c[2] = a.z;
        c[3] = a.w;
        c[4] = b.x;
        c[5] = b.y;
        c[6] = b.z;
        c[7] = b.w;
    }
};

// SAMPLE: points are the subvectors idx[0 .. n); adds each to its nearest
// centroid's fixed-point sums. Else: points are all n subvectors; writes codes.
template <int D, bool SAMPLE>
__global__ void __launch_bounds__(FIT_THREADS) vq_fit_assign_kernel(
    const uint16_t *__restrict__ w, const uint16_t *__restrict__ scales, int cols, long n_sub,
    const float *__restrict__ cent, int K, const int32_t *__restrict__ idx, long n,
    unsigned long long *__restrict__ sums, unsigned int *__restrict__ counts, uint16_t *__restrict__ codes, int *err)
{
    extern __shared__ __align__(16) float sc[];   // [K][D]
    for (int i = threadIdx.x; i < K * D; i += blockDim.x)
        sc[i] = cent[i];
    __syncthreads();
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const long sub = SAMPLE ? (long)idx[i] : i;
        if (sub < 0 || sub >= n_sub) {
            atomicExch(err, 1);
            continue;
        }
        float v[D];
        load_subvector<D>(w, scales, cols, sub, v);
        float best_d = __int_as_float(0x7F800000);   // +inf
        int best = 0;
#pragma unroll 4
        for (int k = 0; k < K; ++k) {
            float c[D];
            Vec<D>::get(sc + k * D, c);
            float dist = 0.f;
#pragma unroll
            for (int t = 0; t < D; ++t) {
                const float diff = __fsub_rn(v[t], c[t]);
                dist = __fadd_rn(dist, __fmul_rn(diff, diff));
            }
            if (dist < best_d) {   // strict: the lower index keeps a tie
                best_d = dist;
                best = k;
            }
        }
        if constexpr (SAMPLE) {
#pragma unroll
            for (int t = 0; t < D; ++t)
                atomicAdd(&sums[(long)best * D + t], (unsigned long long)__float2ll_rn(__fmul_rn(v[t], FIX_SCALE)));
            atomicAdd(&counts[best], 1u);
        } else {
            codes[sub] = (uint16_t)best;
        }
    }
}

template <int D>
__global__ void vq_fit_update_kernel(float *__restrict__ cent, unsigned long long *__restrict__ sums,
                                     unsigned int *__restrict__ counts, int K)
{
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K)
        return;
    const unsigned int cnt = counts[k];
#pragma unroll
    for (int t = 0; t < D; ++t) {
        if (cnt) {
            const double s = __ll2double_rn((long long)sums[(long)k * D + t]);
            cent[(long)k * D + t] = __double2float_rn(__ddiv_rn(s * 0x1p-40, (double)cnt));
        }
        sums[(long)k * D + t] = 0ull;
    }
    counts[k] = 0u;
}

__global__ void vq_fit_round_kernel(float *__restrict__ cent, int n, uint16_t *__restrict__ codebook)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n)
        return;
    const __half h = __float2half_rn(cent[i]);
    codebook[i] = __half_as_ushort(h);
    cent[i] = __half2float(h);
}

struct FitPlan {
    size_t err, cent, sums, counts, total;
};

FitPlan plan_fit(int K, int d)
{
    FitPlan p{};
    size_t o = 0;
    p.err = o; o = align_up(o + 4, 256);
    p.cent = o; o = align_up(o + (size_t)K * d * 4, 256);
    p.sums = o; o = align_up(o + (size_t)K * d * 8, 256);
    p.counts = o; o = align_up(o + (size_t)K * 4, 256);
    p.total = o;
    return p;
}

template <int D>
cudaError_t run_fit_d(const uint16_t *w, int rows, int cols, int K, const int32_t *sample, int n_sample,
                      const int32_t *init, int iters, uint16_t *scales, uint16_t *codebook, uint16_t *codes,
                      void *ws, cudaStream_t s)
{
    const FitPlan p = plan_fit(K, D);
    int *err = ws_at<int>(ws, p.err);
    float *cent = ws_at<float>(ws, p.cent);
    unsigned long long *sums = ws_at<unsigned long long>(ws, p.sums);
    unsigned int *counts = ws_at<unsigned int>(ws, p.counts);
    const long n_sub = (long)rows * (cols / D);
    const int sms = num_sms();
    cudaError_t e = cudaMemsetAsync(ws, 0, p.total, s);   // error word, sums, counts
    if (e != cudaSuccess)
        return e;
    const long ng = (long)rows * (cols / 64);
    vq_fit_scales_kernel<<<(unsigned)std::min<long>((ng + FIT_THREADS - 1) / FIT_THREADS, 32L * sms), FIT_THREADS, 0,
                           s>>>(w, rows, cols, scales);
    vq_fit_init_kernel<D><<<(K + 127) / 128, 128, 0, s>>>(w, scales, cols, n_sub, init, K, cent, err);
    const size_t smem = (size_t)K * D * 4;
    auto ks = vq_fit_assign_kernel<D, true>;
    auto ka = vq_fit_assign_kernel<D, false>;
    if ((e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return e;
    // blocks per SM as shared memory allows (at most 8), a grid of whole waves
    const int per_sm = (int)std::max<size_t>(1, std::min<size_t>(8, (200u * 1024) / std::max<size_t>(smem, 1)));
    const long grid_s = std::min<long>((n_sample + FIT_THREADS - 1) / FIT_THREADS, (long)sms * per_sm);
    const long grid_a = std::min<long>((n_sub + FIT_THREADS - 1) / FIT_THREADS, (long)sms * per_sm);
    for (int it = 0; it < iters; ++it) {
        ks<<<(unsigned)grid_s, FIT_THREADS, smem, s>>>(w, scales, cols, n_sub, cent, K, sample, n_sample, sums, counts,
                                                      nullptr, err);
        vq_fit_update_kernel<D><<<(K + 127) / 128, 128, 0, s>>>(cent, sums, counts, K);
    }
    vq_fit_round_kernel<<<(K * D + 255) / 256, 256, 0, s>>>(cent, K * D, codebook);
    ka<<<(unsigned)grid_a, FIT_THREADS, smem, s>>>(w, scales, cols, n_sub, cent, K, nullptr, n_sub, nullptr, nullptr,
                                                  codes, err);
    return cudaGetLastError();
}

}  // namespace

size_t fit_workspace_size(int K, int d) { return plan_fit(K, d).total; }

vq_status run_fit(const uint16_t *w, int rows, int cols, int d, int K, const int32_t *sample, int n_sample,
                  const int32_t *init, int iters, uint16_t *scales, uint16_t *codebook, uint16_t *codes, void *ws,
                  size_t ws_bytes, cudaStream_t s)
{
    if (K < 2 || K > 65536 || (long)K * d > FIT_MAX_CENTROID_FLOATS || n_sample < K || iters < 0)
        return VQ_ERR_ARG;
    if (ws_bytes < plan_fit(K, d).total)
        return VQ_ERR_WORKSPACE;
    cudaError_t e;
    switch (d) {
    case 1: e = run_fit_d<1>(w, rows, cols, K, sample, n_sample, init, iters, scales, codebook, codes, ws, s); break;
    case 2: e = run_fit_d<2>(w, rows, cols, K, sample, n_sample, init, iters, scales, codebook, codes, ws, s); break;
    case 4: e = run_fit_d<4>(w, rows, cols, K, sample, n_sample, init, iters, scales, codebook, codes, ws, s); break;
    case 8: e = run_fit_d<8>(w, rows, cols, K, sample, n_sample, init, iters, scales, codebook, codes, ws, s); break;
    default: return VQ_ERR_ARG;
    }
    return e == cudaSuccess ? VQ_OK : VQ_ERR_CUDA;
}

}  // namespace vq
