// C ABI of the VQ-MoE library: argument validation, host-side packing,
// workspace layout and kernel dispatch. See include/vq_moe.h.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "vq_internal.h"

namespace vq {

int num_sms()
{
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            sms = 148;
    }
    return sms;
}

namespace {

bool geometry_ok(int d, int bits)
{
#define VQ_GEO_OK(D_, B_) \
    if (d == D_ && bits == B_) return true;
    VQ_GEOMETRIES(VQ_GEO_OK)
#undef VQ_GEO_OK
    return false;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

vq_status check_module(const vq_module *m)
{
    if (!m || !m->codes || !m->scales || !m->codebook)
        return VQ_ERR_ARG;
    if (m->E < 1 || m->rows < 1 || m->cols < 64 || m->cols % 64 != 0)
        return VQ_ERR_ARG;
    if (m->d != 1 && m->d != 2 && m->d != 4 && m->d != 8)
        return VQ_ERR_ARG;
    if (m->cols % (32 * m->d) != 0 || m->bits < 1 || m->bits > 16)
        return VQ_ERR_ARG;
    if (m->live_bitmap && (!m->live_rank || m->live_rows < 1 || m->live_rows > (int64_t)m->E * m->rows))
        return VQ_ERR_ARG;
    if (!geometry_ok(m->d, m->bits))
        return VQ_ERR_UNSUPPORTED;
    if (!aligned(m->codes, 16) || !aligned(m->codebook, 16) || !aligned(m->scales, 2) || !aligned(m->biases, 2))
        return VQ_ERR_ALIGN;
    if ((m->live_bitmap && !aligned(m->live_bitmap, 4)) || (m->live_rank && !aligned(m->live_rank, 4)))
        return VQ_ERR_ALIGN;
    return VQ_OK;
}

vq_status cuda_status(cudaError_t e)
{
    if (e != cudaSuccess && std::getenv("VQ_DEBUG"))
        std::fprintf(stderr, "vq: CUDA error %d: %s\n", (int)e, cudaGetErrorString(e));
    return e == cudaSuccess ? VQ_OK : VQ_ERR_CUDA;
}

struct DecodePlan {
    int T, k, E, H, I;
    int sa, sb;                  // output slices of the gate/up and down passes
    GemvPlan pg, pu, pd;         // GEMV plans of gate, up (pg covers both when they share a launch) and down
    bool gu_shared;              // gate and up in one launch
    RoutingLayout r;
    size_t off_x16, off_xinv, off_G, off_U, off_h, off_wh, off_D;
    size_t total;
};

vq_status check_layer(const vq_moe_layer *L)
{
    if (!L)
        return VQ_ERR_ARG;
    vq_status st;
    if ((st = check_module(&L->gate)) != VQ_OK || (st = check_module(&L->up)) != VQ_OK ||
        (st = check_module(&L->down)) != VQ_OK)
        return st;
    const int E = L->gate.E, H = L->gate.cols, I = L->gate.rows;
    if (L->up.E != E || L->down.E != E || L->up.cols != H || L->up.rows != I || L->down.rows != H ||
        L->down.cols != I)
        return VQ_ERR_ARG;
    return VQ_OK;
}

DecodePlan plan_decode(const vq_moe_layer *L, int T, int k)
{
    DecodePlan p{};
    p.T = T;
    p.k = k;
    p.E = L->gate.E;
    p.H = L->gate.cols;
    p.I = L->gate.rows;
    // expected experts with tokens under uniform routing (the plan's size hint;
    // any actual routing is handled correctly)
    const double n_exp = p.E * (1.0 - std::pow(1.0 - (double)k / p.E, (double)T));
    const ModDev gu[2] = {make_moddev(L->gate), make_moddev(L->up)};
    const ModDev dn = make_moddev(L->down);
    p.gu_shared = gu[0].d == gu[1].d && gu[0].bits == gu[1].bits && gu[0].rep == gu[1].rep &&
                  (gu[0].biases == nullptr) == (gu[1].biases == nullptr);
    if (p.gu_shared) {
        p.pg = p.pu = gemv_plan(gu, 2, n_exp);
    } else {
        const int s = std::max(gemv_plan(&gu[0], 1, n_exp).slices, gemv_plan(&gu[1], 1, n_exp).slices);
        p.pg = gemv_plan(&gu[0], 1, n_exp, s);
        p.pu = gemv_plan(&gu[1], 1, n_exp, s);
    }
    p.pd = gemv_plan(&dn, 1, n_exp);
    p.sa = p.pg.slices;
    p.sb = p.pd.slices;
    size_t o = 0;
    p.r = plan_routing(o, T, k, p.E);
    const size_t tk = (size_t)T * k;
    p.off_x16 = o; o = align_up(o + (size_t)T * p.H * 2, 256);
    p.off_xinv = o; o = align_up(o + (size_t)T * 4, 256);
    p.off_G = o; o = align_up(o + (size_t)p.sa * tk * p.I * 4, 256);
    p.off_U = o; o = align_up(o + (size_t)p.sa * tk * p.I * 4, 256);
    p.off_h = o; o = align_up(o + tk * p.I * 2, 256);
    p.off_wh = o; o = align_up(o + tk * 4, 256);
    p.off_D = o; o = align_up(o + (size_t)p.sb * tk * p.H * 4, 256);
    p.total = o;
    return p;
}

}  // namespace

ModDev make_moddev(const vq_module &m)
{
    ModDev d{};
    d.codes = m.codes;
    d.scales = m.scales;
    d.biases = m.biases;
    d.codebook = m.codebook;
    d.bitmap = m.live_bitmap;
    d.rank = m.live_rank;
    d.E = m.E;
    d.rows = m.rows;
    d.cols = m.cols;
    d.d = m.d;
    d.bits = m.bits;
    d.row_words = (m.cols / m.d / 32) * m.bits;
    d.ngroups = m.cols / 64;
    d.bm_words = (m.rows + 31) / 32;
    d.live_rows = m.live_bitmap ? m.live_rows : (int64_t)m.E * m.rows;
    d.log_rep = codebook_log_rep(m.d, m.bits);
    d.rep = 1 << d.log_rep;
    return d;
}

namespace {
thread_local cudaEvent_t *g_trace = nullptr;
thread_local int g_trace_n = 0;
thread_local uint32_t g_wait_limit = 1u << 22;

std::mutex g_attr_mu;
std::map<std::pair<const void *, int>, int> g_attr_set;   // (kernel, device) -> shared-memory limit set
}  // namespace

void trace_point(int i, cudaStream_t s)
{
    if (g_trace && i < g_trace_n)
        cudaEventRecord(g_trace[i], s);
}

uint32_t current_wait_limit() { return g_wait_limit; }

cudaError_t set_smem_limit_once(const void *kernel, int bytes)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lock(g_attr_mu);
    int &cur = g_attr_set[{kernel, dev}];
    if (cur >= bytes)
        return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        cur = bytes;
    return e;
}

}  // namespace vq

using namespace vq;

extern "C" {

const char *vq_status_str(vq_status s)
{
    switch (s) {
    case VQ_OK: return "VQ_OK";
    case VQ_ERR_ARG: return "VQ_ERR_ARG: invalid argument";
    case VQ_ERR_ALIGN: return "VQ_ERR_ALIGN: misaligned pointer";
    case VQ_ERR_UNSUPPORTED: return "VQ_ERR_UNSUPPORTED: geometry or size not implemented";
    case VQ_ERR_WORKSPACE: return "VQ_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case VQ_ERR_CUDA: return "VQ_ERR_CUDA: CUDA runtime error";
    case VQ_ERR_DEVICE_CHECK: return "VQ_ERR_DEVICE_CHECK: device-side check failed";
    }
    return "unknown vq_status";
}

int vq_geometry_supported(int32_t d, int32_t bits) { return geometry_ok(d, bits) ? 1 : 0; }

vq_status vq_set_trace_events(void *const *events, int32_t n_events)
{
    if (n_events < 0)
        return VQ_ERR_ARG;
    g_trace = events ? (cudaEvent_t *)events : nullptr;
    g_trace_n = events ? n_events : 0;
    return VQ_OK;
}

vq_status vq_set_wait_limit(int64_t polls)
{
    if (polls > 0xFFFFFFFFll)
        return VQ_ERR_ARG;
    g_wait_limit = polls < 0 ? (1u << 22) : (uint32_t)polls;
    return VQ_OK;
}

size_t vq_packed_words(int64_t rows, int32_t ncode, int32_t bits)
{
    if (rows < 0 || ncode <= 0 || ncode % 32 != 0 || bits < 1 || bits > 16)
        return 0;
    return (size_t)rows * (size_t)(ncode / 32) * (size_t)bits;
}

static int bm_live(const uint32_t *bm, int rows, int e, int r)
{
    if (!bm)
        return 1;
    const int nw = (rows + 31) / 32;
    return (bm[(size_t)e * nw + r / 32] >> (r % 32)) & 1;
}

vq_status vq_pack(const uint16_t *codes, int32_t E, int32_t rows, int32_t ncode, int32_t bits,
                  const uint32_t *live_bitmap, uint32_t *out, size_t out_words, size_t *rows_written)
{
    if (!codes || !out || E < 1 || rows < 1 || ncode <= 0 || ncode % 32 != 0 || bits < 1 || bits > 16)
        return VQ_ERR_ARG;
    const size_t rw = vq_packed_words(1, ncode, bits);
    size_t n = 0;
    for (int e = 0; e < E; ++e)
        for (int r = 0; r < rows; ++r)
            if (bm_live(live_bitmap, rows, e, r))
                ++n;
    if (out_words < n * rw)
        return VQ_ERR_ARG;
    const uint32_t lim = 1u << bits;
    size_t row = 0;
    for (int e = 0; e < E; ++e)
        for (int r = 0; r < rows; ++r) {
            if (!bm_live(live_bitmap, rows, e, r))
                continue;
            const uint16_t *src = codes + ((size_t)e * rows + r) * ncode;
            uint32_t *dst = out + row * rw;
            std::memset(dst, 0, rw * sizeof(uint32_t));
            for (int j = 0; j < ncode; ++j) {
                const uint32_t v = src[j];
                if (v >= lim)
                    return VQ_ERR_ARG;
                const size_t bit = (size_t)j * bits;
                const size_t w = bit >> 5;
                const unsigned sh = bit & 31;
                dst[w] |= v << sh;
                if (sh + bits > 32)
                    dst[w + 1] |= v >> (32 - sh);
            }
            ++row;
        }
    if (rows_written)
        *rows_written = n;
    return VQ_OK;
}

vq_status vq_pack_scales(const uint16_t *scales, int32_t E, int32_t rows, int32_t ngroups,
                         const uint32_t *live_bitmap, uint16_t *out, size_t out_elems, size_t *rows_written)
{
    if (!scales || !out || E < 1 || rows < 1 || ngroups < 1)
        return VQ_ERR_ARG;
    size_t n = 0;
    for (int e = 0; e < E; ++e)
        for (int r = 0; r < rows; ++r)
            n += bm_live(live_bitmap, rows, e, r);
    if (out_elems < n * (size_t)ngroups)
        return VQ_ERR_ARG;
    size_t row = 0;
    for (int e = 0; e < E; ++e)
        for (int r = 0; r < rows; ++r)
            if (bm_live(live_bitmap, rows, e, r)) {
                std::memcpy(out + row * ngroups, scales + ((size_t)e * rows + r) * ngroups,
                            (size_t)ngroups * sizeof(uint16_t));
                ++row;
            }
    if (rows_written)
        *rows_written = n;
    return VQ_OK;
}

vq_status vq_live_rank(const uint32_t *live_bitmap, int32_t E, int32_t rows, uint32_t *rank_out)
{
    if (!live_bitmap || !rank_out || E < 1 || rows < 1)
        return VQ_ERR_ARG;
    const int nw = (rows + 31) / 32;
    uint64_t run = 0;
    for (int e = 0; e < E; ++e)
        for (int w = 0; w < nw; ++w) {
            rank_out[(size_t)e * nw + w] = (uint32_t)run;
            uint32_t word = live_bitmap[(size_t)e * nw + w];
            if (w == nw - 1 && rows % 32 != 0 && (word >> (rows % 32)) != 0)
                return VQ_ERR_ARG;
            run += (uint64_t)__builtin_popcount(word);
        }
    if (run > 0xFFFFFFFFull)
        return VQ_ERR_ARG;
    return VQ_OK;
}

vq_status vq_unpack(const vq_module *m, int32_t expert, uint16_t *codes_out, void *stream)
{
    vq_status st = check_module(m);
    if (st != VQ_OK)
        return st;
    if (!codes_out || expert < 0 || expert >= m->E)
        return VQ_ERR_ARG;
    return cuda_status(launch_unpack(make_moddev(*m), expert, codes_out, (cudaStream_t)stream));
}

vq_status vq_dequant(const vq_module *m, int32_t expert, float *w_out, void *stream)
{
    vq_status st = check_module(m);
    if (st != VQ_OK)
        return st;
    if (!w_out || expert < 0 || expert >= m->E)
        return VQ_ERR_ARG;
    return cuda_status(launch_dequant(make_moddev(*m), expert, w_out, (cudaStream_t)stream));
}

vq_status vq_gemv(const vq_module *m, int32_t expert, const uint16_t *x, int32_t T, void *y, int32_t y_dtype,
                  void *stream)
{
    vq_status st = check_module(m);
    if (st != VQ_OK)
        return st;
    if (!x || !y || T < 0 || expert < 0 || expert >= m->E || (y_dtype != VQ_F32 && y_dtype != VQ_BF16))
        return VQ_ERR_ARG;
    if (!aligned(x, 16))
        return VQ_ERR_ALIGN;
    if (T == 0)
        return VQ_OK;
    GemvArgs a{};
    a.mod[0] = make_moddev(*m);
    a.mod[1] = a.mod[0];
    a.nmod = 1;
    a.act = x;
    a.act_bf16 = 1;
    a.act_by_slot = 0;
    a.act_rows = T;
    a.expert = expert;
    a.T = T;
    a.slices = 1;
    a.min_units = 0;
    a.out[0] = y;
    a.out[1] = y;
    a.out_dtype = y_dtype;
    a.out_slice_stride = 0;
    a.err = nullptr;
    return cuda_status(launch_gemv(a, (cudaStream_t)stream, false));
}

size_t vq_gemm_workspace_size(const vq_module *m, int32_t T)
{
    if (check_module(m) != VQ_OK || T < 0)
        return 0;
    return gemm_workspace_size(m, T);
}

vq_status vq_gemm(const vq_module *m0, const vq_module *m1, int32_t expert, const uint16_t *x, int32_t T, float *y0,
                  float *y1, void *workspace, size_t ws_bytes, void *stream)
{
    vq_status st = check_module(m0);
    if (st != VQ_OK || (m1 && (st = check_module(m1)) != VQ_OK))
        return st;
    if (T < 0 || expert < 0 || expert >= m0->E || (T > 0 && (!x || !y0 || (m1 && !y1))))
        return VQ_ERR_ARG;
    if (m1 && (m1->E != m0->E || m1->rows != m0->rows || m1->cols != m0->cols || m1->d != m0->d ||
               m1->bits != m0->bits))
        return VQ_ERR_ARG;
    if (!aligned(x, 16) || !aligned(y0, 16) || !aligned(y1, 16))
        return VQ_ERR_ALIGN;
    if (!workspace || !aligned(workspace, 256))
        return VQ_ERR_WORKSPACE;
    return run_gemm(m0, m1, expert, x, T, y0, y1, workspace, ws_bytes, (cudaStream_t)stream);
}

vq_status vq_route(const float *logits, int32_t T, int32_t E, int32_t top_k, int32_t renorm, int32_t *ids,
                   float *weights, int32_t *offsets, int32_t *perm, void *stream)
{
    if (!logits || !ids || !weights || !offsets || !perm || T < 0 || E < 1 || E > 4096 || top_k < 1 ||
        top_k > std::min(E, 32) || (long)T * top_k >= (1L << 31))
        return VQ_ERR_ARG;
    return cuda_status(launch_route(logits, T, E, top_k, renorm, ids, weights, offsets, perm, nullptr, nullptr,
                                    nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0, nullptr,
                                    (cudaStream_t)stream, false));
}

size_t vq_moe_workspace_size(const vq_moe_layer *L, int32_t T, int32_t top_k, int32_t mode)
{
    if (check_layer(L) != VQ_OK || T < 0 || top_k < 1 || top_k > std::min(L->gate.E, 32))
        return 0;
    if (mode == VQ_MODE_DECODE)
        return plan_decode(L, T, top_k).total;
    if (mode == VQ_MODE_PREFILL)
        return prefill_workspace_size(L, T, top_k);
    return 0;
}

static vq_status check_moe_args(const vq_moe_layer *L, const uint16_t *x, int32_t T, const float *logits,
                                int32_t top_k, void *y, int32_t y_dtype, void *workspace)
{
    vq_status st = check_layer(L);
    if (st != VQ_OK)
        return st;
    // an empty batch launches nothing, so its x, logits and y may be NULL
    if ((T > 0 && (!x || !logits || !y)) || T < 0 || top_k < 1 || top_k > std::min(L->gate.E, 32) ||
        L->gate.E > 4096 || (y_dtype != VQ_F32 && y_dtype != VQ_BF16) || (long)T * top_k >= (1L << 31))
        return VQ_ERR_ARG;
    if (!aligned(x, 16) || !aligned(y, 16))
        return VQ_ERR_ALIGN;
    if (!workspace || !aligned(workspace, 256))
        return VQ_ERR_WORKSPACE;
    return VQ_OK;
}

vq_status vq_moe_decode(const vq_moe_layer *L, const uint16_t *x, int32_t T, const float *logits, int32_t top_k,
                        int32_t renorm, void *y, int32_t y_dtype, void *workspace, size_t ws_bytes, void *stream)
{
    vq_status st = check_moe_args(L, x, T, logits, top_k, y, y_dtype, workspace);
    if (st != VQ_OK)
        return st;
    if (T == 0)
        return VQ_OK;
    const DecodePlan p = plan_decode(L, T, top_k);
    if (ws_bytes < p.total)
        return VQ_ERR_WORKSPACE;
    // the GEMV kernels index their work (token tiles x modules x 256-row blocks x
    // stages) with 32-bit integers
    for (const vq_module *m : {&L->gate, &L->up, &L->down})
        if ((double)max_passes(T, top_k, p.E) * 2.0 * ((m->rows + 255) / 256) * (m->cols / 64) >= 2147483647.0)
            return VQ_ERR_UNSUPPORTED;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t *ids = ws_at<int32_t>(workspace, p.r.ids);
    float *w = ws_at<float>(workspace, p.r.w);
    int32_t *offsets = ws_at<int32_t>(workspace, p.r.offsets);
    int32_t *perm = ws_at<int32_t>(workspace, p.r.perm);
    int32_t *pos = ws_at<int32_t>(workspace, p.r.pos);
    int32_t *active = ws_at<int32_t>(workspace, p.r.active);
    int32_t *nact = ws_at<int32_t>(workspace, p.r.nact);
    int *errw = ws_at<int>(workspace, p.r.err);
    __half *x16 = ws_at<__half>(workspace, p.off_x16);
    float *xinv = ws_at<float>(workspace, p.off_xinv);
    float *G = ws_at<float>(workspace, p.off_G);
    float *U = ws_at<float>(workspace, p.off_U);
    __half *h = ws_at<__half>(workspace, p.off_h);
    float *wh = ws_at<float>(workspace, p.off_wh);
    float *D = ws_at<float>(workspace, p.off_D);
    const long tk = (long)T * top_k;

    trace_point(0, s);
    int2 *passes = ws_at<int2>(workspace, p.r.passes);
    int32_t *npass = ws_at<int32_t>(workspace, p.r.npass);
    // the routing launch clears the partial-sum slices beyond the first; the GEMVs
    // then store only the pieces they compute
    ZeroSpans zs{};
    zs.p[0] = G + tk * p.I;
    zs.n[0] = (long)(p.sa - 1) * tk * p.I;
    zs.p[1] = U + tk * p.I;
    zs.n[1] = (long)(p.sa - 1) * tk * p.I;
    zs.p[2] = D + tk * p.H;
    zs.n[2] = (long)(p.sb - 1) * tk * p.H;
    cudaError_t err = launch_route(logits, T, p.E, top_k, renorm, ids, w, offsets, perm, pos, active, nact, passes,
                                   npass, x, x16, xinv, p.H, errw, s, true, &zs);
    if (err != cudaSuccess)
        return VQ_ERR_CUDA;
    trace_point(1, s);

    // gate and up: one launch when they share a geometry
    GemvArgs a{};
    a.act = x16;
    a.act_bf16 = 0;
    a.act_by_slot = 0;
    a.act_rows = T;
    a.offsets = offsets;
    a.perm = perm;
    a.top_k = top_k;
    a.active = active;
    a.n_active = nact;
    a.passes = passes;
    a.n_passes = npass;
    a.slices = p.sa;
    a.min_units = p.pg.min_units;
    a.slices_zeroed = 1;
    a.out_dtype = VQ_F32;
    a.out_slice_stride = tk * p.I;
    a.err = errw;
    const ModDev mg = make_moddev(L->gate), mu = make_moddev(L->up);
    if (p.gu_shared) {
        a.mod[0] = mg;
        a.mod[1] = mu;
        a.nmod = 2;
        a.out[0] = G;
        a.out[1] = U;
        err = launch_gemv(a, s, true);
    } else {
        a.nmod = 1;
        a.mod[0] = a.mod[1] = mg;
        a.out[0] = a.out[1] = G;
        err = launch_gemv(a, s, true);
        if (err == cudaSuccess) {
            a.mod[0] = a.mod[1] = mu;
            a.min_units = p.pu.min_units;
            a.out[0] = a.out[1] = U;
            err = launch_gemv(a, s, true);
        }
    }
    if (err != cudaSuccess)
        return VQ_ERR_CUDA;

    trace_point(2, s);
    err = launch_swiglu(G, U, p.sa, tk * p.I, (int)tk, p.I, perm, top_k, xinv, w, h, wh, s, true);
    if (err != cudaSuccess)
        return VQ_ERR_CUDA;
    trace_point(3, s);

    GemvArgs b = a;
    const ModDev md = make_moddev(L->down);
    b.mod[0] = b.mod[1] = md;
    b.nmod = 1;
    b.act = h;
    b.act_bf16 = 0;
    b.act_by_slot = 1;
    b.act_rows = tk;
    b.slices = p.sb;
    b.min_units = p.pd.min_units;
    b.out[0] = b.out[1] = D;
    b.out_slice_stride = tk * p.H;
    err = launch_gemv(b, s, true);
    if (err != cudaSuccess)
        return VQ_ERR_CUDA;

    trace_point(4, s);
    err = launch_combine(D, p.sb, tk * p.H, wh, pos, T, top_k, p.H, y, y_dtype, s, true);
    trace_point(5, s);
    return cuda_status(err);
}

size_t vq_fit_workspace_size(int32_t K, int32_t d)
{
    if (K < 2 || K > 65536 || (d != 1 && d != 2 && d != 4 && d != 8))
        return 0;
    return fit_workspace_size(K, d);
}

vq_status vq_fit(const uint16_t *w, int32_t rows, int32_t cols, int32_t d, int32_t K, const int32_t *sample,
                 int32_t n_sample, const int32_t *init, int32_t iters, uint16_t *scales, uint16_t *codebook,
                 uint16_t *codes, void *workspace, size_t ws_bytes, void *stream)
{
    if (!w || !sample || !init || !scales || !codebook || !codes || rows < 1 || cols < 64 || cols % 64 ||
        (d != 1 && d != 2 && d != 4 && d != 8) || n_sample > (1 << 22) || (long)rows * (cols / d) >= (1L << 31))
        return VQ_ERR_ARG;
    if (!aligned(w, 16) || !aligned(scales, 16) || !aligned(codebook, 16) || !aligned(codes, 16) ||
        !aligned(sample, 4) || !aligned(init, 4))
        return VQ_ERR_ALIGN;
    if (!workspace || !aligned(workspace, 256))
        return VQ_ERR_WORKSPACE;
    return run_fit(w, rows, cols, d, K, sample, n_sample, init, iters, scales, codebook, codes, workspace, ws_bytes,
                   (cudaStream_t)stream);
}

vq_status vq_moe_check(const void *workspace, void *stream)
{
    if (!workspace || !aligned(workspace, 256))
        return VQ_ERR_WORKSPACE;
    int word = 0;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return cuda_status(e);
    return word == 0 ? VQ_OK : VQ_ERR_DEVICE_CHECK;
}

vq_status vq_moe_prefill(const vq_moe_layer *L, const uint16_t *x, int32_t T, const float *logits, int32_t top_k,
                         int32_t renorm, void *y, int32_t y_dtype, void *workspace, size_t ws_bytes, void *stream)
{
    vq_status st = check_moe_args(L, x, T, logits, top_k, y, y_dtype, workspace);
    if (st != VQ_OK)
        return st;
    return run_prefill(L, x, T, logits, top_k, renorm, y, y_dtype, workspace, ws_bytes, (cudaStream_t)stream);
}

vq_status vq_moe_prefill_chunked(const vq_moe_layer *L, const uint16_t *x, int32_t T, const float *logits,
                                 int32_t top_k, int32_t renorm, int32_t chunk, void *y, int32_t y_dtype,
                                 void *workspace, size_t ws_bytes, void *stream)
{
    vq_status st = check_moe_args(L, x, T, logits, top_k, y, y_dtype, workspace);
    if (st != VQ_OK)
        return st;
    if (chunk < 1)
        return VQ_ERR_ARG;
    const int H = L->gate.cols, E = L->gate.E;
    const size_t ybytes = y_dtype == VQ_F32 ? 4 : 2;
    for (int64_t c0 = 0; c0 < T; c0 += chunk) {
        const int32_t n = (int32_t)std::min<int64_t>(chunk, T - c0);
        st = run_prefill(L, x + (size_t)c0 * H, n, logits + (size_t)c0 * E, top_k, renorm,
                         static_cast<char *>(y) + (size_t)c0 * H * ybytes, y_dtype, workspace, ws_bytes,
                         (cudaStream_t)stream);
        if (st != VQ_OK)
            return st;
    }
    return VQ_OK;
}

}  // extern "C"
