// vq_moe_decode_noalloc: the decode layer for callers that cannot allocate
// device memory.
//
// Some callers have no way to call cudaMalloc: a host framework that owns
// every device allocation and forbids new ones on its serving path, or a
// program that reaches this library through a thin C FFI with no CUDA memory
// API of its own. For them this entry point takes only inputs and outputs;
// the decode path's scratch (routing tables, fp16 activations, partial sums)
// lives in one file-scope device array, VQ_STATIC_SCRATCH_BYTES large, that
// every GPU which loads the library holds until the process exits.
//
// The array's host-side name is only a stand-in for its device address, so
// the address is looked up with cudaGetSymbolAddress (with the device
// current) on the first call made on each device, and that address is what
// the kernels receive. The cached address belongs to the device's CUDA
// context: it is looked up again when the context has changed since (for
// instance after cudaDeviceReset, which destroys the context and with it the
// array's storage).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "vq_internal.h"

namespace {

constexpr size_t VQ_STATIC_SCRATCH_BYTES = (size_t)16 << 20;   // 16 MiB
constexpr int MAX_DEVICES = 64;

static __device__ __align__(256) unsigned char g_vq_scratch[VQ_STATIC_SCRATCH_BYTES];

struct ScratchSlot {
    void *ptr = nullptr;
    unsigned long long ctx_id = 0;   // context the address belongs to
};

std::mutex g_scratch_mu;
ScratchSlot g_scratch[MAX_DEVICES];

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Id of the calling thread's current context, 0 when there is none or the
// driver cannot say (the address is then looked up again).
unsigned long long current_ctx_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
        resolved = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of g_vq_scratch in the current device's context.
vq_status scratch_on_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return VQ_ERR_CUDA;
    if (dev < 0 || dev >= MAX_DEVICES)
        return VQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchSlot &slot = g_scratch[dev];
    const unsigned long long id = current_ctx_id();
    if (!slot.ptr || id == 0 || id != slot.ctx_id) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_vq_scratch) != cudaSuccess || !p)
            return VQ_ERR_CUDA;
        slot.ptr = p;
        slot.ctx_id = current_ctx_id();   // the lookup has made the context current
    }
    *out = slot.ptr;
    return VQ_OK;
}

}  // namespace

extern "C" vq_status vq_moe_decode_noalloc(const vq_moe_layer *L, const uint16_t *x, int32_t T, const float *logits,
                                           int32_t top_k, int32_t renorm, void *y, int32_t y_dtype, void *stream)
{
    const size_t need = vq_moe_workspace_size(L, T, top_k, VQ_MODE_DECODE);
    if (need == 0)
        return VQ_ERR_ARG;         // invalid layer, T or top_k: no CUDA state is touched
    if (need > VQ_STATIC_SCRATCH_BYTES)
        return VQ_ERR_WORKSPACE;   // this batch needs more scratch than the static array holds
    void *scratch = nullptr;
    const vq_status st = scratch_on_current_device(&scratch);
    if (st != VQ_OK)
        return st;
    // the workspace path validates every argument and writes everything it reads
    return vq_moe_decode(L, x, T, logits, top_k, renorm, y, y_dtype, scratch, VQ_STATIC_SCRATCH_BYTES, stream);
}
