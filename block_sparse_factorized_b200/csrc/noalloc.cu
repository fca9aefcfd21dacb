// noalloc.cu -- backward pass for callers that cannot allocate device memory.
//
// st_attn_bwd needs a workspace (the fp32 dQ accumulator and the per-row D_i) that the caller
// allocates.  Some callers cannot: a plug-in running inside a host application that owns every
// device allocation (a serving process with a fixed memory budget, a framework whose pool must
// not be bypassed), or code on a latency-critical path where cudaMalloc's implicit device
// synchronisation is not acceptable.  st_attn_bwd_noalloc gives them the same backward pass with
// the workspace taken from a fixed array that is part of this library's device image.
//
// The array has a fixed size (ST_NOALLOC_SCRATCH_BYTES) and every GPU that loads the library
// holds it until the process exits.  All calls on a device share it and it keeps the last call's
// contents; the prepare phase rewrites everything the main phase reads (the dQ accumulator is
// zeroed, D recomputed), so no state leaks from one call to the next.  Two calls whose work
// overlaps on the GPU (different streams, or another thread) race on the array.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/st_attn.h"

namespace {

// The scratch array itself.  In host code `scratch` names a host-side stand-in, not a device
// address: the device address comes from cudaGetSymbolAddress, once per device and context.
static __device__ __align__(256) unsigned char scratch[ST_NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex scratch_mutex;
void *scratch_ptr[MAX_DEVICES] = {};
unsigned long long scratch_ctx[MAX_DEVICES] = {};  // context id the address belongs to

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

template <typename F>
F driver_fn(const char *name)
{
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<F>(ptr);
    return nullptr;
}

// Process-unique id of the current context (ids are never reused, unlike context handles), so
// that an address looked up before a cudaDeviceReset is not reused in the context that follows.
st_status_t current_context_id(unsigned long long *id)
{
    static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!get_current || !get_id) return ST_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return ST_ERR_CUDA;
    return get_id(ctx, id) == CUDA_SUCCESS ? ST_OK : ST_ERR_CUDA;
}

// Device address of `scratch` on the current device; looked up on the first call per device
// (and again on the first call after that device's context was replaced).
st_status_t scratch_address(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ST_ERR_CUDA;
    if (dev < 0 || dev >= MAX_DEVICES) return ST_ERR_UNSUPPORTED;
    if (cudaSetDevice(dev) != cudaSuccess) return ST_ERR_CUDA;  // makes the device's primary context current
    unsigned long long ctx = 0;
    const st_status_t s = current_context_id(&ctx);
    if (s != ST_OK) return s;
    std::lock_guard<std::mutex> lock(scratch_mutex);
    if (!scratch_ptr[dev] || scratch_ctx[dev] != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, scratch) != cudaSuccess || !p) return ST_ERR_CUDA;
        scratch_ptr[dev] = p;
        scratch_ctx[dev] = ctx;
    }
    *out = scratch_ptr[dev];
    return ST_OK;
}

}  // namespace

extern "C" st_status_t st_attn_bwd_noalloc(const void *q, const void *k, const void *v,
                                           const void *o, const float *lse, const void *dO,
                                           const st_layout_t *layout, void *dq, void *dk, void *dv,
                                           const st_desc_t *desc, st_stream_t stream)
{
    if (!desc || !layout) return ST_ERR_INVALID_ARG;
    const size_t need = st_attn_bwd_workspace_bytes(desc, layout);
    if (need == 0) return ST_ERR_INVALID_ARG;
    if (need > ST_NOALLOC_SCRATCH_BYTES) return ST_ERR_WORKSPACE;
    void *ws = nullptr;
    const st_status_t s = scratch_address(&ws);
    if (s != ST_OK) return s;
    return st_attn_bwd(q, k, v, o, lse, dO, layout, dq, dk, dv, ws, need, desc, stream);
}
