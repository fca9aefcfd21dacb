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
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/st_attn.h"

namespace {

// The scratch array itself.  In host code `scratch` names a host-side stand-in, not a device
// address: the device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char scratch[ST_NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex scratch_mutex;
void *scratch_ptr[MAX_DEVICES] = {};

// Device address of `scratch` on the current device; looked up on the first call per device.
st_status_t scratch_address(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ST_ERR_CUDA;
    if (dev < 0 || dev >= MAX_DEVICES) return ST_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(scratch_mutex);
    if (!scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, scratch) != cudaSuccess || !p) return ST_ERR_CUDA;
        scratch_ptr[dev] = p;
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
