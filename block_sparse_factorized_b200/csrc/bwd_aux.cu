// bwd_aux.cu -- the memory-bound passes around the backward kernel.
//   bwd_pre:     D_i = dO_i . O_i (fp32), zero the fp32 dQ accumulator, and zero dK/dV of heads
//                whose keys are not all written by the main kernel (fixed pattern-2 heads read
//                only summary positions; every other key gets no gradient).
//   dq_convert:  dQ fp32 accumulator -> output dtype (round to nearest even).
// Both are HBM-bound: 8 threads per 64-wide row, 16-byte accesses, grid sized to the SM count.
#include "kernels.h"
#include "sm100.cuh"

namespace st {
namespace {

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

__global__ void __launch_bounds__(256) bwd_pre_kernel(const PreParams p)
{
    const int64_t sub = threadIdx.x & 7;  // 16-byte slice of the row (8 bf16)
    const int64_t nthr_rows = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 3);
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 3) + (threadIdx.x >> 3);
         r < p.rows; r += nthr_rows) {
        const uint4 a = reinterpret_cast<const uint4 *>(p.o + r * 64)[sub];
        const uint4 b = reinterpret_cast<const uint4 *>(p.dout + r * 64)[sub];
        float s = bf_lo(a.x) * bf_lo(b.x) + bf_hi(a.x) * bf_hi(b.x) + bf_lo(a.y) * bf_lo(b.y) +
                  bf_hi(a.y) * bf_hi(b.y) + bf_lo(a.z) * bf_lo(b.z) + bf_hi(a.z) * bf_hi(b.z) +
                  bf_lo(a.w) * bf_lo(b.w) + bf_hi(a.w) * bf_hi(b.w);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        if (sub == 0) p.delta[r] = s;
        float4 *acc = reinterpret_cast<float4 *>(p.dq_acc + r * 64);
        acc[2 * sub] = make_float4(0.f, 0.f, 0.f, 0.f);
        acc[2 * sub + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
        const int32_t h = static_cast<int32_t>((r / p.n) % p.heads);
        if (p.zero_fill[h]) {
            reinterpret_cast<uint4 *>(p.dk + r * 64)[sub] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4 *>(p.dv + r * 64)[sub] = make_uint4(0, 0, 0, 0);
        }
    }
}

__global__ void __launch_bounds__(256) dq_convert_kernel(const ConvParams p)
{
    const int64_t n8 = p.elems / 8;
    for (int64_t a = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; a < n8;
         a += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 x = reinterpret_cast<const float4 *>(p.dq_acc)[2 * a];
        const float4 y = reinterpret_cast<const float4 *>(p.dq_acc)[2 * a + 1];
        reinterpret_cast<uint4 *>(p.dq)[a] =
            make_uint4(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w), pack_bf16(y.x, y.y), pack_bf16(y.z, y.w));
    }
}

int sm_count()
{
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

}  // namespace

cudaError_t launch_bwd_pre(const PreParams &p, cudaStream_t s)
{
    const int64_t want = (p.rows + 31) / 32;
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    const int blocks = static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
    bwd_pre_kernel<<<blocks, 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_dq_convert(const ConvParams &p, cudaStream_t s)
{
    const int64_t want = (p.elems / 8 + 255) / 256;
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    const int blocks = static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
    dq_convert_kernel<<<blocks, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace st
