// bwd_aux.cu -- the memory-bound passes around the backward kernel.
//   bwd_pre:     D_i = dO_i . O_i (fp32), zero the fp32 dQ accumulator and the split key tiles'
//                arrival counters, and zero dK/dV of heads whose keys are not all written by the
//                main kernel (fixed pattern-2 heads read only summary positions; every other key
//                gets no gradient).
//   dq_convert:  dQ fp32 accumulator -> output dtype (round to nearest even).
//   split_finish: dK/dV of the backward's split key tiles from their chunks' fp32 partials.
//   split:       fp32 tensor -> bf16 high part (round to nearest even) and optionally the bf16
//                low part x - hi, the operands of the split-precision products of fp32 I/O.
// Both are HBM-bound: 8 threads per 64-wide row, 16-byte accesses, grid sized to the SM count.
#include "tiles.cuh"

namespace st {
namespace {


template <bool F32>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const PreParams p)
{
    for (int32_t c = blockIdx.x * blockDim.x + threadIdx.x; c < p.ncounters; c += gridDim.x * blockDim.x)
        p.counters[c] = 0;
    const int64_t sub = threadIdx.x & 7;  // eighth of the 64-wide row
    const int64_t nthr_rows = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 3);
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 3) + (threadIdx.x >> 3);
         r < p.rows; r += nthr_rows) {
        float s;
        if (F32) {
            const float4 *a = reinterpret_cast<const float4 *>(p.o_f32 + r * 64) + 2 * sub;
            const float4 *b = reinterpret_cast<const float4 *>(p.dout_f32 + r * 64) + 2 * sub;
            const float4 a0 = a[0], a1 = a[1], b0 = b[0], b1 = b[1];
            s = a0.x * b0.x + a0.y * b0.y + a0.z * b0.z + a0.w * b0.w + a1.x * b1.x + a1.y * b1.y +
                a1.z * b1.z + a1.w * b1.w;
        } else {
            const uint4 a = reinterpret_cast<const uint4 *>(p.o + r * 64)[sub];
            const uint4 b = reinterpret_cast<const uint4 *>(p.dout + r * 64)[sub];
            s = bf16_lo(a.x) * bf16_lo(b.x) + bf16_hi(a.x) * bf16_hi(b.x) + bf16_lo(a.y) * bf16_lo(b.y) +
                bf16_hi(a.y) * bf16_hi(b.y) + bf16_lo(a.z) * bf16_lo(b.z) + bf16_hi(a.z) * bf16_hi(b.z) +
                bf16_lo(a.w) * bf16_lo(b.w) + bf16_hi(a.w) * bf16_hi(b.w);
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        if (sub == 0) p.delta[r] = s;
        float4 *acc = reinterpret_cast<float4 *>(p.dq_acc + r * 64);
        acc[2 * sub] = make_float4(0.f, 0.f, 0.f, 0.f);
        acc[2 * sub + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
        const int32_t h = static_cast<int32_t>((r / p.n) % p.heads);
        if (p.zero_fill[h]) {
            if (F32) {
                float4 *k4 = reinterpret_cast<float4 *>(p.dk_f32 + r * 64) + 2 * sub;
                float4 *v4 = reinterpret_cast<float4 *>(p.dv_f32 + r * 64) + 2 * sub;
                k4[0] = k4[1] = v4[0] = v4[1] = make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                reinterpret_cast<uint4 *>(p.dk + r * 64)[sub] = make_uint4(0, 0, 0, 0);
                reinterpret_cast<uint4 *>(p.dv + r * 64)[sub] = make_uint4(0, 0, 0, 0);
            }
        }
    }
}

template <bool F32>
__global__ void __launch_bounds__(256) dq_convert_kernel(const ConvParams p)
{
    const int64_t n8 = p.elems / 8;
    for (int64_t a = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; a < n8;
         a += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 x = reinterpret_cast<const float4 *>(p.dq_acc)[2 * a];
        const float4 y = reinterpret_cast<const float4 *>(p.dq_acc)[2 * a + 1];
        if (F32) {
            reinterpret_cast<float4 *>(p.dq_f32)[2 * a] = x;
            reinterpret_cast<float4 *>(p.dq_f32)[2 * a + 1] = y;
        } else {
            reinterpret_cast<uint4 *>(p.dq)[a] = make_uint4(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w),
                                                            pack_bf16(y.x, y.y), pack_bf16(y.z, y.w));
        }
    }
}

__device__ __forceinline__ float bf16_round(float x) { return bf16_lo(pack_bf16(x, 0.f)); }

__global__ void __launch_bounds__(256) split_kernel(const SplitParams p)
{
    const int64_t n8 = p.elems / 8;
    for (int64_t a = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; a < n8;
         a += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 x = reinterpret_cast<const float4 *>(p.src)[2 * a];
        const float4 y = reinterpret_cast<const float4 *>(p.src)[2 * a + 1];
        reinterpret_cast<uint4 *>(p.hi)[a] =
            make_uint4(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w), pack_bf16(y.x, y.y), pack_bf16(y.z, y.w));
        if (p.lo) {
            const float v[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
            float r[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) r[e] = v[e] - bf16_round(v[e]);
            reinterpret_cast<uint4 *>(p.lo)[a] = make_uint4(pack_bf16(r[0], r[1]), pack_bf16(r[2], r[3]),
                                                            pack_bf16(r[4], r[5]), pack_bf16(r[6], r[7]));
        }
    }
}

// One block of 512 threads per (split key tile, batch element, matrix): thread t owns row t % 128,
// columns 16 (t / 128) .. of dK or dV; the chunks' partials are added in chunk order (a fixed
// order: the result does not depend on which chunk finished first), up to four chunks' loads in
// flight at a time.  A slot holds, for each of dK, dV, the 16-byte group q (0..3) of the
// 16-column slice g (0..3) of row r at uint4 ((which * 4 + q) * 4 + g) * 128 + r (the order the
// backward kernel's threads write it in, so that each warp reads 512 contiguous bytes here).
template <bool F32>
__global__ void __launch_bounds__(512) split_finish_kernel(const SplitFinishParams p)
{
    const int32_t which = blockIdx.x & 1, rb = blockIdx.x >> 1;
    const int32_t rec_i = rb / p.batch, b = rb - rec_i * p.batch;
    const SplitRec rec = p.recs[rec_i];
    const Part part = p.parts[rec.part];
    const int32_t row = threadIdx.x & 127, g = threadIdx.x >> 7;
    const int32_t pos = frame_pos(p.g, part.kframe, part.o, rec.tile, row);
    if (pos < 0) return;
    constexpr size_t SLOT4 = 2 * 128 * 64 / 4;  // a slot, in float4
    float a[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) a[e] = 0.f;
    const float4 *base = reinterpret_cast<const float4 *>(p.partials) + ((which * 4) * 4 + g) * 128 + row;
    for (int32_t c0 = 0; c0 < rec.nsplit; c0 += 4) {
        float4 x[4][4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (c0 + c < rec.nsplit) {
                const float4 *src = base + (static_cast<size_t>(rec.first + c0 + c) * p.batch + b) * SLOT4;
#pragma unroll
                for (int q = 0; q < 4; ++q) x[c][q] = src[q * 4 * 128];
            }
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (c0 + c < rec.nsplit)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    a[4 * q] += x[c][q].x;
                    a[4 * q + 1] += x[c][q].y;
                    a[4 * q + 2] += x[c][q].z;
                    a[4 * q + 3] += x[c][q].w;
                }
    }
    const size_t out = (static_cast<size_t>(b * p.heads + part.head) * p.g.n + pos) * 64 + 16 * g;
    if (F32) {
        float4 *d4 = reinterpret_cast<float4 *>((which == 0 ? p.dk_f32 : p.dv_f32) + out);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4 v = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
            if (part.merge) {  // add the first pass's values
                const float4 y = d4[q];
                v.x += y.x;
                v.y += y.y;
                v.z += y.z;
                v.w += y.w;
            }
            d4[q] = v;
        }
    } else {
        uint4 *d4 = reinterpret_cast<uint4 *>((which == 0 ? p.dk : p.dv) + out);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            if (part.merge) {
                const uint4 y = d4[q];
                const uint32_t yy[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    a[8 * q + 2 * e] += bf16_lo(yy[e]);
                    a[8 * q + 2 * e + 1] += bf16_hi(yy[e]);
                }
            }
            d4[q] = make_uint4(pack_bf16(a[8 * q], a[8 * q + 1]), pack_bf16(a[8 * q + 2], a[8 * q + 3]),
                               pack_bf16(a[8 * q + 4], a[8 * q + 5]), pack_bf16(a[8 * q + 6], a[8 * q + 7]));
        }
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

int blocks_for(int64_t work_units)
{
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    return static_cast<int>(work_units < cap ? (work_units > 0 ? work_units : 1) : cap);
}

cudaError_t launch_bwd_pre(const PreParams &p, bool f32, cudaStream_t s)
{
    const int blocks = blocks_for((p.rows + 31) / 32);
    if (f32)
        bwd_pre_kernel<true><<<blocks, 256, 0, s>>>(p);
    else
        bwd_pre_kernel<false><<<blocks, 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_dq_convert(const ConvParams &p, bool f32, cudaStream_t s)
{
    const int blocks = blocks_for((p.elems / 8 + 255) / 256);
    if (f32)
        dq_convert_kernel<true><<<blocks, 256, 0, s>>>(p);
    else
        dq_convert_kernel<false><<<blocks, 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_split(const SplitParams &p, cudaStream_t s)
{
    split_kernel<<<blocks_for((p.elems / 8 + 255) / 256), 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_split_finish(const SplitFinishParams &p, bool f32, cudaStream_t s)
{
    if (p.nrecs == 0) return cudaSuccess;
    const unsigned blocks = static_cast<unsigned>(p.nrecs) * p.batch * 2;
    if (f32)
        split_finish_kernel<true><<<blocks, 512, 0, s>>>(p);
    else
        split_finish_kernel<false><<<blocks, 512, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace st
