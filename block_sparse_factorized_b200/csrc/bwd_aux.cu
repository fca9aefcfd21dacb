// bwd_aux.cu -- the memory-bound passes around the backward kernel.
//   bwd_pre:     D_i = dO_i . O_i (fp32), zero the fp32 dQ accumulator (of heads whose dQ the main
//                kernel does not write directly) and the work counters, and zero dK/dV of heads
//                whose keys are not all written by the main kernel (fixed pattern-2 heads read
//                only summary positions; every other key gets no gradient).
//   dq_convert:  dQ fp32 accumulator -> output dtype (round to nearest even), same heads.
//   split_finish: dK/dV of the backward's split key tiles from their chunks' fp32 partials.
//   split:       fp32 tensor -> bf16 high part (round to nearest even) and optionally the bf16
//                low part x - hi, the operands of the split-precision products of fp32 I/O.
// Both are HBM-bound: 8 threads per 64-wide row, 16-byte accesses, grid sized to the SM count.
#include "tiles.cuh"

namespace st {
namespace {


// Rows (of 64 values) each thread of the two passes below handles, their loads issued together:
// with one 16- or 32-byte load per thread in flight the passes stop well short of HBM bandwidth.
constexpr int UNROLL = 4;

// Grid: x over chunks of 32 UNROLL rows of one batch-head, y over batch-heads (grid-stride both
// ways), so that the per-head flags are read once per block.  Thread: one eighth (8 values) of
// UNROLL rows 32 apart.
template <bool F32>
__global__ void __launch_bounds__(256, 4) bwd_pre_kernel(const PreParams p)
{
    constexpr int U = F32 ? 2 : UNROLL;  // fp32 rows: half as many per thread, in registers
    if (blockIdx.x == 0 && blockIdx.y == 0)
        for (int32_t c = threadIdx.x; c < p.ncounters; c += blockDim.x) p.counters[c] = 0;
    const int32_t sub = threadIdx.x & 7;  // eighth of the 64-wide row
    const int32_t rpb = blockDim.x >> 3;
    for (int64_t bh = blockIdx.y; bh < p.bh; bh += gridDim.y) {
        const int32_t flags = p.head_flags[bh % p.heads];
        const bool zero_dq = (flags & HEAD_DQ_DIRECT) == 0, zero_kv = (flags & HEAD_ZERO_FILL) != 0;
        for (int32_t r0 = blockIdx.x * rpb * U + (threadIdx.x >> 3); r0 < p.n; r0 += gridDim.x * rpb * U) {
            float s[U];
            if (F32) {
                float4 a[U][2], b[U][2];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (r0 + u * rpb < p.n) {
                        const int64_t r = bh * p.n + r0 + u * rpb;
                        const float4 *pa = reinterpret_cast<const float4 *>(p.o_f32 + r * 64) + 2 * sub;
                        const float4 *pb = reinterpret_cast<const float4 *>(p.dout_f32 + r * 64) + 2 * sub;
                        a[u][0] = pa[0];
                        a[u][1] = pa[1];
                        b[u][0] = pb[0];
                        b[u][1] = pb[1];
                    }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    s[u] = 0.f;
                    if (r0 + u * rpb < p.n)
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            s[u] += a[u][h].x * b[u][h].x + a[u][h].y * b[u][h].y + a[u][h].z * b[u][h].z +
                                    a[u][h].w * b[u][h].w;
                }
            } else {
                uint4 a[U], b[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (r0 + u * rpb < p.n) {
                        const int64_t r = bh * p.n + r0 + u * rpb;
                        a[u] = reinterpret_cast<const uint4 *>(p.o + r * 64)[sub];
                        b[u] = reinterpret_cast<const uint4 *>(p.dout + r * 64)[sub];
                    }
#pragma unroll
                for (int u = 0; u < U; ++u)
                    s[u] = (r0 + u * rpb < p.n)
                               ? bf16_lo(a[u].x) * bf16_lo(b[u].x) + bf16_hi(a[u].x) * bf16_hi(b[u].x) +
                                     bf16_lo(a[u].y) * bf16_lo(b[u].y) + bf16_hi(a[u].y) * bf16_hi(b[u].y) +
                                     bf16_lo(a[u].z) * bf16_lo(b[u].z) + bf16_hi(a[u].z) * bf16_hi(b[u].z) +
                                     bf16_lo(a[u].w) * bf16_lo(b[u].w) + bf16_hi(a[u].w) * bf16_hi(b[u].w)
                               : 0.f;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {  // the 8 threads of a row sum their eighths
                s[u] += __shfl_xor_sync(0xffffffffu, s[u], 1);
                s[u] += __shfl_xor_sync(0xffffffffu, s[u], 2);
                s[u] += __shfl_xor_sync(0xffffffffu, s[u], 4);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (r0 + u * rpb >= p.n) continue;
                const int64_t r = bh * p.n + r0 + u * rpb;
                if (sub == 0) p.delta[r] = s[u];
                if (zero_dq) {
                    float4 *acc = reinterpret_cast<float4 *>(p.dq_acc + r * 64);
                    acc[2 * sub] = make_float4(0.f, 0.f, 0.f, 0.f);
                    acc[2 * sub + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                if (zero_kv) {
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
    }
}

// Grid: x over chunks of one batch-head, y over (batch, accumulated head) pairs only -- the
// heads whose dQ the main kernel stores directly get no block.  A thread converts UNROLL groups of
// 8 consecutive values, 256 groups apart.
template <bool F32>
__global__ void __launch_bounds__(256, 4) dq_convert_kernel(const ConvParams p)
{
    const int64_t n8 = static_cast<int64_t>(p.n) * 8;  // 8-value groups per batch-head
    const int64_t pairs = static_cast<int64_t>(p.batch) * p.nacc;
    for (int64_t y = blockIdx.y; y < pairs; y += gridDim.y) {
        const int64_t b = y / p.nacc;
        const int64_t bh = b * p.heads + p.acc_head[y - b * p.nacc];
        const float4 *src = reinterpret_cast<const float4 *>(p.dq_acc) + bh * n8 * 2;
        for (int64_t a0 = static_cast<int64_t>(blockIdx.x) * blockDim.x * UNROLL + threadIdx.x; a0 < n8;
             a0 += static_cast<int64_t>(gridDim.x) * blockDim.x * UNROLL) {
            float4 x[UNROLL], y[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int64_t a = a0 + u * static_cast<int64_t>(blockDim.x);
                if (a < n8) {
                    x[u] = src[2 * a];
                    y[u] = src[2 * a + 1];
                }
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int64_t a = a0 + u * static_cast<int64_t>(blockDim.x);
                if (a >= n8) continue;
                const int64_t e = bh * n8 + a;
                if (F32) {
                    reinterpret_cast<float4 *>(p.dq_f32)[2 * e] = x[u];
                    reinterpret_cast<float4 *>(p.dq_f32)[2 * e + 1] = y[u];
                } else {
                    reinterpret_cast<uint4 *>(p.dq)[e] =
                        make_uint4(pack_bf16(x[u].x, x[u].y), pack_bf16(x[u].z, x[u].w), pack_bf16(y[u].x, y[u].y),
                                   pack_bf16(y[u].z, y[u].w));
                }
            }
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

}  // namespace

int sm_count()
{
    constexpr int MAXDEV = 64;
    static int count[MAXDEV] = {};  // per device, filled on first use
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
    if (dev >= MAXDEV) dev = MAXDEV - 1;
    if (count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        count[dev] = n;
    }
    return count[dev];
}

int blocks_for(int64_t work_units)
{
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    return static_cast<int>(work_units < cap ? (work_units > 0 ? work_units : 1) : cap);
}

// x: chunks of one batch-head's rows (at most 4096 blocks), y: batch-heads (at most 65535)
static dim3 head_grid(int64_t chunks, int64_t bh)
{
    const int64_t x = chunks < 1 ? 1 : (chunks > 4096 ? 4096 : chunks);
    const int64_t y = bh < 1 ? 1 : (bh > 65535 ? 65535 : bh);
    return dim3(static_cast<unsigned>(x), static_cast<unsigned>(y));
}

cudaError_t launch_bwd_pre(const PreParams &p, bool f32, cudaStream_t s)
{
    const dim3 grid = head_grid((p.n + 32 * UNROLL - 1) / (32 * UNROLL), p.bh);
    if (f32)
        bwd_pre_kernel<true><<<grid, 256, 0, s>>>(p);
    else
        bwd_pre_kernel<false><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_dq_convert(const ConvParams &p, bool f32, cudaStream_t s)
{
    if (p.nacc == 0) return cudaSuccess;
    const dim3 grid = head_grid((static_cast<int64_t>(p.n) * 8 + 256 * UNROLL - 1) / (256 * UNROLL),
                                static_cast<int64_t>(p.batch) * p.nacc);
    if (f32)
        dq_convert_kernel<true><<<grid, 256, 0, s>>>(p);
    else
        dq_convert_kernel<false><<<grid, 256, 0, s>>>(p);
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
