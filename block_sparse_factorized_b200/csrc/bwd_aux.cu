// bwd_aux.cu -- the memory-bound passes around the backward kernel.
//   bwd_pre:     D_i = dO_i . O_i (fp32), zero the fp32 dQ accumulator (of heads whose dQ the main
//                kernel does not write directly) and the work counters, and zero dK/dV of heads
//                whose keys are not all written by the main kernel (fixed pattern-2 heads read
//                only summary positions; every other key gets no gradient).
//   dq_convert:  dQ fp32 accumulator -> output dtype (round to nearest even), same heads.
//   split_finish: dK/dV of the backward's split key tiles from their chunks' fp32 partials.
//   split:       fp32 tensor -> bf16 high part (round to nearest even) and optionally the bf16
//                low part x - hi, the operands of the split-precision products of fp32 I/O.
// All are HBM-bound: 8 threads per row, 8- to 32-byte accesses, grid sized to the SM count.
#include "tiles.cuh"

namespace st {
namespace {


// Rows each thread of the two passes below handles, their loads issued together: with one 16-
// or 32-byte load per thread in flight the passes stop well short of HBM bandwidth.
constexpr int UNROLL = 4;

// N bf16 values of a row (an eighth of a row of 8 N), loaded as one 8-byte word (N = 4) or N / 8
// 16-byte words, as bf16 pairs.
template <int N>
struct Bf16Slice {
    static_assert(N == 4 || N % 8 == 0, "slice width");
    uint32_t w[N / 2];
    __device__ __forceinline__ void load(const uint16_t *src)
    {
        if constexpr (N == 4) {
            const uint2 x = *reinterpret_cast<const uint2 *>(src);
            w[0] = x.x;
            w[1] = x.y;
        } else {
#pragma unroll
            for (int l = 0; l < N / 8; ++l) {
                const uint4 x = reinterpret_cast<const uint4 *>(src)[l];
                w[4 * l] = x.x;
                w[4 * l + 1] = x.y;
                w[4 * l + 2] = x.z;
                w[4 * l + 3] = x.w;
            }
        }
    }
};

template <int N>
__device__ __forceinline__ void zero_bf16(uint16_t *dst)
{
    if constexpr (N == 4) {
        *reinterpret_cast<uint2 *>(dst) = make_uint2(0u, 0u);
    } else {
#pragma unroll
        for (int l = 0; l < N / 8; ++l) reinterpret_cast<uint4 *>(dst)[l] = make_uint4(0u, 0u, 0u, 0u);
    }
}

template <int N>
__device__ __forceinline__ void zero_f32(float *dst)
{
#pragma unroll
    for (int l = 0; l < N / 4; ++l) reinterpret_cast<float4 *>(dst)[l] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// Grid: x over chunks of 32 UNROLL rows of one batch-head, y over batch-heads (grid-stride both
// ways), so that the per-head flags are read once per block.  Thread: one eighth of UNROLL rows 32
// apart (DV / 8 values of O and dO; DQK / 8 of the dQ accumulator and dK, DV / 8 of dV).
template <bool F32, int DQK, int DV>
__global__ void __launch_bounds__(256, 4) bwd_pre_kernel(const PreParams p)
{
    constexpr int U = (F32 || DV > 64) ? 2 : UNROLL;  // wide (fp32 or 128-value) rows: half as many per thread
    constexpr int EQ = DQK / 8, EV = DV / 8;
    if (blockIdx.x == 0 && blockIdx.y == 0)
        for (int32_t c = threadIdx.x; c < p.ncounters; c += blockDim.x) p.counters[c] = 0;
    const int32_t sub = threadIdx.x & 7;  // eighth of the row
    const int32_t rpb = blockDim.x >> 3;
    for (int64_t bh = blockIdx.y; bh < p.bh; bh += gridDim.y) {
        const int32_t flags = p.head_flags[bh % p.heads];
        const bool zero_dq = (flags & HEAD_DQ_DIRECT) == 0, zero_kv = (flags & HEAD_ZERO_FILL) != 0;
        for (int32_t r0 = blockIdx.x * rpb * U + (threadIdx.x >> 3); r0 < p.n; r0 += gridDim.x * rpb * U) {
            float s[U];
            if constexpr (F32) {
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
                Bf16Slice<EV> a[U], b[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (r0 + u * rpb < p.n) {
                        const int64_t r = bh * p.n + r0 + u * rpb;
                        a[u].load(p.o + r * DV + EV * sub);
                        b[u].load(p.dout + r * DV + EV * sub);
                    }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float acc = 0.f;
                    if (r0 + u * rpb < p.n)
#pragma unroll
                        for (int e = 0; e < EV / 2; ++e)
                            acc += bf16_lo(a[u].w[e]) * bf16_lo(b[u].w[e]) + bf16_hi(a[u].w[e]) * bf16_hi(b[u].w[e]);
                    s[u] = acc;
                }
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
                if (zero_dq) zero_f32<EQ>(p.dq_acc + r * DQK + EQ * sub);
                if (zero_kv) {
                    if constexpr (F32) {
                        zero_f32<8>(p.dk_f32 + r * 64 + 8 * sub);
                        zero_f32<8>(p.dv_f32 + r * 64 + 8 * sub);
                    } else {
                        zero_bf16<EQ>(p.dk + r * DQK + EQ * sub);
                        zero_bf16<EV>(p.dv + r * DV + EV * sub);
                    }
                }
            }
        }
    }
}

// Grid: x over chunks of one batch-head, y over (batch, accumulated head) pairs only -- the
// heads whose dQ the main kernel stores directly get no block.  A thread converts UNROLL groups of
// 8 consecutive values, 256 groups apart (rows of DQK values, DQK / 8 groups each).
template <bool F32, int DQK>
__global__ void __launch_bounds__(256, 4) dq_convert_kernel(const ConvParams p)
{
    const int64_t n8 = static_cast<int64_t>(p.n) * (DQK / 8);  // 8-value groups per batch-head
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

// One block of 512 threads per (split key tile, batch element, matrix): thread t owns row t % 128
// and the W / 4 ... columns of slice g = t / 128 of dK (W = DQK) or dV (W = DV); the chunks'
// partials are added in chunk order (a fixed order: the result does not depend on which chunk
// finished first), up to four (two for slices wider than 16) chunks' loads in flight at a time.  A slot holds dK's 16-byte group
// q of slice g of row r at uint4 (q * 4 + g) * 128 + r, then dV's the same way (DQK * 32 uint4
// further) -- the order the backward kernel's threads write it in, so that each warp reads 512
// contiguous bytes here.
template <bool F32, int W>
__device__ __forceinline__ void split_finish_one(const SplitFinishParams &p, const SplitRec &rec, const Part &part,
                                                 int32_t b, int32_t row, int32_t g, int32_t pos, size_t slot4,
                                                 size_t part0, uint16_t *out, float *out_f32)
{
    float a[W];
#pragma unroll
    for (int e = 0; e < W; ++e) a[e] = 0.f;
    const float4 *base = reinterpret_cast<const float4 *>(p.partials) + part0 + g * 128 + row;
    constexpr int CB = W > 16 ? 2 : 4;  // chunks whose loads are in flight together (registers)
    for (int32_t c0 = 0; c0 < rec.nsplit; c0 += CB) {
        float4 x[CB][W / 4];
#pragma unroll
        for (int c = 0; c < CB; ++c)
            if (c0 + c < rec.nsplit) {
                const float4 *src = base + (static_cast<size_t>(rec.first + c0 + c) * p.batch + b) * slot4;
#pragma unroll
                for (int q = 0; q < W / 4; ++q) x[c][q] = src[q * 4 * 128];
            }
#pragma unroll
        for (int c = 0; c < CB; ++c)
            if (c0 + c < rec.nsplit)
#pragma unroll
                for (int q = 0; q < W / 4; ++q) {
                    a[4 * q] += x[c][q].x;
                    a[4 * q + 1] += x[c][q].y;
                    a[4 * q + 2] += x[c][q].z;
                    a[4 * q + 3] += x[c][q].w;
                }
    }
    const size_t out_off = (static_cast<size_t>(b * p.heads + part.head) * p.g.n + pos) * (4 * W) + W * g;
    if constexpr (F32) {
        float4 *d4 = reinterpret_cast<float4 *>(out_f32 + out_off);
#pragma unroll
        for (int q = 0; q < W / 4; ++q) {
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
        uint4 *d4 = reinterpret_cast<uint4 *>(out + out_off);
#pragma unroll
        for (int q = 0; q < W / 8; ++q) {
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

template <bool F32, int DQK, int DV>
__global__ void __launch_bounds__(512) split_finish_kernel(const SplitFinishParams p)
{
    const int32_t which = blockIdx.x & 1, rb = blockIdx.x >> 1;
    const int32_t rec_i = rb / p.batch, b = rb - rec_i * p.batch;
    const SplitRec rec = p.recs[rec_i];
    const Part part = p.parts[rec.part];
    const int32_t row = threadIdx.x & 127, g = threadIdx.x >> 7;
    const int32_t pos = frame_pos(p.g, part.kframe, part.o, rec.tile, row);
    if (pos < 0) return;
    constexpr size_t SLOT4 = static_cast<size_t>(128) * (DQK + DV) / 4;  // a slot, in float4
    if (which == 0)
        split_finish_one<F32, DQK / 4>(p, rec, part, b, row, g, pos, SLOT4, 0, p.dk, p.dk_f32);
    else
        split_finish_one<F32, DV / 4>(p, rec, part, b, row, g, pos, SLOT4, static_cast<size_t>(DQK) * 32, p.dv,
                                      p.dv_f32);
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

cudaError_t launch_bwd_pre(const PreParams &p, bool f32, int dqk, int dv, cudaStream_t s)
{
    const dim3 grid = head_grid((p.n + 32 * UNROLL - 1) / (32 * UNROLL), p.bh);
    if (f32 && dqk == 64 && dv == 64)
        bwd_pre_kernel<true, 64, 64><<<grid, 256, 0, s>>>(p);
    else if (!f32 && dqk == 64 && dv == 64)
        bwd_pre_kernel<false, 64, 64><<<grid, 256, 0, s>>>(p);
    else if (!f32 && dqk == 32 && dv == 32)
        bwd_pre_kernel<false, 32, 32><<<grid, 256, 0, s>>>(p);
    else if (!f32 && dqk == 64 && dv == 128)
        bwd_pre_kernel<false, 64, 128><<<grid, 256, 0, s>>>(p);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_dq_convert(const ConvParams &p, bool f32, int dqk, cudaStream_t s)
{
    if (p.nacc == 0) return cudaSuccess;
    const dim3 grid = head_grid((static_cast<int64_t>(p.n) * (dqk / 8) + 256 * UNROLL - 1) / (256 * UNROLL),
                                static_cast<int64_t>(p.batch) * p.nacc);
    if (f32 && dqk == 64)
        dq_convert_kernel<true, 64><<<grid, 256, 0, s>>>(p);
    else if (!f32 && dqk == 64)
        dq_convert_kernel<false, 64><<<grid, 256, 0, s>>>(p);
    else if (!f32 && dqk == 32)
        dq_convert_kernel<false, 32><<<grid, 256, 0, s>>>(p);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_split(const SplitParams &p, cudaStream_t s)
{
    split_kernel<<<blocks_for((p.elems / 8 + 255) / 256), 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_split_finish(const SplitFinishParams &p, bool f32, int dqk, int dv, cudaStream_t s)
{
    if (p.nrecs == 0) return cudaSuccess;
    const unsigned blocks = static_cast<unsigned>(p.nrecs) * p.batch * 2;
    if (f32 && dqk == 64 && dv == 64)
        split_finish_kernel<true, 64, 64><<<blocks, 512, 0, s>>>(p);
    else if (!f32 && dqk == 64 && dv == 64)
        split_finish_kernel<false, 64, 64><<<blocks, 512, 0, s>>>(p);
    else if (!f32 && dqk == 32 && dv == 32)
        split_finish_kernel<false, 32, 32><<<blocks, 512, 0, s>>>(p);
    else if (!f32 && dqk == 64 && dv == 128)
        split_finish_kernel<false, 64, 128><<<blocks, 512, 0, s>>>(p);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace st
