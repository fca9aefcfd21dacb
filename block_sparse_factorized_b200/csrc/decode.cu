// decode.cu -- decode step on sm_100a: one new query row per (batch, head) at position pos against
// the key/value cache rows 0..pos.
//
// "长序列为何不必让每个 token 看见全部历史？…" §11: in incremental decoding each step brings one new query
// row against the cached keys and values plus the new one (Q_LEN = 1, KV_LEN = pos + 1).  The row's
// allowed set is the pattern's A(h, pos) ("Sparse Transformers（稀疏 Transformer）深度解读报告" §2.2;
// a subset of {j <= pos}, §2.1), so the result is row pos of the forward pass.  The work is a
// gather of |A(h, pos)| key and value rows (about l + n/l of them) and a softmax over their scores:
// HBM-bound, no contraction to put on the tensor cores.  Scores and the softmax are computed in
// fp32 (the pages compute Q K^T in fp32 when sampling, §3.6).
//
// Every allowed set is a grid of runs followed by a contiguous range (KeySet, decode.h).  The keys of one
// (batch, head) are split into chunks of DEC_CHUNK = 64 over the CTAs of grid row y; a CTA of 128
// threads works as 16 groups of 8 lanes, a group taking 4 keys with each lane holding an eighth of
// the query-key row (d / 8 components) and of the value row (dv / 8).  All K and V loads of a chunk
// are issued before any is used (the work is one round trip to memory, not a chain of them); then
// scores, their maximum and 2^(s - M) v.  Each CTA leaves (M, L, O) of its chunk in the workspace and
// counts itself in the (batch, head)'s counter; the CTA that completes the count combines the
// chunks by log-sum-exp weights -- one launch per step, the counters zeroed before it.
#include "decode.h"
#include "tiles.cuh"

namespace st {
namespace {

constexpr int DEC_THREADS = 128;
constexpr int DEC_GROUPS = DEC_THREADS / 8;

// Elements N * lane8 .. N * lane8 + N - 1 of row `row` of a [rows, W] tensor, widened to fp32
// (N = W / 8: 4, 8 or 16 elements, one to four 8- or 16-byte loads).
template <bool F32, int W>
__device__ __forceinline__ void load_part(const void *base, int64_t row, int lane8, float (&x)[W / 8])
{
    constexpr int N = W / 8;
    if (F32) {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(base) + row * W + N * lane8);
#pragma unroll
        for (int e = 0; e < N / 4; ++e) {
            const float4 a = p[e];
            x[4 * e] = a.x; x[4 * e + 1] = a.y; x[4 * e + 2] = a.z; x[4 * e + 3] = a.w;
        }
    } else if (N == 4) {
        const uint2 a = *reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(base) + row * W + N * lane8);
        x[0] = bf16_lo(a.x); x[1] = bf16_hi(a.x); x[2] = bf16_lo(a.y); x[3] = bf16_hi(a.y);
    } else {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(base) + row * W + N * lane8);
#pragma unroll
        for (int e = 0; e < N / 8; ++e) {
            const uint4 a = p[e];
            const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                x[8 * e + 2 * t] = bf16_lo(w[t]);
                x[8 * e + 2 * t + 1] = bf16_hi(w[t]);
            }
        }
    }
}

template <bool F32, int D, int DV>
__global__ void __launch_bounds__(DEC_THREADS) decode_kernel(const DecodeParams p)
{
    constexpr int KPG = DEC_CHUNK / DEC_GROUPS;  // keys per group
    constexpr int NQ = D / 8, NV = DV / 8;       // components per lane
    constexpr int PART = dec_part(DV);
    __shared__ float red[DEC_GROUPS][DV + 1];
    __shared__ float wmax[DEC_THREADS / 32];
    const int32_t bh = blockIdx.x, h = bh % p.heads;
    const KeySet ks = key_set(p.kind[h], p.pos, p.l, p.c, p.off[h]);
    const int64_t total = key_count(ks);
    const int64_t e0 = static_cast<int64_t>(blockIdx.y) * DEC_CHUNK;
    const int grp = threadIdx.x >> 3, l8 = threadIdx.x & 7;
    const size_t cache = static_cast<size_t>(bh) * p.n;  // first cache row of this (batch, head)
    float q[NQ];
    load_part<F32, D>(p.q, bh, l8, q);
#pragma unroll
    for (int e = 0; e < NQ; ++e) q[e] *= p.scale_log2;  // scores in log2 units
    // The group's keys e0 + grp + 16 r (r < KPG): every K and V load first, so that one round trip
    // to memory serves the whole chunk.
    float k[KPG][NQ], v[KPG][NV];
    bool valid[KPG];
#pragma unroll
    for (int r = 0; r < KPG; ++r) {
        const int64_t e = e0 + grp + DEC_GROUPS * r;
        valid[r] = e < total;
        if (valid[r]) {
            const int64_t row = cache + key_at(ks, e);
            load_part<F32, D>(p.k, row, l8, k[r]);
            load_part<F32, DV>(p.v, row, l8, v[r]);
        }
    }
    // scores (every lane runs every shuffle: the groups of a warp share them) and their maximum
    float s[KPG], m = -INFINITY;
#pragma unroll
    for (int r = 0; r < KPG; ++r) {
        float x = 0.f;
        if (valid[r])
#pragma unroll
            for (int t = 0; t < NQ; ++t) x = fmaf(q[t], k[r][t], x);
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        s[r] = valid[r] ? x : -INFINITY;
        m = fmaxf(m, s[r]);
    }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    const float M = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
    // sum of 2^(s - M) and of 2^(s - M) v (every lane of a group adds the same weight)
    float acc[NV], lsum = 0.f;
#pragma unroll
    for (int t = 0; t < NV; ++t) acc[t] = 0.f;
#pragma unroll
    for (int r = 0; r < KPG; ++r)
        if (valid[r]) {
            const float w = ex2(s[r] - M);
            lsum += w;
#pragma unroll
            for (int t = 0; t < NV; ++t) acc[t] = fmaf(w, v[r][t], acc[t]);
        }
#pragma unroll
    for (int t = 0; t < NV; ++t) red[grp][NV * l8 + t] = acc[t];
    if (l8 == 0) red[grp][DV] = lsum;
    __syncthreads();
    const int32_t nsplit = static_cast<int32_t>(gridDim.y);
    float *parts = p.part + static_cast<size_t>(bh) * nsplit * PART;
    float *part = parts + static_cast<size_t>(blockIdx.y) * PART;
    for (int c = threadIdx.x; c < DV + 1; c += DEC_THREADS) {
        float sum = 0.f;
        for (int g = 0; g < DEC_GROUPS; ++g) sum += red[g][c];  // fixed order
        part[c < DV ? 4 + c : 1] = sum;  // O (DV columns, 16-byte aligned at 4) and L at 1
    }
    if (threadIdx.x == 0) part[0] = M;  // -inf for a chunk without keys
    // count this chunk; the CTA that brings the count to nsplit combines (the fences order every
    // CTA's part before its count, and the counts before the combining CTA's reads)
    __shared__ int32_t is_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(&p.cnt[bh], 1) == nsplit - 1;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // O = sum_c 2^(M_c - M) O_c / L, L = sum_c 2^(M_c - M) L_c, lse = (M + log2 L) ln 2; a row
    // without keys gets O = 0, lse = -inf.  The parts are read through L2 (ld.global.cg: other CTAs
    // wrote them), spread over all threads so that each makes few independent loads: thread
    // (group g, quad q) adds, for the chunks c = g, g + G, ..., their weighted columns 4qd .. 4qd + 3
    // (and, for qd = 0, their L); the G group sums are then added in group order (deterministic).
    constexpr int NQD = DV / 4;                 // 16-byte quads of a value row
    constexpr int G = DEC_THREADS / NQD;        // chunk groups
    __shared__ float osum[G][DV + 1];
    float mloc = -INFINITY;
    for (int c = threadIdx.x; c < nsplit; c += DEC_THREADS) mloc = fmaxf(mloc, __ldcg(parts + c * PART));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mloc;
    __syncthreads();
    const float Mall = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
    const int g = threadIdx.x / NQD, qd = threadIdx.x % NQD;
    float4 oq = make_float4(0.f, 0.f, 0.f, 0.f);
    float lacc = 0.f;
    if (Mall != -INFINITY)
        for (int c = g; c < nsplit; c += G) {
            const float *pc = parts + static_cast<size_t>(c) * PART;
            const float mc = __ldcg(pc);
            const float4 x = __ldcg(reinterpret_cast<const float4 *>(pc + 4) + qd);
            const float w = mc == -INFINITY ? 0.f : ex2(mc - Mall);
            oq.x = fmaf(w, x.x, oq.x);
            oq.y = fmaf(w, x.y, oq.y);
            oq.z = fmaf(w, x.z, oq.z);
            oq.w = fmaf(w, x.w, oq.w);
            if (qd == 0) lacc = fmaf(w, __ldcg(pc + 1), lacc);
        }
    osum[g][4 * qd] = oq.x;
    osum[g][4 * qd + 1] = oq.y;
    osum[g][4 * qd + 2] = oq.z;
    osum[g][4 * qd + 3] = oq.w;
    if (qd == 0) osum[g][DV] = lacc;
    __syncthreads();
    for (int t = threadIdx.x; t < DV; t += DEC_THREADS) {
        float L = 0.f, o = 0.f;
        for (int gg = 0; gg < G; ++gg) {  // fixed order
            L += osum[gg][DV];
            o += osum[gg][t];
        }
        const bool has = L > 0.f;
        o = has ? o / L : 0.f;
        if (F32)
            static_cast<float *>(p.o)[static_cast<size_t>(bh) * DV + t] = o;
        else
            static_cast<uint16_t *>(p.o)[static_cast<size_t>(bh) * DV + t] =
                static_cast<uint16_t>(pack_bf16(o, 0.f) & 0xFFFFu);
        if (t == 0) p.lse[bh] = has ? (Mall + lg2(L)) * LN2 : -INFINITY;
    }
}

template <bool F32, int D, int DV>
cudaError_t launch_w(const DecodeParams &p, int32_t nsplit, cudaStream_t s)
{
    const dim3 grid(static_cast<unsigned>(p.bh), static_cast<unsigned>(nsplit));
    decode_kernel<F32, D, DV><<<grid, DEC_THREADS, 0, s>>>(p);
    return cudaGetLastError();
}

template <bool F32>
cudaError_t launch_f(const DecodeParams &p, int32_t nsplit, int d, int dv, cudaStream_t s)
{
    if (d == 32 && dv == 32) return launch_w<F32, 32, 32>(p, nsplit, s);
    if (d == 64 && dv == 64) return launch_w<F32, 64, 64>(p, nsplit, s);
    if (d == 128 && dv == 128) return launch_w<F32, 128, 128>(p, nsplit, s);
    if (d == 64 && dv == 128) return launch_w<F32, 64, 128>(p, nsplit, s);
    return cudaErrorInvalidValue;
}

}  // namespace

bool decode_widths_supported(int d, int dv)
{
    return (d == dv && (d == 32 || d == 64 || d == 128)) || (d == 64 && dv == 128);
}

cudaError_t launch_decode(const DecodeParams &p, int32_t nsplit, bool f32, int d, int dv, cudaStream_t s)
{
    return f32 ? launch_f<true>(p, nsplit, d, dv, s) : launch_f<false>(p, nsplit, d, dv, s);
}

}  // namespace st
