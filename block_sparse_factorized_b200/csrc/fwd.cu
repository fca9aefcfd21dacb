// fwd.cu -- fused forward pass of factorized sparse attention on sm_100a.
//
// One CTA computes one 128-row query tile of one part of one (batch, head) over the contiguous
// run of 128-key tiles its work item lists ("Sparse Transformers（稀疏 Transformer）深度解读报告"
// §3.5: blocked computation, softmax fused into the kernel, upper triangle never computed; "长序列
// 为何不必让每个 token 看见全部历史？…" §05: only selected block pairs enter the kernel, boundary
// blocks keep an element mask).  Roles:
//   warp 0      TMA producer: the Q tile, then K/V tiles through an NST-stage ring
//   warp 1      MMA issuer (one thread): S = Q K^T into TMEM (128 x 128 fp32), then O += P V
//               into TMEM (128 x 64 fp32) once the softmax has written P (bf16) to SMEM
//   warps 2..5  softmax, one query row per thread (TMEM lane = row): interval mask, running
//               max m and sum l with exp2, P to SMEM, O rescale in TMEM when m grows, and the
//               epilogue O / l, lse = (m + log2 l) ln 2, stored through TMA.
// Arithmetic follows "长序列为何不必让每个 token 看见全部历史？…" §01-§02: S = Q K^T / sqrt(d),
// softmax over the allowed keys only, O = P V; the log-sum-exp is kept for the backward pass
// (recomputation, "Sparse Transformers 深度解读报告" §3.4).  A row with no allowed key gets O = 0
// and lse = -inf.  A merge part (second pass of a merged head) combines its (O, lse) with the
// first pass's by log-sum-exp weights.
#include "tiles.cuh"

namespace st {
namespace {

constexpr int NST = 2;                         // K/V ring depth
constexpr uint32_t TB = TILE_BYTES;            // one 128 x 64 bf16 tile, 16 KB
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 256;            // S: columns 0..127, O: 128..191

// Shared-memory plan.  SPLIT (fp32 I/O) adds the low bf16 parts of Q and of each K tile.
//   Q [, Q_lo] | NST x (K, V [, K_lo]) | P (two 128 x 64 halves: keys 0-63, 64-127) | barriers
// The Q tile doubles as the O staging tile of the epilogue.
template <bool SPLIT>
struct Plan {
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_QL = TB;
    static constexpr uint32_t OFF_STAGE = (SPLIT ? 2 : 1) * TB;
    static constexpr uint32_t STAGE = (SPLIT ? 3 : 2) * TB;     // K at +0, V at +TB, K_lo at +2TB
    static constexpr uint32_t OFF_P = OFF_STAGE + NST * STAGE;
    static constexpr uint32_t OFF_BAR = OFF_P + 2 * TB;
    static constexpr uint32_t SMEM_BYTES = OFF_BAR + 128;
    static constexpr int MIN_BLOCKS = SPLIT ? 1 : 2;
};

struct Bars {
    uint64_t q_full, s_full, p_full, o_done;
    uint64_t kv_full[NST], kv_empty[NST];
    uint32_t tmem_base;
    int32_t abort;
};
static_assert(sizeof(Bars) <= 128, "barrier block");

template <bool SPLIT>
__global__ void __launch_bounds__(THREADS, Plan<SPLIT>::MIN_BLOCKS)
    fwd_kernel(const __grid_constant__ FwdParams p)
{
    using L = Plan<SPLIT>;
    constexpr uint32_t OFF_Q = L::OFF_Q, OFF_P = L::OFF_P, OFF_BAR = L::OFF_BAR;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Bars *bars = reinterpret_cast<Bars *>(smem + OFF_BAR);
    volatile int32_t *abort = &bars->abort;

    const int32_t item = blockIdx.x / p.batch, b = blockIdx.x - item * p.batch;
    const WorkItem w = p.items[item];
    const Part part = p.parts[w.part];
    const int32_t bh = b * p.heads + part.head;
    const int32_t nkt = w.end - w.begin;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->p_full, 128);
        mbar_init(&bars->o_done, 1);
        for (int s = 0; s < NST; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        // the 128-byte swizzle needs 1024-byte aligned tiles
        bars->abort = (smem_u32(smem) & 1023u) ? 1 : 0;
        if (bars->abort) atomicOr(p.err, 2);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = bars->tmem_base;
    const bool run = (*abort == 0) && nkt > 0;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0 && run) {
            const FrameMaps &mq = p.q, &mk = p.k, &mv = p.v;
            tma_prefetch(frame_map(mq, part.qframe));
            tma_prefetch(frame_map(mk, part.kframe));
            tma_prefetch(frame_map(mv, part.kframe));
            mbar_arrive_expect_tx(&bars->q_full, (SPLIT ? 2 : 1) * TB);
            load_tile(mq, part.qframe, p.g, part.o, w.tile, bh, smem + OFF_Q, &bars->q_full);
            if (SPLIT)
                load_tile(p.ql, part.qframe, p.g, part.o, w.tile, bh, smem + L::OFF_QL, &bars->q_full);
            int it = 0;
            for (; it < nkt; ++it) {
                const int s = it % NST;
                if (it >= NST && !mbar_wait(&bars->kv_empty[s], ((it / NST) - 1) & 1, abort, p.err))
                    break;
                uint8_t *stage = smem + L::OFF_STAGE + s * L::STAGE;
                mbar_arrive_expect_tx(&bars->kv_full[s], L::STAGE);
                load_tile(mk, part.kframe, p.g, part.o, w.begin + it, bh, stage, &bars->kv_full[s]);
                load_tile(mv, part.kframe, p.g, part.o, w.begin + it, bh, stage + TB, &bars->kv_full[s]);
                if (SPLIT)
                    load_tile(p.kl, part.kframe, p.g, part.o, w.begin + it, bh, stage + 2 * TB,
                              &bars->kv_full[s]);
            }
            if (*abort) {  // drain the copies still in flight before the CTA leaves
                volatile int32_t never = 0;
                mbar_wait(&bars->q_full, 0, &never, p.err);
                for (int j = (it > NST ? it - NST : 0); j < it; ++j)
                    mbar_wait(&bars->kv_full[j % NST], (j / NST) & 1, &never, p.err);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0 && run) {
            const uint32_t tS = tbase, tO = tbase + 128;
            constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idO = idesc_bf16(128, 64, false, true);
            const uint32_t sQ = smem_u32(smem + OFF_Q), sP = smem_u32(smem + OFF_P);
            if (mbar_wait(&bars->q_full, 0, abort, p.err)) {
                for (int it = 0; it < nkt; ++it) {
                    const int s = it % NST;
                    if (!mbar_wait(&bars->kv_full[s], (it / NST) & 1, abort, p.err)) break;
                    tc_fence_after();
                    const uint32_t sK = smem_u32(smem + L::OFF_STAGE + s * L::STAGE);
                    const uint32_t sV = sK + TB;
                    // S = Q K^T: both operands K-major, 16 elements (32 bytes) of d per step.
                    // Split precision adds Q_hi K_lo^T + Q_lo K_hi^T into the same accumulator.
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16_ss(tS, desc_sw128(sQ + 32 * k, 16, 1024),
                                    desc_sw128(sK + 32 * k, 16, 1024), idS, k > 0 ? 1u : 0u);
                    if (SPLIT) {
                        const uint32_t sQl = smem_u32(smem + L::OFF_QL), sKl = sK + 2 * TB;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            mma_bf16_ss(tS, desc_sw128(sQ + 32 * k, 16, 1024),
                                        desc_sw128(sKl + 32 * k, 16, 1024), idS, 1u);
                            mma_bf16_ss(tS, desc_sw128(sQl + 32 * k, 16, 1024),
                                        desc_sw128(sK + 32 * k, 16, 1024), idS, 1u);
                        }
                    }
                    mma_commit(&bars->s_full);
                    if (!mbar_wait(&bars->p_full, it & 1, abort, p.err)) break;
                    tc_fence_after();
                    // O += P V: P K-major (two 64-key halves), V MN-major (16 keys = 2048 bytes)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16_ss(tO, desc_sw128(sP + (k >> 2) * TB + (k & 3) * 32, 16, 1024),
                                    desc_sw128(sV + k * 2048, TB, 1024), idO,
                                    (it > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&bars->kv_empty[s]);
                }
                mma_commit(&bars->o_done);
            }
        }
    } else {
        // ---------------- softmax + epilogue (warps 2..5) ----------------
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        int32_t lo_abs, hi_abs;
        const int32_t i = row_interval(p.g, part, w.tile, row, lo_abs, hi_abs);
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tbase + lane_off, tO = tbase + 128 + lane_off;
        const uint32_t sP = smem_u32(smem + OFF_P);
        const float sc = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = run;
        uint32_t v[32];
        for (int it = 0; ok && it < nkt; ++it) {
            // warp-uniform wait: every lane must agree before warp-collective TMEM accesses
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, it & 1, abort, p.err))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int32_t kt = w.begin + it;
            const int32_t lo = lo_abs - kt * TILE, hi = hi_abs - kt * TILE;
            const bool full = (lo <= 0) && (hi >= TILE - 1);
            float mx = -INFINITY;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                tmem_ld32(tS + ch * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int c = ch * 32 + e;
                    const bool keep = full || (c >= lo && c <= hi);
                    mx = keep ? fmaxf(mx, __uint_as_float(v[e]) * sc) : mx;
                }
            }
            const float m_new = fmaxf(m, mx);
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = (m == -INFINITY) ? 0.f : ex2(m - m_use);
            if (it > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                // running max grew: rescale this row's partial O (PV of the previous tile is
                // complete: the S commit of this tile covers every earlier MMA)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    tmem_ld32(tO + h * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                    tmem_st32(tO + h * 32, v);
                }
                tmem_wait_st();
            }
            float sum = 0.f;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                tmem_ld32(tS + ch * 32, v);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int c0 = ch * 32 + 2 * e, c1 = c0 + 1;
                    const bool k0 = full || (c0 >= lo && c0 <= hi);
                    const bool k1 = full || (c1 >= lo && c1 <= hi);
                    const float p0 = k0 ? ex2(__uint_as_float(v[2 * e]) * sc - m_use) : 0.f;
                    const float p1 = k1 ? ex2(__uint_as_float(v[2 * e + 1]) * sc - m_use) : 0.f;
                    sum += p0 + p1;
                    pk[e] = pack_bf16(p0, p1);
                }
                const uint32_t half = sP + (ch >> 1) * TB;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    st_shared_v4(half + sw128_off(row, (ch & 1) * 4 + j), pk[4 * j], pk[4 * j + 1],
                                 pk[4 * j + 2], pk[4 * j + 3]);
            }
            l = l * alpha + sum;
            m = m_new;
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->p_full);
        }
        // ---------------- epilogue ----------------
        float acc[64];
        const bool o_ready =
            ok && nkt > 0 && __all_sync(0xffffffffu, mbar_wait(&bars->o_done, 0, abort, p.err));
        if (o_ready) {
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                tmem_ld32(tO + h * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) acc[h * 32 + e] = __uint_as_float(v[e]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 64; ++e) acc[e] = 0.f;
        }
        const bool has = l > 0.f;
        float w2 = has ? 1.f / l : 0.f;                     // weight of this part's acc
        float lse2 = has ? m + lg2(l) : -INFINITY;          // log2 units
        float w1 = 0.f;
        const size_t rowoff = (static_cast<size_t>(bh) * p.g.n + (i < 0 ? 0 : i));
        if (part.merge && i >= 0) {
            const float L1 = p.lse[rowoff] * LOG2E;
            const float Lm = fmaxf(L1, lse2);
            if (Lm == -INFINITY) {
                w2 = 0.f;
                lse2 = -INFINITY;
            } else {
                const float e1 = ex2(L1 - Lm), e2 = ex2(lse2 - Lm), tot = e1 + e2;
                w1 = e1 / tot;
                w2 = w2 * (e2 / tot);
                lse2 = Lm + lg2(tot);
            }
        }
        if (i >= 0) p.lse[rowoff] = lse2 * LN2;
#pragma unroll
        for (int e = 0; e < 64; ++e) acc[e] *= w2;
        if (w1 != 0.f) {  // add the first pass's output with its log-sum-exp weight
            if (SPLIT) {
                const float4 *src = reinterpret_cast<const float4 *>(p.o_prev_f32 + rowoff * 64);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float4 u = src[j];
                    acc[4 * j] += w1 * u.x;
                    acc[4 * j + 1] += w1 * u.y;
                    acc[4 * j + 2] += w1 * u.z;
                    acc[4 * j + 3] += w1 * u.w;
                }
            } else {
                const uint4 *src = reinterpret_cast<const uint4 *>(p.o_prev + rowoff * 64);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 u = src[j];
                    const uint32_t pw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc[8 * j + 2 * e] += w1 * bf16_lo(pw[e]);
                        acc[8 * j + 2 * e + 1] += w1 * bf16_hi(pw[e]);
                    }
                }
            }
        }
        if (SPLIT) {
            // fp32 output: row by row (64 floats = 256 bytes per row)
            if (i >= 0 && *abort == 0) {
                float4 *dst = reinterpret_cast<float4 *>(p.o_f32 + rowoff * 64);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    dst[j] = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
            }
        } else {
            const uint32_t sO = smem_u32(smem + OFF_Q);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                st_shared_v4(sO + sw128_off(row, j), pack_bf16(acc[8 * j], acc[8 * j + 1]),
                             pack_bf16(acc[8 * j + 2], acc[8 * j + 3]),
                             pack_bf16(acc[8 * j + 4], acc[8 * j + 5]),
                             pack_bf16(acc[8 * j + 6], acc[8 * j + 7]));
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (row == 0 && *abort == 0) {
                store_tile(p.o, part.qframe, p.g, part.o, w.tile, bh, smem + OFF_Q);
                bulk_commit();
                bulk_wait_all();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

template <bool SPLIT>
cudaError_t launch_fwd_t(const FwdParams &p, cudaStream_t s)
{
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(fwd_kernel<SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Plan<SPLIT>::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    if (p.nitems == 0) return cudaSuccess;
    fwd_kernel<SPLIT><<<dim3(static_cast<unsigned>(p.nitems) * p.batch), THREADS, Plan<SPLIT>::SMEM_BYTES, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd(const FwdParams &p, bool split, cudaStream_t s)
{
    return split ? launch_fwd_t<true>(p, s) : launch_fwd_t<false>(p, s);
}

}  // namespace st
