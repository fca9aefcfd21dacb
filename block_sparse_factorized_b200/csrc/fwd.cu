// fwd.cu -- fused forward pass of factorized sparse attention on sm_100a.
//
// One CTA computes one 128-row query tile of one part of one (batch, head) over the contiguous
// run of 128-key tiles its work item lists ("Sparse Transformers（稀疏 Transformer）深度解读报告"
// §3.5: blocked computation, softmax fused into the kernel, upper triangle never computed; "长序列
// 为何不必让每个 token 看见全部历史？…" §05: only selected block pairs enter the kernel, boundary
// blocks keep an element mask).
//
// Arithmetic ("长序列为何不必让每个 token 看见全部历史？…" §01-§02): S = Q K^T / sqrt(d), softmax over
// the allowed keys only, O = P V, and the log-sum-exp saved for the recomputing backward pass
// ("Sparse Transformers 深度解读报告" §3.4).  A row with no allowed key gets O = 0, lse = -inf.
//
// Each 128-key tile is split into two 64-key halves, each owned by its own softmax warpgroup with
// its own running max m_h, running sum l_h and its own O accumulator in TMEM: the halves are two
// independent online softmaxes over disjoint key sets, combined once in the epilogue by
//   M = max(m_0, m_1), L = sum_h 2^(m_h - M) l_h, O = sum_h 2^(m_h - M) O_h / L, lse = M + log2 L
// (log2 units).  No per-tile exchange between the warpgroups is needed.
//
// Roles (320 threads):
//   warp 0       TMA producer: Q (and its low part for split precision), K/V tiles, NST-stage ring
//   warp 1       MMA issuer (one thread): S = Q K^T into TMEM (128 x 128 fp32); then per half h,
//                once warpgroup h wrote P_h (bf16, SMEM): O_h += P_h V_h (128 x 64 fp32 in TMEM)
//   warps 2..5   softmax of key half 0, warps 6..9 of key half 1; one query row per thread
//                (TMEM lane = row): interval mask, max, exp2, P_h to SMEM, and a rescale of O_h
//                only when the row max grew by more than 2^8 (otherwise the stale max is kept:
//                numerator and denominator use the same max, so the result is unchanged)
//   epilogue     both warpgroups: combine the halves (each writes 32 of the 64 output columns),
//                a merge part folds in the first pass's (O, lse), TMA store in the query frame.
#include "tiles.cuh"

namespace st {
namespace {

constexpr int NST = 2;                         // K/V ring depth
constexpr uint32_t TB = TILE_BYTES;            // one 128 x 64 bf16 tile, 16 KB
constexpr int THREADS = 320;
constexpr uint32_t TMEM_COLS = 256;            // S: 0..127, O_0: 128..191, O_1: 192..255
constexpr float RESCALE_LOG2 = 8.0f;           // keep a stale max while it is within 2^8

// Shared-memory plan.  SPLIT (fp32 I/O) adds the low bf16 parts of Q and of each K tile.
//   Q [, Q_lo] | NST x (K, V [, K_lo]) | P (two 128 x 64 halves: keys 0-63, 64-127) | barriers
// The Q tile doubles as the O staging tile and the P area as the (m, l) exchange in the epilogue.
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
    uint64_t q_full, s_full, o_done;
    uint64_t p_full[2], pv_done[2];
    uint64_t kv_full[NST], kv_empty[NST];
    uint32_t tmem_base;
    int32_t abort;
};
static_assert(sizeof(Bars) <= 128, "barrier block");

// Row max of 64 scores: eight independent partial maxima folded with three-input max (short
// dependency chains, about one instruction per two scores).
__device__ __forceinline__ float max64(const uint32_t (&v)[64])
{
    float a[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = fmaxf(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
#pragma unroll
    for (int c = 16; c < 64; c += 2)
        a[(c >> 1) & 7] = max3f(a[(c >> 1) & 7], __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
    return max3f(max3f(a[0], a[1], a[2]), max3f(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
}

template <bool SPLIT>
__global__ void __launch_bounds__(THREADS, Plan<SPLIT>::MIN_BLOCKS)
    fwd_kernel(const __grid_constant__ FwdParams p)
{
    using L = Plan<SPLIT>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Bars *bars = reinterpret_cast<Bars *>(smem + L::OFF_BAR);
    volatile int32_t *abort = &bars->abort;

    const int32_t item = blockIdx.x / p.batch, b = blockIdx.x - item * p.batch;
    const WorkItem w = p.items[item];
    const Part part = p.parts[w.part];
    const int32_t bh = b * p.heads + part.head;
    const int32_t nkt = w.end - w.begin;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->p_full[0], 128);
        mbar_init(&bars->p_full[1], 128);
        mbar_init(&bars->pv_done[0], 1);
        mbar_init(&bars->pv_done[1], 1);
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
            load_tile(mq, part.qframe, p.g, part.o, w.tile, bh, smem + L::OFF_Q, &bars->q_full);
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
            const uint32_t tS = tbase;
            constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idO = idesc_bf16(128, 64, false, true);
            const uint32_t sQ = smem_u32(smem + L::OFF_Q), sP = smem_u32(smem + L::OFF_P);
            // S = Q K^T: both operands K-major, 16 elements (32 bytes) of d per step.  Split
            // precision adds Q_hi K_lo^T + Q_lo K_hi^T into the same accumulator.
            auto issue_s = [&](int it) {
                const uint32_t sK = smem_u32(smem + L::OFF_STAGE + (it % NST) * L::STAGE);
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
            };
            // O_h += P_h V_h: P_h K-major (64 keys, 32 bytes per step), V_h MN-major (rows 64h..,
            // 16 keys = 2048 bytes per step)
            auto issue_pv = [&](int it, int h) {
                const uint32_t sV = smem_u32(smem + L::OFF_STAGE + (it % NST) * L::STAGE) + TB;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_ss(tbase + 128 + 64 * h, desc_sw128(sP + h * TB + k * 32, 16, 1024),
                                desc_sw128(sV + h * 8192 + k * 2048, TB, 1024), idO,
                                (it > 0 || k > 0) ? 1u : 0u);
                mma_commit(&bars->pv_done[h]);
            };
            // Order per key tile: PV_0(it) | S(it+1) | PV_1(it): the next scores are computed as
            // soon as both halves have read S(it), while half 1's PV is still pending.
            bool go = mbar_wait(&bars->q_full, 0, abort, p.err) &&
                      mbar_wait(&bars->kv_full[0], 0, abort, p.err);
            if (go) {
                tc_fence_after();
                issue_s(0);
            }
            for (int it = 0; go && it < nkt; ++it) {
                if (!mbar_wait(&bars->p_full[0], it & 1, abort, p.err)) break;
                tc_fence_after();
                issue_pv(it, 0);
                if (!mbar_wait(&bars->p_full[1], it & 1, abort, p.err)) break;
                tc_fence_after();
                if (it + 1 < nkt) {
                    if (!mbar_wait(&bars->kv_full[(it + 1) % NST], ((it + 1) / NST) & 1, abort, p.err)) break;
                    tc_fence_after();
                    issue_s(it + 1);
                }
                issue_pv(it, 1);
                mma_commit(&bars->kv_empty[it % NST]);
            }
            if (go) mma_commit(&bars->o_done);
        }
    } else {
        // ---------------- softmax of one key half + epilogue (warps 2..9) ----------------
        const int h = (warp - 2) >> 2;                 // key half owned by this warpgroup
        const int q4 = warp & 3;                       // TMEM lane quarter of this warp
        const int row = q4 * 32 + lane;
        const int wg_tid = threadIdx.x - 64 - 128 * h; // 0..127 within the warpgroup
        int32_t lo_abs, hi_abs;
        const int32_t i = row_interval(p.g, part, w.tile, row, lo_abs, hi_abs);
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tbase + lane_off + 64 * h;
        const uint32_t tO = tbase + lane_off + 128 + 64 * h;
        const uint32_t sPh = smem_u32(smem + L::OFF_P) + h * TB;
        const float sc = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = run;
        uint32_t v[64];
        for (int it = 0; ok && it < nkt; ++it) {
            // warp-uniform wait: every lane must agree before warp-collective TMEM accesses
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, it & 1, abort, p.err))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int32_t base = (w.begin + it) * TILE + 64 * h;
            const int32_t lo = lo_abs - base, hi = hi_abs - base;   // allowed columns of this half
            tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
            tmem_wait_ld();
            if (!(lo <= 0 && hi >= 63)) {  // boundary tile for this row: interval mask
                const uint32_t span = static_cast<uint32_t>(hi - lo);
                const bool none = hi < lo;
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const bool keep = !none && static_cast<uint32_t>(c - lo) <= span;
                    v[c] = keep ? v[c] : 0xFF800000u;  // -inf
                }
            }
            const float m_tile = max64(v) * sc;
            const float m_new = fmaxf(m, m_tile);
            const bool grow = m_new > m + RESCALE_LOG2;   // also true for the first finite max
            const float m_use = grow ? m_new : m;
            const float alpha = grow ? ex2(m - m_use) : 1.f;  // 0 when nothing was seen yet
            const float nb = (m_use == -INFINITY) ? 0.f : -m_use;
            float ps[4] = {0.f, 0.f, 0.f, 0.f};  // four partial sums
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
                // p = exp2(s log2e / sqrt(d) - m)
                const float p0 = ex2(fmaf(__uint_as_float(v[c]), sc, nb));
                const float p1 = ex2(fmaf(__uint_as_float(v[c + 1]), sc, nb));
                ps[(c >> 1) & 3] += p0 + p1;
                v[c >> 1] = pack_bf16(p0, p1);
            }
            // PV of the previous tile must be done with P_h and O_h before they change
            if (it > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[h], (it - 1) & 1, abort, p.err))) {
                ok = false;
                break;
            }
            if (it > 0) tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                st_shared_v4(sPh + sw128_off(row, j), v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            if (it > 0 && __any_sync(0xffffffffu, grow)) {
                // rescale this half's partial O (complete: pv_done above; PV of this tile waits
                // for p_full)
                uint32_t o[32];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    tmem_ld32(tO + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(tO + 32 * c, o);
                }
                tmem_wait_st();
            }
            l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
            m = m_use;
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->p_full[h]);
        }
        // ---------------- epilogue: combine the halves ----------------
        const bool o_ready =
            ok && nkt > 0 && __all_sync(0xffffffffu, mbar_wait(&bars->o_done, 0, abort, p.err));
        if (o_ready) tc_fence_after();
        // (m, l) exchange through the P area (free once every MMA is done)
        float2 *stats = reinterpret_cast<float2 *>(smem + L::OFF_P);
        stats[h * 128 + row] = make_float2(m, l);
        named_bar_sync(1, 256);
        const float2 other = stats[(1 - h) * 128 + row];
        const float m0 = h == 0 ? m : other.x, l0 = h == 0 ? l : other.y;
        const float m1 = h == 0 ? other.x : m, l1 = h == 0 ? other.y : l;
        const float M = fmaxf(m0, m1);
        const float w0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M);
        const float w1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M);
        const float Lsum = l0 * w0 + l1 * w1;
        const bool has = Lsum > 0.f;
        float lse2 = has ? M + lg2(Lsum) : -INFINITY;       // log2 units
        float c0 = has ? w0 / Lsum : 0.f, c1 = has ? w1 / Lsum : 0.f, cprev = 0.f;
        const size_t rowoff = (static_cast<size_t>(bh) * p.g.n + (i < 0 ? 0 : i));
        if (part.merge && i >= 0) {
            const float L1 = p.lse[rowoff] * LOG2E;
            const float Lm = fmaxf(L1, lse2);
            if (Lm == -INFINITY) {
                c0 = c1 = 0.f;
                lse2 = -INFINITY;
            } else {
                const float e1 = ex2(L1 - Lm), e2 = ex2(lse2 - Lm), tot = e1 + e2;
                cprev = e1 / tot;
                c0 *= e2 / tot;
                c1 *= e2 / tot;
                lse2 = Lm + lg2(tot);
            }
        }
        // this warpgroup writes output columns 32h .. 32h + 31
        float acc[32];
        if (o_ready) {
            uint32_t o[32];
            tmem_ld32(tbase + lane_off + 128 + 32 * h, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] = c0 * __uint_as_float(o[e]);
            tmem_ld32(tbase + lane_off + 192 + 32 * h, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] = fmaf(c1, __uint_as_float(o[e]), acc[e]);
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] = 0.f;
        }
        if (cprev != 0.f) {  // add the first pass's output with its log-sum-exp weight
            if (SPLIT) {
                const float4 *src = reinterpret_cast<const float4 *>(p.o_prev_f32 + rowoff * 64 + 32 * h);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 u = src[j];
                    acc[4 * j] += cprev * u.x;
                    acc[4 * j + 1] += cprev * u.y;
                    acc[4 * j + 2] += cprev * u.z;
                    acc[4 * j + 3] += cprev * u.w;
                }
            } else {
                const uint4 *src = reinterpret_cast<const uint4 *>(p.o_prev + rowoff * 64 + 32 * h);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 u = src[j];
                    const uint32_t pw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc[8 * j + 2 * e] += cprev * bf16_lo(pw[e]);
                        acc[8 * j + 2 * e + 1] += cprev * bf16_hi(pw[e]);
                    }
                }
            }
        }
        // every thread has read its previous output and lse: the tile may now be overwritten
        named_bar_sync(1, 256);
        if (h == 0 && i >= 0) p.lse[rowoff] = lse2 * LN2;
        if (SPLIT) {
            // fp32 output: row by row, this warpgroup's 32 columns (128 bytes)
            if (i >= 0 && *abort == 0) {
                float4 *dst = reinterpret_cast<float4 *>(p.o_f32 + rowoff * 64 + 32 * h);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    dst[j] = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
            }
        } else {
            const uint32_t sO = smem_u32(smem + L::OFF_Q);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                st_shared_v4(sO + sw128_off(row, 4 * h + j), pack_bf16(acc[8 * j], acc[8 * j + 1]),
                             pack_bf16(acc[8 * j + 2], acc[8 * j + 3]),
                             pack_bf16(acc[8 * j + 4], acc[8 * j + 5]),
                             pack_bf16(acc[8 * j + 6], acc[8 * j + 7]));
            fence_proxy_async_smem();
            named_bar_sync(1, 256);
            if (wg_tid == 0 && h == 0 && *abort == 0) {
                store_tile(p.o, part.qframe, p.g, part.o, w.tile, bh, smem + L::OFF_Q);
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
