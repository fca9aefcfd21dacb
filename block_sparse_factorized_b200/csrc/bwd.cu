// bwd.cu -- backward pass of factorized sparse attention on sm_100a, with recomputation.
//
// "Sparse Transformers（稀疏 Transformer）深度解读报告" §3.4: attention weights are not stored;
// the backward pass rebuilds them.  Here P_ij = exp(S_ij - lse_i) from the saved log-sum-exp,
// then (plain calculus of O = softmax(Q K^T / sqrt d) V over the allowed keys)
//   dV_j += P_ij dO_i,  dP_ij = dO_i . v_j,  dS_ij = P_ij (dP_ij - D_i),  D_i = dO_i . O_i,
//   dK_j += dS_ij q_i / sqrt(d),  dQ_i += dS_ij k_j / sqrt(d).
// One CTA owns one 128-key tile (of one part, one batch-head) and walks the contiguous run of
// query tiles that read it, so dK and dV accumulate in TMEM and are written once; dQ of each
// (query tile, key tile) pair is added to an fp32 accumulator with vector atomics.
// Roles:
//   warp 0      TMA: K and V of the key tile once, then Q and dO per query tile (2-stage ring)
//   warp 1      MMA issuer: S = Q K^T and dP = dO V^T (TMEM, 128 x 128 fp32 each), then after
//               the softmax warps wrote P and dS (bf16, SMEM): dV += P^T dO, dK += dS^T Q
//               (TMEM 128 x 64 each, resident for the whole item) and dQ = dS K (TMEM 128 x 64)
//   warps 2..9  two warpgroups, one query row per thread, warpgroup h owning score columns
//               64h..64h+63 (no row reduction is needed here: P comes from the saved lse):
//               interval mask, P, dS; drain dQ columns 32h.. with atomics; at the end one key
//               row per thread: dK, dV columns 32h.. to bf16 and a TMA store.
// A merge part (second pass of a merged head) adds the dK/dV the first pass wrote.
#include "tiles.cuh"

namespace st {
namespace {

constexpr uint32_t TB = TILE_BYTES;
constexpr int NST = 2;                             // Q/dO ring depth
constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = OFF_K + TB;
constexpr uint32_t OFF_Q = OFF_V + TB;             // NST tiles
constexpr uint32_t OFF_DO = OFF_Q + NST * TB;      // NST tiles
constexpr uint32_t OFF_P = OFF_DO + NST * TB;      // 2 halves; dK/dV staging at the end
constexpr uint32_t OFF_DS = OFF_P + 2 * TB;        // 2 halves
constexpr uint32_t OFF_BAR = OFF_DS + 2 * TB;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256;
constexpr int THREADS = 320;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 320, COL_DQ = 384;

struct Bars {
    uint64_t kv_full, s_full, p_full, dq_full, dq_empty;
    uint64_t qdo_full[NST], qdo_empty[NST];
    uint32_t tmem_base;
    int32_t abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// F32: fp32 I/O -- dK and dV are written row by row in fp32 (the MMAs run on bf16 copies).
template <bool F32>
__global__ void __launch_bounds__(THREADS, 1) bwd_kernel(const __grid_constant__ BwdParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Bars *bars = reinterpret_cast<Bars *>(smem + OFF_BAR);
    volatile int32_t *abort = &bars->abort;

    const int32_t item = blockIdx.x / p.batch, b = blockIdx.x - item * p.batch;
    const WorkItem w = p.items[item];
    const Part part = p.parts[w.part];
    const int32_t bh = b * p.heads + part.head;
    const int32_t kt = w.tile;
    const int32_t nq = w.end - w.begin;

    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->p_full, 256);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, 256);
        for (int s = 0; s < NST; ++s) {
            mbar_init(&bars->qdo_full[s], 1);
            mbar_init(&bars->qdo_empty[s], 1);
        }
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
    const bool run = (*abort == 0) && nq > 0;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0 && run) {
            tma_prefetch(frame_map(p.q, part.qframe));
            tma_prefetch(frame_map(p.dout, part.qframe));
            mbar_arrive_expect_tx(&bars->kv_full, 2 * TB);
            load_tile(p.k, part.kframe, p.g, part.o, kt, bh, smem + OFF_K, &bars->kv_full);
            load_tile(p.v, part.kframe, p.g, part.o, kt, bh, smem + OFF_V, &bars->kv_full);
            int j = 0;
            for (; j < nq; ++j) {
                const int s = j % NST;
                if (j >= NST && !mbar_wait(&bars->qdo_empty[s], ((j / NST) - 1) & 1, abort, p.err))
                    break;
                mbar_arrive_expect_tx(&bars->qdo_full[s], 2 * TB);
                load_tile(p.q, part.qframe, p.g, part.o, w.begin + j, bh, smem + OFF_Q + s * TB,
                          &bars->qdo_full[s]);
                load_tile(p.dout, part.qframe, p.g, part.o, w.begin + j, bh,
                          smem + OFF_DO + s * TB, &bars->qdo_full[s]);
            }
            if (*abort) {  // drain the copies still in flight before the CTA leaves
                volatile int32_t never = 0;
                mbar_wait(&bars->kv_full, 0, &never, p.err);
                for (int jj = (j > NST ? j - NST : 0); jj < j; ++jj)
                    mbar_wait(&bars->qdo_full[jj % NST], (jj / NST) & 1, &never, p.err);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0 && run) {
            constexpr uint32_t id_nn = idesc_bf16(128, 128, false, false);  // S, dP
            constexpr uint32_t id_tt = idesc_bf16(128, 64, true, true);     // dV, dK
            constexpr uint32_t id_kt = idesc_bf16(128, 64, false, true);    // dQ
            const uint32_t sK = smem_u32(smem + OFF_K), sV = smem_u32(smem + OFF_V);
            const uint32_t sP = smem_u32(smem + OFF_P), sDS = smem_u32(smem + OFF_DS);
            if (mbar_wait(&bars->kv_full, 0, abort, p.err)) {
                for (int j = 0; j < nq; ++j) {
                    const int s = j % NST;
                    if (!mbar_wait(&bars->qdo_full[s], (j / NST) & 1, abort, p.err)) break;
                    tc_fence_after();
                    const uint32_t sQ = smem_u32(smem + OFF_Q + s * TB);
                    const uint32_t sDO = smem_u32(smem + OFF_DO + s * TB);
                    // S = Q K^T, dP = dO V^T (all K-major over d)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16_ss(tbase + COL_S, desc_sw128(sQ + 32 * k, 16, 1024),
                                    desc_sw128(sK + 32 * k, 16, 1024), id_nn, k > 0 ? 1u : 0u);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16_ss(tbase + COL_DP, desc_sw128(sDO + 32 * k, 16, 1024),
                                    desc_sw128(sV + 32 * k, 16, 1024), id_nn, k > 0 ? 1u : 0u);
                    mma_commit(&bars->s_full);
                    if (!mbar_wait(&bars->p_full, j & 1, abort, p.err)) break;
                    if (j > 0 && !mbar_wait(&bars->dq_empty, (j - 1) & 1, abort, p.err)) break;
                    tc_fence_after();
                    // dV += P^T dO, dK += dS^T Q: A = P^T / dS^T MN-major (two 64-key atoms,
                    // 16 KB apart), B = dO / Q MN-major; 16 queries (2048 bytes) per step
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16_ss(tbase + COL_DV, desc_sw128(sP + k * 2048, TB, 1024),
                                    desc_sw128(sDO + k * 2048, TB, 1024), id_tt,
                                    (j > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16_ss(tbase + COL_DK, desc_sw128(sDS + k * 2048, TB, 1024),
                                    desc_sw128(sQ + k * 2048, TB, 1024), id_tt,
                                    (j > 0 || k > 0) ? 1u : 0u);
                    // dQ = dS K: A = dS K-major (two 64-key halves), B = K MN-major
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16_ss(tbase + COL_DQ, desc_sw128(sDS + (k >> 2) * TB + (k & 3) * 32, 16, 1024),
                                    desc_sw128(sK + k * 2048, TB, 1024), id_kt, k > 0 ? 1u : 0u);
                    mma_commit(&bars->dq_full);
                    mma_commit(&bars->qdo_empty[s]);
                }
            }
        }
    } else {
        // ------- P, dS, dQ drain, epilogue (warps 2..9: warpgroup h owns columns 64h..64h+63) -------
        const int h = (warp - 2) >> 2;
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const int wg_tid = threadIdx.x - 64 - 128 * h;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tbase + COL_S + lane_off + 64 * h, tDP = tbase + COL_DP + lane_off + 64 * h;
        const uint32_t tDQ = tbase + COL_DQ + lane_off + 32 * h;
        const uint32_t sPh = smem_u32(smem + OFF_P) + h * TB, sDSh = smem_u32(smem + OFF_DS) + h * TB;
        const float sc = p.scale_log2, dsc = p.ds_scale;
        const size_t head_base = static_cast<size_t>(bh) * p.g.n;
        bool ok = run;
        uint32_t sv[32], dv[32];
        for (int j = 0; ok && j < nq; ++j) {
            const int32_t qt = w.begin + j;
            int32_t lo_abs, hi_abs;
            const int32_t i = row_interval(p.g, part, qt, row, lo_abs, hi_abs);
            float nlse = 0.f, nD = 0.f;  // -lse (log2 units) and -D_i / sqrt(d) of this row
            if (i >= 0) {
                const float lse = p.lse[head_base + i];
                // a row with no allowed key (lse = -inf) has every entry masked to -inf below;
                // keep its base finite so that -inf + base stays -inf instead of NaN
                nlse = lse == -INFINITY ? 0.f : -lse * LOG2E;
                nD = -p.delta[head_base + i] * dsc;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, j & 1, abort, p.err))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int32_t base = kt * TILE + 64 * h;
            const int32_t lo = lo_abs - base, hi = hi_abs - base;   // allowed columns of this half
            const bool full = (lo <= 0) && (hi >= 63);
            const uint32_t span = static_cast<uint32_t>(hi - lo);
            const bool none = hi < lo;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                tmem_ld32(tS + ch * 32, sv);
                tmem_ld32(tDP + ch * 32, dv);
                tmem_wait_ld();
                if (!full) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const bool keep = !none && static_cast<uint32_t>(ch * 32 + e - lo) <= span;
                        sv[e] = keep ? sv[e] : 0xFF800000u;  // -inf: P = 0, dS = 0
                    }
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    // P = exp2(S log2e / sqrt(d) - lse log2e);  dS = P (dP - D) / sqrt(d)
                    const float p0 = ex2(fmaf(__uint_as_float(sv[2 * e]), sc, nlse));
                    const float p1 = ex2(fmaf(__uint_as_float(sv[2 * e + 1]), sc, nlse));
                    const float d0 = p0 * fmaf(__uint_as_float(dv[2 * e]), dsc, nD);
                    const float d1 = p1 * fmaf(__uint_as_float(dv[2 * e + 1]), dsc, nD);
                    sv[e] = pack_bf16(p0, p1);
                    dv[e] = pack_bf16(d0, d1);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t off = sw128_off(row, ch * 4 + q);
                    st_shared_v4(sPh + off, sv[4 * q], sv[4 * q + 1], sv[4 * q + 2], sv[4 * q + 3]);
                    st_shared_v4(sDSh + off, dv[4 * q], dv[4 * q + 1], dv[4 * q + 2], dv[4 * q + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->p_full);
            // drain dQ columns 32h .. 32h+31 of this (query tile, key tile) pair
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->dq_full, j & 1, abort, p.err))) {
                ok = false;
                break;
            }
            tc_fence_after();
            tmem_ld32(tDQ, sv);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars->dq_empty);
            if (i >= 0) {
                float4 *dst = reinterpret_cast<float4 *>(p.dq_acc + (head_base + i) * 64 + 32 * h);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    atomicAdd(dst + e, make_float4(__uint_as_float(sv[4 * e]), __uint_as_float(sv[4 * e + 1]),
                                                   __uint_as_float(sv[4 * e + 2]), __uint_as_float(sv[4 * e + 3])));
            }
        }
        // ------- dK, dV epilogue: one key row per thread, warpgroup h writes columns 32h.. -------
        if (ok) {
            const int32_t pos = frame_pos(p.g, part.kframe, part.o, kt, row);
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t tacc = tbase + (which == 0 ? COL_DK : COL_DV) + lane_off + 32 * h;
                float acc[32];
                tmem_ld32(tacc, sv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) acc[e] = __uint_as_float(sv[e]);
                if (F32) {
                    if (pos >= 0 && *abort == 0) {
                        const float *pf = which == 0 ? p.dk_prev_f32 : p.dv_prev_f32;
                        float *of = (which == 0 ? p.dk_f32 : p.dv_f32) + (head_base + pos) * 64 + 32 * h;
                        if (part.merge) {
                            const float4 *src = reinterpret_cast<const float4 *>(pf + (head_base + pos) * 64 + 32 * h);
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float4 u = src[q];
                                acc[4 * q] += u.x;
                                acc[4 * q + 1] += u.y;
                                acc[4 * q + 2] += u.z;
                                acc[4 * q + 3] += u.w;
                            }
                        }
                        float4 *d4 = reinterpret_cast<float4 *>(of);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            d4[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
                    }
                    continue;
                }
                if (part.merge && pos >= 0) {
                    const uint16_t *prev = which == 0 ? p.dk_prev : p.dv_prev;
                    const uint4 *src = reinterpret_cast<const uint4 *>(prev + (head_base + pos) * 64 + 32 * h);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 u = src[q];
                        const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            acc[8 * q + 2 * e] += bf16_lo(uu[e]);
                            acc[8 * q + 2 * e + 1] += bf16_hi(uu[e]);
                        }
                    }
                }
                const uint32_t dst = smem_u32(smem + OFF_P) + which * TB;  // staging: dK, dV tiles
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    st_shared_v4(dst + sw128_off(row, 4 * h + q), pack_bf16(acc[8 * q], acc[8 * q + 1]),
                                 pack_bf16(acc[8 * q + 2], acc[8 * q + 3]),
                                 pack_bf16(acc[8 * q + 4], acc[8 * q + 5]),
                                 pack_bf16(acc[8 * q + 6], acc[8 * q + 7]));
            }
            fence_proxy_async_smem();
        }
        named_bar_sync(1, 256);
        if (!F32 && h == 0 && wg_tid == 0 && ok && *abort == 0) {
            store_tile(p.dk, part.kframe, p.g, part.o, kt, bh, smem + OFF_P);
            store_tile(p.dv, part.kframe, p.g, part.o, kt, bh, smem + OFF_P + TB);
            bulk_commit();
            bulk_wait_all();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

template <bool F32>
cudaError_t launch_bwd_t(const BwdParams &p, cudaStream_t s)
{
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(bwd_kernel<F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    if (p.nitems == 0) return cudaSuccess;
    bwd_kernel<F32><<<dim3(static_cast<unsigned>(p.nitems) * p.batch), THREADS, SMEM_BYTES, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(const BwdParams &p, bool f32, cudaStream_t s)
{
    return f32 ? launch_bwd_t<true>(p, s) : launch_bwd_t<false>(p, s);
}

}  // namespace st
