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
//   warps 2..17 four warpgroups, one query row per thread, warpgroup g owning score columns
//               32g..32g+31 (no row reduction is needed here: P comes from the saved lse):
//               interval mask, P, dS; dQ columns 16g.. staged per warp and added to the fp32
//               accumulator with a TMA reduce; at the end one key row per thread: dK, dV
//               columns 16g.. to bf16 and a TMA store.
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
constexpr uint32_t OFF_DQ = OFF_DS + 2 * TB;       // dQ staging: 2 x (128 rows x 32 fp32)
constexpr uint32_t OFF_BAR = OFF_DQ + 2 * TB;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256;
constexpr int NWG = 4;                             // softmax warpgroups
constexpr int THREADS = 64 + 128 * NWG;
constexpr int CW = 128 / NWG;                       // score columns per warpgroup (32)
constexpr int OW = 64 / NWG;                        // dQ / dK / dV columns per warpgroup (16)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 320, COL_DQ = 384;

struct Bars {
    uint64_t kv_full, s_full, dp_full, p_ready, ds_ready, dq_full, dq_empty;
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
        mbar_init(&bars->dp_full, 1);
        mbar_init(&bars->p_ready, 128 * NWG);
        mbar_init(&bars->ds_ready, 128 * NWG);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, 128 * NWG);
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
            // Per query tile j the tensor core runs, in order:
            //   dV += P_j^T dO_j | S_{j+1} | dK += dS_j^T Q_j, dQ_j = dS_j K | dP_{j+1}
            // so that it computes dV_j and S_{j+1} while the softmax warps build dS_j, and dK_j,
            // dQ_j, dP_{j+1} while they drain dQ_j and build P_{j+1}.
            auto issue_s = [&](uint32_t sQ) {  // S = Q K^T (both K-major over d)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_ss(tbase + COL_S, desc_sw128(sQ + 32 * k, 16, 1024),
                                desc_sw128(sK + 32 * k, 16, 1024), id_nn, k > 0 ? 1u : 0u);
                mma_commit(&bars->s_full);
            };
            auto issue_dp = [&](uint32_t sDO) {  // dP = dO V^T
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_ss(tbase + COL_DP, desc_sw128(sDO + 32 * k, 16, 1024),
                                desc_sw128(sV + 32 * k, 16, 1024), id_nn, k > 0 ? 1u : 0u);
                mma_commit(&bars->dp_full);
            };
            bool go = mbar_wait(&bars->kv_full, 0, abort, p.err) &&
                      mbar_wait(&bars->qdo_full[0], 0, abort, p.err);
            if (go) {
                tc_fence_after();
                issue_s(smem_u32(smem + OFF_Q));
                issue_dp(smem_u32(smem + OFF_DO));
            }
            for (int j = 0; go && j < nq; ++j) {
                const int s = j % NST, s1 = (j + 1) % NST;
                const uint32_t sQ = smem_u32(smem + OFF_Q + s * TB);
                const uint32_t sDO = smem_u32(smem + OFF_DO + s * TB);
                const bool next = j + 1 < nq;
                if (!mbar_wait(&bars->p_ready, j & 1, abort, p.err)) break;
                tc_fence_after();
                // dV += P^T dO: A = P^T MN-major (two 64-key atoms 16 KB apart), B = dO
                // MN-major; 16 queries (2048 bytes) per step
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16_ss(tbase + COL_DV, desc_sw128(sP + k * 2048, TB, 1024),
                                desc_sw128(sDO + k * 2048, TB, 1024), id_tt, (j > 0 || k > 0) ? 1u : 0u);
                if (next) {  // S of the next query tile: the softmax warps are done reading S_j
                    if (!mbar_wait(&bars->qdo_full[s1], ((j + 1) / NST) & 1, abort, p.err)) break;
                    tc_fence_after();
                    issue_s(smem_u32(smem + OFF_Q + s1 * TB));
                }
                if (!mbar_wait(&bars->ds_ready, j & 1, abort, p.err)) break;
                if (j > 0 && !mbar_wait(&bars->dq_empty, (j - 1) & 1, abort, p.err)) break;
                tc_fence_after();
                // dK += dS^T Q (as dV), dQ = dS K: A = dS K-major (two 64-key halves), B = K MN-major
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16_ss(tbase + COL_DK, desc_sw128(sDS + k * 2048, TB, 1024),
                                desc_sw128(sQ + k * 2048, TB, 1024), id_tt, (j > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16_ss(tbase + COL_DQ, desc_sw128(sDS + (k >> 2) * TB + (k & 3) * 32, 16, 1024),
                                desc_sw128(sK + k * 2048, TB, 1024), id_kt, k > 0 ? 1u : 0u);
                mma_commit(&bars->dq_full);
                mma_commit(&bars->qdo_empty[s]);
                if (next) issue_dp(smem_u32(smem + OFF_DO + s1 * TB));  // dP_j already consumed
            }
        }
    } else {
        // ------- P, dS, dQ drain, epilogue (warps 2..: warpgroup g owns score columns CW g..) -------
        const int g = (warp - 2) >> 2;
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const int wg_tid = threadIdx.x - 64 - 128 * g;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tbase + COL_S + lane_off + CW * g, tDP = tbase + COL_DP + lane_off + CW * g;
        const uint32_t tDQ = tbase + COL_DQ + lane_off + OW * g;
        // P and dS live in two 128 x 64 swizzled halves; this warpgroup's 32 columns are four
        // 16-byte chunks of half g/2
        const uint32_t sPg = smem_u32(smem + OFF_P) + (g >> 1) * TB, sDSg = smem_u32(smem + OFF_DS) + (g >> 1) * TB;
        const uint32_t chunk0 = (g & 1) * 4;
        const uint32_t warp_slot = (g * 4 + q4) * 2048;     // this warp's dQ staging (32 x 64 B)
        const uint32_t sDQw = smem_u32(smem + OFF_DQ) + warp_slot;
        const float sc = p.scale_log2, dsc = p.ds_scale;
        const size_t head_base = static_cast<size_t>(bh) * p.g.n;
        bool ok = run;
        uint32_t sv[32], dv[32];
        float pr[CW];                  // P of this row's CW columns, kept from P_j to dS_j
        float nlse = 0.f, nD = 0.f;    // -lse (log2 units) and -D_i / sqrt(d) of the row
        int32_t lo = 1, hi = 0;        // allowed columns of this slice, relative to the slice
        // Order per query tile: P_0; then for each j: dS_j, P_{j+1}, drain dQ_j.  Building P_{j+1}
        // while the tensor core computes dK_j and dQ_j hides their latency.  Buffer safety comes
        // from commit order: S_{j+1} is issued after dV_j (so s_full(j+1) means P_j was read) and
        // dP_{j+1} after dK_j, dQ_j (so dp_full(j+1) means dS_j was read).
        auto wait_all = [&](uint64_t *bar, int parity) {
            ok = ok && __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, p.err));
            if (ok) tc_fence_after();
            return ok;
        };
        // Row data of query tile j (interval, -lse, -D).  The loads are issued just before the
        // wait for S_j: issued any earlier they would sit in front of the proxy fences of the dS
        // phase, which wait for them.
        float nlse_n = 0.f, nD_n = 0.f;
        int32_t lo_n = 1, hi_n = 0;
        auto prefetch = [&](int j) {
            int32_t lo_abs, hi_abs;
            const int32_t i = row_interval(p.g, part, w.begin + j, row, lo_abs, hi_abs);
            nlse_n = 0.f;
            nD_n = 0.f;
            if (i >= 0) {
                const float lse = p.lse[head_base + i];
                // a row with no allowed key (lse = -inf) has every entry masked to -inf below;
                // keep its base finite so that -inf + base stays -inf instead of NaN
                nlse_n = lse == -INFINITY ? 0.f : -lse * LOG2E;
                nD_n = -p.delta[head_base + i] * dsc;
            }
            const int32_t base = kt * TILE + CW * g;
            lo_n = lo_abs - base;
            hi_n = hi_abs - base;
        };
        auto p_phase = [&](int j) {    // P_j = exp2(S log2e / sqrt(d) - lse log2e) -> SMEM
            prefetch(j);
            nlse = nlse_n;
            nD = nD_n;
            lo = lo_n;
            hi = hi_n;
            if (!wait_all(&bars->s_full, j & 1)) return;
            tmem_ld32(tS, sv);
            tmem_wait_ld();
            if (!(lo <= 0 && hi >= CW - 1)) {
                const uint32_t span = static_cast<uint32_t>(hi - lo);
                const bool none = hi < lo;
#pragma unroll
                for (int e = 0; e < CW; ++e) {
                    const bool keep = !none && static_cast<uint32_t>(e - lo) <= span;
                    sv[e] = keep ? sv[e] : 0xFF800000u;  // -inf: P = 0, dS = 0
                }
            }
            {
                const uint64_t sc2 = f32x2(sc, sc), nl2 = f32x2(nlse, nlse);
#pragma unroll
                for (int e = 0; e < CW; e += 2) {
                    float x0, x1;
                    f32x2_split(fma2(f32x2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2, nl2), x0, x1);
                    pr[e] = ex2(x0);
                    pr[e + 1] = ex2(x1);
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
                st_shared_v4(sPg + sw128_off(row, chunk0 + q), pack_bf16(pr[8 * q], pr[8 * q + 1]),
                             pack_bf16(pr[8 * q + 2], pr[8 * q + 3]), pack_bf16(pr[8 * q + 4], pr[8 * q + 5]),
                             pack_bf16(pr[8 * q + 6], pr[8 * q + 7]));
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->p_ready);
        };
        auto ds_phase = [&](int j) {   // dS_j = P (dP - D) / sqrt(d) -> SMEM
            if (!wait_all(&bars->dp_full, j & 1)) return;
            tmem_ld32(tDP, dv);
            tmem_wait_ld();
            const uint64_t dsc2 = f32x2(dsc, dsc), nD2 = f32x2(nD, nD);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = 8 * q + 2 * e;
                    // dS = P (dP - D) / sqrt(d), two entries per f32x2 instruction
                    const uint64_t t = fma2(f32x2(__uint_as_float(dv[c]), __uint_as_float(dv[c + 1])), dsc2, nD2);
                    float d0, d1;
                    f32x2_split(mul2(f32x2(pr[c], pr[c + 1]), t), d0, d1);
                    pk[e] = pack_bf16(d0, d1);
                }
                st_shared_v4(sDSg + sw128_off(row, chunk0 + q), pk[0], pk[1], pk[2], pk[3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->ds_ready);
        };
        auto drain = [&](int j) {      // dQ_j columns OW g.. : TMEM -> SMEM -> TMA reduce-add
            if (!wait_all(&bars->dq_full, j & 1)) return;
            uint32_t dq[16];
            tmem_ld16(tDQ, dq);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars->dq_empty);
            // per-warp staging (32 rows x 64 bytes, 64-byte swizzle): no cross-warp barrier
            if (lane == 0) bulk_wait_read_all();  // this warp's previous reduce has read it
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q)
                st_shared_v4(sDQw + sw64_off(lane, q), dq[4 * q], dq[4 * q + 1], dq[4 * q + 2], dq[4 * q + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                reduce_warp_f32(p.dq_red, part.qframe, p.g, w.begin + j, bh, OW * g, q4,
                                smem + OFF_DQ + warp_slot);
                bulk_commit();
            }
        };
        if (ok) p_phase(0);
        for (int j = 0; ok && j < nq; ++j) {
            ds_phase(j);
            if (ok && j + 1 < nq) p_phase(j + 1);
            if (ok) drain(j);
        }
        if (lane == 0) bulk_wait_read_all();  // this warp's dQ reduces have read their staging
        // ------- dK, dV epilogue: one key row per thread, warpgroup g writes columns OW g.. -------
        if (ok) {
            const int32_t pos = frame_pos(p.g, part.kframe, part.o, kt, row);
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                uint32_t a16[16];
                tmem_ld16(tbase + (which == 0 ? COL_DK : COL_DV) + lane_off + OW * g, a16);
                tmem_wait_ld();
                float acc[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] = __uint_as_float(a16[e]);
                if (F32) {
                    if (pos >= 0 && *abort == 0) {
                        const float *pf = which == 0 ? p.dk_prev_f32 : p.dv_prev_f32;
                        float *of = (which == 0 ? p.dk_f32 : p.dv_f32) + (head_base + pos) * 64 + OW * g;
                        if (part.merge) {
                            const float4 *src = reinterpret_cast<const float4 *>(pf + (head_base + pos) * 64 + OW * g);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float4 u = src[q];
                                acc[4 * q] += u.x;
                                acc[4 * q + 1] += u.y;
                                acc[4 * q + 2] += u.z;
                                acc[4 * q + 3] += u.w;
                            }
                        }
                        float4 *d4 = reinterpret_cast<float4 *>(of);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            d4[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
                    }
                    continue;
                }
                if (part.merge && pos >= 0) {
                    const uint16_t *prev = which == 0 ? p.dk_prev : p.dv_prev;
                    const uint4 *src = reinterpret_cast<const uint4 *>(prev + (head_base + pos) * 64 + OW * g);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
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
                for (int q = 0; q < 2; ++q)
                    st_shared_v4(dst + sw128_off(row, 2 * g + q), pack_bf16(acc[8 * q], acc[8 * q + 1]),
                                 pack_bf16(acc[8 * q + 2], acc[8 * q + 3]),
                                 pack_bf16(acc[8 * q + 4], acc[8 * q + 5]),
                                 pack_bf16(acc[8 * q + 6], acc[8 * q + 7]));
            }
            fence_proxy_async_smem();
        }
        named_bar_sync(1, 128 * NWG);
        if (!F32 && g == 0 && wg_tid == 0 && ok && *abort == 0) {
            store_tile(p.dk, part.kframe, p.g, part.o, kt, bh, smem + OFF_P);
            store_tile(p.dv, part.kframe, p.g, part.o, kt, bh, smem + OFF_P + TB);
            bulk_commit();
            bulk_wait_read_all();  // the CTA may leave once the copy engine has read SMEM
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
