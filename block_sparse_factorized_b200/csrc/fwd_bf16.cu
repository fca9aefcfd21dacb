// fwd_bf16.cu -- fused forward pass of factorized sparse attention on sm_100a, bf16 I/O.
//
// Same work units as the split-precision kernel in fwd.cu: one 128-row query tile of one part of
// one (batch, head) over the contiguous run of 128-key tiles its work item lists
// ("Sparse Transformers（稀疏 Transformer）深度解读报告" §3.5: blocked computation, softmax fused,
// upper triangle never computed; "长序列为何不必让每个 token 看见全部历史？…" §05: only selected
// block pairs enter the kernel, boundary blocks keep an element mask).  Arithmetic ("长序列为何不必
// 让每个 token 看见全部历史？…" §01-§02): S = Q K^T / sqrt(d), softmax over the allowed keys, O = P V,
// and the log-sum-exp saved for the recomputing backward pass ("Sparse Transformers 深度解读报告"
// §3.4).  A row with no allowed key gets O = 0, lse = -inf.
//
// Layout of one CTA (two per SM, persistent, claiming units longest first from a global counter):
//   warp 0      TMA producer: Q (two buffers: the next unit's Q loads while this unit runs), K and
//               V tiles in NST-slot rings with separate barriers
//   warp 1      MMA issuer (one thread): S = Q K^T (128 x 128 fp32 in TMEM), issued for the next
//               key tile as soon as the softmax holds the current S in registers; once the
//               softmax wrote P (bf16 pairs, its own 64 TMEM columns), O += P V with P read from
//               TMEM.  TMEM: S 128 columns, O 64, P 64 -- the 256 a CTA allocates.
//   warps 2..5  softmax, one query row per thread over all 128 columns of the tile: interval
//               mask, row max, exp2, P to TMEM, and a rescale of O only when the row max grew by
//               more than 2^8 (a stale max is kept otherwise: numerator and denominator share it);
//               at the end of a unit, O / l and lse, written row by row (a merge part folds in
//               the first pass's (O, lse) by log-sum-exp weights)
// While one CTA's softmax runs, the other CTA on the SM uses the tensor core, and the reverse.
#include "tiles.cuh"

namespace st {
namespace {

constexpr int NST = 2;                         // K/V ring depth
constexpr int NQB = 2;                         // Q buffers
constexpr int NSCHED = 4;                      // claimed-unit ring depth
constexpr int THREADS = 192;
constexpr float RESCALE_LOG2 = 8.0f;           // keep a stale max while it is within 2^8

// Query-key rows of width DQK, value rows of width DV.
template <int DQK, int DV>
struct Cfg {
    static constexpr uint32_t QB = Tile<DQK>::BYTES, VB = Tile<DV>::BYTES;
    static constexpr uint32_t COL_S = 0;                       // S: 128 fp32 columns
    static constexpr uint32_t COL_O = 128;                     // O: DV fp32 columns
    static constexpr uint32_t COL_P = 128 + DV;                // P: 128 bf16 as 64 columns of pairs
    static constexpr uint32_t COLS_USED = COL_P + 64;
    static constexpr int CTAS_PER_SM = COLS_USED <= 256 ? 2 : 1;
    static constexpr uint32_t TMEM_COLS = CTAS_PER_SM == 2 ? 256 : 512;
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + NQB * QB;
    static constexpr uint32_t OFF_V = OFF_K + NST * QB;
    // a merge epilogue's per-warp staging of its 32 output rows (DV * 2 bytes each)
    static constexpr uint32_t OFF_STG = OFF_V + NST * VB;
    static constexpr uint32_t STG_ROW = DV * 2;
    static constexpr uint32_t OFF_BAR = OFF_STG + 4 * 32 * STG_ROW;
    static constexpr uint32_t OFF_UNITS = OFF_BAR + 256;
    static constexpr uint32_t SMEM_BYTES = OFF_UNITS + 4 * 96;
    static_assert(SMEM_BYTES * CTAS_PER_SM <= 228 * 1024 - CTAS_PER_SM * 1024, "shared memory per SM");
};

struct Bars {
    uint64_t q_full[NQB], q_empty[NQB];
    uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
    uint64_t s_full, s_free, p_full, pv_done, o_done, o_free;
    uint64_t mma_idle;           // every MMA this CTA issued has completed (before teardown)
    uint64_t sched_full[NSCHED], sched_empty[NSCHED];
    int32_t sched[NSCHED];       // unit index claimed by the producer, -1 = no more units
    uint32_t tmem_base;
    int32_t abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct Unit {
    WorkItem w;
    Part part;
    int32_t bh, nkt;
};
static_assert(sizeof(Unit) <= 96, "unit slot");

__device__ __forceinline__ Unit load_unit(const FwdParams &p, int32_t u)
{
    Unit r;
    const int32_t item = u / p.batch, b = u - item * p.batch;
    r.w = p.items[item];
    r.part = p.parts[r.w.part];
    r.bh = b * p.heads + r.part.head;
    r.nkt = r.w.end - r.w.begin;
    return r;
}

// The j-th unit this CTA processes, as claimed by the producer, with its fields copied out of
// the shared slot j % NSCHED (the producer refills a slot once every consumer has arrived):
// -1 when the list is exhausted, -2 when the wait gave up.  Called by the MMA thread
// (warp_wide false) or by whole softmax warps.
__device__ __forceinline__ int32_t next_unit(Bars *bars, const Unit *slots, int32_t j, bool warp_wide,
                                             volatile int32_t *abort, int32_t *err, Unit &U)
{
    const int s = j % NSCHED;
    bool ok = mbar_wait(&bars->sched_full[s], (j / NSCHED) & 1, abort, err);
    if (warp_wide) ok = __all_sync(0xffffffffu, ok);
    if (!ok) return -2;
    const int32_t u = *reinterpret_cast<volatile int32_t *>(&bars->sched[s]);
    if (u >= 0) U = slots[s];
    if (warp_wide) __syncwarp();
    if (!warp_wide || (threadIdx.x & 31) == 0) mbar_arrive(&bars->sched_empty[s]);
    return u;
}

// Row max of 128 scores: eight independent partial maxima folded with three-input max.
__device__ __forceinline__ float max128(const uint32_t (&v)[128])
{
    float a[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = fmaxf(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
#pragma unroll
    for (int c = 16; c < 128; c += 2)
        a[(c >> 1) & 7] = max3f(a[(c >> 1) & 7], __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
    return max3f(max3f(a[0], a[1], a[2]), max3f(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
}

// The 32 registers of v starting at e, as an array reference for the TMEM load/store helpers.
__device__ __forceinline__ uint32_t (&part32(uint32_t (&v)[128], int e))[32]
{
    return *reinterpret_cast<uint32_t(*)[32]>(&v[e]);
}

template <int DQK, int DV>
__global__ void __launch_bounds__(THREADS, (Cfg<DQK, DV>::CTAS_PER_SM)) fwd_bf16_kernel(const __grid_constant__ FwdParams p)
{
    using C = Cfg<DQK, DV>;
    constexpr uint32_t OFF_Q = C::OFF_Q, OFF_K = C::OFF_K, OFF_V = C::OFF_V, OFF_BAR = C::OFF_BAR,
                       OFF_UNITS = C::OFF_UNITS, QB = C::QB, VB = C::VB, TMEM_COLS = C::TMEM_COLS,
                       COL_S = C::COL_S, COL_O = C::COL_O, COL_P = C::COL_P;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Bars *bars = reinterpret_cast<Bars *>(smem + OFF_BAR);
    Unit *slots = reinterpret_cast<Unit *>(smem + OFF_UNITS);
    volatile int32_t *abort = &bars->abort;
    const int32_t nunits = p.nitems * p.batch;

    if (threadIdx.x == 0) {
        for (int b = 0; b < NQB; ++b) {
            mbar_init(&bars->q_full[b], 1);
            mbar_init(&bars->q_empty[b], 1);
        }
        for (int s = 0; s < NST; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, 4);  // one arrival per softmax warp once S is in registers
        mbar_init(&bars->p_full, 128);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->o_free, 128);
        mbar_init(&bars->mma_idle, 1);
        for (int s = 0; s < NSCHED; ++s) {
            mbar_init(&bars->sched_full[s], 1);
            mbar_init(&bars->sched_empty[s], 1 + 4);  // the MMA thread and the 4 softmax warps
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
    const bool run = (*abort == 0);

    // Phase bookkeeping shared by every role: T counts key tiles processed so far by this CTA,
    // kq counts units with at least one key tile (the ones that use Q, O and the o_* barriers).
    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0 && run) {
            tma_prefetch(&p.q.nat);
            tma_prefetch(&p.k.nat);
            tma_prefetch(&p.v.nat);
            // K(t) and V(t) sit in ring slot t % NST with their own barriers: a K slot is free
            // once S(t) is done, a V slot once O += P(t) V(t) is done; K(t + 1) is requested
            // ahead of V(t), since the MMA issuer needs it first.
            int32_t TK = 0, TV = 0, kq = 0;  // K tiles, V tiles and Q tiles issued
            auto load_k = [&](const Unit &U, int32_t tile) {
                const int s = TK % NST;
                if (TK >= NST && !mbar_wait(&bars->k_empty[s], ((TK / NST) - 1) & 1, abort, p.err)) return false;
                mbar_arrive_expect_tx(&bars->k_full[s], QB);
                load_tile_w<DQK>(p.k, U.part.kframe, p.g, U.part.o, tile, U.bh, smem + OFF_K + s * QB, &bars->k_full[s]);
                ++TK;
                return true;
            };
            auto load_v = [&](const Unit &U, int32_t tile) {
                const int s = TV % NST;
                if (TV >= NST && !mbar_wait(&bars->v_empty[s], ((TV / NST) - 1) & 1, abort, p.err)) return false;
                mbar_arrive_expect_tx(&bars->v_full[s], VB);
                load_tile_w<DV>(p.v, U.part.kframe, p.g, U.part.o, tile, U.bh, smem + OFF_V + s * VB, &bars->v_full[s]);
                ++TV;
                return true;
            };
            bool fail = false;
            for (int32_t j = 0; !fail; ++j) {
                const int s = j % NSCHED;
                if (j >= NSCHED && !mbar_wait(&bars->sched_empty[s], ((j / NSCHED) - 1) & 1, abort, p.err))
                    break;
                int32_t u = atomicAdd(p.sched, 1);
                if (u >= nunits) u = -1;
                bars->sched[s] = u;
                Unit U;
                if (u >= 0) {
                    U = load_unit(p, u);
                    slots[s] = U;
                }
                mbar_arrive(&bars->sched_full[s]);
                if (u < 0) break;
                if (U.nkt == 0) continue;
                // Q buffer kq % NQB: free once every S of the unit that last used it is done
                const int qb = kq % NQB;
                if (kq >= NQB && !mbar_wait(&bars->q_empty[qb], ((kq / NQB) - 1) & 1, abort, p.err)) break;
                ++kq;
                mbar_arrive_expect_tx(&bars->q_full[qb], QB);
                load_tile_w<DQK>(p.q, U.part.qframe, p.g, U.part.o, U.w.tile, U.bh, smem + OFF_Q + qb * QB, &bars->q_full[qb]);
                fail = !load_k(U, U.w.begin);
                for (int it = 0; !fail && it < U.nkt; ++it)
                    fail = (it + 1 < U.nkt && !load_k(U, U.w.begin + it + 1)) || !load_v(U, U.w.begin + it);
            }
            if (*abort) {  // drain the copies still in flight before the CTA leaves
                volatile int32_t never = 0;
                for (int32_t i = (kq > NQB ? kq - NQB : 0); i < kq; ++i)
                    mbar_wait(&bars->q_full[i % NQB], (i / NQB) & 1, &never, p.err);
                for (int32_t i = (TK > NST ? TK - NST : 0); i < TK; ++i)
                    mbar_wait(&bars->k_full[i % NST], (i / NST) & 1, &never, p.err);
                for (int32_t i = (TV > NST ? TV - NST : 0); i < TV; ++i)
                    mbar_wait(&bars->v_full[i % NST], (i / NST) & 1, &never, p.err);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0 && run) {
            constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idO = idesc_bf16(128, DV, false, true);
            // S = Q K^T: both operands K-major, DQK / 16 steps of 16 elements
            auto issue_s = [&](int32_t t, int qb) {
                const uint32_t sQ = smem_u32(smem + OFF_Q + qb * QB), sK = smem_u32(smem + OFF_K + (t % NST) * QB);
#pragma unroll
                for (int k = 0; k < DQK / 16; ++k)
                    mma_bf16_ss(tbase + COL_S, Tile<DQK>::kmajor(sQ, k), Tile<DQK>::kmajor(sK, k), idS,
                                k > 0 ? 1u : 0u);
                mma_commit(&bars->s_full);
                mma_commit(&bars->k_empty[t % NST]);
            };
            // O += P V: P from TMEM (8 columns of bf16 pairs = 16 keys per step), V MN-major
            // (16 keys per step); the first tile of a unit overwrites O
            auto issue_pv = [&](int32_t t, bool first) {
                const uint32_t sV = smem_u32(smem + OFF_V + (t % NST) * VB);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16_ts(tbase + COL_O, tbase + COL_P + 8 * k, Tile<DV>::mnmajor(sV, k), idO,
                                (!first || k > 0) ? 1u : 0u);
                mma_commit(&bars->pv_done);
                mma_commit(&bars->v_empty[t % NST]);
            };
            // S(t) may overwrite S(t-1) once every softmax warp holds S(t-1) in registers
            auto wait_s_free = [&](int32_t t) { return t < 1 || mbar_wait(&bars->s_free, (t - 1) & 1, abort, p.err); };
            int32_t T = 0, kq = 0;
            bool fail = false;
            for (int32_t j = 0; !fail; ++j) {
                Unit U;
                const int32_t u = next_unit(bars, slots, j, false, abort, p.err, U);
                if (u < 0) break;
                if (U.nkt == 0) continue;
                // Order per key tile t: S(t+1) | O += P(t) V(t).  The tensor core computes the
                // next scores while the softmax of this tile runs; a unit's first S follows the
                // previous unit's last s_free the same way (its Q is in the other buffer).
                const int qb = kq % NQB;
                if (!mbar_wait(&bars->q_full[qb], (kq / NQB) & 1, abort, p.err) ||
                    !mbar_wait(&bars->k_full[T % NST], (T / NST) & 1, abort, p.err) || !wait_s_free(T))
                    break;
                tc_fence_after();
                issue_s(T, qb);
                if (U.nkt == 1) mma_commit(&bars->q_empty[qb]);  // every S of this unit issued
                for (int it = 0; it < U.nkt; ++it) {
                    const int32_t t = T + it;
                    if (it + 1 < U.nkt) {
                        if (!mbar_wait(&bars->k_full[(t + 1) % NST], ((t + 1) / NST) & 1, abort, p.err) ||
                            !wait_s_free(t + 1)) {
                            fail = true;
                            break;
                        }
                        tc_fence_after();
                        issue_s(t + 1, qb);
                        if (it + 2 == U.nkt) mma_commit(&bars->q_empty[qb]);
                    }
                    if (!mbar_wait(&bars->v_full[t % NST], (t / NST) & 1, abort, p.err) ||
                        !mbar_wait(&bars->p_full, t & 1, abort, p.err)) {
                        fail = true;
                        break;
                    }
                    // the previous unit's epilogue must have read O before the first product
                    if (it == 0 && kq > 0 && !mbar_wait(&bars->o_free, (kq - 1) & 1, abort, p.err)) {
                        fail = true;
                        break;
                    }
                    tc_fence_after();
                    issue_pv(t, it == 0);
                }
                if (fail) break;
                mma_commit(&bars->o_done);
                T += U.nkt;
                ++kq;
            }
            // no product may still be running when TMEM is released (also after an abort)
            mma_commit(&bars->mma_idle);
            volatile int32_t never = 0;
            mbar_wait(&bars->mma_idle, 0, &never, p.err);
        }
    } else {
        // ---------------- softmax + epilogue (warps 2..5, one query row per thread) ----------------
        const int q4 = warp & 3;                       // TMEM lane quarter of this warp
        const int row = q4 * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tbase + lane_off + COL_S, tO = tbase + lane_off + COL_O, tP = tbase + lane_off + COL_P;
        const float sc = p.scale_log2;
        bool ok = run;
        uint32_t v[128];
        int32_t T = 0, kq = 0;
        // what a unit's epilogue needs: row, tile, batch-head, merge flag, O-unit index, (m, l)
        struct Pending {
            int32_t i, bh, merge, kq;
            float m, l;
        };
        // O / l (and the first pass's output for a merge part) and lse, written row by row.
        // Reads O from TMEM, then frees it.
        auto epilogue = [&](const Pending &e, bool has_o) {
            if (has_o) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done, e.kq & 1, abort, p.err))) {
                    ok = false;
                    return;
                }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < DV / 32; ++c) tmem_ld32(tO + 32 * c, part32(v, 32 * c));
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&bars->o_free);  // the next unit's first product may now overwrite O
            }
            const size_t rowoff = static_cast<size_t>(e.bh) * p.g.n + (e.i < 0 ? 0 : e.i);
            const bool has = e.l > 0.f;
            float lse2 = has ? e.m + lg2(e.l) : -INFINITY;  // log2 units
            float cnew = has ? 1.f / e.l : 0.f, cprev = 0.f;
            if (e.merge) {  // fold in the first pass's (O, lse) by log-sum-exp weights
                const float L1 = e.i >= 0 ? p.lse[rowoff] * LOG2E : -INFINITY;
                const float Lm = fmaxf(L1, lse2);
                if (Lm == -INFINITY) {
                    cnew = 0.f;
                    lse2 = -INFINITY;
                } else {
                    const float e1 = ex2(L1 - Lm), e2 = ex2(lse2 - Lm), tot = e1 + e2;
                    cprev = e1 / tot;
                    cnew *= e2 / tot;
                    lse2 = Lm + lg2(tot);
                }
            }
            const bool live = e.i >= 0 && *abort == 0;  // not a grid-frame padding row
            if (!__any_sync(0xffffffffu, cprev != 0.f)) {
                // no first-pass output to fold in: 8 columns (16 bytes) at a time, row by row
                if (live) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.o + rowoff * DV);
#pragma unroll
                    for (int q = 0; q < DV / 8; ++q) {
                        float a[8];
#pragma unroll
                        for (int c = 0; c < 8; ++c) a[c] = has_o ? cnew * __uint_as_float(v[8 * q + c]) : 0.f;
                        dst[q] = make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]),
                                            pack_bf16(a[6], a[7]));
                    }
                    p.lse[rowoff] = lse2 * LN2;
                }
                return;
            }
            // A merge: the warp's 32 rows go through its shared staging, so that the first pass's
            // rows are read whole (a warp instruction reads RPI complete rows of DV * 2 bytes, not
            // 16 bytes of each of 32 rows scattered over the grid frame) and written back whole.
            // Chunk c (16 bytes) of staged row r sits at stg_off(r, c), swizzled so that both
            // access patterns are free of bank conflicts.
            constexpr int CPR = DV / 8;                 // 16-byte chunks per row
            constexpr int RPI = 32 / CPR;               // rows per warp instruction
            const uint32_t stg = smem_u32(smem + C::OFF_STG) + q4 * 32 * C::STG_ROW;
            auto stg_off = [&](uint32_t r, uint32_t c) {
                return CPR >= 8 ? r * C::STG_ROW + ((c ^ (r & 7u)) << 4) : sw64_off(r, c);
            };
            const int32_t sub_row = lane / CPR, sub_c = lane % CPR;
#pragma unroll
            for (int r0 = 0; r0 < 32; r0 += RPI) {
                const int32_t r = r0 + sub_row;
                const int32_t ir = __shfl_sync(0xffffffffu, live ? e.i : -1, r);
                uint4 x = make_uint4(0u, 0u, 0u, 0u);
                if (ir >= 0)
                    x = reinterpret_cast<const uint4 *>(p.o_prev + (static_cast<size_t>(e.bh) * p.g.n + ir) * DV)[sub_c];
                st_shared_v4(stg + stg_off(r, sub_c), x.x, x.y, x.z, x.w);
            }
            __syncwarp();
            // this thread's row: O / l plus the first pass's share, as bf16, into the staging
#pragma unroll
            for (int q = 0; q < DV / 8; ++q) {
                float a[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) a[c] = has_o ? cnew * __uint_as_float(v[8 * q + c]) : 0.f;
                const uint4 x = ld_shared_v4(stg + stg_off(lane, q));
                const uint32_t pw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    a[2 * c] = fmaf(cprev, bf16_lo(pw[c]), a[2 * c]);
                    a[2 * c + 1] = fmaf(cprev, bf16_hi(pw[c]), a[2 * c + 1]);
                }
                st_shared_v4(stg + stg_off(lane, q), pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]),
                             pack_bf16(a[6], a[7]));
            }
            __syncwarp();
            // whole rows to global memory (rows of the grid frame's padding are skipped)
#pragma unroll
            for (int r0 = 0; r0 < 32; r0 += RPI) {
                const int32_t r = r0 + sub_row;
                const int32_t ir = __shfl_sync(0xffffffffu, live ? e.i : -1, r);
                const uint4 x = ld_shared_v4(stg + stg_off(r, sub_c));
                if (ir >= 0)
                    reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(e.bh) * p.g.n + ir) * DV)[sub_c] = x;
            }
            __syncwarp();  // the staging is reused by this warp's next epilogue
            if (live) p.lse[rowoff] = lse2 * LN2;
        };
        for (int32_t j = 0; ok; ++j) {
            Unit U;
            const int32_t u = next_unit(bars, slots, j, true, abort, p.err, U);
            if (u < 0) break;
            int32_t lo_abs, hi_abs;
            const int32_t i = row_interval(p.g, U.part, U.w.tile, row, lo_abs, hi_abs);
            if (U.nkt == 0 && U.part.merge) continue;  // no key tile: nothing to add to the first pass
            float m = -INFINITY, l = 0.f;              // (a unit without one writes O = 0, lse = -inf)
            for (int it = 0; ok && it < U.nkt; ++it) {
                const int32_t t = T + it;
                // warp-uniform wait: every lane must agree before warp-collective TMEM accesses
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, t & 1, abort, p.err))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, part32(v, 32 * c));
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s_free);  // the next S may overwrite this one
                const int32_t base = (U.w.begin + it) * TILE;
                const int32_t lo = lo_abs - base, hi = hi_abs - base;  // allowed columns of the tile
                if (!(lo <= 0 && hi >= TILE - 1)) {  // boundary tile for this row: interval mask
                    const uint64_t k01 = interval_bits64(lo, hi), k23 = interval_bits64(lo - 64, hi - 64);
                    const uint32_t kw[4] = {static_cast<uint32_t>(k01), static_cast<uint32_t>(k01 >> 32),
                                            static_cast<uint32_t>(k23), static_cast<uint32_t>(k23 >> 32)};
#pragma unroll
                    for (int c = 0; c < 128; ++c) v[c] = (kw[c >> 5] & (1u << (c & 31))) ? v[c] : 0xFF800000u;
                }
                const float m_tile = max128(v) * sc;
                const float m_new = fmaxf(m, m_tile);
                const bool grow = m_new > m + RESCALE_LOG2;   // also true for the first finite max
                const float m_use = grow ? m_new : m;
                const float alpha = grow ? ex2(m - m_use) : 1.f;  // 0 when nothing was seen yet
                const float nb = (m_use == -INFINITY) ? 0.f : -m_use;
                // p = exp2(s log2e / sqrt(d) - m), two columns per f32x2 instruction; P packed as
                // bf16 pairs (column c of the TMEM operand holds keys 2c, 2c + 1) into v[0..63]
                const uint64_t sc2 = f32x2(sc, sc), nb2 = f32x2(nb, nb);
                uint64_t ps2[2] = {0ull, 0ull};
#pragma unroll
                for (int c = 0; c < 128; c += 2) {
                    float x0, x1;
                    f32x2_split(fma2(f32x2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), sc2, nb2), x0, x1);
                    const float p0 = ex2(x0), p1 = ex2(x1);
                    ps2[(c >> 1) & 1] = add2(ps2[(c >> 1) & 1], f32x2(p0, p1));
                    v[c >> 1] = pack_bf16(p0, p1);
                }
                // the previous product (possibly the previous unit's) must be done reading P, and
                // with O before a rescale
                if (t > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars->pv_done, (t - 1) & 1, abort, p.err))) {
                    ok = false;
                    break;
                }
                if (t > 0) tc_fence_after();
                if (it > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
                    for (int c = 0; c < DV / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tO + 32 * c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(tO + 32 * c, o);
                    }
                }
                tmem_st32(tP, part32(v, 0));
                tmem_st32(tP + 32, part32(v, 32));
                tmem_wait_st();
                float s0, s1, s2, s3;
                f32x2_split(ps2[0], s0, s1);
                f32x2_split(ps2[1], s2, s3);
                l = l * alpha + ((s0 + s1) + (s2 + s3));
                m = m_use;
                tc_fence_before();
                mbar_arrive(&bars->p_full);
            }
            if (!ok) break;
            epilogue(Pending{i, U.bh, U.part.merge, kq, m, l}, U.nkt > 0);
            if (U.nkt > 0) {
                T += U.nkt;
                ++kq;
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


template <int DQK, int DV>
cudaError_t launch_w(const FwdParams &p, cudaStream_t s)
{
    using C = Cfg<DQK, DV>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(fwd_bf16_kernel<DQK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const int64_t units = static_cast<int64_t>(p.nitems) * p.batch;
    if (units == 0) return cudaSuccess;
    const int64_t cap = static_cast<int64_t>(sm_count()) * C::CTAS_PER_SM;
    fwd_bf16_kernel<DQK, DV><<<static_cast<unsigned>(units < cap ? units : cap), THREADS, C::SMEM_BYTES, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

// Row widths (query-key, value) with a kernel: (32, 32), (64, 64), (128, 128), (64, 128).
bool fwd_bf16_widths_supported(int dqk, int dv)
{
    return (dqk == dv && (dqk == 32 || dqk == 64 || dqk == 128)) || (dqk == 64 && dv == 128);
}

cudaError_t launch_fwd_bf16(const FwdParams &p, int dqk, int dv, cudaStream_t s)
{
    if (dqk == 32 && dv == 32) return launch_w<32, 32>(p, s);
    if (dqk == 64 && dv == 64) return launch_w<64, 64>(p, s);
    if (dqk == 128 && dv == 128) return launch_w<128, 128>(p, s);
    if (dqk == 64 && dv == 128) return launch_w<64, 128>(p, s);
    return cudaErrorInvalidValue;
}

}  // namespace st
