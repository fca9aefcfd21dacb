// fwd.cu -- fused forward pass of factorized sparse attention on sm_100a, fp32 I/O.
//
// fp32 inputs are split into bf16 high and low parts (hi = bf16(x), lo = bf16(x - hi)) and the
// scores take three products, S = Q_hi K_hi^T + Q_hi K_lo^T + Q_lo K_hi^T, all accumulated in
// fp32 in TMEM; P V runs on bf16 P and V_hi.  (bf16 I/O runs the kernel in fwd_bf16.cu.)
//
// Each work unit is one 128-row query tile of one part of one (batch, head) over the contiguous
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
// independent online softmaxes over disjoint key sets, combined once per unit by
//   M = max(m_0, m_1), L = sum_h 2^(m_h - M) l_h, O = sum_h 2^(m_h - M) O_h / L, lse = M + log2 L
// (log2 units).  No per-tile exchange between the warpgroups is needed.
//
// The kernel is persistent: one CTA per SM (the high and low parts fill the shared memory of two)
// claims units from the longest-first list through a global counter (greedy list scheduling).
// Barrier phases run on across units, so the next unit's Q load and first S product overlap the
// current unit's last softmax and epilogue.  Roles (320 threads):
//   warp 0       TMA producer: Q and its low part, K (with its low part) and V tiles in NST-slot
//                rings with separate barriers
//   warp 1       MMA issuer (one thread): S = Q K^T into TMEM (128 x 128 fp32), issued for the
//                next key tile as soon as the softmax warps hold the current S in registers;
//                per half h, once warpgroup h wrote P_h (bf16, SMEM): O_h += P_h V_h (128 x 64
//                fp32 in TMEM)
//   warps 2..5   softmax of key half 0, warps 6..9 of key half 1; one query row per thread
//                (TMEM lane = row): interval mask, max, exp2, P_h to SMEM, and a rescale of O_h
//                only when the row max grew by more than 2^8 (otherwise the stale max is kept:
//                numerator and denominator use the same max, so the result is unchanged);
//                then the unit's epilogue: combine the halves (each warpgroup writes 32 of the 64
//                fp32 output columns straight to global memory), a merge part folds in the first
//                pass's (O, lse).
#include "tiles.cuh"

namespace st {
namespace {

constexpr int NST = 2;                         // K/V ring depth
constexpr int NSCHED = 4;                      // claimed-unit ring depth
constexpr uint32_t TB = TILE_BYTES;            // one 128 x 64 bf16 tile, 16 KB
constexpr int THREADS = 320;
constexpr uint32_t TMEM_COLS = 256;            // S: 0..127, O_0: 128..191, O_1: 192..255
constexpr float RESCALE_LOG2 = 8.0f;           // keep a stale max while it is within 2^8

// Shared-memory plan, with the bf16 high and low parts of Q and of each K tile:
//   Q, Q_lo | NST x (K, V, K_lo) | P (two 128 x 64 halves: keys 0-63, 64-127) | barriers
// The P area doubles as the (m, l) exchange of the epilogue.
struct Plan {
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_QL = TB;
    static constexpr uint32_t QBYTES = 2 * TB;
    static constexpr uint32_t OFF_STAGE = QBYTES;
    static constexpr uint32_t STAGE = 3 * TB;                   // K at +0, V at +TB, K_lo at +2TB
    static constexpr uint32_t OFF_P = OFF_STAGE + NST * STAGE;
    static constexpr uint32_t OFF_BAR = OFF_P + 2 * TB;
    static constexpr uint32_t OFF_UNITS = OFF_BAR + 256;  // the claimed units' fields, NSCHED entries
    static constexpr uint32_t SMEM_BYTES = OFF_UNITS + NSCHED * 96;
};

struct Bars {
    uint64_t q_full, q_empty, s_full, s_free, o_done, o_free;
    uint64_t st_full, st_read;   // epilogue (m, l) exchange between the two warpgroups
    uint64_t mma_idle;           // every MMA this CTA issued has completed (before teardown)
    uint64_t p_full[2], pv_done[2];
    uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
    uint64_t sched_full[NSCHED], sched_empty[NSCHED];
    int32_t sched[NSCHED];       // unit index claimed by the producer, -1 = no more units
    uint32_t tmem_base;
    int32_t abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

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
// the shared slot j % NSCHED (which the producer fills; it may refill it once every consumer has
// arrived): -1 when the list is exhausted, -2 when the wait gave up.  Called by the MMA thread
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

__global__ void __launch_bounds__(THREADS, 1)
    fwd_split_kernel(const __grid_constant__ FwdParams p)
{
    using L = Plan;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Bars *bars = reinterpret_cast<Bars *>(smem + L::OFF_BAR);
    Unit *slots = reinterpret_cast<Unit *>(smem + L::OFF_UNITS);
    volatile int32_t *abort = &bars->abort;
    const int32_t nunits = p.nitems * p.batch;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, 8);  // one arrival per softmax warp once S is in registers
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->o_free, 256);
        mbar_init(&bars->st_full, 256);
        mbar_init(&bars->st_read, 256);
        mbar_init(&bars->mma_idle, 1);
        for (int h = 0; h < 2; ++h) {
            mbar_init(&bars->p_full[h], 128);
            mbar_init(&bars->pv_done[h], 1);
        }
        for (int s = 0; s < NST; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        for (int s = 0; s < NSCHED; ++s) {
            mbar_init(&bars->sched_full[s], 1);
            mbar_init(&bars->sched_empty[s], 1 + 8);  // the MMA thread and the 8 softmax warps
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
            // K(t) and V(t) sit in ring slot t % NST but have their own barriers: a K slot is
            // free once S(t) is done, a V slot once PV(t) is done, and K(t + 1) is requested
            // ahead of V(t), since the MMA issuer needs it first.
            int32_t TK = 0, TV = 0, kq = 0;  // K tiles, V tiles and Q tiles issued
            auto load_k = [&](const Unit &U, int32_t tile) {
                const int s = TK % NST;
                if (TK >= NST && !mbar_wait(&bars->k_empty[s], ((TK / NST) - 1) & 1, abort, p.err)) return false;
                uint8_t *stage = smem + L::OFF_STAGE + s * L::STAGE;
                mbar_arrive_expect_tx(&bars->k_full[s], 2 * TB);
                load_tile(p.k, U.part.kframe, p.g, U.part.o, tile, U.bh, stage, &bars->k_full[s]);
                load_tile(p.kl, U.part.kframe, p.g, U.part.o, tile, U.bh, stage + 2 * TB, &bars->k_full[s]);
                ++TK;
                return true;
            };
            auto load_v = [&](const Unit &U, int32_t tile) {
                const int s = TV % NST;
                if (TV >= NST && !mbar_wait(&bars->v_empty[s], ((TV / NST) - 1) & 1, abort, p.err)) return false;
                uint8_t *stage = smem + L::OFF_STAGE + s * L::STAGE;
                mbar_arrive_expect_tx(&bars->v_full[s], TB);
                load_tile(p.v, U.part.kframe, p.g, U.part.o, tile, U.bh, stage + TB, &bars->v_full[s]);
                ++TV;
                return true;
            };
            bool fail = false;
            // Units are claimed from a global counter in list order (longest first), so the
            // CTAs share the list greedily, and broadcast to the other roles through sched[].
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
                // the previous unit's S products must be done reading Q before it is replaced
                if (kq > 0 && !mbar_wait(&bars->q_empty, (kq - 1) & 1, abort, p.err)) break;
                ++kq;
                mbar_arrive_expect_tx(&bars->q_full, L::QBYTES);
                load_tile(p.q, U.part.qframe, p.g, U.part.o, U.w.tile, U.bh, smem + L::OFF_Q, &bars->q_full);
                load_tile(p.ql, U.part.qframe, p.g, U.part.o, U.w.tile, U.bh, smem + L::OFF_QL, &bars->q_full);
                fail = !load_k(U, U.w.begin);
                for (int it = 0; !fail && it < U.nkt; ++it)
                    fail = (it + 1 < U.nkt && !load_k(U, U.w.begin + it + 1)) || !load_v(U, U.w.begin + it);
            }
            if (*abort) {  // drain the copies still in flight before the CTA leaves
                volatile int32_t never = 0;
                if (kq > 0) mbar_wait(&bars->q_full, (kq - 1) & 1, &never, p.err);
                for (int32_t j = (TK > NST ? TK - NST : 0); j < TK; ++j)
                    mbar_wait(&bars->k_full[j % NST], (j / NST) & 1, &never, p.err);
                for (int32_t j = (TV > NST ? TV - NST : 0); j < TV; ++j)
                    mbar_wait(&bars->v_full[j % NST], (j / NST) & 1, &never, p.err);
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
            auto issue_s = [&](int32_t t) {
                const uint32_t sK = smem_u32(smem + L::OFF_STAGE + (t % NST) * L::STAGE);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_ss(tS, desc_sw128(sQ + 32 * k, 16, 1024),
                                desc_sw128(sK + 32 * k, 16, 1024), idS, k > 0 ? 1u : 0u);
                {
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
                mma_commit(&bars->k_empty[t % NST]);
            };
            // O_h += P_h V_h: P_h K-major (64 keys, 32 bytes per step), V_h MN-major (rows 64h..,
            // 16 keys = 2048 bytes per step); the first tile of a unit overwrites O_h
            auto issue_pv = [&](int32_t t, int h, bool first) {
                const uint32_t sV = smem_u32(smem + L::OFF_STAGE + (t % NST) * L::STAGE) + TB;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_ss(tbase + 128 + 64 * h, desc_sw128(sP + h * TB + k * 32, 16, 1024),
                                desc_sw128(sV + h * 8192 + k * 2048, TB, 1024), idO,
                                (!first || k > 0) ? 1u : 0u);
                mma_commit(&bars->pv_done[h]);
            };
            int32_t T = 0, kq = 0;
            bool fail = false;
            for (int32_t j = 0; !fail; ++j) {
                Unit U;
                const int32_t u = next_unit(bars, slots, j, false, abort, p.err, U);
                if (u < 0) break;
                if (U.nkt == 0) continue;
                // Order per key tile: S(t+1) | PV_0(t) | PV_1(t).  S(t+1) overwrites S(t) as soon
                // as both halves hold S(t) in registers (s_free), so the tensor pipe computes the
                // next scores while the softmax of this tile runs; the next unit's first S
                // follows the last tile's s_free the same way.
                auto wait_s_free = [&](int32_t t) { return t < 0 || mbar_wait(&bars->s_free, t & 1, abort, p.err); };
                if (!mbar_wait(&bars->q_full, kq & 1, abort, p.err) ||
                    !mbar_wait(&bars->k_full[T % NST], (T / NST) & 1, abort, p.err) || !wait_s_free(T - 1))
                    break;
                tc_fence_after();
                issue_s(T);
                for (int it = 0; it < U.nkt; ++it) {
                    const int32_t t = T + it;
                    if (it + 1 < U.nkt) {
                        if (!mbar_wait(&bars->k_full[(t + 1) % NST], ((t + 1) / NST) & 1, abort, p.err) ||
                            !wait_s_free(t)) {
                            fail = true;
                            break;
                        }
                        tc_fence_after();
                        issue_s(t + 1);
                    } else {
                        mma_commit(&bars->q_empty);  // every S of this unit has been issued
                    }
                    if (!mbar_wait(&bars->v_full[t % NST], (t / NST) & 1, abort, p.err) ||
                        !mbar_wait(&bars->p_full[0], t & 1, abort, p.err)) {
                        fail = true;
                        break;
                    }
                    // the previous unit's epilogue must have read O before the first PV
                    if (it == 0 && kq > 0 && !mbar_wait(&bars->o_free, (kq - 1) & 1, abort, p.err)) {
                        fail = true;
                        break;
                    }
                    tc_fence_after();
                    issue_pv(t, 0, it == 0);
                    if (!mbar_wait(&bars->p_full[1], t & 1, abort, p.err)) { fail = true; break; }
                    tc_fence_after();
                    issue_pv(t, 1, it == 0);
                    mma_commit(&bars->v_empty[t % NST]);
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
        // ---------------- softmax of one key half + epilogue (warps 2..9) ----------------
        const int h = (warp - 2) >> 2;                 // key half owned by this warpgroup
        const int q4 = warp & 3;                       // TMEM lane quarter of this warp
        const int row = q4 * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tbase + lane_off + 64 * h;
        const uint32_t tO = tbase + lane_off + 128 + 64 * h;
        const uint32_t sPh = smem_u32(smem + L::OFF_P) + h * TB;
        const float sc = p.scale_log2;
        bool ok = run;
        uint32_t v[64];
        int32_t T = 0, kq = 0;
        for (int32_t j = 0; ok; ++j) {
            Unit U;
            const int32_t u = next_unit(bars, slots, j, true, abort, p.err, U);
            if (u < 0) break;
            int32_t lo_abs, hi_abs;
            const int32_t i = row_interval(p.g, U.part, U.w.tile, row, lo_abs, hi_abs);
            float m = -INFINITY, l = 0.f;
            for (int it = 0; ok && it < U.nkt; ++it) {
                const int32_t t = T + it;
                // warp-uniform wait: every lane must agree before warp-collective TMEM accesses
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, t & 1, abort, p.err))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int32_t base = (U.w.begin + it) * TILE + 64 * h;
                const int32_t lo = lo_abs - base, hi = hi_abs - base;   // allowed columns of this half
                tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s_free);  // the next S may overwrite this one
                if (!(lo <= 0 && hi >= 63)) {  // boundary tile for this row: interval mask
                    const uint64_t keep = interval_bits64(lo, hi);
                    const uint32_t k0 = static_cast<uint32_t>(keep), k1 = static_cast<uint32_t>(keep >> 32);
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        v[c] = ((c < 32 ? k0 : k1) & (1u << (c & 31))) ? v[c] : 0xFF800000u;  // -inf
                }
                const float m_tile = max64(v) * sc;
                const float m_new = fmaxf(m, m_tile);
                const bool grow = m_new > m + RESCALE_LOG2;   // also true for the first finite max
                const float m_use = grow ? m_new : m;
                const float alpha = grow ? ex2(m - m_use) : 1.f;  // 0 when nothing was seen yet
                const float nb = (m_use == -INFINITY) ? 0.f : -m_use;
                // p = exp2(s log2e / sqrt(d) - m), two columns per f32x2 instruction; two
                // f32x2 partial sums
                const uint64_t sc2 = f32x2(sc, sc), nb2 = f32x2(nb, nb);
                uint64_t ps2[2] = {0ull, 0ull};
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    float x0, x1;
                    f32x2_split(fma2(f32x2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), sc2, nb2), x0, x1);
                    const float p0 = ex2(x0), p1 = ex2(x1);
                    ps2[(c >> 1) & 1] = add2(ps2[(c >> 1) & 1], f32x2(p0, p1));
                    v[c >> 1] = pack_bf16(p0, p1);
                }
                float ps[4];
                f32x2_split(ps2[0], ps[0], ps[1]);
                f32x2_split(ps2[1], ps[2], ps[3]);
                // the previous PV of this half (possibly the previous unit's) must be done with
                // P_h, and with O_h before a rescale
                if (t > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[h], (t - 1) & 1, abort, p.err))) {
                    ok = false;
                    break;
                }
                if (t > 0) tc_fence_after();
                if (it == 0 && kq > 0 &&
                    !__all_sync(0xffffffffu, mbar_wait(&bars->st_read, (kq - 1) & 1, abort, p.err))) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st_shared_v4(sPh + sw128_off(row, c), v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                if (it > 0 && __any_sync(0xffffffffu, grow)) {
                    // rescale this half's partial O (PV of this tile waits for p_full)
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
            if (!ok) break;
            // ---------------- epilogue of the unit: combine the halves ----------------
            const bool has_o = U.nkt > 0;
            if (!has_o && U.part.merge) continue;  // nothing to add to the first pass's result
            const size_t rowoff = (static_cast<size_t>(U.bh) * p.g.n + (i < 0 ? 0 : i));
            // merge part: the first pass's lse, read by both warpgroups before either writes it
            const float L1 = (U.part.merge && i >= 0) ? p.lse[rowoff] * LOG2E : -INFINITY;
            float2 other = make_float2(-INFINITY, 0.f);
            if (has_o) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done, kq & 1, abort, p.err))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // (m, l) exchange through the P area: every PV of this unit is done (o_done);
                // the next P stores of either warpgroup wait for st_read
                float2 *stats = reinterpret_cast<float2 *>(smem + L::OFF_P);
                stats[h * 128 + row] = make_float2(m, l);
                mbar_arrive(&bars->st_full);
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->st_full, kq & 1, abort, p.err))) {
                    ok = false;
                    break;
                }
                other = stats[(1 - h) * 128 + row];
                mbar_arrive(&bars->st_read);
            }
            const float m0 = h == 0 ? m : other.x, l0 = h == 0 ? l : other.y;
            const float m1 = h == 0 ? other.x : m, l1 = h == 0 ? other.y : l;
            const float M = fmaxf(m0, m1);
            const float w0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M);
            const float w1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M);
            const float Lsum = l0 * w0 + l1 * w1;
            const bool has = Lsum > 0.f;
            float lse2 = has ? M + lg2(Lsum) : -INFINITY;       // log2 units
            float c0 = has ? w0 / Lsum : 0.f, c1 = has ? w1 / Lsum : 0.f, cprev = 0.f;
            if (U.part.merge) {
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
            // this warpgroup writes output columns 32h .. 32h + 31 of both halves' O
            float acc[32];
            if (has_o) {
                uint32_t o[32];
                tmem_ld32(tbase + lane_off + 128 + 32 * h, o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) acc[e] = c0 * __uint_as_float(o[e]);
                tmem_ld32(tbase + lane_off + 192 + 32 * h, o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) acc[e] = fmaf(c1, __uint_as_float(o[e]), acc[e]);
                tc_fence_before();
                mbar_arrive(&bars->o_free);  // the next unit's first PV may now overwrite O
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) acc[e] = 0.f;
            }
            if (i >= 0 && *abort == 0) {
                if (cprev != 0.f) {  // add the first pass's output with its log-sum-exp weight
                    const float4 *src = reinterpret_cast<const float4 *>(p.o_prev_f32 + rowoff * 64 + 32 * h);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 q = src[j];
                        acc[4 * j] += cprev * q.x;
                        acc[4 * j + 1] += cprev * q.y;
                        acc[4 * j + 2] += cprev * q.z;
                        acc[4 * j + 3] += cprev * q.w;
                    }
                }
                // one row, this warpgroup's 32 columns, straight to global memory: the first
                // pass's values of these columns were read above by this same thread
                float4 *dst = reinterpret_cast<float4 *>(p.o_f32 + rowoff * 64 + 32 * h);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    dst[j] = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
                if (h == 0) p.lse[rowoff] = lse2 * LN2;
            }
            T += U.nkt;
            if (has_o) ++kq;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

cudaError_t launch_fwd_split(const FwdParams &p, cudaStream_t s)
{
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(fwd_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Plan::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const int64_t units = static_cast<int64_t>(p.nitems) * p.batch;
    if (units == 0) return cudaSuccess;
    const int64_t cap = sm_count();
    const unsigned grid = static_cast<unsigned>(units < cap ? units : cap);
    fwd_split_kernel<<<grid, THREADS, Plan::SMEM_BYTES, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd(const FwdParams &p, bool split, int dqk, int dv, cudaStream_t s)
{
    if (split) return (dqk == 64 && dv == 64) ? launch_fwd_split(p, s) : cudaErrorInvalidValue;
    return launch_fwd_bf16(p, dqk, dv, s);
}

}  // namespace st
