// bwd.cu -- backward pass of factorized sparse attention on sm_100a, with recomputation.
//
// "Sparse Transformers（稀疏 Transformer）深度解读报告" §3.4: attention weights are not stored;
// the backward pass rebuilds them.  Here P_ij = exp(S_ij - lse_i) from the saved log-sum-exp,
// then (plain calculus of O = softmax(Q K^T / sqrt d) V over the allowed keys)
//   dV_j += P_ij dO_i,  dP_ij = dO_i . v_j,  dS_ij = P_ij (dP_ij - D_i),  D_i = dO_i . O_i,
//   dK_j += dS_ij q_i / sqrt(d),  dQ_i += dS_ij k_j / sqrt(d).
// A work item is one 128-key tile (of one part, one batch-head) with the contiguous run of query
// tiles that read it (at most a fixed number: a longer run is split into chunks, whose fp32
// partials a pass after this kernel sums in chunk order).  dK and dV accumulate in TMEM and are
// written once per item; dQ of each (query tile, key tile) pair is added to an fp32 accumulator
// with TMA reduce-adds.
//
// The kernel is persistent (one CTA per SM) and claims items, longest first, from a global
// counter.  Both the MMA issuer and the softmax warps walk one flat sequence of query tiles over
// all the items they claim, so the next item's S and dP (K and V have two buffers) and its first P
// overlap the current item's last tile and its dK/dV epilogue, even for an item of one tile.
// Roles (576 threads):
//   warp 0      TMA: K and V of each item (KVS slots), Q and dO per query tile (2-stage ring)
//   warp 1      MMA issuer: S = Q K^T and dP = dO V^T (TMEM, 128 x 128 fp32 each), then after
//               the softmax warps wrote P and dS (bf16, SMEM): dV += P^T dO, dK += dS^T Q
//               (TMEM 128 x 64 each, resident for the whole item) and dQ = dS K (TMEM 128 x 64)
//   warps 2..17 four warpgroups, one query row per thread, warpgroup g owning score columns
//               32g..32g+31 (no row reduction is needed here: P comes from the saved lse):
//               interval mask, P, dS; dQ columns 16g.. staged per warp and added to the fp32
//               accumulator with a TMA reduce (or, where this item is the only one that reads
//               the query tile, written to dQ directly); at the end of an item one key row per
//               thread: dK, dV columns 16g.. staged per warp (32 rows) in the warp's dQ slot for
//               two TMA stores (bf16), written row by row (fp32), or stored as the fp32 partial
//               of a split key tile.
// A merge part (second pass of a merged head) adds the dK/dV the first pass wrote.
#include <type_traits>

#include "tiles.cuh"

namespace st {
namespace {

constexpr uint32_t TB = TILE_BYTES;              // a 128 x 128 bf16 operand half (P, dS): 16 KB
constexpr int NSCHED = 4;                          // claimed-item ring depth
constexpr int NWG = 4;                             // softmax warpgroups
constexpr int NSM = 128 * NWG;                     // softmax threads
constexpr int THREADS = 64 + NSM;
constexpr int CW = 128 / NWG;                      // score columns per warpgroup (32)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256;
constexpr int MAX_STAGES = 2;                      // ring depths are at most this

// Query-key rows of width DQK, value rows of width DV.
template <int DQK, int DV>
struct BCfg {
    static constexpr uint32_t QB = Tile<DQK>::BYTES, VB = Tile<DV>::BYTES;  // Q or K tile, V or dO tile
    // ring depths: 128-wide value rows fit shared memory only with single buffers
    static constexpr int KVS = DV > 64 ? 1 : 2;    // K/V slots (items in flight)
    static constexpr int NST = DV > 64 ? 1 : 2;    // Q/dO ring depth
    static constexpr int OWQ = DQK / NWG;          // dQ / dK columns per warpgroup
    static constexpr int OWV = DV / NWG;           // dV columns per warpgroup
    // per-warp staging: the dQ slice (32 rows x OWQ fp32), or the dK and dV slices (bf16)
    static constexpr uint32_t STG_DQ = 32 * OWQ * 4, STG_DK = 32 * OWQ * 2, STG_DV = 32 * OWV * 2;
    static constexpr uint32_t STG = STG_DQ > STG_DK + STG_DV ? STG_DQ : STG_DK + STG_DV;
    static constexpr uint32_t OFF_K = 0;                       // KVS slots
    static constexpr uint32_t OFF_V = OFF_K + KVS * QB;        // KVS slots
    static constexpr uint32_t OFF_Q = OFF_V + KVS * VB;        // NST tiles
    static constexpr uint32_t OFF_DO = OFF_Q + NST * QB;       // NST tiles
    static constexpr uint32_t OFF_P = OFF_DO + NST * VB;       // 2 halves
    static constexpr uint32_t OFF_DS = OFF_P + 2 * TB;         // 2 halves
    static constexpr uint32_t OFF_DQ = OFF_DS + 2 * TB;        // staging, NSM / 32 warps
    static constexpr uint32_t OFF_BAR = OFF_DQ + (NSM / 32) * ((STG + 1023) & ~1023u);
    static constexpr uint32_t OFF_ITEMS = OFF_BAR + 256;       // the claimed items' fields
    static constexpr uint32_t SMEM_BYTES = OFF_ITEMS + NSCHED * 96;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static constexpr uint32_t COL_DK = COL_DV + DV, COL_DQ = COL_DK + DQK;
    static_assert(COL_DQ + DQK <= TMEM_COLS, "tensor memory");
};

struct Bars {
    uint64_t kv_full[MAX_STAGES], kv_empty[MAX_STAGES];
    uint64_t qdo_full[MAX_STAGES], qdo_empty[MAX_STAGES];
    uint64_t s_full, dp_full, p_ready, ds_ready, dq_full, dq_empty;
    uint64_t acc_free;             // the epilogue has read dK and dV of the item from TMEM
    uint64_t mma_idle;             // every MMA this CTA issued has completed (before teardown)
    uint64_t sched_full[NSCHED], sched_empty[NSCHED];
    int32_t sched[NSCHED];         // claimed item (index into items x batch), -1 = none left
    uint32_t tmem_base;
    int32_t abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct Item {
    WorkItem w;
    Part part;
    int32_t b, bh, nq;
};
static_assert(sizeof(Item) <= 96, "item slot");

__device__ __forceinline__ Item load_item(const BwdParams &p, int32_t u)
{
    Item r;
    const int32_t item = u / p.batch;
    r.b = u - item * p.batch;
    r.w = p.items[item];
    r.part = p.parts[r.w.part];
    r.bh = r.b * p.heads + r.part.head;
    r.nq = r.w.end - r.w.begin;
    return r;
}

// The j-th item this CTA processes, as claimed by the producer (its fields are in the shared
// item slot j % NSCHED until the caller releases it with done_item): -1 when the list is
// exhausted, -2 when the wait gave up.  Called by the MMA thread (warp_wide false) or by whole
// softmax warps.
__device__ __forceinline__ int32_t next_item(Bars *bars, int32_t j, bool warp_wide, volatile int32_t *abort,
                                             int32_t *err)
{
    const int s = j % NSCHED;
    bool ok = mbar_wait(&bars->sched_full[s], (j / NSCHED) & 1, abort, err);
    if (warp_wide) ok = __all_sync(0xffffffffu, ok);
    if (!ok) return -2;
    return *reinterpret_cast<volatile int32_t *>(&bars->sched[s]);
}
__device__ __forceinline__ void done_item(Bars *bars, int32_t j, bool warp_wide)
{
    if (warp_wide) __syncwarp();
    if (!warp_wide || (threadIdx.x & 31) == 0) mbar_arrive(&bars->sched_empty[j % NSCHED]);
}

// F32: fp32 I/O -- dK and dV are written in fp32 (the MMAs run on bf16 copies; query-key and
// value rows of 64).  DQK, DV: the widths of the query-key and value rows.
template <bool F32, int DQK, int DV>
__global__ void __launch_bounds__(THREADS, 1) bwd_kernel(const __grid_constant__ BwdParams p)
{
    using C = BCfg<DQK, DV>;
    constexpr int KVS = C::KVS, NST = C::NST, OWQ = C::OWQ, OWV = C::OWV;
    constexpr uint32_t QB = C::QB, VB = C::VB, OFF_K = C::OFF_K, OFF_V = C::OFF_V, OFF_Q = C::OFF_Q,
                       OFF_DO = C::OFF_DO, OFF_P = C::OFF_P, OFF_DS = C::OFF_DS, OFF_DQ = C::OFF_DQ,
                       OFF_BAR = C::OFF_BAR, OFF_ITEMS = C::OFF_ITEMS, COL_DK = C::COL_DK,
                       COL_DQ = C::COL_DQ;
    static_assert(!F32 || (DQK == 64 && DV == 64), "fp32 I/O has rows of 64");
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Bars *bars = reinterpret_cast<Bars *>(smem + OFF_BAR);
    volatile int32_t *abort = &bars->abort;
    const int32_t nunits = p.nitems * p.batch;

    if (threadIdx.x == 0) {
        for (int s = 0; s < KVS; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int s = 0; s < NST; ++s) {
            mbar_init(&bars->qdo_full[s], 1);
            mbar_init(&bars->qdo_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->dp_full, 1);
        mbar_init(&bars->p_ready, NSM);
        mbar_init(&bars->ds_ready, NSM);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, NSM);
        mbar_init(&bars->acc_free, NSM);
        mbar_init(&bars->mma_idle, 1);
        for (int s = 0; s < NSCHED; ++s) {
            mbar_init(&bars->sched_full[s], 1);
            mbar_init(&bars->sched_empty[s], 1 + NSM / 32);  // the MMA thread and each softmax warp
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
    const bool run = (*abort == 0);

    // Phase bookkeeping shared by every role: I counts items processed by this CTA (K/V slot
    // I % 2, the dK/dV hand-off), J counts query tiles over all of them (Q/dO ring, per-tile
    // barriers).
    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0 && run) {
            tma_prefetch(&p.q.nat);
            tma_prefetch(&p.dout.nat);
            tma_prefetch(&p.k.nat);
            tma_prefetch(&p.v.nat);
            int32_t I = 0, J = 0;  // K/V loads and Q/dO loads issued
            bool fail = false;
            for (int32_t j = 0; !fail; ++j) {
                // items are claimed from a global counter in list order (longest first) and
                // broadcast to the other roles through sched[]
                const int s = j % NSCHED;
                if (j >= NSCHED && !mbar_wait(&bars->sched_empty[s], ((j / NSCHED) - 1) & 1, abort, p.err))
                    break;
                int32_t u = atomicAdd(p.sched, 1);
                if (u >= nunits) u = -1;
                bars->sched[s] = u;
                Item *slot = reinterpret_cast<Item *>(smem + OFF_ITEMS) + s;
                if (u >= 0) *slot = load_item(p, u);
                mbar_arrive(&bars->sched_full[s]);
                if (u < 0) break;
                const Item it = *slot;
                const int ks = I % KVS;
                if (I >= KVS && !mbar_wait(&bars->kv_empty[ks], ((I / KVS) - 1) & 1, abort, p.err)) break;
                mbar_arrive_expect_tx(&bars->kv_full[ks], QB + VB);
                load_tile_w<DQK>(p.k, it.part.kframe, p.g, it.part.o, it.w.tile, it.bh, smem + OFF_K + ks * QB,
                                 &bars->kv_full[ks]);
                load_tile_w<DV>(p.v, it.part.kframe, p.g, it.part.o, it.w.tile, it.bh, smem + OFF_V + ks * VB,
                                &bars->kv_full[ks]);
                ++I;
                for (int32_t jj = 0; jj < it.nq; ++jj, ++J) {
                    const int qs = J % NST;
                    if (J >= NST && !mbar_wait(&bars->qdo_empty[qs], ((J / NST) - 1) & 1, abort, p.err)) {
                        fail = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->qdo_full[qs], QB + VB);
                    load_tile_w<DQK>(p.q, it.part.qframe, p.g, it.part.o, it.w.begin + jj, it.bh,
                                     smem + OFF_Q + qs * QB, &bars->qdo_full[qs]);
                    load_tile_w<DV>(p.dout, it.part.qframe, p.g, it.part.o, it.w.begin + jj, it.bh,
                                    smem + OFF_DO + qs * VB, &bars->qdo_full[qs]);
                }
            }
            if (*abort) {  // drain the copies still in flight before the CTA leaves
                volatile int32_t never = 0;
                for (int32_t i = (I > KVS ? I - KVS : 0); i < I; ++i)
                    mbar_wait(&bars->kv_full[i % KVS], (i / KVS) & 1, &never, p.err);
                for (int32_t i = (J > NST ? J - NST : 0); i < J; ++i)
                    mbar_wait(&bars->qdo_full[i % NST], (i / NST) & 1, &never, p.err);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0 && run) {
            constexpr uint32_t id_nn = idesc_bf16(128, 128, false, false);  // S, dP
            constexpr uint32_t id_tv = idesc_bf16(128, DV, true, true);     // dV
            constexpr uint32_t id_tk = idesc_bf16(128, DQK, true, true);    // dK
            constexpr uint32_t id_kt = idesc_bf16(128, DQK, false, true);   // dQ
            const uint32_t sP = smem_u32(smem + OFF_P), sDS = smem_u32(smem + OFF_DS);
            auto sQ = [&](int32_t t) { return smem_u32(smem + OFF_Q + (t % NST) * QB); };
            auto sDO = [&](int32_t t) { return smem_u32(smem + OFF_DO + (t % NST) * VB); };
            auto sKs = [&](int32_t slot) { return smem_u32(smem + OFF_K + slot * QB); };
            auto sVs = [&](int32_t slot) { return smem_u32(smem + OFF_V + slot * VB); };
            // Per query tile t the tensor core runs, in order:
            //   dV += P_t^T dO_t | S_{t+1} | dQ_t = dS_t K, dK += dS_t^T Q_t | dP_{t+1}
            // so that it computes dV_t and S_{t+1} while the softmax warps build dS_t, and dK_t,
            // dQ_t, dP_{t+1} while they drain dQ_t and build P_{t+1}.  An item's first S and dP
            // follow the previous item's last dQ.
            auto issue_s = [&](uint32_t q, uint32_t k) {  // S = Q K^T (both K-major over DQK)
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk)
                    mma_bf16_ss(tbase + COL_S, Tile<DQK>::kmajor(q, kk), Tile<DQK>::kmajor(k, kk), id_nn,
                                kk > 0 ? 1u : 0u);
                mma_commit(&bars->s_full);
            };
            auto issue_dp = [&](uint32_t o, uint32_t v) {  // dP = dO V^T (both K-major over DV)
#pragma unroll
                for (int kk = 0; kk < DV / 16; ++kk)
                    mma_bf16_ss(tbase + COL_DP, Tile<DV>::kmajor(o, kk), Tile<DV>::kmajor(v, kk), id_nn,
                                kk > 0 ? 1u : 0u);
                mma_commit(&bars->dp_full);
            };
            // One flat loop over the query tiles of all items this CTA claims: the tile after the
            // last one of an item is the next item's first, so the next item's S and dP are
            // issued as early as within an item (after dV and after dK, dQ of the current tile).
            auto item_nq = [&](int32_t jj_slot) {
                return (reinterpret_cast<const Item *>(smem + OFF_ITEMS) + jj_slot % NSCHED)->nq;
            };
            int32_t j = 0, I = 0, J = 0;  // current item (claim index), items started, tiles done
            int32_t u = next_item(bars, 0, false, abort, p.err);
            if (u >= 0) {
                int32_t nq = item_nq(0), jj = 0, ks = 0;
                bool ok = mbar_wait(&bars->kv_full[0], 0, abort, p.err) &&
                          mbar_wait(&bars->qdo_full[0], 0, abort, p.err);
                if (ok) {
                    tc_fence_after();
                    issue_s(sQ(0), sKs(0));
                    issue_dp(sDO(0), sVs(0));
                }
                while (ok) {
                    const int32_t t = J;
                    const bool last = jj + 1 == nq;
                    // the next tile: this item's next query tile, or the next item's first
                    int32_t nks = ks;
                    bool has_next = !last;
                    if (last) {
                        const int32_t un = next_item(bars, j + 1, false, abort, p.err);
                        if (un == -2) break;
                        has_next = un >= 0;
                        nks = (I + 1) % KVS;
                    }
                    if (!mbar_wait(&bars->p_ready, t & 1, abort, p.err)) break;
                    // the previous item's epilogue must have read dK and dV before they restart
                    if (jj == 0 && I > 0 && !mbar_wait(&bars->acc_free, (I - 1) & 1, abort, p.err)) break;
                    tc_fence_after();
                    // dV += P^T dO: A = P^T MN-major (two 64-key atoms 16 KB apart), B = dO
                    // MN-major; 16 queries per step
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ss(tbase + COL_DV, desc_sw128(sP + kk * 2048, TB, 1024), Tile<DV>::mnmajor(sDO(t), kk),
                                    id_tv, (jj > 0 || kk > 0) ? 1u : 0u);
                    // S of the next tile: the softmax warps are done reading S_t.  With single
                    // buffers (a one-stage Q/dO ring, or one K/V slot at an item's last tile) the
                    // next tile's Q or K takes the slot of this tile's, so its S follows dK below.
                    const bool late_s = NST == 1 || (last && KVS == 1);
                    auto next_s = [&]() {
                        if (!mbar_wait(&bars->qdo_full[(t + 1) % NST], ((t + 1) / NST) & 1, abort, p.err) ||
                            (last && !mbar_wait(&bars->kv_full[nks], ((I + 1) / KVS) & 1, abort, p.err)))
                            return false;
                        tc_fence_after();
                        issue_s(sQ(t + 1), sKs(nks));
                        return true;
                    };
                    if (has_next && !late_s && !next_s()) break;
                    if (!mbar_wait(&bars->ds_ready, t & 1, abort, p.err) ||
                        (t > 0 && !mbar_wait(&bars->dq_empty, (t - 1) & 1, abort, p.err)))
                        break;
                    tc_fence_after();
                    const uint32_t sK = sKs(ks);
                    // dQ = dS K (A = dS K-major, two 64-key halves; B = K MN-major), signalled at once
                    // so that the drain can start, then dK += dS^T Q (as dV); on an item's last tile
                    // dq_full waits for dK too, since the epilogue reads it
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ss(tbase + COL_DQ, desc_sw128(sDS + (kk >> 2) * TB + (kk & 3) * 32, 16, 1024),
                                    Tile<DQK>::mnmajor(sK, kk), id_kt, kk > 0 ? 1u : 0u);
                    if (!last) mma_commit(&bars->dq_full);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ss(tbase + COL_DK, desc_sw128(sDS + kk * 2048, TB, 1024), Tile<DQK>::mnmajor(sQ(t), kk),
                                    id_tk, (jj > 0 || kk > 0) ? 1u : 0u);
                    if (last) mma_commit(&bars->dq_full);  // also: dK, dV of the item complete
                    mma_commit(&bars->qdo_empty[t % NST]);
                    if (last) {
                        mma_commit(&bars->kv_empty[ks]);  // K and V of this item are no longer read
                        done_item(bars, j, false);
                    }
                    if (has_next && late_s && !next_s()) break;
                    if (has_next) issue_dp(sDO(t + 1), sVs(nks));  // dP_t consumed
                    ++J;
                    if (!has_next) break;
                    if (last) {
                        ++j;
                        ++I;
                        nq = item_nq(j);
                        jj = 0;
                        ks = nks;
                    } else {
                        ++jj;
                    }
                }
            }
            // no product may still be running when TMEM is released (also after an abort)
            mma_commit(&bars->mma_idle);
            volatile int32_t never = 0;
            mbar_wait(&bars->mma_idle, 0, &never, p.err);
        }
    } else {
        // ------- P, dS, dQ drain, epilogue (warps 2..: warpgroup g owns score columns CW g..) -------
        const int g = (warp - 2) >> 2;
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tbase + COL_S + lane_off + CW * g, tDP = tbase + COL_DP + lane_off + CW * g;
        const uint32_t tDQ = tbase + COL_DQ + lane_off + OWQ * g;
        // P and dS live in two 128 x 64 swizzled halves; this warpgroup's 32 columns are four
        // 16-byte chunks of half g/2
        const uint32_t sPg = smem_u32(smem + OFF_P) + (g >> 1) * TB, sDSg = smem_u32(smem + OFF_DS) + (g >> 1) * TB;
        const uint32_t chunk0 = (g & 1) * 4;
        // this warp's staging: its dQ slice (32 rows x OWQ fp32) or its dK and dV slices (bf16)
        const uint32_t warp_slot = (g * 4 + q4) * ((C::STG + 1023) & ~1023u);
        const uint32_t sDQw = smem_u32(smem + OFF_DQ) + warp_slot;
        const float sc = p.scale_log2, dsc = p.ds_scale;
        bool ok = run;
        uint32_t sv[32], dv[32];
        float pr[CW];                  // P of this row's CW columns, kept from P_t to dS_t
        float nlse = 0.f, nD = 0.f;    // -lse (log2 units) and -D_i / sqrt(d) of the row
        int32_t lo = 1, hi = 0;        // allowed columns of this slice, relative to the slice
        const Item *cur = nullptr;     // the item being processed (its shared slot: the fields
                                       // are read where needed, to keep registers free)
        size_t head_base = 0;          // first row of its batch-head
        // Order per query tile: P_0; then for each t: dS_t, P_{t+1}, drain dQ_t.  Building P_{t+1}
        // while the tensor core computes dK_t and dQ_t hides their latency.  Buffer safety comes
        // from commit order: S_{t+1} is issued after dV_t (so s_full(t+1) means P_t was read) and
        // dP_{t+1} after dK_t, dQ_t (so dp_full(t+1) means dS_t was read).
        auto wait_all = [&](uint64_t *bar, int parity) {
            ok = ok && __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, p.err));
            if (ok) tc_fence_after();
            return ok;
        };
        // Row data of query tile jj of the item (interval, -lse, -D).  The loads are issued just
        // before the wait for S: issued any earlier they would sit in front of the proxy fences of
        // the dS phase, which wait for them.
        auto p_phase = [&](int32_t t, const Item *it, int32_t jj) {  // P_t = exp2(S log2e / sqrt(d) - lse log2e) -> SMEM
            int32_t lo_abs, hi_abs;
            const int32_t i = row_interval(p.g, it->part, it->w.begin + jj, row, lo_abs, hi_abs);
            const size_t hb = static_cast<size_t>(it->bh) * p.g.n;
            nlse = 0.f;
            nD = 0.f;
            if (i >= 0) {
                const float lse = p.lse[hb + i];
                // a row with no allowed key (lse = -inf) has every entry masked to -inf below;
                // keep its base finite so that -inf + base stays -inf instead of NaN
                nlse = lse == -INFINITY ? 0.f : -lse * LOG2E;
                nD = -p.delta[hb + i] * dsc;
            }
            const int32_t base = it->w.tile * TILE + CW * g;
            lo = lo_abs - base;
            hi = hi_abs - base;
            if (!wait_all(&bars->s_full, t & 1)) return;
            tmem_ld32(tS, sv);
            tmem_wait_ld();
            if (!(lo <= 0 && hi >= CW - 1)) {
                const uint32_t keep = interval_bits32(lo, hi);
#pragma unroll
                for (int e = 0; e < CW; ++e) sv[e] = (keep & (1u << e)) ? sv[e] : 0xFF800000u;  // -inf: P = 0, dS = 0
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
        auto ds_phase = [&](int32_t t) {  // dS_t = P (dP - D) / sqrt(d) -> SMEM
            if (!wait_all(&bars->dp_full, t & 1)) return;
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
                    const uint64_t x = fma2(f32x2(__uint_as_float(dv[c]), __uint_as_float(dv[c + 1])), dsc2, nD2);
                    float d0, d1;
                    f32x2_split(mul2(f32x2(pr[c], pr[c + 1]), x), d0, d1);
                    pk[e] = pack_bf16(d0, d1);
                }
                st_shared_v4(sDSg + sw128_off(row, chunk0 + q), pk[0], pk[1], pk[2], pk[3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->ds_ready);
        };
        auto drain = [&](int32_t t, int32_t jj) {  // dQ_t columns OWQ g.. : TMEM -> SMEM -> TMA reduce-add
            if (!wait_all(&bars->dq_full, t & 1)) return;
            uint32_t dq[OWQ];
            tmem_ld_n<OWQ>(tDQ, dq);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars->dq_empty);
            // per-warp staging (32 rows, swizzled as the TMA map of the slice): no cross-warp barrier
            if (lane == 0) bulk_wait_read_all();  // this warp's previous reduce / store has read it
            __syncwarp();
            const bool direct = cur->part.dq_direct != 0;  // the only contribution to these rows
            if (!F32 && direct) {  // bf16 dQ itself: 32 rows x 2 OWQ bytes
#pragma unroll
                for (int q = 0; q < OWQ / 8; ++q)
                    st_shared_v4(sDQw + swz_off<2 * OWQ>(lane, q),
                                 pack_bf16(__uint_as_float(dq[8 * q]), __uint_as_float(dq[8 * q + 1])),
                                 pack_bf16(__uint_as_float(dq[8 * q + 2]), __uint_as_float(dq[8 * q + 3])),
                                 pack_bf16(__uint_as_float(dq[8 * q + 4]), __uint_as_float(dq[8 * q + 5])),
                                 pack_bf16(__uint_as_float(dq[8 * q + 6]), __uint_as_float(dq[8 * q + 7])));
            } else {  // fp32: 32 rows x 4 OWQ bytes
#pragma unroll
                for (int q = 0; q < OWQ / 4; ++q)
                    st_shared_v4(sDQw + swz_off<4 * OWQ>(lane, q), dq[4 * q], dq[4 * q + 1], dq[4 * q + 2], dq[4 * q + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (direct)  // a natural-frame query part: a plain TMA store of the slice
                    tma_store_3d(&p.dq_direct, smem + OFF_DQ + warp_slot, OWQ * g,
                                 (cur->w.begin + jj) * TILE + 32 * q4, cur->bh);
                else
                    reduce_warp_f32(p.dq_red, cur->part.qframe, p.g, cur->w.begin + jj, cur->bh, OWQ * g, q4,
                                    smem + OFF_DQ + warp_slot);
                bulk_commit();
            }
        };
        // One flat loop over the query tiles of all items, as the MMA issuer's: per tile t, dS_t,
        // then P of the next tile (the next item's first after an item's last tile), then the
        // drain of dQ_t, and after an item's last tile its dK/dV epilogue -- so that building the
        // next P covers the wait for dK_t, dQ_t even when an item has a single query tile.
        int32_t J = 0, j = 0;  // query tiles processed, current item (claim index)
        const Item *slot0 = reinterpret_cast<const Item *>(smem + OFF_ITEMS);
        if (next_item(bars, 0, true, abort, p.err) >= 0) {
            cur = slot0;
            head_base = static_cast<size_t>(cur->bh) * p.g.n;
            int32_t nq = cur->nq, jj = 0;
            p_phase(0, cur, 0);
            while (ok) {
                const int32_t t = J;
                const bool last = jj + 1 == nq;
                const Item *nxt = cur;
                int32_t njj = jj + 1;
                bool has_next = !last;
                if (last) {
                    const int32_t un = next_item(bars, j + 1, true, abort, p.err);
                    if (un == -2) {
                        ok = false;
                        break;
                    }
                    has_next = un >= 0;
                    nxt = slot0 + (j + 1) % NSCHED;
                    njj = 0;
                }
                ds_phase(t);
                if (ok && has_next) p_phase(t + 1, nxt, njj);
                if (ok) drain(t, jj);
                if (!ok) break;
                if (!last) {
                    ++J;
                    ++jj;
                    continue;
                }
                // ------- dK, dV of the item: one key row per thread, warpgroup g owns dK columns
                // OWQ g.. and dV columns OWV g.. -------
                // (the last drain waited for dq_full of the item's last tile, whose commit covers
                // every dK and dV product of the item).  The next item's P_0 is already built; its
                // first dV product waits for acc_free, arrived below.
                const int32_t pos = frame_pos(p.g, cur->part.kframe, cur->part.o, cur->w.tile, row);
                // Chunk of a split key tile: store the fp32 partial in this chunk's slot (a pass after
                // the kernel adds the chunks' slots in chunk order and writes dK and dV), in thread
                // order: dK's 16-byte group q of slice g of row r at uint4 (q * 4 + g) * 128 + r, dV's
                // after all of dK's (DQK * 32 uint4 further), so that each warp store is 512
                // contiguous bytes.  bf16 output: each warp stages its 32 rows of dK and dV in its
                // own staging slot and writes them with two TMA stores (no cross-warp barrier; the
                // warp's next dQ drain waits for their reads as for a reduce).
                constexpr size_t SLOT = static_cast<size_t>(128) * (DQK + DV);
                const bool split = cur->w.slot >= 0;
                const bool staged = !F32 && !split;
                if (staged) {
                    if (lane == 0) bulk_wait_read_all();  // this warp's last reduce has read the slot
                    __syncwarp();
                }
                // one of the two outputs: W columns from TMEM column col, partial-slot offset part0
                // (uint4), first-pass values and output rows of `width` elements at out / out_f32,
                // staging at stg
                auto emit = [&](auto Wc, uint32_t col, size_t part0, uint16_t *out, float *out_f32, int32_t width,
                                uint32_t stg) {
                    constexpr int W = decltype(Wc)::value;
                    uint32_t a16[W];
                    tmem_ld_n<W>(tbase + col + lane_off + W * g, a16);
                    tmem_wait_ld();
                    if (*abort != 0) return;
                    if (split) {
                        uint4 *dst = reinterpret_cast<uint4 *>(p.partials + (static_cast<size_t>(cur->w.slot) * p.batch + cur->b) * SLOT) + part0;
#pragma unroll
                        for (int q = 0; q < W / 4; ++q)
                            dst[(q * 4 + g) * 128 + row] = make_uint4(a16[4 * q], a16[4 * q + 1], a16[4 * q + 2], a16[4 * q + 3]);
                        return;
                    }
                    float a[W];
#pragma unroll
                    for (int e = 0; e < W; ++e) a[e] = __uint_as_float(a16[e]);
                    if (pos < 0) return;  // frame padding
                    const size_t off = (head_base + pos) * width + W * g;
                    if (F32) {  // rows of the fp32 output, the first pass's values added by this thread
                        float4 *d4 = reinterpret_cast<float4 *>(out_f32 + off);
#pragma unroll
                        for (int q = 0; q < W / 4; ++q) {
                            float4 v = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
                            if (cur->part.merge) {
                                const float4 x = d4[q];
                                v.x += x.x;
                                v.y += x.y;
                                v.z += x.z;
                                v.w += x.w;
                            }
                            d4[q] = v;
                        }
                        return;
                    }
                    if (cur->part.merge) {  // add the first pass's values
                        const uint4 *src = reinterpret_cast<const uint4 *>(out + off);
#pragma unroll
                        for (int q = 0; q < W / 8; ++q) {
                            const uint4 x = src[q];
                            const uint32_t xx[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                a[8 * q + 2 * e] += bf16_lo(xx[e]);
                                a[8 * q + 2 * e + 1] += bf16_hi(xx[e]);
                            }
                        }
                    }
                    // this warp's slice: 32 rows x 2 W bytes, swizzled as the slice's TMA map
#pragma unroll
                    for (int q = 0; q < W / 8; ++q)
                        st_shared_v4(stg + swz_off<2 * W>(lane, q), pack_bf16(a[8 * q], a[8 * q + 1]),
                                     pack_bf16(a[8 * q + 2], a[8 * q + 3]), pack_bf16(a[8 * q + 4], a[8 * q + 5]),
                                     pack_bf16(a[8 * q + 6], a[8 * q + 7]));
                };
                emit(std::integral_constant<int, OWQ>(), COL_DK, 0, p.dk_out, p.dk_f32, DQK, sDQw);
                emit(std::integral_constant<int, OWV>(), COL_DV, static_cast<size_t>(DQK) * 32, p.dv_out, p.dv_f32, DV,
                     sDQw + C::STG_DK);
                tc_fence_before();
                mbar_arrive(&bars->acc_free);  // the next item's first dV, dK may overwrite them
                if (staged) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        store_warp_slice(p.dk_w, cur->part.kframe, p.g, cur->part.o, cur->w.tile, cur->bh, OWQ * g, q4,
                                         smem + OFF_DQ + warp_slot);
                        store_warp_slice(p.dv_w, cur->part.kframe, p.g, cur->part.o, cur->w.tile, cur->bh, OWV * g, q4,
                                         smem + OFF_DQ + warp_slot + C::STG_DK);
                        bulk_commit();
                    }
                }
                done_item(bars, j, true);
                ++J;
                if (!has_next) break;
                ++j;
                cur = nxt;
                head_base = static_cast<size_t>(cur->bh) * p.g.n;
                nq = cur->nq;
                jj = 0;
            }
        }
        if (lane == 0) bulk_wait_read_all();  // this warp's reduces and stores have read its slot
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

template <bool F32, int DQK, int DV>
cudaError_t launch_bwd_t(const BwdParams &p, cudaStream_t s)
{
    constexpr uint32_t SMEM = BCfg<DQK, DV>::SMEM_BYTES;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(bwd_kernel<F32, DQK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const int64_t units = static_cast<int64_t>(p.nitems) * p.batch;
    if (units == 0) return cudaSuccess;
    const int64_t cap = sm_count();
    bwd_kernel<F32, DQK, DV><<<static_cast<unsigned>(units < cap ? units : cap), THREADS, SMEM, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool bwd_widths_supported(int dqk, int dv)
{
    return (dqk == 64 && dv == 64) || (dqk == 32 && dv == 32) || (dqk == 64 && dv == 128);
}

cudaError_t launch_bwd(const BwdParams &p, bool f32, int dqk, int dv, cudaStream_t s)
{
    if (f32) return dqk == 64 && dv == 64 ? launch_bwd_t<true, 64, 64>(p, s) : cudaErrorInvalidValue;
    if (dqk == 64 && dv == 64) return launch_bwd_t<false, 64, 64>(p, s);
    if (dqk == 32 && dv == 32) return launch_bwd_t<false, 32, 32>(p, s);
    if (dqk == 64 && dv == 128) return launch_bwd_t<false, 64, 128>(p, s);
    return cudaErrorInvalidValue;
}

}  // namespace st
