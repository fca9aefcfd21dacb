// layout.cu -- host construction of the block layout (natural-frame CSR with element masks, and
// the execution-frame work lists the kernels run), its device upload and its queries.
//
// Block-sparse layout: "长序列为何不必让每个 token 看见全部历史？滑动窗口、块稀疏与全局 token" §05
// (only selected block pairs enter the kernel; boundary blocks keep an element mask).  Sets:
// "Sparse Transformers（稀疏 Transformer）深度解读报告" §2.2 (strided, fixed) and §3.1 (merged =
// union, Eq.7; per-head, Eq.8); the causal restriction j <= i from its §2.1, and the upper
// triangle is never scheduled (§3.5).
#include <cuda_runtime.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <unordered_map>

#include "layout.h"

namespace {

// ---- allowed sets as runs of consecutive keys (natural frame) --------------------------------
// Calls f(j0, j1) for inclusive runs covering A(i) (runs may overlap for merged kinds).
template <class F>
void for_each_run(int kind, int64_t i, int64_t l, int64_t c, int64_t o, F f)
{
    auto band = [&]() { f(i - l > 0 ? i - l : 0, i); };
    auto stride = [&]() {
        for (int64_t j = i % l; j <= i; j += l) f(j, j);
    };
    auto block = [&]() { f((i / l) * l, i); };
    auto summary = [&]() {
        const int64_t s = (l - c - o) > 0 ? (l - c - o) : 0, e = l - 1 - o;
        if (e < s) return;
        for (int64_t u = 0; u * l + s <= i; ++u) f(u * l + s, std::min(u * l + e, i));
    };
    switch (kind) {
    case ST_KIND_SA1: band(); break;
    case ST_KIND_SA2: stride(); break;
    case ST_KIND_SU: band(); stride(); break;
    case ST_KIND_FA1: block(); break;
    case ST_KIND_FA2: summary(); break;
    case ST_KIND_FU: block(); summary(); break;
    default: break;
    }
}

uint64_t hash_words(const uint32_t *w, size_t nw)
{
    uint64_t h = 1469598103934665603ull;
    for (size_t a = 0; a < nw; ++a) {
        h ^= w[a];
        h *= 1099511628211ull;
    }
    return h;
}

void build_nat_plan(NatPlan &P, int64_t n, int64_t l, int64_t c, int32_t B)
{
    const int64_t nqb = (n + B - 1) / B;
    const size_t nw = static_cast<size_t>(B) * B / 32;
    std::vector<std::vector<uint32_t>> pool;
    std::vector<int32_t> slot_of(static_cast<size_t>(nqb), -1);
    std::vector<int32_t> touched;
    std::unordered_map<uint64_t, std::vector<int32_t>> dedup;
    P.row_ptr.assign(1, 0);
    for (int64_t qb = 0; qb < nqb; ++qb) {
        touched.clear();
        int32_t used = 0;
        for (int32_t r = 0; r < B; ++r) {
            const int64_t i = qb * B + r;
            if (i >= n) break;
            for_each_run(P.kind, i, l, c, P.o, [&](int64_t j0, int64_t j1) {
                for (int64_t j = j0; j <= j1;) {
                    const int64_t kb = j / B;
                    const int64_t end = std::min(j1, kb * B + B - 1);
                    int32_t &s = slot_of[static_cast<size_t>(kb)];
                    if (s < 0) {
                        if (used == static_cast<int32_t>(pool.size())) pool.emplace_back(nw, 0u);
                        s = used++;
                        std::fill(pool[s].begin(), pool[s].end(), 0u);
                        touched.push_back(static_cast<int32_t>(kb));
                    }
                    uint32_t *w = pool[s].data();
                    for (int64_t jj = j; jj <= end; ++jj) {
                        const int64_t bit = static_cast<int64_t>(r) * B + (jj - kb * B);
                        w[bit >> 5] |= 1u << (bit & 31);
                    }
                    j = end + 1;
                }
            });
        }
        std::sort(touched.begin(), touched.end());
        for (int32_t kb : touched) {
            int32_t &s = slot_of[static_cast<size_t>(kb)];
            const uint32_t *w = pool[s].data();
            bool full = true;
            for (size_t a = 0; a < nw && full; ++a) full = (w[a] == 0xFFFFFFFFu);
            int32_t id = -1;
            if (!full) {
                const uint64_t h = hash_words(w, nw);
                auto &cand = dedup[h];
                for (int32_t m : cand)
                    if (memcmp(&P.masks[static_cast<size_t>(m) * nw], w, nw * 4) == 0) { id = m; break; }
                if (id < 0) {
                    id = P.n_masks++;
                    P.masks.insert(P.masks.end(), w, w + nw);
                    cand.push_back(id);
                }
            }
            P.col_idx.push_back(kb);
            P.mask_id.push_back(id);
            s = -1;
        }
        P.row_ptr.push_back(static_cast<int32_t>(P.col_idx.size()));
    }
}

int32_t next_pow2(int32_t x)
{
    int32_t p = 1;
    while (p < x) p <<= 1;
    return p;
}

bool is_pow2(int32_t x) { return x > 0 && (x & (x - 1)) == 0; }

// Execution plan: frames, parts, work lists (see frames.cuh).  Returns ST_ERR_UNSUPPORTED when
// the kernels cannot run this layout (the natural-frame CSR is still built and exportable).
st_status_t build_exec(st_layout &L)
{
    const int64_t n = L.n;
    const int32_t l = L.l, c = L.c, H = L.pat.num_heads;
    if (n % st::TILE != 0 || n % l != 0 || n > (1ll << 30) || H > 64) return ST_ERR_UNSUPPORTED;
    st::Geom &g = L.geom;
    memset(&g, 0, sizeof(g));
    g.n = static_cast<int32_t>(n);
    g.l = l;
    g.c = c;
    g.R = static_cast<int32_t>(n / l);
    if (g.R >= st::TILE) {
        g.Rt = st::TILE;
        g.cpt = 1;
        g.tpc = (g.R + st::TILE - 1) / st::TILE;
    } else {
        g.Rt = next_pow2(g.R);
        g.cpt = st::TILE / g.Rt;
        g.tpc = 1;
    }
    g.ngroups = (l + g.cpt - 1) / g.cpt;
    g.div_l = st::make_fastdiv(static_cast<uint32_t>(l));
    g.div_c = st::make_fastdiv(static_cast<uint32_t>(c > 0 ? c : 1));
    g.div_tpc = st::make_fastdiv(static_cast<uint32_t>(g.tpc));
    g.div_Rt = st::make_fastdiv(static_cast<uint32_t>(g.Rt));
    if (L.pat.family == ST_FIXED) {
        if (!is_pow2(c) || c > st::TILE || c > l) return ST_ERR_UNSUPPORTED;
        g.upt = st::TILE / c;
        for (int32_t h = 0; h < H; ++h)
            if (L.head_off[h] + c > l) return ST_ERR_UNSUPPORTED;
    }
    L.parts.clear();
    for (int32_t h = 0; h < H; ++h) {
        st::Part p;
        memset(&p, 0, sizeof(p));
        p.head = h;
        p.o = L.head_off[h];
        auto add = [&](int32_t rule, int32_t qf, int32_t kf, int32_t lo, int32_t hi, int32_t merge) {
            st::Part q = p;
            q.rule = rule;
            q.qframe = qf;
            q.kframe = kf;
            q.lo_off = lo;
            q.hi_off = hi;
            q.merge = merge;
            q.nq = st::frame_tiles(g, qf);
            q.nk = st::frame_tiles(g, kf);
            L.parts.push_back(q);
        };
        switch (L.head_kind[h]) {
        case ST_KIND_SA1: add(st::RU_BAND, st::FR_NAT, st::FR_NAT, l, 0, 0); break;
        case ST_KIND_SA2: add(st::RU_COL, st::FR_COL, st::FR_COL, 0, 0, 0); break;
        case ST_KIND_SU:  // A1 \ A2 = {max(0, i-l+1) .. i-1} (natural), then A2 on the grid view
            add(st::RU_BAND, st::FR_NAT, st::FR_NAT, l - 1, 1, 0);
            add(st::RU_COL, st::FR_COL, st::FR_COL, 0, 0, 1);
            break;
        case ST_KIND_FA1: add(st::RU_BLOCK, st::FR_NAT, st::FR_NAT, 0, 0, 0); break;
        case ST_KIND_FA2: add(st::RU_SUM, st::FR_NAT, st::FR_SUM, 0, 0, 0); break;
        case ST_KIND_FU:  // same block (natural), then earlier blocks' summary runs (compacted)
            add(st::RU_BLOCK, st::FR_NAT, st::FR_NAT, 0, 0, 0);
            add(st::RU_SUMPREV, st::FR_NAT, st::FR_SUM, 0, 0, 1);
            break;
        default: return ST_ERR_INTERNAL;
        }
    }
    L.passes = 1;
    for (auto &p : L.parts)
        if (p.merge) L.passes = 2;

    int32_t max_q = 0;
    for (auto &p : L.parts) max_q = std::max(max_q, p.nq);
    L.fwd_item_of.assign(L.parts.size() * static_cast<size_t>(max_q), -1);
    for (int a = 0; a < 2; ++a) { L.fwd_items[a].clear(); L.bwd_items[a].clear(); }
    L.bwd_slots = 0;
    L.bwd_splits = 0;
    L.bwd_split_recs[0].clear();
    L.bwd_split_recs[1].clear();
    L.exec_tiles = 0;
    L.allowed_pairs = 0;
    std::vector<std::vector<st::WorkItem>> fwd_by_part(L.parts.size());
    for (size_t pi = 0; pi < L.parts.size(); ++pi) {
        const st::Part &p = L.parts[pi];
        for (int32_t qt = 0; qt < p.nq; ++qt) {
            int32_t tmin = INT32_MAX, tmax = -1;
            for (int32_t rho = 0; rho < st::TILE; ++rho) {
                int32_t lo, hi;
                st::row_interval(g, p, qt, rho, lo, hi);
                if (lo > hi) continue;
                if (hi >= p.nk * st::TILE || lo < 0) return ST_ERR_INTERNAL;
                L.allowed_pairs += hi - lo + 1;
                tmin = std::min(tmin, lo / st::TILE);
                tmax = std::max(tmax, hi / st::TILE);
            }
            st::WorkItem w{static_cast<int32_t>(pi), qt, tmax < 0 ? 0 : tmin, tmax < 0 ? 0 : tmax + 1, -1, 1, -1, -1};
            L.exec_tiles += w.end - w.begin;
            fwd_by_part[pi].push_back(w);
        }
    }
    // backward: for each key tile, the contiguous range of query tiles that reference it
    for (size_t pi = 0; pi < L.parts.size(); ++pi) {
        const st::Part &p = L.parts[pi];
        std::vector<int32_t> qmin(static_cast<size_t>(p.nk), INT32_MAX), qmax(static_cast<size_t>(p.nk), -1);
        for (const auto &w : fwd_by_part[pi])
            for (int32_t kt = w.begin; kt < w.end; ++kt) {
                qmin[kt] = std::min(qmin[kt], w.tile);
                qmax[kt] = std::max(qmax[kt], w.tile);
            }
        for (int32_t kt = 0; kt < p.nk; ++kt) {
            if (qmax[kt] < 0) continue;
            for (int32_t qt = qmin[kt]; qt <= qmax[kt]; ++qt) {
                const auto &w = fwd_by_part[pi][qt];
                if (!(w.begin <= kt && kt < w.end)) return ST_ERR_INTERNAL;  // not contiguous
            }
            const int32_t len = qmax[kt] + 1 - qmin[kt];
            if (len <= st::BWD_CHUNK) {
                L.bwd_items[p.merge].push_back(
                    st::WorkItem{static_cast<int32_t>(pi), kt, qmin[kt], qmax[kt] + 1, -1, 1, -1, -1});
                continue;
            }
            // near-equal chunks, each with its own partial-sum slot, sharing one counter
            const int32_t nch = (len + st::BWD_CHUNK - 1) / st::BWD_CHUNK;
            for (int32_t ch = 0; ch < nch; ++ch) {
                const int32_t b0 = qmin[kt] + static_cast<int32_t>(static_cast<int64_t>(len) * ch / nch);
                const int32_t b1 = qmin[kt] + static_cast<int32_t>(static_cast<int64_t>(len) * (ch + 1) / nch);
                L.bwd_items[p.merge].push_back(st::WorkItem{static_cast<int32_t>(pi), kt, b0, b1,
                                                            L.bwd_slots + ch, nch, L.bwd_slots, L.bwd_splits});
            }
            L.bwd_split_recs[p.merge].push_back(st::SplitRec{static_cast<int32_t>(pi), kt, L.bwd_slots, nch});
            L.bwd_slots += nch;
            L.bwd_splits += 1;
        }
        for (const auto &w : fwd_by_part[pi]) {
            L.fwd_item_of[pi * static_cast<size_t>(max_q) + w.tile] = 0;
            L.fwd_items[p.merge].push_back(w);
        }
    }
    // longest-processing-time-first order: the block scheduler then hands out heavy items first
    auto by_cost = [](const st::WorkItem &a, const st::WorkItem &b) {
        return (a.end - a.begin) > (b.end - b.begin);
    };
    for (int a = 0; a < 2; ++a) {
        std::stable_sort(L.fwd_items[a].begin(), L.fwd_items[a].end(), by_cost);
        std::stable_sort(L.bwd_items[a].begin(), L.bwd_items[a].end(), by_cost);
    }
    for (int a = 0; a < 2; ++a)
        for (size_t k = 0; k < L.fwd_items[a].size(); ++k) {
            const auto &w = L.fwd_items[a][k];
            L.fwd_item_of[static_cast<size_t>(w.part) * max_q + w.tile] =
                static_cast<int32_t>(a * 1000000000 + k);
        }
    // heads whose pass-0 backward leaves some key unwritten need a zero fill first
    L.head_flags.assign(static_cast<size_t>(H), 0);
    std::vector<uint8_t> cov(static_cast<size_t>(n));
    for (int32_t h = 0; h < H; ++h) {
        std::fill(cov.begin(), cov.end(), 0);
        for (const auto &w : L.bwd_items[0]) {
            const st::Part &p = L.parts[w.part];
            if (p.head != h) continue;
            for (int32_t rho = 0; rho < st::TILE; ++rho) {
                const int32_t pos = st::frame_pos(g, p.kframe, p.o, w.tile, rho);
                if (pos >= 0) cov[pos] = 1;
            }
        }
        for (int64_t j = 0; j < n; ++j)
            if (!cov[j]) { L.head_flags[h] |= st::HEAD_ZERO_FILL; break; }
    }
    // heads whose every (natural-frame) query tile is read by exactly one backward item, of
    // either pass: that item's dQ tile is the whole gradient of its rows and is written directly,
    // with no fp32 accumulation
    std::vector<int32_t> qcnt(static_cast<size_t>(n / st::TILE));
    for (int32_t h = 0; h < H; ++h) {
        bool nat = true;
        for (const auto &p : L.parts)
            if (p.head == h && p.qframe != st::FR_NAT) nat = false;
        if (!nat) continue;
        std::fill(qcnt.begin(), qcnt.end(), 0);
        for (int a = 0; a < 2; ++a)
            for (const auto &w : L.bwd_items[a])
                if (L.parts[w.part].head == h)
                    for (int32_t qt = w.begin; qt < w.end; ++qt) ++qcnt[qt];
        if (std::all_of(qcnt.begin(), qcnt.end(), [](int32_t x) { return x == 1; })) {
            L.head_flags[h] |= st::HEAD_DQ_DIRECT;
            for (auto &p : L.parts)
                if (p.head == h) p.dq_direct = 1;
        }
    }
    return ST_OK;
}

}  // namespace

extern "C" {

st_status_t st_layout_build(const st_pattern_t *pattern, int64_t n, int32_t l, int32_t c,
                            int32_t block, st_layout_t **out)
{
    if (!pattern || !out) return ST_ERR_INVALID_ARG;
    const st_pattern_t &P = *pattern;
    if (P.family != ST_STRIDED && P.family != ST_FIXED) return ST_ERR_INVALID_ARG;
    if (P.head_mode < ST_PER_HEAD_ALTERNATING || P.head_mode > ST_SINGLE_A2) return ST_ERR_INVALID_ARG;
    if (P.num_heads < 1 || n < 1 || l < 1 || (block != 64 && block != 128)) return ST_ERR_INVALID_ARG;
    if (n > (1ll << 31) - 1) return ST_ERR_INVALID_ARG;
    if (P.family == ST_FIXED && (c < 1 || c > l)) return ST_ERR_INVALID_ARG;
    st_layout *L = new (std::nothrow) st_layout();
    if (!L) return ST_ERR_OOM;
    try {
        L->pat = P;
        L->n = n;
        L->l = l;
        L->c = (P.family == ST_FIXED) ? c : 0;
        L->block = block;
        const int32_t H = P.num_heads;
        const int64_t step = P.a2_offset_step > 0 ? P.a2_offset_step : L->c;
        L->head_kind.resize(H);
        L->head_off.resize(H);
        L->head_plan.resize(H);
        for (int32_t h = 0; h < H; ++h) {
            int second;  // -1 merged, 0 head 1, 1 head 2
            int64_t k;   // pattern-2 head number
            switch (P.head_mode) {
            case ST_PER_HEAD_ALTERNATING: second = h & 1; k = h / 2; break;
            case ST_MERGED: second = -1; k = h; break;
            case ST_SINGLE_A1: second = 0; k = h; break;
            default: second = 1; k = h; break;
            }
            int32_t kind;
            if (P.family == ST_STRIDED)
                kind = second < 0 ? ST_KIND_SU : (second ? ST_KIND_SA2 : ST_KIND_SA1);
            else
                kind = second < 0 ? ST_KIND_FU : (second ? ST_KIND_FA2 : ST_KIND_FA1);
            const bool uses_off = (kind == ST_KIND_FA2 || kind == ST_KIND_FU);
            L->head_kind[h] = kind;
            L->head_off[h] = uses_off ? static_cast<int32_t>((k * step) % l) : 0;
            int32_t found = -1;
            for (size_t a = 0; a < L->plans.size(); ++a)
                if (L->plans[a].kind == kind && L->plans[a].o == L->head_off[h]) found = static_cast<int32_t>(a);
            if (found < 0) {
                NatPlan np;
                np.kind = kind;
                np.o = L->head_off[h];
                L->plans.push_back(std::move(np));
                found = static_cast<int32_t>(L->plans.size() - 1);
            }
            L->head_plan[h] = found;
        }
        const st_status_t es = build_exec(*L);
        if (es == ST_ERR_INTERNAL) { delete L; return ST_ERR_INTERNAL; }
        L->exec_ok = (es == ST_OK);
    } catch (const std::bad_alloc &) {
        delete L;
        return ST_ERR_OOM;
    }
    *out = L;
    return ST_OK;
}

st_status_t st_layout_upload(st_layout_t *L, st_stream_t stream)
{
    if (!L) return ST_ERR_INVALID_ARG;
    if (!L->exec_ok) return ST_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ST_ERR_CUDA;
    if (L->uploaded && dev != L->device) return ST_ERR_INVALID_ARG;
    const size_t np = L->parts.size() * sizeof(st::Part);
    const size_t nf0 = L->fwd_items[0].size() * sizeof(st::WorkItem);
    const size_t nf1 = L->fwd_items[1].size() * sizeof(st::WorkItem);
    const size_t nb0 = L->bwd_items[0].size() * sizeof(st::WorkItem);
    const size_t nb1 = L->bwd_items[1].size() * sizeof(st::WorkItem);
    const size_t nz = L->head_flags.size() * sizeof(int32_t);
    const size_t ns0 = L->bwd_split_recs[0].size() * sizeof(st::SplitRec);
    const size_t ns1 = L->bwd_split_recs[1].size() * sizeof(st::SplitRec);
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t off_f0 = up(np), off_f1 = off_f0 + up(nf0), off_b0 = off_f1 + up(nf1),
                 off_b1 = off_b0 + up(nb0), off_z = off_b1 + up(nb1), off_s0 = off_z + up(nz),
                 off_s1 = off_s0 + up(ns0), off_e = off_s1 + up(ns1), total = off_e + 256;
    if (!L->uploaded) {
        if (cudaMalloc(&L->d_buf, total) != cudaSuccess) return ST_ERR_OOM;
        if (cudaMemsetAsync(L->d_buf, 0, total, stream) != cudaSuccess) return ST_ERR_CUDA;
        L->device = dev;
        char *b = static_cast<char *>(L->d_buf);
        L->d_parts = reinterpret_cast<st::Part *>(b);
        L->d_fwd[0] = reinterpret_cast<st::WorkItem *>(b + off_f0);
        L->d_fwd[1] = reinterpret_cast<st::WorkItem *>(b + off_f1);
        L->d_bwd[0] = reinterpret_cast<st::WorkItem *>(b + off_b0);
        L->d_bwd[1] = reinterpret_cast<st::WorkItem *>(b + off_b1);
        L->d_head_flags = reinterpret_cast<int32_t *>(b + off_z);
        L->d_split[0] = reinterpret_cast<st::SplitRec *>(b + off_s0);
        L->d_split[1] = reinterpret_cast<st::SplitRec *>(b + off_s1);
        L->d_err = reinterpret_cast<int32_t *>(b + off_e);
    }
    auto cp = [&](void *dst, const void *src, size_t bytes) {
        return bytes == 0 || cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, stream) == cudaSuccess;
    };
    if (!cp(L->d_parts, L->parts.data(), np) || !cp(L->d_fwd[0], L->fwd_items[0].data(), nf0) ||
        !cp(L->d_fwd[1], L->fwd_items[1].data(), nf1) || !cp(L->d_bwd[0], L->bwd_items[0].data(), nb0) ||
        !cp(L->d_bwd[1], L->bwd_items[1].data(), nb1) || !cp(L->d_head_flags, L->head_flags.data(), nz) ||
        !cp(L->d_split[0], L->bwd_split_recs[0].data(), ns0) || !cp(L->d_split[1], L->bwd_split_recs[1].data(), ns1))
        return ST_ERR_CUDA;
    L->uploaded = true;
    return ST_OK;
}

st_status_t st_layout_head_kind(const st_layout_t *L, int32_t head, int32_t *kind, int32_t *offset)
{
    if (!L || head < 0 || head >= L->pat.num_heads) return ST_ERR_INVALID_ARG;
    if (kind) *kind = L->head_kind[head];
    if (offset) *offset = L->head_off[head];
    return ST_OK;
}

st_status_t st_layout_export(const st_layout_t *L, int32_t head, const int32_t **row_ptr,
                             const int32_t **col_idx, const int32_t **mask_id,
                             const uint32_t **masks, int32_t *n_qblk, int32_t *nnz, int32_t *n_masks)
{
    if (!L || head < 0 || head >= L->pat.num_heads) return ST_ERR_INVALID_ARG;
    NatPlan &P = L->plans[L->head_plan[head]];
    try {
        std::lock_guard<std::mutex> lock(L->plans_mu);
        if (!P.built) {
            build_nat_plan(P, L->n, L->l, L->c, L->block);
            P.built = true;
        }
    } catch (const std::bad_alloc &) {
        return ST_ERR_OOM;
    }
    if (row_ptr) *row_ptr = P.row_ptr.data();
    if (col_idx) *col_idx = P.col_idx.data();
    if (mask_id) *mask_id = P.mask_id.data();
    if (masks) *masks = P.masks.data();
    if (n_qblk) *n_qblk = static_cast<int32_t>(P.row_ptr.size() - 1);
    if (nnz) *nnz = static_cast<int32_t>(P.col_idx.size());
    if (n_masks) *n_masks = P.n_masks;
    return ST_OK;
}

st_status_t st_layout_info(const st_layout_t *L, st_layout_info_t *info)
{
    if (!L || !info) return ST_ERR_INVALID_ARG;
    if (!L->exec_ok) return ST_ERR_UNSUPPORTED;
    memset(info, 0, sizeof(*info));
    info->fwd_items = static_cast<int64_t>(L->fwd_items[0].size() + L->fwd_items[1].size());
    info->bwd_items = static_cast<int64_t>(L->bwd_items[0].size() + L->bwd_items[1].size());
    info->exec_tiles = L->exec_tiles;
    info->allowed_pairs = L->allowed_pairs;
    info->passes = L->passes;
    info->split_passes = (L->bwd_split_recs[0].empty() ? 0 : 1) + (L->bwd_split_recs[1].empty() ? 0 : 1);
    for (const int32_t f : L->head_flags)
        if (f & st::HEAD_DQ_DIRECT) ++info->dq_direct_heads;
    return ST_OK;
}

st_status_t st_layout_exec_row(const st_layout_t *L, int32_t head, int64_t i, int64_t *keys, int64_t *count)
{
    if (!L || !keys || !count || head < 0 || head >= L->pat.num_heads || i < 0 || i >= L->n)
        return ST_ERR_INVALID_ARG;
    if (!L->exec_ok) return ST_ERR_UNSUPPORTED;
    const st::Geom &g = L->geom;
    int32_t max_q = 0;
    for (auto &p : L->parts) max_q = std::max(max_q, p.nq);
    int64_t cnt = 0;
    for (size_t pi = 0; pi < L->parts.size(); ++pi) {
        const st::Part &p = L->parts[pi];
        if (p.head != head) continue;
        // locate the query tile and row holding natural position i in the part's query frame
        int32_t t = -1, rho = -1;
        for (int32_t tt = 0; tt < p.nq && t < 0; ++tt)
            for (int32_t rr = 0; rr < st::TILE; ++rr)
                if (st::frame_pos(g, p.qframe, p.o, tt, rr) == i) { t = tt; rho = rr; break; }
        if (t < 0) return ST_ERR_INTERNAL;
        const int32_t code = L->fwd_item_of[pi * static_cast<size_t>(max_q) + t];
        if (code < 0) return ST_ERR_INTERNAL;
        const st::WorkItem &w = L->fwd_items[code / 1000000000][code % 1000000000];
        int32_t lo, hi;
        st::row_interval(g, p, t, rho, lo, hi);
        for (int32_t kt = w.begin; kt < w.end; ++kt)
            for (int32_t kr = 0; kr < st::TILE; ++kr) {
                const int32_t kidx = kt * st::TILE + kr;
                if (kidx < lo || kidx > hi) continue;
                const int32_t pos = st::frame_pos(g, p.kframe, p.o, kt, kr);
                if (pos < 0) return ST_ERR_INTERNAL;
                keys[cnt++] = pos;
            }
    }
    std::sort(keys, keys + cnt);
    *count = cnt;
    return ST_OK;
}

st_status_t st_layout_check(st_layout_t *L, st_stream_t stream)
{
    if (!L) return ST_ERR_INVALID_ARG;
    if (!L->uploaded) return ST_ERR_NOT_UPLOADED;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return ST_ERR_CUDA;
    int32_t e = 0;
    if (cudaMemcpy(&e, L->d_err, sizeof(e), cudaMemcpyDeviceToHost) != cudaSuccess) return ST_ERR_CUDA;
    if (e != 0) {
        if (cudaMemset(L->d_err, 0, sizeof(int32_t)) != cudaSuccess) return ST_ERR_CUDA;
        return ST_ERR_DEVICE_TIMEOUT;
    }
    return ST_OK;
}

void st_layout_destroy(st_layout_t *L)
{
    if (!L) return;
    if (L->d_buf) cudaFree(L->d_buf);
    delete L;
}

}  // extern "C"
