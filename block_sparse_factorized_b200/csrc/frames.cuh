// frames.cuh -- execution frames and per-row key intervals (host and device).
//
// Every head kind is run as one or two "parts".  A part pairs a query frame with a key frame:
// a frame lists the sequence positions in tiles of 128 rows, and for every query row the
// allowed keys of the part form ONE contiguous interval of key-frame indices.  That makes every
// boundary mask an interval test and lets a tile be classified full/partial/empty per row.
//
//   FR_NAT  natural order: tile t holds positions 128 t .. 128 t + 127.
//   FR_COL  the (n/l) x l grid view of the sequence (row r, column col holds position r*l+col),
//           read column-wise.  The strided pattern-2 set {j <= i : (i-j) mod l == 0} is "same
//           column, grid row <= mine", i.e. plain causal attention inside each column ("稀疏与局部
//           注意力：Longformer、BigBird、Sparse Transformer" §二: strided attention equals row and
//           column attention on a 2-D grid).  A column of R = n/l rows occupies a slot of Rt
//           rows (Rt = R rounded up to a power of two when R < 128, else 128); a tile holds
//           cpt = 128/Rt column slots, or one 128-row piece of a column when R > 128.
//   FR_SUM  the fixed pattern-2 keys compacted: only the c summary positions of each block,
//           (l-c-o) .. (l-1-o) within the block, in order; tile t holds 128/c blocks' runs.
//           Fixed pattern-2 becomes plain causal attention from natural queries onto them.
//
// Interval rules (query at natural position i; key-frame index kappa):
//   RU_BAND   kappa = j in [max(0, i - lo_off), i - hi_off]   strided head 1 (lo 0 .. l) and
//                                                            the merged band part (l-1 .. 1)
//   RU_BLOCK  kappa = j in [floor(i/l) l, i]                  fixed head 1
//   RU_COL    same column slot, grid row <= the query's       strided head 2 (and merged part 2)
//   RU_SUM    kappa in [0, count(i) - 1], count(i) = number of summary positions <= i
//                                                            fixed head 2
//   RU_SUMPREV kappa in [0, floor(i/l) c - 1]: summary runs of earlier blocks only (the part
//             of a merged fixed head not already in the same-block part)
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define ST_HD __host__ __device__ __forceinline__
#else
#define ST_HD inline
#endif

namespace st {

constexpr int32_t TILE = 128;

enum Frame : int32_t { FR_NAT = 0, FR_COL = 1, FR_SUM = 2 };
enum Rule : int32_t { RU_BAND = 0, RU_BLOCK = 1, RU_COL = 2, RU_SUM = 3, RU_SUMPREV = 4 };

// Division by a runtime constant d >= 1 as a multiply-high and a shift (valid for 0 <= x < 2^31):
// with s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1,  x / d = (umulhi(x, m) + x) >> s.
struct FastDiv {
    uint32_t mul, shift;
};

inline FastDiv make_fastdiv(uint32_t d)
{
    uint32_t s = 0;
    while ((1ull << s) < d) ++s;
    const uint64_t m = ((((1ull << s) - d) << 32) / d) + 1;
    return FastDiv{static_cast<uint32_t>(m), s};
}

ST_HD int32_t fdiv(int32_t x, FastDiv f)
{
#if defined(__CUDA_ARCH__)
    const uint32_t hi = __umulhi(static_cast<uint32_t>(x), f.mul);
#else
    const uint32_t hi = static_cast<uint32_t>((static_cast<uint64_t>(static_cast<uint32_t>(x)) * f.mul) >> 32);
#endif
    return static_cast<int32_t>((hi + static_cast<uint32_t>(x)) >> f.shift);
}

struct Geom {
    int32_t n, l, c;
    int32_t R;        // n / l grid rows
    int32_t Rt;       // rows per column slot in a column-frame tile (a power of two)
    int32_t cpt;      // column slots per column-frame tile
    int32_t tpc;      // column-frame tiles per column group
    int32_t ngroups;  // column groups
    int32_t upt;      // summary blocks per summary-frame tile (128 / c)
    int32_t pad[3];
    FastDiv div_l, div_c, div_tpc, div_Rt;  // for the per-row frame arithmetic
};

struct Part {
    int32_t head;
    int32_t rule;          // Rule
    int32_t qframe, kframe;
    int32_t o;             // fixed pattern-2 sub-block offset
    int32_t lo_off, hi_off;
    int32_t merge;         // 1: second pass, merges into what the first pass wrote
    int32_t nq, nk;        // tiles in the query / key frame
    int32_t dq_direct;     // 1: each query tile of the head is read by exactly one backward item
                           // (of any pass), so that item writes its dQ rows directly
    int32_t pad;
};

// Per-head flags of the backward pass.
constexpr int32_t HEAD_ZERO_FILL = 1;   // some key is written by no pass-0 item: dK, dV zeroed first
constexpr int32_t HEAD_DQ_DIRECT = 2;   // dQ written by the main kernel (see Part::dq_direct)

struct WorkItem {          // fwd: tile = query tile, [begin,end) key tiles; bwd: the converse
    int32_t part, tile, begin, end;
    // bwd only: a key tile whose query run is long is split into chunks processed by separate
    // CTAs.  slot: this chunk's fp32 partial-sum slot (-1: not split); nsplit: chunks of the key
    // tile; first: slot of its chunk 0 (chunks use consecutive slots); split: its SplitRec.
    int32_t slot, nsplit, first, split;
};
static_assert(sizeof(WorkItem) == 32, "work item layout");

// A split key tile: its dK/dV are the sum, in chunk order, of slots first .. first + nsplit - 1.
struct SplitRec {
    int32_t part, tile, first, nsplit;
};

// Longest query run one backward CTA walks; longer runs are split into near-equal chunks.
constexpr int32_t BWD_CHUNK = 48;

ST_HD int32_t imin(int32_t a, int32_t b) { return a < b ? a : b; }
ST_HD int32_t imax(int32_t a, int32_t b) { return a > b ? a : b; }

ST_HD int32_t frame_tiles(const Geom &g, int32_t fr)
{
    if (fr == FR_NAT) return g.n / TILE;
    if (fr == FR_COL) return g.ngroups * g.tpc;
    return (g.R * g.c + TILE - 1) / TILE;
}

// Natural position of row rho of tile t in frame fr (o: summary offset), or -1 for padding.
ST_HD int32_t frame_pos(const Geom &g, int32_t fr, int32_t o, int32_t t, int32_t rho)
{
    if (fr == FR_NAT) return t * TILE + rho;
    if (fr == FR_COL) {
        const int32_t grp = fdiv(t, g.div_tpc), rt = t - grp * g.tpc;
        const int32_t a = fdiv(rho, g.div_Rt), rr = rho - a * g.Rt;
        const int32_t col = grp * g.cpt + a, r = rt * TILE + rr;
        return (col < g.l && r < g.R) ? r * g.l + col : -1;
    }
    const int32_t kappa = t * TILE + rho;
    const int32_t u = fdiv(kappa, g.div_c), s = kappa - u * g.c;
    return u < g.R ? u * g.l + (g.l - g.c - o) + s : -1;
}

// Allowed key interval [lo, hi] (absolute key-frame indices) of query row rho of query tile t.
// Padding rows and rows with no allowed key get lo > hi.  Returns the natural position or -1.
ST_HD int32_t row_interval(const Geom &g, const Part &p, int32_t t, int32_t rho, int32_t &lo,
                           int32_t &hi)
{
    const int32_t i = frame_pos(g, p.qframe, p.o, t, rho);
    if (i < 0) { lo = 1; hi = 0; return -1; }
    switch (p.rule) {
    case RU_BAND:
        lo = imax(0, i - p.lo_off);
        hi = i - p.hi_off;
        break;
    case RU_BLOCK:
        lo = fdiv(i, g.div_l) * g.l;
        hi = i;
        break;
    case RU_COL: {
        const int32_t grp = fdiv(t, g.div_tpc), rt = t - grp * g.tpc;
        const int32_t a = fdiv(rho, g.div_Rt), rr = rho - a * g.Rt;
        lo = grp * g.tpc * TILE + a * g.Rt;
        hi = lo + rt * TILE + rr;
        break;
    }
    case RU_SUMPREV:
        lo = 0;
        hi = fdiv(i, g.div_l) * g.c - 1;
        break;
    default: {  // RU_SUM
        const int32_t blk = fdiv(i, g.div_l);
        int32_t w = i - blk * g.l - (g.l - g.c - p.o) + 1;
        w = imax(0, imin(w, g.c));
        lo = 0;
        hi = blk * g.c + w - 1;
        break;
    }
    }
    return i;
}

}  // namespace st
