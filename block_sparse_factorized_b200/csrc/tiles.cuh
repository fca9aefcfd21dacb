// tiles.cuh -- frame-aware TMA tile transfers and fast exp2/log2, shared by the kernels.
#pragma once
#include "frames.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace st {

constexpr uint32_t TILE_BYTES = 128 * 64 * 2;  // one 128 x 64 bf16 tile, 16 KB
constexpr float LN2 = 0.6931471805599453f;
constexpr float LOG2E = 1.4426950408889634f;

// Hardware base-2 exponential / logarithm (MUFU ex2 / lg2), flush-to-zero.
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Columns lo..hi of a 64-column slice as a bit mask (bit c = column c allowed); lo and hi are
// relative to the slice and may lie outside it; hi < lo is the empty interval.
__device__ __forceinline__ uint64_t interval_bits64(int32_t lo, int32_t hi)
{
    if (hi < lo || hi < 0 || lo > 63) return 0ull;
    const uint64_t up = hi >= 63 ? ~0ull : ((2ull << hi) - 1ull);
    const uint64_t dn = lo <= 0 ? ~0ull : (~0ull << lo);
    return up & dn;
}

// The same for a 32-column slice.
__device__ __forceinline__ uint32_t interval_bits32(int32_t lo, int32_t hi)
{
    if (hi < lo || hi < 0 || lo > 31) return 0u;
    const uint32_t up = hi >= 31 ? ~0u : ((2u << hi) - 1u);
    const uint32_t dn = lo <= 0 ? ~0u : (~0u << lo);
    return up & dn;
}

__device__ __forceinline__ const CUtensorMap *frame_map(const FrameMaps &m, int32_t fr)
{
    return fr == FR_NAT ? &m.nat : (fr == FR_COL ? &m.col : &m.sum);
}

// TMA load of columns x .. x + box - 1 (the map's box width) of tile t of frame fr (summary
// offset o) of batch-head bh into dst.
__device__ __forceinline__ void load_tile_x(const FrameMaps &m, int32_t fr, const Geom &g, int32_t o, int32_t t,
                                            int32_t bh, int32_t x, void *dst, uint64_t *bar)
{
    if (fr == FR_NAT) {
        tma_load_3d(dst, &m.nat, bar, x, t * TILE, bh);
    } else if (fr == FR_COL) {
        const int32_t grp = fdiv(t, g.div_tpc), rt = t - grp * g.tpc;
        tma_load_4d(dst, &m.col, bar, x, rt * TILE, grp * g.cpt, bh);
    } else {
        tma_load_4d(dst, &m.sum, bar, x, g.l - g.c - o, t * g.upt, bh);
    }
}

// TMA load of tile t of frame fr (summary offset o) of batch-head bh into dst (16 KB).
__device__ __forceinline__ void load_tile(const FrameMaps &m, int32_t fr, const Geom &g, int32_t o,
                                          int32_t t, int32_t bh, void *dst, uint64_t *bar)
{
    load_tile_x(m, fr, g, o, t, bh, 0, dst, bar);
}

// TMA store of a 16 KB tile; rows outside the tensor (padding of the grid and summary frames)
// are clipped by the copy engine.
__device__ __forceinline__ void store_tile(const FrameMaps &m, int32_t fr, const Geom &g, int32_t o,
                                           int32_t t, int32_t bh, const void *src)
{
    if (fr == FR_NAT) {
        tma_store_3d(&m.nat, src, 0, t * TILE, bh);
    } else if (fr == FR_COL) {
        const int32_t grp = fdiv(t, g.div_tpc), rt = t - grp * g.tpc;
        tma_store_4d(&m.col, src, 0, rt * TILE, grp * g.cpt, bh);
    } else {
        tma_store_4d(&m.sum, src, 0, g.l - g.c - o, t * g.upt, bh);
    }
}

// TMA reduce-add of one warp's 32 rows (tile rows 32 q4 .. 32 q4 + 31) x 16 fp32 columns
// (col0 .. col0 + 15) of query tile t.  The reduce maps' boxes are 16 columns by 32 rows:
// {16, 32, 1} in the natural frame, {16, min(Rt, 32), max(1, 32 / Rt), 1} in the grid frame.
__device__ __forceinline__ void reduce_warp_f32(const FrameMaps &m, int32_t fr, const Geom &g, int32_t t,
                                                int32_t bh, int32_t col0, int32_t q4, const void *src)
{
    if (fr == FR_NAT) {
        tma_reduce_add_3d(&m.nat, src, col0, t * TILE + 32 * q4, bh);
    } else {
        const int32_t grp = fdiv(t, g.div_tpc), rt = t - grp * g.tpc;
        const int32_t rho0 = 32 * q4, a0 = fdiv(rho0, g.div_Rt), r0 = rho0 - a0 * g.Rt;
        tma_reduce_add_4d(&m.col, src, col0, rt * TILE + r0, grp * g.cpt + a0, bh);
    }
}

// TMA store of one warp's 32 rows (tile rows 32 q4 .. 32 q4 + 31) x 16 bf16 columns (col0 ..
// col0 + 15) of key tile t in frame fr (summary offset o).  The maps' boxes are 16 columns by 32
// rows: {16, 32, 1} natural, {16, min(Rt, 32), max(1, 32 / Rt), 1} grid, {16, min(c, 32),
// max(1, 32 / c), 1} summary (c a power of two, so the 32 rows are one part of a run or whole
// runs).  Rows past the tensor (frame padding) are dropped.
__device__ __forceinline__ void store_warp_slice(const FrameMaps &m, int32_t fr, const Geom &g, int32_t o,
                                                 int32_t t, int32_t bh, int32_t col0, int32_t q4, const void *src)
{
    const int32_t rho0 = 32 * q4;
    if (fr == FR_NAT) {
        tma_store_3d(&m.nat, src, col0, t * TILE + rho0, bh);
    } else if (fr == FR_COL) {
        const int32_t grp = fdiv(t, g.div_tpc), rt = t - grp * g.tpc;
        const int32_t a0 = fdiv(rho0, g.div_Rt), r0 = rho0 - a0 * g.Rt;
        tma_store_4d(&m.col, src, col0, rt * TILE + r0, grp * g.cpt + a0, bh);
    } else {
        const int32_t kappa = t * TILE + rho0, u = fdiv(kappa, g.div_c), s0 = kappa - u * g.c;
        tma_store_4d(&m.sum, src, col0, g.l - g.c - o + s0, u, bh);
    }
}

// Per-width tile geometry.  A 128-row bf16 tile of W columns is loaded as NBOX TMA boxes of BOX
// columns, each one swizzle span wide (64-byte swizzle for W = 32, 128-byte otherwise), stored
// one after another: box b holds columns b*BOX .. b*BOX + BOX - 1 of every row.
template <int W>
struct Tile {
    static_assert(W == 32 || W == 64 || W == 128, "row width");
    static constexpr int BOX = W < 64 ? W : 64;
    static constexpr int NBOX = W / BOX;
    static constexpr uint32_t SPAN = BOX * 2;                // bytes per row of a box (swizzle span)
    static constexpr uint32_t BOX_BYTES = 128 * SPAN;
    static constexpr uint32_t BYTES = NBOX * BOX_BYTES;
    static constexpr uint32_t LAYOUT = W < 64 ? UMMA_SW64 : UMMA_SW128;
    // K-major operand (rows = M or N, K = the W columns): the K16 step k starts 32 bytes further
    // in the same box, or in the next box once a box's columns are used up; 8-row groups are
    // 8 * SPAN bytes apart.
    __device__ static uint64_t kmajor(uint32_t base, int k)
    {
        const int col = 16 * k;
        return desc_swz(base + (col / BOX) * BOX_BYTES + (col % BOX) * 2, 16, 8 * SPAN, LAYOUT);
    }
    // MN-major operand (K = the 128 rows, N = the W columns): the K16 step k starts 16 rows
    // further; 8-row groups are 8 * SPAN bytes apart (SBO) and the N atoms are the boxes (LBO).
    __device__ static uint64_t mnmajor(uint32_t base, int k)
    {
        return desc_swz(base + 16 * k * SPAN, BOX_BYTES, 8 * SPAN, LAYOUT);
    }
};

// TMA load of tile t of frame fr of batch-head bh into dst: NBOX boxes, one transaction count.
template <int W>
__device__ __forceinline__ void load_tile_w(const FrameMaps &m, int32_t fr, const Geom &g, int32_t o, int32_t t,
                                            int32_t bh, uint8_t *dst, uint64_t *bar)
{
#pragma unroll
    for (int b = 0; b < Tile<W>::NBOX; ++b)
        load_tile_x(m, fr, g, o, t, bh, b * Tile<W>::BOX, dst + b * Tile<W>::BOX_BYTES, bar);
}

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

}  // namespace st
