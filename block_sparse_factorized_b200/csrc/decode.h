// decode.h -- the decode step's key enumeration (host and device) and kernel parameters.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "frames.cuh"

namespace st {

constexpr int DEC_CHUNK = 64;   // keys per CTA (16 groups x 4 keys)
// floats per chunk result for value rows of width dv: M, L, (pad, pad), O[dv] -- O 16-byte aligned
__host__ __device__ constexpr int dec_part(int dv) { return dv + 4; }

// Allowed keys of one row: nu runs, run u covering g0 + u * gs .. + glen - 1 (the last run cut to
// glast keys), and the range r0 .. r0 + nr - 1.  Runs and range are disjoint and every run lies
// below the range, so runs-then-range is increasing order.
struct KeySet {
    int64_t r0, nr, g0, gs, nu, glen, glast;
};

// A(i) of set kind `kind` (st_kind_t numbering) for pattern parameters l, c and sub-block offset o
// ("Sparse Transformers 深度解读报告" §2.2, with j <= i on every set, §2.1):
//   local band  max(0, i - l) .. i          stride       i, i - l, i - 2l, ...
//   same block  floor(i/l) l .. i           summary      j mod l in [l - c - o, l - 1 - o], j <= i
// merged kinds: the band (resp. the block) as the range, the rest of the other set as the runs.
ST_HD KeySet key_set(int32_t kind, int64_t i, int64_t l, int64_t c, int64_t o)
{
    KeySet k{0, 0, 0, 1, 0, 1, 1};
    const int64_t blk = i / l;
    switch (kind) {
    case 1:  // sA1
    case 3:  // sU: the band, then i - m l for m >= 2 (m = 0, 1 lie in the band)
        k.r0 = i - l > 0 ? i - l : 0;
        k.nr = i - k.r0 + 1;
        if (kind == 3 && blk >= 2) {
            k.g0 = i - blk * l;
            k.gs = l;
            k.nu = blk - 1;
        }
        break;
    case 2:  // sA2
        k.g0 = i - blk * l;
        k.gs = l;
        k.nu = blk + 1;
        break;
    case 4:  // fA1
    case 6:  // fU: the block, then the summary runs of the earlier blocks
        k.r0 = blk * l;
        k.nr = i - k.r0 + 1;
        if (kind == 6) {
            k.g0 = l - c - o;
            k.gs = l;
            k.glen = k.glast = c;
            k.nu = blk;
        }
        break;
    case 5: {  // fA2: the runs of blocks 0 .. blk that start at or before i
        k.g0 = l - c - o;
        k.gs = l;
        k.glen = k.glast = c;
        const int64_t start = blk * l + k.g0;
        if (start <= i) {
            k.nu = blk + 1;
            k.glast = i - start + 1 < c ? i - start + 1 : c;
        } else {
            k.nu = blk;
        }
        break;
    }
    default:
        break;
    }
    return k;
}

ST_HD int64_t key_count(const KeySet &k) { return k.nr + (k.nu > 0 ? (k.nu - 1) * k.glen + k.glast : 0); }

// The e-th key of the set in increasing order (the runs, then the range).
ST_HD int64_t key_at(const KeySet &k, int64_t e)
{
    const int64_t ng = key_count(k) - k.nr;
    if (e >= ng) return k.r0 + (e - ng);
    const int64_t u = e / k.glen;
    return k.g0 + u * k.gs + (e - u * k.glen);
}

struct DecodeParams {
    const void *q;      // [B*H, d] one query row per (batch, head)
    const void *k;      // [B*H, n, d] key cache (rows past pos unread)
    const void *v;      // [B*H, n, dv] value cache (rows past pos unread)
    void *o;            // [B*H, dv]
    float *lse;         // [B*H], natural log
    float *part;        // [B*H, nsplit, dec_part(dv)] chunk results (workspace)
    int32_t *cnt;       // [B*H] chunks finished (workspace, zero before the launch)
    int32_t kind[64], off[64];
    int64_t pos, n, l, c;
    int32_t bh, heads;
    float scale_log2;   // log2(e) / sqrt(d)
};

// Row widths (query-key d, value dv) with a decode kernel: (32, 32), (64, 64), (128, 128), (64, 128).
bool decode_widths_supported(int d, int dv);
cudaError_t launch_decode(const DecodeParams &p, int32_t nsplit, bool f32, int d, int dv, cudaStream_t s);

}  // namespace st
