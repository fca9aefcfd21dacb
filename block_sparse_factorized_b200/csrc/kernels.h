// kernels.h -- parameter blocks and launch wrappers of the sm_100a kernels (internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "frames.cuh"

namespace st {

// Tensor maps of one [B*H, n, 64] tensor in the three frames (see frames.cuh):
//   nat: dims {64, n, BH},       box {64, 128, 1}
//   col: dims {64, R, l, BH},    box {64, Rt, cpt, 1}   (grid view, read column-wise)
//   sum: dims {64, l, R, BH},    box {64, c, 128/c, 1}  (summary runs of each block)
struct FrameMaps {
    CUtensorMap nat, col, sum;
};

struct FwdParams {
    FrameMaps q, k, v;
    FrameMaps ql, kl;            // split precision (fp32 I/O): low bf16 parts of Q and K
    const Part *parts;
    const WorkItem *items;
    int32_t nitems, batch, heads;
    Geom g;
    float scale_log2;            // log2(e) / sqrt(d)
    float *lse;                  // [B*H, n]
    uint16_t *o;                 // [B*H, n, 64] bf16 output, written row by row
    const uint16_t *o_prev;      // merge pass: the output (bf16) written by the first pass
    float *o_f32;                // fp32 I/O: output written row by row
    const float *o_prev_f32;     // fp32 I/O merge pass: the first pass's output
    int32_t *err;                // device error word
    int32_t *sched;              // unit counter, zero at launch
};

struct BwdParams {
    FrameMaps q, k, v, dout;
    FrameMaps dk_w, dv_w;        // bf16 I/O: dK, dV in the key frames, 16-column x 32-row boxes
                                 // (one softmax warp's slice; 32-byte swizzle)
    FrameMaps dq_red;            // fp32 dQ accumulator in the query frames, box 16 columns by
                                 // 32 rows (reduce-add target; nat and col only)
    CUtensorMap dq_direct;       // dQ output (natural frame), box 16 columns by 32 rows: one
                                 // warp's slice of a dq_direct part (fp32: 64-byte swizzle,
                                 // bf16: 32-byte swizzle)
    const Part *parts;
    const WorkItem *items;
    int32_t nitems, batch, heads;
    Geom g;
    float scale_log2;            // log2(e) / sqrt(d)
    float ds_scale;              // 1 / sqrt(d), folded into dS
    const float *lse;            // [B*H, n] natural-log lse of the forward
    const float *delta;          // [B*H, n] D_i = dO_i . O_i
    float *dq_acc;               // [B*H, n, 64] fp32, zeroed before the main kernel
    float *partials;             // [slots, B, 2, 128, 64] fp32 dK/dV partials of split key tiles
    int32_t *sched;              // item counter of this pass, zeroed before the main kernel
    uint16_t *dk_out, *dv_out;   // bf16 I/O: dK, dV [B*H, n, 64], written row by row
    float *dk_f32, *dv_f32;      // fp32 I/O: outputs written row by row
    int32_t *err;
};

struct PreParams {
    const uint16_t *o, *dout;    // bf16 [B*H, n, 64]
    const float *o_f32, *dout_f32;  // fp32 I/O instead of o, dout
    float *dk_f32, *dv_f32;         // fp32 I/O instead of dk, dv
    float *delta;                // [B*H, n]
    float *dq_acc;               // [B*H, n, 64] zeroed here (heads without HEAD_DQ_DIRECT)
    uint16_t *dk, *dv;           // zero-filled for heads flagged HEAD_ZERO_FILL
    const int32_t *head_flags;   // [H]
    int32_t *counters;           // zeroed here
    int32_t ncounters;
    int64_t bh;                  // B*H
    int32_t n, heads;
};

struct ConvParams {
    const float *dq_acc;
    uint16_t *dq;
    float *dq_f32;               // fp32 I/O: plain copy instead of rounding to bf16
    int32_t acc_head[64];        // the heads whose dQ is accumulated (not HEAD_DQ_DIRECT)
    int32_t nacc;                // how many
    int32_t batch, n, heads;
};

// dK/dV of split key tiles: sum of the chunks' fp32 partials in chunk order, plus the first
// pass's values for a merge part, written at the tile's rows.
struct SplitFinishParams {
    const float *partials;       // [slots, B, 2, 128, 64]
    const SplitRec *recs;
    const Part *parts;
    int32_t nrecs, batch, heads;
    Geom g;
    uint16_t *dk, *dv;           // bf16 I/O
    float *dk_f32, *dv_f32;      // fp32 I/O
};

// fp32 -> bf16 hi (round to nearest even) and, if lo != nullptr, lo = bf16(x - hi)
struct SplitParams {
    const float *src;
    uint16_t *hi, *lo;
    int64_t elems;
};

// Streaming multiprocessors of the current device (queried once per device).
int sm_count();

// Forward launch: the split-precision kernel (fp32 I/O, 64-wide rows) or the bf16 kernel for
// query-key rows of width dqk and value rows of width dv.
cudaError_t launch_fwd(const FwdParams &p, bool split, int dqk, int dv, cudaStream_t s);
cudaError_t launch_fwd_bf16(const FwdParams &p, int dqk, int dv, cudaStream_t s);
bool fwd_bf16_widths_supported(int dqk, int dv);
// Backward row widths (query-key dqk, value dv): bf16 (64, 64), (32, 32), (64, 128); fp32 I/O (64, 64).
bool bwd_widths_supported(int dqk, int dv);
cudaError_t launch_bwd(const BwdParams &p, bool f32, int dqk, int dv, cudaStream_t s);
cudaError_t launch_bwd_pre(const PreParams &p, bool f32, int dqk, int dv, cudaStream_t s);
cudaError_t launch_dq_convert(const ConvParams &p, bool f32, int dqk, cudaStream_t s);
cudaError_t launch_split(const SplitParams &p, cudaStream_t s);
cudaError_t launch_split_finish(const SplitFinishParams &p, bool f32, int dqk, int dv, cudaStream_t s);

}  // namespace st
