// api.cu -- C ABI entry points: argument checks, TMA descriptors, launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <atomic>

#include "decode.h"
#include "kernels.h"
#include "layout.h"

namespace {

// Forward workspace head: one int32 unit counter per pass (zeroed by every call), padded so the
// fp32 copies that follow stay 256-byte aligned.
constexpr size_t FWD_SCHED_BYTES = 256;

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

int64_t value_width(const st_desc_t *desc) { return desc->dv == 0 ? desc->d : desc->dv; }

// Backward workspace: fp32 dK/dV partial sums of the chunks of split key tiles (one slot of 128
// rows x (d + dv) values per chunk and batch element) and the item counters of the two passes of
// the persistent kernel.
size_t bwd_partial_bytes(const st_desc_t *desc, const st_layout_t *layout)
{
    return static_cast<size_t>(layout->bwd_slots) * desc->batch * 128 * (desc->d + value_width(desc)) * sizeof(float);
}
size_t bwd_counter_bytes(const st_desc_t *, const st_layout_t *)
{
    return 2 * sizeof(int32_t);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lookup_encode()
{
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<EncodeTiledFn>(ptr);
    return nullptr;
}

// The driver's tensor-map encoder, looked up once (thread-safe static initialisation; a failed
// lookup is retried by the next call).
EncodeTiledFn encode_fn()
{
    static std::atomic<EncodeTiledFn> fn{lookup_encode()};
    EncodeTiledFn f = fn.load(std::memory_order_acquire);
    if (!f && (f = lookup_encode())) fn.store(f, std::memory_order_release);
    return f;
}

bool encode(CUtensorMap *m, const void *base, CUtensorMapDataType dt, cuuint32_t rank,
            const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box,
            CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B)
{
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return encode_fn()(m, dt, rank, const_cast<void *>(base), dims, strides, box, es,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps of a bf16 [BH, n, W] tensor in the natural, grid-column and summary frames.  A box
// is 128 rows by one swizzle span of columns: W = 32 columns (64 bytes, 64-byte swizzle) or 64
// columns (128 bytes, 128-byte swizzle); a 128-wide row is loaded as two boxes.
bool make_maps(st::FrameMaps &m, const void *base, const st::Geom &g, int64_t BH, bool col, bool sum, int W = 64)
{
    memset(&m, 0, sizeof(m));
    const cuuint64_t w = static_cast<cuuint64_t>(W), row = w * 2, n = static_cast<cuuint64_t>(g.n),
                     l = static_cast<cuuint64_t>(g.l);
    const cuuint32_t bx = static_cast<cuuint32_t>(W < 64 ? W : 64);
    const CUtensorMapSwizzle swz = W < 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    const CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    {
        const cuuint64_t dims[3] = {w, n, static_cast<cuuint64_t>(BH)};
        const cuuint64_t str[2] = {row, n * row};
        const cuuint32_t box[3] = {bx, 128, 1};
        if (!encode(&m.nat, base, dt, 3, dims, str, box, swz)) return false;
    }
    if (col) {
        const cuuint64_t dims[4] = {w, static_cast<cuuint64_t>(g.R), l, static_cast<cuuint64_t>(BH)};
        const cuuint64_t str[3] = {l * row, row, n * row};
        const cuuint32_t box[4] = {bx, static_cast<cuuint32_t>(g.Rt), static_cast<cuuint32_t>(g.cpt), 1};
        if (!encode(&m.col, base, dt, 4, dims, str, box, swz)) return false;
    }
    if (sum) {
        const cuuint64_t dims[4] = {w, l, static_cast<cuuint64_t>(g.R), static_cast<cuuint64_t>(BH)};
        const cuuint64_t str[3] = {row, l * row, n * row};
        const cuuint32_t box[4] = {bx, static_cast<cuuint32_t>(g.c), static_cast<cuuint32_t>(g.upt), 1};
        if (!encode(&m.sum, base, dt, 4, dims, str, box, swz)) return false;
    }
    return true;
}

// The swizzle of a box whose rows are `bytes` wide (16: none; 32, 64, 128: the same span), as the
// backward kernel's per-warp staging writes them.
CUtensorMapSwizzle swizzle_for(uint32_t bytes)
{
    return bytes >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                        : (bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                       : (bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE));
}

// [BH, n, W] maps with `bx`-column, 32-row boxes in the natural, grid-column and (if sum) summary
// frames, for one backward warp's slice of rows: the fp32 dQ accumulator as a reduce target
// (bx = W / 4 fp32), or a warp's slice of a dK or dV tile (bf16).
bool make_maps_slice(st::FrameMaps &m, const void *base, const st::Geom &g, int64_t BH, bool col, bool sum,
                     uint32_t W, uint32_t bx, bool f32)
{
    memset(&m, 0, sizeof(m));
    const cuuint64_t es = f32 ? 4 : 2, row = W * es, n = static_cast<cuuint64_t>(g.n), l = static_cast<cuuint64_t>(g.l);
    const CUtensorMapDataType dt = f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle swz = swizzle_for(static_cast<uint32_t>(bx * es));
    {
        const cuuint64_t dims[3] = {W, n, static_cast<cuuint64_t>(BH)};
        const cuuint64_t str[2] = {row, n * row};
        const cuuint32_t box[3] = {bx, 32, 1};
        if (!encode(&m.nat, base, dt, 3, dims, str, box, swz)) return false;
    }
    if (col) {
        const cuuint64_t dims[4] = {W, static_cast<cuuint64_t>(g.R), l, static_cast<cuuint64_t>(BH)};
        const cuuint64_t str[3] = {l * row, row, n * row};
        const cuuint32_t rows = static_cast<cuuint32_t>(g.Rt < 32 ? g.Rt : 32);
        const cuuint32_t slots = static_cast<cuuint32_t>(g.Rt < 32 ? 32 / g.Rt : 1);
        const cuuint32_t box[4] = {bx, rows, slots, 1};
        if (!encode(&m.col, base, dt, 4, dims, str, box, swz)) return false;
    }
    if (sum) {
        const cuuint64_t dims[4] = {W, l, static_cast<cuuint64_t>(g.R), static_cast<cuuint64_t>(BH)};
        const cuuint64_t str[3] = {row, l * row, n * row};
        const cuuint32_t rows = static_cast<cuuint32_t>(g.c < 32 ? g.c : 32);
        const cuuint32_t runs = static_cast<cuuint32_t>(g.c < 32 ? 32 / g.c : 1);
        const cuuint32_t box[4] = {bx, rows, runs, 1};
        if (!encode(&m.sum, base, dt, 4, dims, str, box, swz)) return false;
    }
    return true;
}

// The dQ output [BH, n, W] in the natural frame with a W / 4-column, 32-row box: one warp's slice
// of a query tile whose dQ the backward kernel stores directly (fp32 or bf16, swizzled as the
// kernel stages it).
bool make_map_dq_direct(CUtensorMap *m, const void *base, const st::Geom &g, int64_t BH, bool f32, uint32_t W)
{
    const cuuint64_t es = f32 ? 4 : 2, row = W * es, n = static_cast<cuuint64_t>(g.n);
    const cuuint64_t dims[3] = {W, n, static_cast<cuuint64_t>(BH)};
    const cuuint64_t str[2] = {row, n * row};
    const cuuint32_t box[3] = {W / 4, 32, 1};
    return encode(m, base, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dims, str,
                  box, swizzle_for(static_cast<uint32_t>(W / 4 * es)));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Frames {
    bool qcol = false, kcol = false, ksum = false;
};

Frames frames_used(const st_layout &L)
{
    Frames f;
    for (const auto &p : L.parts) {
        f.qcol |= (p.qframe == st::FR_COL);
        f.kcol |= (p.kframe == st::FR_COL);
        f.ksum |= (p.kframe == st::FR_SUM);
    }
    return f;
}

// Row widths the kernels are built for (query-key, value).  bf16 forward: (32, 32), (64, 64),
// (128, 128), (64, 128); bf16 backward: (32, 32), (64, 64), (64, 128); fp32 I/O: (64, 64).
bool widths_supported(const st_desc_t *desc, bool fwd = false)
{
    const int64_t dv = value_width(desc);
    if (desc->dtype == ST_BF16 && desc->d <= 128 && dv <= 128)
        return fwd ? st::fwd_bf16_widths_supported(static_cast<int>(desc->d), static_cast<int>(dv))
                   : st::bwd_widths_supported(static_cast<int>(desc->d), static_cast<int>(dv));
    return desc->d == 64 && dv == 64;
}

// Sizes every call and workspace query accepts: positive, and few enough rows (batch x heads x n
// <= 2^40) that no byte count below can wrap.
bool sizes_valid(const st_desc_t *desc)
{
    return desc->dv >= 0 && desc->batch >= 1 && desc->heads >= 1 && desc->n >= 1 && desc->d >= 1 &&
           desc->batch <= (1ll << 30) && desc->heads <= (1ll << 30) && desc->n <= (1ll << 40) &&
           desc->batch * desc->heads <= (1ll << 40) / desc->n;
}

st_status_t check_common(const st_layout *L, const st_desc_t *desc, bool fwd = false)
{
    if (!L || !desc) return ST_ERR_INVALID_ARG;
    if (!sizes_valid(desc)) return ST_ERR_INVALID_ARG;
    if (desc->dtype != ST_BF16 && desc->dtype != ST_FP32) return ST_ERR_INVALID_ARG;
    if (desc->heads != L->pat.num_heads || desc->n != L->n) return ST_ERR_INVALID_ARG;
    if (!L->exec_ok) return ST_ERR_UNSUPPORTED;
    if (!widths_supported(desc, fwd)) return ST_ERR_UNSUPPORTED;
    if (desc->batch * desc->heads > (1ll << 30)) return ST_ERR_UNSUPPORTED;
    if (!L->uploaded) return ST_ERR_NOT_UPLOADED;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ST_ERR_CUDA;
    if (dev != L->device) return ST_ERR_INVALID_ARG;
    if (!encode_fn()) return ST_ERR_CUDA;
    return ST_OK;
}

constexpr float LOG2E = 1.4426950408889634f;

size_t bf16_copy_bytes(const st_desc_t *desc)
{
    const size_t b = static_cast<size_t>(desc->batch) * desc->heads * desc->n * 64 * 2;
    return (b + 255) & ~size_t(255);
}

// fp32 I/O: round src to bf16 (and its residual) in the workspace.
bool split_copy(const void *src, void *hi, void *lo, const st_desc_t *desc, st_stream_t stream)
{
    st::SplitParams sp;
    sp.src = static_cast<const float *>(src);
    sp.hi = static_cast<uint16_t *>(hi);
    sp.lo = static_cast<uint16_t *>(lo);
    sp.elems = desc->batch * desc->heads * desc->n * 64;
    return st::launch_split(sp, stream) == cudaSuccess;
}

}  // namespace

extern "C" {

size_t st_attn_fwd_workspace_bytes(const st_desc_t *desc, const st_layout_t *layout)
{
    if (!desc || !layout || !sizes_valid(desc)) return 0;
    // the unit counters of the two passes; fp32 I/O adds bf16 copies Q_hi, Q_lo, K_hi, K_lo, V_hi
    return FWD_SCHED_BYTES + (desc->dtype == ST_FP32 ? 5 * bf16_copy_bytes(desc) : 0);
}

size_t st_attn_bwd_workspace_bytes(const st_desc_t *desc, const st_layout_t *layout)
{
    if (!desc || !layout || !sizes_valid(desc)) return 0;
    const size_t rows = static_cast<size_t>(desc->batch) * desc->heads * desc->n;
    const size_t dq = rows * desc->d * sizeof(float);
    const size_t dl = rows * sizeof(float);
    const size_t base = round256(dq) + round256(dl) + round256(bwd_partial_bytes(desc, layout)) +
                        round256(bwd_counter_bytes(desc, layout));
    // fp32 I/O adds bf16 copies of Q, K, V and dO for the tensor-core operands
    return desc->dtype == ST_FP32 ? base + 4 * bf16_copy_bytes(desc) : base;
}

st_status_t st_attn_fwd(const void *q, const void *k, const void *v, const st_layout_t *layout,
                        void *o, float *lse, void *workspace, size_t workspace_bytes,
                        const st_desc_t *desc, st_stream_t stream)
{
    if (!q || !k || !v || !o || !lse) return ST_ERR_INVALID_ARG;
    const st_status_t cs = check_common(layout, desc, true);
    if (cs != ST_OK) return cs;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ST_ERR_ALIGNMENT;
    const st_layout &L = *layout;
    const int64_t BH = desc->batch * desc->heads;
    const Frames f = frames_used(L);
    const bool f32 = desc->dtype == ST_FP32;
    const int dqk = static_cast<int>(desc->d), dv = static_cast<int>(value_width(desc));
    st::FwdParams p;
    memset(&p, 0, sizeof(p));
    if (!workspace || workspace_bytes < st_attn_fwd_workspace_bytes(desc, layout)) return ST_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ST_ERR_ALIGNMENT;
    int32_t *sched = static_cast<int32_t *>(workspace);
    if (cudaMemsetAsync(sched, 0, 2 * sizeof(int32_t), stream) != cudaSuccess) return ST_ERR_CUDA;
    if (f32) {
        const size_t cb = bf16_copy_bytes(desc);
        char *w = static_cast<char *>(workspace) + FWD_SCHED_BYTES;
        void *qh = w, *ql = w + cb, *kh = w + 2 * cb, *kl = w + 3 * cb, *vh = w + 4 * cb;
        if (!split_copy(q, qh, ql, desc, stream) || !split_copy(k, kh, kl, desc, stream) ||
            !split_copy(v, vh, nullptr, desc, stream))
            return ST_ERR_CUDA;
        if (!make_maps(p.q, qh, L.geom, BH, f.qcol, false) || !make_maps(p.ql, ql, L.geom, BH, f.qcol, false) ||
            !make_maps(p.k, kh, L.geom, BH, f.kcol, f.ksum) || !make_maps(p.kl, kl, L.geom, BH, f.kcol, f.ksum) ||
            !make_maps(p.v, vh, L.geom, BH, f.kcol, f.ksum))
            return ST_ERR_CUDA;
        p.o_f32 = static_cast<float *>(o);
        p.o_prev_f32 = static_cast<const float *>(o);
    } else if (!make_maps(p.q, q, L.geom, BH, f.qcol, false, dqk) ||
               !make_maps(p.k, k, L.geom, BH, f.kcol, f.ksum, dqk) ||
               !make_maps(p.v, v, L.geom, BH, f.kcol, f.ksum, dv)) {
        return ST_ERR_CUDA;
    }
    p.parts = L.d_parts;
    p.batch = static_cast<int32_t>(desc->batch);
    p.heads = static_cast<int32_t>(desc->heads);
    p.g = L.geom;
    p.scale_log2 = LOG2E / sqrtf(static_cast<float>(dqk));  // log2(e) / sqrt(d)
    p.lse = lse;
    if (!f32) p.o = static_cast<uint16_t *>(o);
    p.o_prev = static_cast<const uint16_t *>(o);
    p.err = L.d_err;
    for (int pass = 0; pass < 2; ++pass) {
        p.items = L.d_fwd[pass];
        p.nitems = static_cast<int32_t>(L.fwd_items[pass].size());
        p.sched = sched + pass;
        if (st::launch_fwd(p, f32, dqk, dv, stream) != cudaSuccess) return ST_ERR_CUDA;
    }
    return ST_OK;
}

namespace {

struct BwdWs {
    float *dq_acc, *delta;
    float *partials;   // split key tiles: dK/dV partial sums
    int32_t *counters; // split key tiles: chunks finished
    char *copies;      // fp32 I/O: bf16 Q, K, V, dO
};

st_status_t bwd_workspace(const st_desc_t *desc, const st_layout_t *layout, void *workspace,
                          size_t workspace_bytes, BwdWs &ws)
{
    if (!workspace || workspace_bytes < st_attn_bwd_workspace_bytes(desc, layout)) return ST_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ST_ERR_ALIGNMENT;
    const size_t rows = static_cast<size_t>(desc->batch) * desc->heads * desc->n;
    char *w = static_cast<char *>(workspace);
    ws.dq_acc = reinterpret_cast<float *>(w);
    w += round256(rows * desc->d * sizeof(float));
    ws.delta = reinterpret_cast<float *>(w);
    w += round256(rows * sizeof(float));
    ws.partials = reinterpret_cast<float *>(w);
    w += round256(bwd_partial_bytes(desc, layout));
    ws.counters = reinterpret_cast<int32_t *>(w);
    w += round256(bwd_counter_bytes(desc, layout));
    ws.copies = w;
    return ST_OK;
}

}  // namespace

st_status_t st_attn_bwd_prepare(const void *o, const void *dO, const st_layout_t *layout, void *dk,
                                void *dv, void *workspace, size_t workspace_bytes,
                                const st_desc_t *desc, st_stream_t stream)
{
    if (!o || !dO || !dk || !dv) return ST_ERR_INVALID_ARG;
    st_status_t cs = check_common(layout, desc);
    if (cs != ST_OK) return cs;
    BwdWs ws;
    if ((cs = bwd_workspace(desc, layout, workspace, workspace_bytes, ws)) != ST_OK) return cs;
    if (!aligned16(o) || !aligned16(dO) || !aligned16(dk) || !aligned16(dv)) return ST_ERR_ALIGNMENT;
    st::PreParams pre;
    memset(&pre, 0, sizeof(pre));
    const bool f32 = desc->dtype == ST_FP32;
    pre.o = static_cast<const uint16_t *>(o);
    pre.dout = static_cast<const uint16_t *>(dO);
    if (f32) {
        pre.o_f32 = static_cast<const float *>(o);
        pre.dout_f32 = static_cast<const float *>(dO);
        pre.dk_f32 = static_cast<float *>(dk);
        pre.dv_f32 = static_cast<float *>(dv);
    }
    pre.delta = ws.delta;
    pre.dq_acc = ws.dq_acc;
    pre.dk = static_cast<uint16_t *>(dk);
    pre.dv = static_cast<uint16_t *>(dv);
    pre.head_flags = layout->d_head_flags;
    pre.counters = ws.counters;
    pre.ncounters = 2;
    pre.bh = desc->batch * desc->heads;
    pre.n = static_cast<int32_t>(desc->n);
    pre.heads = static_cast<int32_t>(desc->heads);
    return st::launch_bwd_pre(pre, f32, static_cast<int>(desc->d), static_cast<int>(value_width(desc)), stream) ==
                   cudaSuccess
               ? ST_OK
               : ST_ERR_CUDA;
}

st_status_t st_attn_bwd_main(const void *q, const void *k, const void *v, const float *lse,
                             const void *dO, const st_layout_t *layout, void *dq, void *dk, void *dv,
                             void *workspace, size_t workspace_bytes, const st_desc_t *desc,
                             st_stream_t stream)
{
    if (!q || !k || !v || !lse || !dO || !dq || !dk || !dv) return ST_ERR_INVALID_ARG;
    st_status_t cs = check_common(layout, desc);
    if (cs != ST_OK) return cs;
    BwdWs ws;
    if ((cs = bwd_workspace(desc, layout, workspace, workspace_bytes, ws)) != ST_OK) return cs;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(lse) || !aligned16(dO) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return ST_ERR_ALIGNMENT;
    const st_layout &L = *layout;
    const int64_t BH = desc->batch * desc->heads;
    const Frames f = frames_used(L);
    st::BwdParams p;
    memset(&p, 0, sizeof(p));
    const bool f32 = desc->dtype == ST_FP32;
    const void *qb = q, *kb = k, *vb = v, *dob = dO;
    if (f32) {
        const size_t cb = bf16_copy_bytes(desc);
        char *c = ws.copies;
        if (!split_copy(q, c, nullptr, desc, stream) || !split_copy(k, c + cb, nullptr, desc, stream) ||
            !split_copy(v, c + 2 * cb, nullptr, desc, stream) || !split_copy(dO, c + 3 * cb, nullptr, desc, stream))
            return ST_ERR_CUDA;
        qb = c;
        kb = c + cb;
        vb = c + 2 * cb;
        dob = c + 3 * cb;
        p.dk_f32 = static_cast<float *>(dk);
        p.dv_f32 = static_cast<float *>(dv);
    }
    const uint32_t dqk = static_cast<uint32_t>(desc->d), dvw = static_cast<uint32_t>(value_width(desc));
    if (!make_map_dq_direct(&p.dq_direct, dq, L.geom, BH, f32, dqk)) return ST_ERR_CUDA;
    if (!make_maps_slice(p.dq_red, ws.dq_acc, L.geom, BH, f.qcol, false, dqk, dqk / 4, true)) return ST_ERR_CUDA;
    if (!f32 && (!make_maps_slice(p.dk_w, dk, L.geom, BH, f.kcol, f.ksum, dqk, dqk / 4, false) ||
                 !make_maps_slice(p.dv_w, dv, L.geom, BH, f.kcol, f.ksum, dvw, dvw / 4, false)))
        return ST_ERR_CUDA;
    if (!make_maps(p.q, qb, L.geom, BH, f.qcol, false, dqk) || !make_maps(p.dout, dob, L.geom, BH, f.qcol, false, dvw) ||
        !make_maps(p.k, kb, L.geom, BH, f.kcol, f.ksum, dqk) || !make_maps(p.v, vb, L.geom, BH, f.kcol, f.ksum, dvw))
        return ST_ERR_CUDA;
    p.parts = L.d_parts;
    p.batch = static_cast<int32_t>(desc->batch);
    p.heads = static_cast<int32_t>(desc->heads);
    p.g = L.geom;
    p.scale_log2 = LOG2E / sqrtf(static_cast<float>(dqk));  // log2(e) / sqrt(d)
    p.ds_scale = 1.0f / sqrtf(static_cast<float>(dqk));
    p.lse = lse;
    p.delta = ws.delta;
    p.dq_acc = ws.dq_acc;
    p.partials = ws.partials;
    if (!f32) {
        p.dk_out = static_cast<uint16_t *>(dk);
        p.dv_out = static_cast<uint16_t *>(dv);
    }
    p.err = L.d_err;
    for (int pass = 0; pass < 2; ++pass) {
        p.items = L.d_bwd[pass];
        p.nitems = static_cast<int32_t>(L.bwd_items[pass].size());
        p.sched = ws.counters + pass;
        if (st::launch_bwd(p, f32, static_cast<int>(dqk), static_cast<int>(dvw), stream) != cudaSuccess)
            return ST_ERR_CUDA;
        // split key tiles of this pass: the next pass (a merge) reads their dK/dV
        st::SplitFinishParams sf;
        memset(&sf, 0, sizeof(sf));
        sf.partials = ws.partials;
        sf.recs = L.d_split[pass];
        sf.parts = L.d_parts;
        sf.nrecs = static_cast<int32_t>(L.bwd_split_recs[pass].size());
        sf.batch = p.batch;
        sf.heads = p.heads;
        sf.g = L.geom;
        sf.dk = static_cast<uint16_t *>(dk);
        sf.dv = static_cast<uint16_t *>(dv);
        if (f32) {
            sf.dk_f32 = static_cast<float *>(dk);
            sf.dv_f32 = static_cast<float *>(dv);
        }
        if (st::launch_split_finish(sf, f32, static_cast<int>(dqk), static_cast<int>(dvw), stream) != cudaSuccess)
            return ST_ERR_CUDA;
    }
    return ST_OK;
}

st_status_t st_attn_bwd_finish(const st_layout_t *layout, void *dq, void *workspace,
                               size_t workspace_bytes, const st_desc_t *desc, st_stream_t stream)
{
    if (!dq) return ST_ERR_INVALID_ARG;
    st_status_t cs = check_common(layout, desc);
    if (cs != ST_OK) return cs;
    BwdWs ws;
    if ((cs = bwd_workspace(desc, layout, workspace, workspace_bytes, ws)) != ST_OK) return cs;
    if (!aligned16(dq)) return ST_ERR_ALIGNMENT;
    st::ConvParams cv;
    cv.dq_acc = ws.dq_acc;
    cv.dq = static_cast<uint16_t *>(dq);
    cv.dq_f32 = static_cast<float *>(dq);
    cv.nacc = 0;
    for (int32_t h = 0; h < desc->heads; ++h)
        if (!(layout->head_flags[h] & st::HEAD_DQ_DIRECT)) cv.acc_head[cv.nacc++] = h;
    cv.batch = static_cast<int32_t>(desc->batch);
    cv.n = static_cast<int32_t>(desc->n);
    cv.heads = static_cast<int32_t>(desc->heads);
    return st::launch_dq_convert(cv, desc->dtype == ST_FP32, static_cast<int>(desc->d), stream) == cudaSuccess
               ? ST_OK
               : ST_ERR_CUDA;
}

st_status_t st_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                        const float *lse, const void *dO, const st_layout_t *layout, void *dq,
                        void *dk, void *dv, void *workspace, size_t workspace_bytes,
                        const st_desc_t *desc, st_stream_t stream)
{
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return ST_ERR_INVALID_ARG;
    st_status_t cs = check_common(layout, desc);
    if (cs != ST_OK) return cs;
    BwdWs ws;
    if ((cs = bwd_workspace(desc, layout, workspace, workspace_bytes, ws)) != ST_OK) return cs;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return ST_ERR_ALIGNMENT;
    if ((cs = st_attn_bwd_prepare(o, dO, layout, dk, dv, workspace, workspace_bytes, desc, stream)) != ST_OK)
        return cs;
    if ((cs = st_attn_bwd_main(q, k, v, lse, dO, layout, dq, dk, dv, workspace, workspace_bytes, desc,
                               stream)) != ST_OK)
        return cs;
    return st_attn_bwd_finish(layout, dq, workspace, workspace_bytes, desc, stream);
}

size_t st_attn_decode_workspace_bytes(const st_desc_t *desc, const st_layout_t *layout)
{
    if (!desc || !layout || !sizes_valid(desc)) return 0;
    const size_t nsplit = static_cast<size_t>((desc->n + st::DEC_CHUNK - 1) / st::DEC_CHUNK);
    const size_t part = static_cast<size_t>(value_width(desc)) + 4;  // dec_part(dv) floats per chunk
    const size_t bh = static_cast<size_t>(desc->batch) * desc->heads;
    // the per-(batch, head) chunk counters, then the chunk results
    return round256(bh * sizeof(int32_t)) + round256(bh * nsplit * part * sizeof(float));
}

st_status_t st_attn_decode(const void *q, const void *k_cache, const void *v_cache, const st_layout_t *layout,
                           int64_t pos, void *o, float *lse, void *workspace, size_t workspace_bytes,
                           const st_desc_t *desc, st_stream_t stream)
{
    if (!q || !k_cache || !v_cache || !o || !lse || !layout || !desc) return ST_ERR_INVALID_ARG;
    const st_layout &L = *layout;
    if (!sizes_valid(desc)) return ST_ERR_INVALID_ARG;
    if (desc->dtype != ST_BF16 && desc->dtype != ST_FP32) return ST_ERR_INVALID_ARG;
    if (desc->heads != L.pat.num_heads || desc->n != L.n || pos < 0 || pos >= L.n) return ST_ERR_INVALID_ARG;
    const int64_t dv = value_width(desc);
    if (desc->d > 128 || dv > 128 || !st::decode_widths_supported(static_cast<int>(desc->d), static_cast<int>(dv)) ||
        desc->heads > 64 || desc->batch * desc->heads > (1ll << 30))
        return ST_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) || !aligned16(lse))
        return ST_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < st_attn_decode_workspace_bytes(desc, layout)) return ST_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ST_ERR_ALIGNMENT;
    st::DecodeParams p;
    memset(&p, 0, sizeof(p));
    p.q = q;
    p.k = k_cache;
    p.v = v_cache;
    p.o = o;
    p.lse = lse;
    const size_t bh = static_cast<size_t>(desc->batch) * desc->heads;
    p.cnt = static_cast<int32_t *>(workspace);
    p.part = reinterpret_cast<float *>(static_cast<char *>(workspace) + round256(bh * sizeof(int32_t)));
    int64_t most = 1;
    for (int32_t h = 0; h < desc->heads; ++h) {
        p.kind[h] = L.head_kind[h];
        p.off[h] = L.head_off[h];
        const int64_t cnt = st::key_count(st::key_set(p.kind[h], pos, L.l, L.c, p.off[h]));
        if (cnt > most) most = cnt;
    }
    p.pos = pos;
    p.n = L.n;
    p.l = L.l;
    p.c = L.c;
    p.bh = static_cast<int32_t>(desc->batch * desc->heads);
    p.heads = static_cast<int32_t>(desc->heads);
    p.scale_log2 = LOG2E / sqrtf(static_cast<float>(desc->d));  // log2(e) / sqrt(d)
    const int64_t nsplit = (most + st::DEC_CHUNK - 1) / st::DEC_CHUNK;
    if (nsplit > 65535) return ST_ERR_UNSUPPORTED;  // grid dimension y: a row with over 4 M allowed keys
    if (cudaMemsetAsync(p.cnt, 0, bh * sizeof(int32_t), stream) != cudaSuccess) return ST_ERR_CUDA;
    return st::launch_decode(p, static_cast<int32_t>(nsplit), desc->dtype == ST_FP32, static_cast<int>(desc->d),
                             static_cast<int>(dv), stream) == cudaSuccess
               ? ST_OK
               : ST_ERR_CUDA;
}

st_status_t st_decode_row_keys(const st_layout_t *layout, int32_t head, int64_t pos, int64_t *keys, int64_t *count)
{
    if (!layout || !keys || !count || head < 0 || head >= layout->pat.num_heads || pos < 0 || pos >= layout->n)
        return ST_ERR_INVALID_ARG;
    const st::KeySet ks = st::key_set(layout->head_kind[head], pos, layout->l, layout->c, layout->head_off[head]);
    const int64_t cnt = st::key_count(ks);
    for (int64_t e = 0; e < cnt; ++e) keys[e] = st::key_at(ks, e);
    *count = cnt;
    return ST_OK;
}

const char *st_status_string(st_status_t s)
{
    switch (s) {
    case ST_OK: return "ok";
    case ST_ERR_INVALID_ARG: return "invalid argument";
    case ST_ERR_UNSUPPORTED: return "unsupported by the kernels";
    case ST_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case ST_ERR_NOT_UPLOADED: return "layout not uploaded";
    case ST_ERR_CUDA: return "CUDA error";
    case ST_ERR_OOM: return "out of memory";
    case ST_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case ST_ERR_WORKSPACE: return "workspace missing or too small";
    case ST_ERR_INTERNAL: return "internal error";
    }
    return "unknown status";
}

const char *st_version(void) { return "st_attn 0.1 (sm_100a)"; }

}  // extern "C"
