// layout.h -- internal definition of st_layout (host tables + device copy).
#pragma once
#include <stdint.h>

#include <mutex>
#include <vector>

#include "../../include/st_attn.h"
#include "frames.cuh"

// Natural-frame block CSR of one distinct (kind, offset): the exported, bit-exact contract.
struct NatPlan {
    int32_t kind = 0, o = 0;
    bool built = false;  // built on the first export (the kernels never read it)
    std::vector<int32_t> row_ptr, col_idx, mask_id;
    std::vector<uint32_t> masks;
    int32_t n_masks = 0;
};

struct st_layout {
    st_pattern_t pat{};
    int64_t n = 0;
    int32_t l = 0, c = 0, block = 0;
    std::vector<int32_t> head_kind, head_off, head_plan;
    mutable std::vector<NatPlan> plans;
    mutable std::mutex plans_mu;

    // execution plan (only when the kernels can run this layout)
    bool exec_ok = false;
    st::Geom geom{};
    std::vector<st::Part> parts;
    std::vector<int32_t> head_flags;       // HEAD_ZERO_FILL | HEAD_DQ_DIRECT per head
    std::vector<st::WorkItem> fwd_items[2], bwd_items[2];
    int32_t passes = 1;
    int32_t bwd_slots = 0, bwd_splits = 0;  // partial-sum slots and split key tiles (bwd)
    std::vector<st::SplitRec> bwd_split_recs[2];  // split key tiles of each pass
    int64_t exec_tiles = 0, allowed_pairs = 0;
    std::vector<int32_t> fwd_item_of;      // part * max_tiles + q tile -> fwd item index

    // device copy
    bool uploaded = false;
    int device = -1;
    void *d_buf = nullptr;
    st::Part *d_parts = nullptr;
    st::WorkItem *d_fwd[2] = {nullptr, nullptr};
    st::WorkItem *d_bwd[2] = {nullptr, nullptr};
    int32_t *d_head_flags = nullptr;
    st::SplitRec *d_split[2] = {nullptr, nullptr};
    int32_t *d_err = nullptr;
};
