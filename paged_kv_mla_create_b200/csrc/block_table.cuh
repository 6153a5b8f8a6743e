// Page table kernel (SGLang FlashMLA backend page, flashmla_backend.py,
// init_forward_metadata: block_kv_indices [bs, cdiv(max L, 64)], -1 padded, filled
// from req_to_token / req_pool_indices / seq_lens).
//
// One thread per (request, page) entry: it reads the request's length and row index, one
// req_to_token entry (the first slot of its page) and writes one int32.  The same entry
// routine serves the page-table kernel (grid: x = requests, y = chunks of 256 pages) and
// the one-launch metadata kernel, whose CTA 0 plans the splits while the others fill the
// table.
#pragma once
#include "planner.cuh"
#include "ptx.cuh"

namespace mla {

template <typename IdxT, typename LenT>
__device__ __forceinline__ void block_table_entry(int b, int p, const int32_t* __restrict__ req_to_token,
                                                  int64_t r2t_rows, int64_t r2t_stride,
                                                  const IdxT* __restrict__ req_pool_indices,
                                                  const LenT* __restrict__ seq_lens, int32_t seq_len_add,
                                                  int32_t* __restrict__ block_table, int64_t bt_stride,
                                                  int32_t max_pages, int32_t fill_tail) {
    constexpr int kPage = 64;
    const int64_t row = static_cast<int64_t>(req_pool_indices[b]);
    int64_t L = static_cast<int64_t>(seq_lens[b]) + seq_len_add;
    if (L < 0) L = 0;
    int64_t npages = (L + kPage - 1) / kPage;
    const bool row_ok = row >= 0 && row < r2t_rows;
    // Positions beyond the row or beyond the table are clamped (and reported).
    const int64_t max_pages_row = r2t_stride / kPage + ((r2t_stride % kPage) ? 1 : 0);
    if (npages > max_pages || npages > max_pages_row) {
        if (p == 0) raise_error(4 /* MLA_DEVERR_LEN_OUT_OF_RANGE */);
        npages = npages > max_pages ? max_pages : npages;
        npages = npages > max_pages_row ? max_pages_row : npages;
    }
    if (!row_ok) {
        if (p == 0) raise_error(2 /* MLA_DEVERR_ROW_OUT_OF_RANGE */);
        if (fill_tail) block_table[b * bt_stride + p] = -1;
        return;
    }
    int32_t* dst = block_table + b * bt_stride + p;
    if (p < npages) {
        const int32_t slot = __ldg(req_to_token + row * r2t_stride + static_cast<int64_t>(p) * kPage);
        // Slots are non-negative and page-aligned at the start of each page (the pool viewed
        // [-1, 64, 1, 576] holds a page's 64 slots in order); division maps a slot to its page.
        if (slot < 0 || (slot & (kPage - 1)) != 0) raise_error(64 /* MLA_DEVERR_SLOT_INVALID */);
        *dst = slot >= 0 ? slot / kPage : -1;
    } else if (fill_tail) {
        *dst = -1;
    }
}

template <typename IdxT, typename LenT>
__global__ void __launch_bounds__(256)
build_block_table_kernel(const int32_t* __restrict__ req_to_token, int64_t r2t_rows,
                         int64_t r2t_stride, const IdxT* __restrict__ req_pool_indices,
                         const LenT* __restrict__ seq_lens, int32_t seq_len_add,
                         int32_t* __restrict__ block_table, int64_t bt_stride,
                         int32_t max_pages, int32_t fill_tail) {
    pdl_launch_dependents();   // a programmatic dependent waits for this grid's completion
    const int b = blockIdx.x;
    const int p = blockIdx.y * blockDim.x + threadIdx.x;
    if (p >= max_pages) return;
    block_table_entry(b, p, req_to_token, r2t_rows, r2t_stride, req_pool_indices, seq_lens, seq_len_add,
                      block_table, bt_stride, max_pages, fill_tail);
}

// The whole metadata step in one launch: CTA 0 computes the split plan (and the int32
// cache_seqlens = seq_lens + seq_len_add the attention call takes), CTAs 1.. fill the page
// table, 256 entries each in row-major order.
template <typename IdxT, typename LenT>
__global__ void __launch_bounds__(kPlannerThreads)
decode_metadata_kernel(const int32_t* __restrict__ req_to_token, int64_t r2t_rows, int64_t r2t_stride,
                       const IdxT* __restrict__ req_pool_indices, const LenT* __restrict__ seq_lens,
                       int32_t seq_len_add, int32_t bs, int32_t* __restrict__ block_table,
                       int64_t bt_stride, int32_t max_pages, int32_t fill_tail, int32_t parts,
                       int32_t* __restrict__ cache_seqlens, int32_t* __restrict__ md,
                       int32_t* __restrict__ num_splits) {
    // The attention grid, launched as a programmatic dependent, may be scheduled now: it sets
    // itself up and then waits for this grid to complete before it reads any of its outputs.
    pdl_launch_dependents();
    if (blockIdx.x == 0) {
        __shared__ PlannerSmem sm;
        plan_parts(
            [&](int b) -> int32_t {
                const int64_t L = static_cast<int64_t>(seq_lens[b]) + seq_len_add;
                return L < 0 ? 0 : (L > INT32_MAX ? INT32_MAX : static_cast<int32_t>(L));
            },
            bs, parts, md, num_splits, cache_seqlens, sm);
        return;
    }
    const int64_t idx = static_cast<int64_t>(blockIdx.x - 1) * kPlannerThreads + threadIdx.x;
    if (idx >= static_cast<int64_t>(bs) * max_pages) return;
    const int b = static_cast<int>(idx / max_pages);
    const int p = static_cast<int>(idx - static_cast<int64_t>(b) * max_pages);
    block_table_entry(b, p, req_to_token, r2t_rows, r2t_stride, req_pool_indices, seq_lens, seq_len_add,
                      block_table, bt_stride, max_pages, fill_tail);
}

}  // namespace mla
