// Page table kernel (SGLang FlashMLA backend page, flashmla_backend.py,
// init_forward_metadata: block_kv_indices [bs, cdiv(max L, 64)], -1 padded, filled
// from req_to_token / req_pool_indices / seq_lens).
//
// One thread per (request, page) entry.  Grid: x = requests, y = chunks of 256 pages.
// The request's length and row index are read once per CTA; each thread reads one
// req_to_token entry (the first slot of its page) and writes one int32.
#pragma once
#include "ptx.cuh"

namespace mla {

template <typename IdxT, typename LenT>
__global__ void __launch_bounds__(256)
build_block_table_kernel(const int32_t* __restrict__ req_to_token, int64_t r2t_rows,
                         int64_t r2t_stride, const IdxT* __restrict__ req_pool_indices,
                         const LenT* __restrict__ seq_lens, int32_t seq_len_add,
                         int32_t* __restrict__ block_table, int64_t bt_stride,
                         int32_t max_pages, int32_t fill_tail) {
    constexpr int kPage = 64;
    const int b = blockIdx.x;
    const int p = blockIdx.y * blockDim.x + threadIdx.x;
    if (p >= max_pages) return;
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

}  // namespace mla
