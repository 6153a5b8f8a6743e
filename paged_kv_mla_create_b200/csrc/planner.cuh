// Split-KV scheduler kernel in the role of get_mla_metadata (SGLang FlashMLA backend
// page, flashmla_backend.py: tile_scheduler_metadata [num_sm_parts, 8] int32 and
// num_splits [bs+1] int32, recomputed for every batch on the device so that the whole
// metadata step can live inside a CUDA graph without a host round trip).
//
// The plan is a greedy balanced partition of 64-token blocks: every piece of a request
// costs its blocks plus kFixedOverhead; total = sum_b (blocks_b + kFixedOverhead) and
// each part gets the budget cdiv(total, parts) + kFixedOverhead, filled in request order.
// A request that fits in what is left of the budget is taken whole; otherwise the part
// takes (budget - kFixedOverhead) blocks of it when that is positive, and ends.
//
// One CTA: 256 threads stage the lengths in shared memory (as block counts) and reduce
// the total; thread 0 then walks the parts, O(bs + parts) steps of a few instructions
// each, with the next request's block count read one step ahead.
#pragma once
#include "ptx.cuh"

namespace mla {

constexpr int kFixedOverhead = 5;        // blocks of cost charged per piece
constexpr int kPlannerThreads = 256;
constexpr int kPlannerSmemLens = 8192;   // requests staged in shared memory (32 KB)
constexpr int kPlannerSmemParts = 320;   // scheduler rows staged in shared memory (10 KB)

__global__ void __launch_bounds__(kPlannerThreads)
get_mla_metadata_kernel(const int32_t* __restrict__ cache_seqlens, int32_t bs, int32_t parts,
                        int32_t* __restrict__ md, int32_t* __restrict__ num_splits) {
    // s_blocks[b] holds request b's block count until the walk passes it, then
    // num_splits[b + 1] (the walk reads entry b before it writes it).
    __shared__ int32_t s_blocks[kPlannerSmemLens + 1];
    __shared__ int4 s_rows[kPlannerSmemParts * 2];
    __shared__ long long s_warp_sum[kPlannerThreads / 32];
    const bool staged = bs <= kPlannerSmemLens;
    const bool rows_staged = parts <= kPlannerSmemParts;
    long long local = 0;
    for (int b = threadIdx.x; b < bs; b += blockDim.x) {
        const int32_t L = cache_seqlens[b];
        const int32_t nb = L > 0 ? (L + 63) / 64 : 0;
        if (staged) s_blocks[b] = nb;
        local += nb + kFixedOverhead;
    }
    if (staged && threadIdx.x == 0) s_blocks[bs] = 0;
    for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(0xffffffffu, local, off);
    if ((threadIdx.x & 31) == 0) s_warp_sum[threadIdx.x >> 5] = local;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long total = 0;
#pragma unroll
        for (int w = 0; w < kPlannerThreads / 32; ++w) total += s_warp_sum[w];
        // Budgets fit in 32 bits for any table a decode step can address (< 2^31 blocks).
        const int payload = (int)((total + parts - 1) / parts) + kFixedOverhead;
        auto blocks_of = [&](int b) -> int {
            if (staged) return s_blocks[b];
            if (b >= bs) return 0;
            const int32_t L = cache_seqlens[b];
            return L > 0 ? (L + 63) / 64 : 0;
        };
        int b = 0, k = 0, s = 0, cum = 0;
        int nb = bs > 0 ? blocks_of(0) : 0;  // blocks of request b, read one step ahead
        for (int i = 0; i < parts; ++i) {
            const int begin_b = b, begin_k = k, begin_s = s;
            int budget = payload;
            while (b < bs) {
                const int rem = nb - k;
                if (budget >= rem + kFixedOverhead) {
                    cum += s + 1;
                    if (staged)
                        s_blocks[b] = cum;
                    else
                        num_splits[b + 1] = cum;
                    budget -= rem + kFixedOverhead;
                    ++b;
                    nb = blocks_of(b);
                    k = 0;
                    s = 0;
                } else {
                    if (budget > kFixedOverhead) {
                        k += budget - kFixedOverhead;
                        ++s;
                    }
                    break;
                }
            }
            const int4 r0 = make_int4(begin_b, begin_k, b, k);
            const int4 r1 = make_int4(begin_s, 0, 0, 0);
            if (rows_staged) {
                s_rows[2 * i] = r0;
                s_rows[2 * i + 1] = r1;
            } else {
                int4* row = reinterpret_cast<int4*>(md + 8 * static_cast<int64_t>(i));
                row[0] = r0;
                row[1] = r1;
            }
        }
    }
    __syncthreads();
    // coalesced write-back of what the walk staged
    if (threadIdx.x == 0) num_splits[0] = 0;
    if (staged)
        for (int b = threadIdx.x; b < bs; b += blockDim.x) num_splits[b + 1] = s_blocks[b];
    if (rows_staged)
        for (int i = threadIdx.x; i < 2 * parts; i += blockDim.x)
            reinterpret_cast<int4*>(md)[i] = s_rows[i];
}

}  // namespace mla
