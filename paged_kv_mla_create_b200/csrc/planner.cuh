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
// One CTA: 1024 threads stage the lengths in shared memory (as block counts) and reduce
// the total; thread 0 then walks the parts.  The walk is O(bs + parts) shared-memory
// steps, a few microseconds at bs = 4096.
#pragma once
#include "ptx.cuh"

namespace mla {

constexpr int kFixedOverhead = 5;       // blocks of cost charged per piece
constexpr int kPlannerThreads = 1024;
constexpr int kPlannerSmemLens = 11264; // requests whose block counts fit in shared memory (44 KB)

__global__ void __launch_bounds__(kPlannerThreads)
get_mla_metadata_kernel(const int32_t* __restrict__ cache_seqlens, int32_t bs, int32_t parts,
                        int32_t* __restrict__ md, int32_t* __restrict__ num_splits) {
    __shared__ int32_t s_blocks[kPlannerSmemLens];
    __shared__ long long s_warp_sum[kPlannerThreads / 32];
    const bool staged = bs <= kPlannerSmemLens;
    long long local = 0;
    for (int b = threadIdx.x; b < bs; b += blockDim.x) {
        int32_t L = cache_seqlens[b];
        int32_t nb = L > 0 ? (L + 63) / 64 : 0;
        if (staged) s_blocks[b] = nb;
        local += nb + kFixedOverhead;
    }
    for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(0xffffffffu, local, off);
    if ((threadIdx.x & 31) == 0) s_warp_sum[threadIdx.x >> 5] = local;
    __syncthreads();
    if (threadIdx.x != 0) return;
    long long total = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) total += s_warp_sum[w];
    const long long payload = (total + parts - 1) / parts + kFixedOverhead;
    auto blocks_of = [&](int b) -> long long {
        if (staged) return s_blocks[b];
        int32_t L = cache_seqlens[b];
        return L > 0 ? (L + 63) / 64 : 0;
    };
    int b = 0;
    long long k = 0, s = 0, cum = 0;
    num_splits[0] = 0;
    for (int i = 0; i < parts; ++i) {
        const int begin_b = b;
        const long long begin_k = k, begin_s = s;
        long long budget = payload;
        while (b < bs) {
            const long long rem = blocks_of(b) - k;
            if (budget >= rem + kFixedOverhead) {
                cum += s + 1;
                num_splits[b + 1] = static_cast<int32_t>(cum);
                budget -= rem + kFixedOverhead;
                ++b;
                k = 0;
                s = 0;
            } else {
                if (budget - kFixedOverhead > 0) {
                    k += budget - kFixedOverhead;
                    ++s;
                }
                break;
            }
        }
        int4* row = reinterpret_cast<int4*>(md + 8 * static_cast<int64_t>(i));
        row[0] = make_int4(begin_b, static_cast<int>(begin_k), b, static_cast<int>(k));
        row[1] = make_int4(static_cast<int>(begin_s), 0, 0, 0);
    }
}

}  // namespace mla
