// Split-KV scheduler kernel in the role of get_mla_metadata (SGLang FlashMLA backend
// page, flashmla_backend.py: tile_scheduler_metadata [num_sm_parts, 8] int32 and
// num_splits [bs+1] int32, recomputed for every batch on the device so that the whole
// metadata step can live inside a CUDA graph without a host round trip).
//
// The plan is a greedy balanced partition of 64-token blocks: every piece of a request
// costs its blocks plus kFixedOverhead; total = sum_b (blocks_b + kFixedOverhead) and
// each part gets the budget P = cdiv(total, parts) + kFixedOverhead, filled in request
// order.  A request that fits in what is left of the budget is taken whole; otherwise the
// part takes (budget - kFixedOverhead) blocks of it when that is positive, and ends.
//
// The walk is computed per request rather than per part: entering request b with r of
// part i's budget left, either it fits (r >= blocks + F), or, after skipping to a fresh
// part when r <= F, its first piece takes r - F blocks, the following parts take
// Q = P - F blocks each, and the last piece takes the rest (1..Q blocks) -- a closed form
// whose one division is needed only when a request spans more than two further parts.  One
// thread runs that O(bs) recurrence, a short chain of compares per request; then one thread
// per request writes the fields of the part rows that begin or end inside it.  Batches
// larger than kPlannerSmemLens take the part-by-part walk instead, reading the lengths from
// global memory.
#pragma once
#include "ptx.cuh"

namespace mla {

constexpr int kFixedOverhead = 5;        // blocks of cost charged per piece
constexpr int kPlannerThreads = 256;
constexpr int kPlannerSmemLens = 2048;   // requests handled by the per-request walk

struct PlannerSmem {
    int32_t nb[kPlannerSmemLens + 1];   // blocks of request b
    int32_t fp[kPlannerSmemLens];       // first part of request b
    int32_t lp[kPlannerSmemLens];       // last part of request b
    int32_t x0[kPlannerSmemLens];       // blocks of its first piece
    int32_t cum[kPlannerSmemLens];      // num_splits[b + 1]
    long long warp_sum[kPlannerThreads / 32];
};

// The plan, computed by one CTA of kPlannerThreads threads.  len_of(b) is request b's KV
// length (read once per request, by the first loop); cache_seqlens_out, when not null,
// receives those lengths as int32.
template <typename LenFn>
__device__ __forceinline__ void plan_parts(LenFn len_of, int32_t bs, int32_t parts,
                                           int32_t* __restrict__ md, int32_t* __restrict__ num_splits,
                                           int32_t* __restrict__ cache_seqlens_out, PlannerSmem& sm) {
    int32_t* s_nb = sm.nb;
    int32_t* s_fp = sm.fp;
    int32_t* s_lp = sm.lp;
    int32_t* s_x0 = sm.x0;
    int32_t* s_cum = sm.cum;
    long long* s_warp_sum = sm.warp_sum;
    const bool staged = bs <= kPlannerSmemLens;
    long long local = 0;
    for (int b = threadIdx.x; b < bs; b += blockDim.x) {
        const int32_t L = len_of(b);
        if (cache_seqlens_out) cache_seqlens_out[b] = L;
        const int32_t nb = L > 0 ? (L + 63) / 64 : 0;
        if (staged) s_nb[b] = nb;
        local += nb + kFixedOverhead;
    }
    if (staged && threadIdx.x == 0) s_nb[bs] = 0;
    for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(0xffffffffu, local, off);
    if ((threadIdx.x & 31) == 0) s_warp_sum[threadIdx.x >> 5] = local;
    __syncthreads();
    long long total = 0;
#pragma unroll
    for (int w = 0; w < kPlannerThreads / 32; ++w) total += s_warp_sum[w];
    // Budgets fit in 32 bits for any table a decode step can address (< 2^31 blocks).
    const int P = (int)((total + parts - 1) / parts) + kFixedOverhead;
    const int Q = P - kFixedOverhead;   // >= 1

    if (!staged) {
        // part-by-part walk, lengths from global memory
        if (threadIdx.x == 0) {
            auto blocks_of = [&](int b) -> int {
                if (b >= bs) return 0;
                const int32_t L = len_of(b);
                return L > 0 ? (L + 63) / 64 : 0;
            };
            num_splits[0] = 0;
            int b = 0, k = 0, s = 0, cum = 0;
            int nb = blocks_of(0);
            for (int i = 0; i < parts; ++i) {
                const int begin_b = b, begin_k = k, begin_s = s;
                int budget = P;
                while (b < bs) {
                    const int rem = nb - k;
                    if (budget >= rem + kFixedOverhead) {
                        cum += s + 1;
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
                int4* row = reinterpret_cast<int4*>(md + 8 * static_cast<int64_t>(i));
                row[0] = make_int4(begin_b, begin_k, b, k);
                row[1] = make_int4(begin_s, 0, 0, 0);
            }
        }
        return;
    }

    if (threadIdx.x == 0) {
        // The walk's loop-carried state is (i, r): the part and what is left of its budget.
        // Entering request b of c = blocks + F: a part with r <= F and r < c ends unused; the
        // request then fits (r >= c) or is split: its first piece takes r - F blocks, m full
        // middle parts take Q blocks each and the last piece the rest, last = rem - m Q with
        // rem = c - r, leaving Q - last.  m = (rem - 1) / Q is 0 or 1 unless the request spans
        // more than two further parts, so the division stays off the common path: a request
        // about as long as a part's budget often spans two, and a float-estimate quotient or a
        // modulo on that path cost ~30 cycles a request more (bs 64, budget 44 blocks).
        int i = 0, r = P, cum = 0;
        int nb = s_nb[0];
#pragma unroll 4
        for (int b = 0; b < bs; ++b) {
            const int nb_next = s_nb[b + 1];
            const int c = nb + kFixedOverhead;
            if (r < c && r <= kFixedOverhead) {
                r = P;
                ++i;
            }
            s_fp[b] = i;
            if (r >= c) {
                r -= c;
                s_x0[b] = nb;
                cum += 1;
            } else {
                const int rem = c - r;                                   // >= 1
                int m = rem > Q ? 1 : 0;
                if (rem > 2 * Q) m = (rem - 1) / Q;
                s_x0[b] = r - kFixedOverhead;                            // 1 <= x0 < nb
                i += 1 + m;
                r = Q - (rem - m * Q);
                cum += 2 + m;
            }
            s_lp[b] = i;
            s_cum[b] = cum;
            nb = nb_next;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) num_splits[0] = 0;
    // The part rows, scattered from the per-request results without a search.  Part i begins
    // in the first request whose last part is >= i: request b for i in (lp[b-1], lp[b]].  It
    // ends in the last request whose first part is <= i: request b for i in [fp[b], fp[b+1]),
    // no further than lp[b].  Every part up to lp[bs-1] has one of each (no part in between is
    // left empty: a request starts in the part the previous one ended in, or the next one);
    // the parts after it are unused.
    for (int b = threadIdx.x; b < bs; b += blockDim.x) {
        num_splits[b + 1] = s_cum[b];
        const int fpb = s_fp[b], lpb = s_lp[b], x0b = s_x0[b];
        const int lp_prev = b > 0 ? s_lp[b - 1] : -1;
        // (every index stays below parts, which the walk guarantees; the bounds only make sure)
        const int last = min(lpb, parts - 1);
        const int end_last = b + 1 < bs ? min(s_fp[b + 1] - 1, last) : last;
        for (int i = lp_prev + 1; i <= last; ++i) {   // parts that begin in request b
            int32_t* row = md + 8 * static_cast<int64_t>(i);
            const int begin_s = i > fpb ? i - fpb : 0;
            row[0] = b;
            row[1] = begin_s > 0 ? x0b + (begin_s - 1) * Q : 0;
            *reinterpret_cast<int4*>(row + 4) = make_int4(begin_s, 0, 0, 0);
        }
        for (int i = fpb; i <= end_last; ++i) {      // parts that end in request b
            int32_t* row = md + 8 * static_cast<int64_t>(i);
            const bool inside = lpb > i;
            *reinterpret_cast<int2*>(row + 2) = make_int2(inside ? b : b + 1, inside ? x0b + (i - fpb) * Q : 0);
        }
    }
    const int used = bs > 0 ? min(s_lp[bs - 1] + 1, parts) : 0;
    for (int i = used + threadIdx.x; i < parts; i += blockDim.x) {
        int4* row = reinterpret_cast<int4*>(md + 8 * static_cast<int64_t>(i));
        row[0] = make_int4(bs, 0, bs, 0);
        row[1] = make_int4(0, 0, 0, 0);
    }
}

__global__ void __launch_bounds__(kPlannerThreads)
get_mla_metadata_kernel(const int32_t* __restrict__ cache_seqlens, int32_t bs, int32_t parts,
                        int32_t* __restrict__ md, int32_t* __restrict__ num_splits) {
    __shared__ PlannerSmem sm;
    pdl_launch_dependents();   // a programmatic dependent waits for this grid's completion
    plan_parts([&](int b) -> int32_t { return cache_seqlens[b]; }, bs, parts, md, num_splits, nullptr, sm);
}

}  // namespace mla
