// Log-sum-exp merge of split-KV partial results: the step implied by get_mla_metadata's
// num_splits in the SGLang FlashMLA backend page (flashmla_backend.py) and written out
// as merge_state on the FlashInfer backend page (flashinfer_backend.py, forward_extend):
//     lse = ln sum_i exp(lse_i),   o = sum_i exp(lse_i - lse) * o_i.
//
// Requests of 2 .. kFusedMergeMaxPieces pieces are merged inside the attention kernel, by the
// piece that arrives last (merge_rows_cta_bulk, or folded into that piece's own epilogue); the
// merge kernel takes requests of more pieces, a warp per 64-column slice of a query row: it reads
// the pieces' lse values once, then streams the pieces' columns of its slice (2 per lane; 32
// pieces' loads in flight at once, read once, evict-first) and writes bf16.
#pragma once
#include "ptx.cuh"

namespace mla {

constexpr int kCombineWarps = 8;
// Requests of 2 .. kFusedMergeMaxPieces pieces are merged inside the attention kernel by the
// CTA whose piece arrives last; the merge kernel serves requests of more pieces.
constexpr int kFusedMergeMaxPieces = 4;

// The merge kernel's unit of work: one 64-column slice of one query row, a warp, lane l holding
// columns 64 slice + 2l, + 1.  A row's eight slices go to eight warps, so that a request of many
// pieces (a long request split over every part) spreads over the whole grid: a warp per row left
// its 128 rows to 16 of the 148 SMs, each warp streaming ~70 pieces x 2 KB in turn.
constexpr int kMergeSliceCols = 64;
constexpr int kMergeSlices = 512 / kMergeSliceCols;
constexpr int kMergeRegPieces = 128;   // pieces whose lse values stay in registers (4 per lane)

// Merge the n partial states (o_i, lse_i) of one query row (pieces s0 .. s0 + n - 1 of the
// split slots) into bf16 o, columns of `slice` only, and (slice 0) its lse.  Lane l reads the lse
// of pieces l + 32k once; piece i's weight exp(lse_i - lse) is computed by lane i % 32 and
// shuffled to the others.  The pieces go in rounds of 32 with all their loads in flight, and each
// column sums w_i o_i in piece order.  The partials were written by an earlier grid, so the
// read-only path serves them.
__device__ __forceinline__ void merge_row_slice(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                                int s0, int n, int rows, int row, int slice,
                                                __nv_bfloat16* __restrict__ out_row, float* __restrict__ lse_out,
                                                int lane, uint64_t read_pol) {
    auto load_lse = [&](int i) -> float {
        const float* ptr = part_lse + (int64_t)(s0 + i) * rows + row;
        return *ptr;
    };
    const int col = kMergeSliceCols * slice + 2 * lane;
    float lr[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) lr[k] = lane + 32 * k < n ? load_lse(lane + 32 * k) : -INFINITY;
    float m = fmaxf(fmaxf(lr[0], lr[1]), fmaxf(lr[2], lr[3]));
    for (int i = lane + kMergeRegPieces; i < n; i += 32) m = fmaxf(m, load_lse(i));
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (m == -INFINITY) {
        reinterpret_cast<uint32_t*>(out_row)[col >> 1] = 0u;
        if (slice == 0 && lane == 0) *lse_out = -INFINITY;
        return;
    }
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (lane + 32 * k < n) sum += expf(lr[k] - m);
    for (int i = lane + kMergeRegPieces; i < n; i += 32) sum += expf(load_lse(i) - m);
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float lse = m + logf(sum);
    float a0 = 0.f, a1 = 0.f;
    // pieces c0 .. c0 + 31, lane l holding the weight of piece c0 + l
    auto merge_round = [&](int c0, float wl) {
        float2 v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
            v[j] = c0 + j < n ? ld_global_nc_v2_hint(reinterpret_cast<const float2*>(
                                    part_o + ((int64_t)(s0 + c0 + j) * rows + row) * 512 + col), read_pol)
                              : make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const float w = __shfl_sync(0xffffffffu, wl, j);
            a0 += w * v[j].x;
            a1 += w * v[j].y;
        }
    };
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (32 * k < n) merge_round(32 * k, lane + 32 * k < n ? expf(lr[k] - lse) : 0.f);
    for (int c0 = kMergeRegPieces; c0 < n; c0 += 32)
        merge_round(c0, c0 + lane < n ? expf(load_lse(c0 + lane) - lse) : 0.f);
    reinterpret_cast<uint32_t*>(out_row)[col >> 1] = pack_bf16x2(a0, a1);
    if (slice == 0 && lane == 0) *lse_out = lse;
}

// Merge, with a whole CTA of kThreadsCta threads whose shared memory is idle, the n (2 ..
// kFusedMergeMaxPieces) pieces' partial states of nrows <= 64 consecutive query rows
// (row_base ..) of one request.  A piece's rows are contiguous, so each pass brings in, for every
// piece, as many consecutive rows as fit into `stage` (stage_bytes of shared memory) with one
// bulk copy per piece: a bulk copy costs the TMA unit ~70 cycles whatever its size, which made
// one copy per 2 KB row slower than the rows' transfer.  The first pass's copies are issued before
// the pieces' log-sum-exps are read, so that the two overlap.  `bar` is an mbarrier of count 1
// whose phase advances once per pass (`phase` counts the passes run on it), `wait` a bounded wait
// on it; scratch: 256 floats.  Returns false if a wait gave up.
template <int kThreadsCta, typename WaitFn>
__device__ __forceinline__ bool merge_rows_cta_bulk(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                                    int s0, int n, int rows, int row_base, int nrows,
                                                    __nv_bfloat16* __restrict__ out_base, float* __restrict__ lse_base,
                                                    float* scratch, uint32_t stage, uint32_t stage_bytes, uint32_t bar,
                                                    uint32_t& phase, WaitFn wait, int tid) {
    constexpr int kRowBytes = 512 * 4;
    int per_pass = (int)(stage_bytes / (uint32_t)(n * kRowBytes));
    if (per_pass > nrows) per_pass = nrows;
    auto issue = [&](int r0) {
        const int R = min(per_pass, nrows - r0);
        if (tid == 0) mbar_arrive_expect_tx(bar, (uint32_t)(R * n * kRowBytes));
        if (tid < n) {
            fence_proxy_async_global();   // the partials were written by other CTAs' generic stores
            bulk_load(stage + (uint32_t)(tid * R) * kRowBytes,
                      part_o + ((int64_t)(s0 + tid) * rows + row_base + r0) * 512, (uint32_t)(R * kRowBytes), bar);
        }
    };
    issue(0);
    float* w = scratch;             // [4][64]: the pieces' lse, then their weights
    if (tid < 64 * n) {
        const int r = tid & 63, i = tid >> 6;
        w[i * 64 + r] = r < nrows ? __ldcg(part_lse + (int64_t)(s0 + i) * rows + row_base + r) : -INFINITY;
    }
    __syncthreads();
    if (tid < nrows) {
        float m = -INFINITY;
        for (int i = 0; i < n; ++i) m = fmaxf(m, w[i * 64 + tid]);
        float lse = -INFINITY;
        if (m == -INFINITY) {
            for (int i = 0; i < n; ++i) w[i * 64 + tid] = 0.f;   // no key in any piece: o = 0
        } else {
            float sum = 0.f;
            for (int i = 0; i < n; ++i) sum += expf(w[i * 64 + tid] - m);
            lse = m + logf(sum);
            for (int i = 0; i < n; ++i) w[i * 64 + tid] = expf(w[i * 64 + tid] - lse);
        }
        lse_base[tid] = lse;
    }
    __syncthreads();
    for (int r0 = 0; r0 < nrows; r0 += per_pass) {
        const int R = min(per_pass, nrows - r0);
        if (r0 > 0) {
            __syncthreads();   // the previous pass has read the stage
            issue(r0);
        }
        const bool ok = wait(bar, phase & 1u);
        ++phase;
        if (!ok) return false;
        // one 16-byte column group of one row per thread and step: row r, columns 4q .. 4q + 3
        for (int x = tid; x < R * 128; x += kThreadsCta) {
            const int r = x >> 7, q = x & 127;
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int i = 0; i < n; ++i) {
                const float wi = w[i * 64 + r0 + r];
                const float4 v = ld_shared_v4f(stage + (uint32_t)(i * R + r) * kRowBytes + 16u * (uint32_t)q);
                a.x += wi * v.x;
                a.y += wi * v.y;
                a.z += wi * v.z;
                a.w += wi * v.w;
            }
            reinterpret_cast<uint2*>(out_base + (int64_t)(r0 + r) * 512)[q] =
                make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
        }
    }
    return true;
}

// The rows of requests of more than kFusedMergeMaxPieces pieces (the others were written whole or
// merged by the attention kernel, so the launch needs no host knowledge of the plan): each CTA
// first stages num_splits in shared memory (one coalesced read, for up to kCombineStagedRequests
// requests) and notes whether any request has that many pieces, then waits for the attention
// grid; its warps then take (request, query row, column slice) units in turn, or the CTA returns
// at once when nothing is left to merge.  num_splits comes from the metadata step: the attention
// kernel lets this grid in only after its own wait for that step to complete, so num_splits is
// final and is read while the attention kernel still runs.
constexpr int kCombineStagedRequests = 4096;

__global__ void __launch_bounds__(kCombineWarps * 32)
combine_splits_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                      const int32_t* __restrict__ num_splits, int32_t rows, int32_t bs,
                      __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out) {
    __shared__ int32_t s_ns[kCombineStagedRequests + 1];
    const bool staged = bs <= kCombineStagedRequests;
    int many = 0;   // some request of this thread's has more pieces than the attention kernel merges
    if (staged) {
        for (int b = threadIdx.x; b <= bs; b += blockDim.x) s_ns[b] = num_splits[b];
        __syncthreads();
        for (int b = threadIdx.x; b < bs; b += blockDim.x) many |= s_ns[b + 1] - s_ns[b] > kFusedMergeMaxPieces;
    } else {
        for (int b = threadIdx.x; b < bs; b += blockDim.x)
            many |= num_splits[b + 1] - num_splits[b] > kFusedMergeMaxPieces;
    }
    many = __syncthreads_or(many);
    // launched as a programmatic dependent of the attention kernel: wait for all of it (also when
    // there is nothing to merge, so that this grid never completes before the one it follows)
    pdl_wait_prerequisites();
    if (!many) return;
    const uint64_t read_pol = l2_policy_evict_first();   // the partials are read once
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * kCombineWarps;
    const int64_t per_req = (int64_t)rows * kMergeSlices;
    const int64_t total = (int64_t)bs * per_req;
    for (int64_t idx = (int64_t)blockIdx.x * kCombineWarps + (threadIdx.x >> 5); idx < total; idx += warps) {
        const int b = (int)(idx / per_req);
        const int rs = (int)(idx - (int64_t)b * per_req);
        const int row = rs / kMergeSlices, slice = rs - row * kMergeSlices;
        const int s0 = staged ? s_ns[b] : num_splits[b];
        const int n = (staged ? s_ns[b + 1] : num_splits[b + 1]) - s0;
        if (n <= kFusedMergeMaxPieces) continue;
        const int64_t out_row = (int64_t)b * rows + row;
        merge_row_slice(part_o, part_lse, s0, n, rows, row, slice, out + out_row * 512, lse_out + out_row, lane,
                        read_pol);
    }
}

}  // namespace mla
