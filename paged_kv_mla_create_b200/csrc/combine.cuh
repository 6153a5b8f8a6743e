// Log-sum-exp merge of split-KV partial results: the step implied by get_mla_metadata's
// num_splits in the SGLang FlashMLA backend page (flashmla_backend.py) and written out
// as merge_state on the FlashInfer backend page (flashinfer_backend.py, forward_extend):
//     lse = ln sum_i exp(lse_i),   o = sum_i exp(lse_i - lse) * o_i.
//
// A warp merges one query row: it reads the pieces' lse values, then streams the pieces'
// 512 fp32 columns (16 per lane, as 4 float4; four pieces' loads in flight at once) and
// writes bf16; the pieces' rows, kept in L2 by the attention kernel's stores, are then
// dropped from L2 without a write-back (requests of up to kDiscardMaxPieces pieces).
// Requests of 2 .. kFusedMergeMaxPieces pieces are merged that way inside the attention
// kernel by the CTA whose piece arrives last; the merge kernel takes the rest.
#pragma once
#include "ptx.cuh"

namespace mla {

constexpr int kCombineWarps = 8;
constexpr int kDiscardMaxPieces = 4;   // requests of up to this many pieces drop their rows from L2
// Requests of 2 .. kFusedMergeMaxPieces pieces are merged inside the attention kernel by the
// CTA whose piece arrives last; the merge kernel serves requests of more pieces.
constexpr int kFusedMergeMaxPieces = 4;

// Merge the n partial states (o_i, lse_i) of one query row (pieces s0 .. s0 + n - 1 of the
// split slots) into bf16 o and its lse; one warp, lane l holding columns 4l + 128k + [0, 4).
// kCoherent reads through L2 only (the partials were written by other CTAs of the same
// kernel); otherwise through the read-only path with the given L2 policy.
template <bool kCoherent>
__device__ __forceinline__ void merge_row(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                          int s0, int n, int rows, int row, __nv_bfloat16* __restrict__ out_row,
                                          float* __restrict__ lse_out, int lane, uint64_t read_pol) {
    auto load_lse = [&](int i) -> float {
        const float* ptr = part_lse + (int64_t)(s0 + i) * rows + row;
        return kCoherent ? __ldcg(ptr) : *ptr;
    };
    float m = -INFINITY;
    for (int i = lane; i < n; i += 32) m = fmaxf(m, load_lse(i));
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (m == -INFINITY) {
        for (int c = lane; c < 64; c += 32) reinterpret_cast<uint4*>(out_row)[c] = make_uint4(0, 0, 0, 0);
        if (lane == 0) *lse_out = -INFINITY;
        return;
    }
    float sum = 0.f;
    for (int i = lane; i < n; i += 32) sum += expf(load_lse(i) - m);
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float lse = m + logf(sum);
    // A request of few pieces drops its rows' L2 lines once merged (they need no write-back);
    // the loads of a many-piece request (a long serial loop here) only lower their L2
    // priority, which measured faster than dropping each line.
    const bool discard = n <= kDiscardMaxPieces;
    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = 0.f;
    // pieces four at a time, all of their loads in flight before any is used
    for (int i0 = 0; i0 < n; i0 += 4) {
        float4 v[4][4];
        float w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j;
            w[j] = 0.f;
            if (i < n) {
                w[j] = expf(load_lse(i) - lse);
                const float4* src = reinterpret_cast<const float4*>(part_o + ((int64_t)(s0 + i) * rows + row) * 512);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    v[j][k] = kCoherent ? __ldcg(src + lane + 32 * k)
                                        : (discard ? __ldg(src + lane + 32 * k)
                                                   : ld_global_nc_v4_hint(src + lane + 32 * k, read_pol));
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) v[j][k] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                acc[4 * k + 0] += w[j] * v[j][k].x;
                acc[4 * k + 1] += w[j] * v[j][k].y;
                acc[4 * k + 2] += w[j] * v[j][k].z;
                acc[4 * k + 3] += w[j] * v[j][k].w;
            }
        if (discard) {
            // every lane's loads have returned (consumed above): the pieces' rows are dead, so
            // their L2 lines go without a write-back (lane l < 16 takes line l of a 2 KB row)
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (i0 + j < n && lane < 16)
                    discard_l2_line(part_o + ((int64_t)(s0 + i0 + j) * rows + row) * 512 + 32 * lane);
        }
    }
    uint2* dst = reinterpret_cast<uint2*>(out_row);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        dst[lane + 32 * k] = make_uint2(pack_bf16x2(acc[4 * k], acc[4 * k + 1]),
                                        pack_bf16x2(acc[4 * k + 2], acc[4 * k + 3]));
    if (lane == 0) *lse_out = lse;
}

// Streams the N pieces' partial rows of one CTA's query rows and writes bf16 o: thread t
// takes float4 column t % 128 of rows t / 128 + kGroups j, R rows at a time with all R x N
// loads in flight (24 float4 per thread).  w: per-piece weights [N][64] in shared memory.
template <int N, int kThreadsCta>
__device__ __forceinline__ void merge_rows_stream(const float* __restrict__ part_o, const float* w, int s0,
                                                  int rows, int row_base, int nrows,
                                                  __nv_bfloat16* __restrict__ out_base, int tid) {
    constexpr int kGroups = kThreadsCta / 128;
    constexpr int R = 24 / N;
    const int q = tid & 127, g = tid / 128;
    if (g >= kGroups) return;
    for (int r0 = g; r0 < nrows; r0 += kGroups * R) {
        float4 v[R][N];
#pragma unroll
        for (int b = 0; b < R; ++b) {
            const int r = r0 + kGroups * b;
#pragma unroll
            for (int i = 0; i < N; ++i)
                v[b][i] = r < nrows ? __ldcg(reinterpret_cast<const float4*>(
                                          part_o + ((int64_t)(s0 + i) * rows + row_base + r) * 512) + q)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int b = 0; b < R; ++b) {
            const int r = r0 + kGroups * b;
            if (r < nrows) {
                float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int i = 0; i < N; ++i) {
                    const float wi = w[i * 64 + r];
                    a.x += wi * v[b][i].x;
                    a.y += wi * v[b][i].y;
                    a.z += wi * v[b][i].z;
                    a.w += wi * v[b][i].w;
                }
                reinterpret_cast<uint2*>(out_base + (int64_t)r * 512)[q] =
                    make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
            }
        }
    }
}

// Merge, with a whole CTA of kThreadsCta threads (a multiple of 128), the n (2 ..
// kFusedMergeMaxPieces) pieces' partial states of nrows <= 64 consecutive query rows
// (row_base ..) of one request: the pieces' log-sum-exps first (one load per piece and
// row, all in flight), then the weights and each row's lse, then the rows streamed with
// many loads in flight, then their L2 lines dropped (dead, no write-back).  scratch: 320
// floats of shared memory.  The partials were written by other CTAs of the same kernel, so
// every read goes through L2 only.
template <int kThreadsCta>
__device__ __forceinline__ void merge_rows_cta(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                               int s0, int n, int rows, int row_base, int nrows,
                                               __nv_bfloat16* __restrict__ out_base, float* __restrict__ lse_base,
                                               float* scratch, int tid) {
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
    if (n == 2)
        merge_rows_stream<2, kThreadsCta>(part_o, w, s0, rows, row_base, nrows, out_base, tid);
    else if (n == 3)
        merge_rows_stream<3, kThreadsCta>(part_o, w, s0, rows, row_base, nrows, out_base, tid);
    else
        merge_rows_stream<4, kThreadsCta>(part_o, w, s0, rows, row_base, nrows, out_base, tid);
    __syncthreads();
    // every partial line of these rows has been read: drop them without a write-back
    for (int i = 0; i < n; ++i)
        for (int l = tid; l < nrows * 16; l += kThreadsCta)
            discard_l2_line(part_o + ((int64_t)(s0 + i) * rows + row_base + l / 16) * 512 + (l % 16) * 32);
}

// One warp per (request, query row), for requests of more than kFusedMergeMaxPieces pieces;
// the others were written whole or merged by the attention kernel, so the launch needs no
// host knowledge of the plan.
__global__ void __launch_bounds__(kCombineWarps * 32)
combine_splits_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                      const int32_t* __restrict__ num_splits, int32_t rows,
                      __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out) {
    // launched as a programmatic dependent of the attention kernel: wait for all of it
    pdl_wait_prerequisites();
    const uint64_t read_pol = l2_policy_evict_first();   // the partials are read once
    const int b = blockIdx.y;
    const int row = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const int s0 = num_splits[b];
    const int n = num_splits[b + 1] - s0;
    if (n <= kFusedMergeMaxPieces) return;
    const int64_t out_row = (int64_t)b * rows + row;
    merge_row<false>(part_o, part_lse, s0, n, rows, row, out + out_row * 512, lse_out + out_row, lane, read_pol);
}

}  // namespace mla
