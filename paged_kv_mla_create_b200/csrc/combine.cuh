// Log-sum-exp merge of split-KV partial results: the step implied by get_mla_metadata's
// num_splits in the SGLang FlashMLA backend page (flashmla_backend.py) and written out
// as merge_state on the FlashInfer backend page (flashinfer_backend.py, forward_extend):
//     lse = ln sum_i exp(lse_i),   o = sum_i exp(lse_i - lse) * o_i.
//
// One warp per (request, query row).  Requests with a single piece were written
// directly by the attention kernel and are skipped here, so the launch needs no host
// knowledge of the plan.  A warp reads its pieces' lse values, then streams the
// pieces' 512 fp32 columns (16 per lane, as 4 float4; four pieces' loads in flight at once)
// and writes bf16; the pieces' rows, kept in L2 by the attention kernel's stores, are then
// dropped from L2 without a write-back (requests of up to kDiscardMaxPieces pieces).
#pragma once
#include "ptx.cuh"

namespace mla {

constexpr int kCombineWarps = 8;
constexpr int kDiscardMaxPieces = 4;   // requests of up to this many pieces drop their rows from L2

__global__ void __launch_bounds__(kCombineWarps * 32)
combine_splits_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                      const int32_t* __restrict__ num_splits, int32_t rows,
                      __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out) {
    const uint64_t read_pol = l2_policy_evict_first();   // the partials are read once
    const int b = blockIdx.y;
    const int row = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const int s0 = num_splits[b];
    const int n = num_splits[b + 1] - s0;
    if (n <= 1) return;
    float m = -INFINITY;
    for (int i = lane; i < n; i += 32) m = fmaxf(m, part_lse[(int64_t)(s0 + i) * rows + row]);
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const int64_t out_row = (int64_t)b * rows + row;
    if (m == -INFINITY) {
        for (int c = lane; c < 64; c += 32)
            reinterpret_cast<uint4*>(out + out_row * 512)[c] = make_uint4(0, 0, 0, 0);
        if (lane == 0) lse_out[out_row] = -INFINITY;
        return;
    }
    float sum = 0.f;
    for (int i = lane; i < n; i += 32) sum += expf(part_lse[(int64_t)(s0 + i) * rows + row] - m);
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
                w[j] = expf(part_lse[(int64_t)(s0 + i) * rows + row] - lse);
                const float4* src = reinterpret_cast<const float4*>(part_o + ((int64_t)(s0 + i) * rows + row) * 512);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    v[j][k] = discard ? __ldg(src + lane + 32 * k) : ld_global_nc_v4_hint(src + lane + 32 * k, read_pol);
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
    uint2* dst = reinterpret_cast<uint2*>(out + out_row * 512);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        dst[lane + 32 * k] = make_uint2(pack_bf16x2(acc[4 * k], acc[4 * k + 1]),
                                        pack_bf16x2(acc[4 * k + 2], acc[4 * k + 3]));
    if (lane == 0) lse_out[out_row] = lse;
}

}  // namespace mla
