// Extend (prefill with a cached prefix) as the FlashInfer backend page writes it
// (flashinfer_backend.py, forward_extend): the new tokens' queries attend the new tokens
// themselves, causally (prefill_wrapper_ragged.forward_return_lse -> o1, s1), and the cached
// prefix, all of it (prefill_wrapper_paged.forward_return_lse -> o2, s2); the two partial
// results are merged by merge_state(o1, s1, o2, s2).  For MLA the keys are the 576-wide latent
// rows and the values their first 512 columns.  Both attention parts run on the paged decode
// kernel; this file holds the two small kernels around it: the view that presents the new
// tokens' rows as a paged pool, and merge_state.
#pragma once
#include "ptx.cuh"

namespace mla {

constexpr int kExtendThreads = 256;
constexpr int kMergeStateWarps = 8;

// Request b's new rows k_new[b, 0 .. e) (576 bf16 each) as a paged pool: pool rows
// b * e_pad + [0, e), e_pad = 64 * cdiv(e, 64), so that page j of request b is
// b * (e_pad / 64) + j.  `pool` is null when the caller's rows already have that layout
// (e == e_pad): only the page table and the lengths are written then.
__global__ void __launch_bounds__(kExtendThreads)
extend_ragged_view_kernel(const uint4* __restrict__ k_new, int32_t bs, int32_t e, int32_t e_pad,
                          uint4* __restrict__ pool, int32_t* __restrict__ block_table,
                          int32_t* __restrict__ cache_seqlens) {
    constexpr int kUnits = 576 * 2 / 16;   // 16-byte units of a row
    const int pages = e_pad / 64;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = tid; i < (int64_t)bs * pages; i += stride) block_table[i] = (int32_t)i;
    for (int64_t i = tid; i < bs; i += stride) cache_seqlens[i] = e;
    if (pool) {
        const int64_t units = (int64_t)bs * e * kUnits;
        for (int64_t u = tid; u < units; u += stride) {
            const int64_t row = u / kUnits;               // b * e + i
            const int64_t b = row / e, i = row - b * e;
            pool[(b * e_pad + i) * kUnits + (u - row * kUnits)] = __ldg(k_new + u);
        }
    }
}

// merge_state: per row, lse = ln(exp(lse_a) + exp(lse_b)) and
// o = exp(lse_a - lse) o_a + exp(lse_b - lse) o_b, bf16 o of 512 columns, fp32 natural-log lse
// (-inf for a part with no key; a row with no key in either part gets o = 0, lse = -inf).
// One warp per row, lane l holding columns 8l + 256k + [0, 8).
__global__ void __launch_bounds__(kMergeStateWarps * 32)
merge_state_kernel(const __nv_bfloat16* __restrict__ o_a, const float* __restrict__ lse_a,
                   const __nv_bfloat16* __restrict__ o_b, const float* __restrict__ lse_b, int64_t rows,
                   __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
    const int64_t row = (int64_t)blockIdx.x * kMergeStateWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float la = lse_a[row], lb = lse_b[row];
    const float m = fmaxf(la, lb);
    uint4* dst = reinterpret_cast<uint4*>(o + row * 512);
    if (m == -INFINITY) {
        dst[lane] = make_uint4(0, 0, 0, 0);
        dst[lane + 32] = make_uint4(0, 0, 0, 0);
        if (lane == 0) lse[row] = -INFINITY;
        return;
    }
    const float wa0 = expf(la - m), wb0 = expf(lb - m);
    const float sum = wa0 + wb0;
    const float wa = wa0 / sum, wb = wb0 / sum;
    const uint4* sa = reinterpret_cast<const uint4*>(o_a + row * 512);
    const uint4* sb = reinterpret_cast<const uint4*>(o_b + row * 512);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint4 a = __ldg(sa + lane + 32 * k), b = __ldg(sb + lane + 32 * k);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
        uint32_t r[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float lo = __uint_as_float(aw[j] << 16) * wa + __uint_as_float(bw[j] << 16) * wb;
            const float hi = __uint_as_float(aw[j] & 0xFFFF0000u) * wa + __uint_as_float(bw[j] & 0xFFFF0000u) * wb;
            r[j] = pack_bf16x2(lo, hi);
        }
        dst[lane + 32 * k] = make_uint4(r[0], r[1], r[2], r[3]);
    }
    if (lane == 0) lse[row] = m + logf(sum);
}

}  // namespace mla
