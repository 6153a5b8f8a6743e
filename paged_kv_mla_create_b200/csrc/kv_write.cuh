// KV-cache write in the role of token_to_kv_pool.set_kv_buffer(layer, cache_loc, k, v) as the
// SGLang FlashMLA backend page (flashmla_backend.py, forward_decode / forward_extend) calls it
// before attention: each new token's 576-wide latent row (kv_lora_rank 512 + rope 64; in MLA the
// value is the row's first 512 columns, so only k is stored) goes to pool row cache_loc[i].  A
// bf16 pool stores the row as it is; an fp8 pool (float8_e4m3fn or float8_e5m2, the two the
// page's __init__ accepts) stores k / k_scale rounded to nearest even, saturated to the format's
// largest finite value.
//
// One warp per token: 72 sixteen-byte units of bf16 in, 72 units out (bf16) or 72 eight-byte
// units (fp8); the division is IEEE single precision, correctly rounded.
#pragma once
#include "ptx.cuh"

namespace mla {

constexpr int kKvWriteWarps = 8;

// Eight floats -> eight codes of the 8-bit format (first value in the lowest byte).
template <int kFmt>
__device__ __forceinline__ uint2 floats_to_fp8x8(const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint16_t h;
        if constexpr (kFmt == 1)
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(f[2 * i + 1]), "f"(f[2 * i]));
        else
            asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(h) : "f"(f[2 * i + 1]), "f"(f[2 * i]));
        w[i] = h;
    }
    return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

template <int kFmt, typename LocT>
__global__ void __launch_bounds__(kKvWriteWarps * 32)
set_kv_buffer_kernel(uint8_t* __restrict__ pool, int64_t num_slots, const LocT* __restrict__ cache_loc,
                     int32_t n_tokens, const __nv_bfloat16* __restrict__ k, int64_t k_stride,
                     const float* __restrict__ k_scale) {
    constexpr int kDim = 576;
    constexpr int kUnits = kDim / 8;   // eight values per unit
    const int token = blockIdx.x * kKvWriteWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (token >= n_tokens) return;
    const int64_t slot = static_cast<int64_t>(cache_loc[token]);
    if (slot < 0 || slot >= num_slots) {
        if (lane == 0) raise_error(256 /* MLA_DEVERR_SLOT_OUT_OF_RANGE */);
        return;
    }
    const uint4* src = reinterpret_cast<const uint4*>(k + token * k_stride);
    if constexpr (kFmt == 0) {
        uint4* dst = reinterpret_cast<uint4*>(pool + slot * (2 * kDim));
        for (int u = lane; u < kUnits; u += 32) dst[u] = __ldg(src + u);
    } else {
        const float s = k_scale ? *k_scale : 1.0f;
        const bool scaled = k_scale != nullptr;
        uint2* dst = reinterpret_cast<uint2*>(pool + slot * kDim);
        for (int u = lane; u < kUnits; u += 32) {
            const uint4 v = __ldg(src + u);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            float f[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                f[2 * i] = __uint_as_float(w[i] << 16);
                f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            }
            if (scaled) {
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = __fdiv_rn(f[i], s);
            }
            dst[u] = floats_to_fp8x8<kFmt>(f);
        }
    }
}

}  // namespace mla
