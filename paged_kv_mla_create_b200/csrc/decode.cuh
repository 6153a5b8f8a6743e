// Paged MLA decode attention for sm_100a, in the role of flash_mla_with_kvcache as the
// SGLang FlashMLA backend page (flashmla_backend.py, forward_decode / forward_extend)
// calls it: q [bs, q_len, h_q, 576] against the latent cache viewed [-1, 64, 1, 576],
// head_dim_v = kv_lora_rank = 512, softmax_scale, causal, fp8 descales; output o and lse.
//
// Design (one 2-CTA cluster per scheduler part and 128-row query tile):
//   * The 128 query rows of a tile (q_len * h_q flattened, heads fastest) share every KV
//     tile, so QK^T and PV are dense tensor-core contractions: M = 128 rows, N = 64 tokens
//     for S = Q K^T, and M = 128, N = 256 output columns for O = P V.
//   * The fp32 accumulator of O (128 x 512) would fill all of one SM's tensor memory, so
//     the pair splits it: CTA r owns output columns [256r, 256r + 256).  Each CTA also owns
//     half of the 576 reduction columns of S (r = 0: 0..287, r = 1: 288..575) and computes a
//     partial S with its half of Q held in tensor memory; the two partials are exchanged
//     through distributed shared memory and summed (fp32 addition is commutative, so both
//     CTAs hold bit-identical S and take identical softmax decisions).  KV bytes are read
//     from HBM once: CTA r loads columns [256r, 256r + 320) of each page (the 64 shared
//     columns come from L2 for the second CTA).
//   * Tensor memory per CTA: O half (256 cols), Q half (144 cols, bf16 pairs), S (64),
//     P (32, bf16 pairs) = 496 of 512 columns.
//   * Roles: warp 0 issues TMA page loads (one 64-row tile per page, five 64-column boxes
//     with 128-byte swizzle) through the block table into a 4-stage ring; warp 1 issues the
//     tcgen05 MMAs from one thread; warps 4..7 (one thread per query row = TMEM lane) load
//     Q into tensor memory, run the online softmax with a conditional rescale of O, write
//     P into tensor memory, and run the epilogue.
//   * A unit whose block range is a whole request writes bf16 o and lse directly; a split
//     piece writes fp32 partials that combine_splits_kernel merges.
//   * Every wait is bounded (see mbar_wait_bounded); out-of-range page ids never fault:
//     the TMA reads zeros for out-of-range coordinates and the error word records it.
#pragma once
#include "ptx.cuh"

namespace mla {
namespace decode {

constexpr int kRows = 128;                 // query rows per tile (TMEM lanes)
constexpr int kBlock = 64;                 // tokens per KV tile = one page
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kHalfK = 288;                // reduction columns of S per CTA
constexpr int kHalfV = 256;                // output columns per CTA
constexpr int kQkSteps = kHalfK / 16;      // 18 MMAs of K = 16 per S tile
constexpr int kPvSteps = kBlock / 16;      // 4 MMAs of K = 16 per PV tile
constexpr int kBoxCols = 64;               // bf16 columns per 128-byte swizzle box
constexpr int kBoxes = 5;                  // 320 columns per CTA, from column 256 * rank
constexpr int kBoxBytes = kBlock * 128;    // 8 KB
constexpr int kStageBytes = kBoxes * kBoxBytes;  // 40 KB
constexpr int kStages = 4;
constexpr int kXbufBytes = kRows * kBlock * 4;   // one fp32 partial S tile (32 KB)
constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may reach 2^8 before O is rescaled

// Tensor-memory column map (512 columns allocated).
constexpr uint32_t kTmemO = 0;
constexpr uint32_t kTmemQ = 256;
constexpr uint32_t kTmemS = 400;
constexpr uint32_t kTmemP = 464;
constexpr uint32_t kTmemCols = 512;

// Barrier slots (8 bytes each) after the exchange buffer.
enum : int {
    kBarKvFull = 0,
    kBarKvEmpty = kBarKvFull + kStages,
    kBarQFull = kBarKvEmpty + kStages,
    kBarQEmpty,
    kBarSFull,
    kBarSFree,
    kBarPFull,
    kBarPvDone,
    kBarOFull,
    kBarOEmpty,
    kBarXFull,
    kBarXEmpty,
    kNumBars
};

constexpr int kSmemBytes = kStages * kStageBytes + kXbufBytes + kNumBars * 8 + 16 + 1024;

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, false, true);

struct Params {
    const __nv_bfloat16* q;        // [bs, rows, 576]
    const uint8_t* kv_fp8;         // [num_pages * 64, 576] e4m3 (fp8 path only)
    const int32_t* block_table;    // [bs, bt_stride]
    int64_t bt_stride;
    int32_t max_pages;
    const int32_t* cache_seqlens;  // [bs]
    const int32_t* md;             // [num_parts, 8]
    const int32_t* num_splits;     // [bs + 1]
    int32_t bs, q_len, h_q, rows;
    int64_t num_pages;
    float scale_log2;              // softmax_scale * log2(e)
    const float* descale_q;        // nullable
    const float* descale_k;        // nullable
    int32_t causal;
    __nv_bfloat16* out;            // [bs, rows, 512]
    float* lse;                    // [bs, rows]
    float* part_o;                 // [splits, rows, 512]
    float* part_lse;               // [splits, rows]
};

// The work units of a part, identical in every role: request b, block range [kb0, kb1).
struct UnitIter {
    int b, b1, k0, k1, bs;
    const int32_t* seqlens;
    int max_pages;
    __device__ bool next(int& ub, int& kb0, int& kb1) {
        while (b <= b1 && b < bs) {
            if (b == b1 && k1 == 0) return false;
            int L = seqlens[b];
            int nb = L > 0 ? (L + kBlock - 1) / kBlock : 0;
            if (nb > max_pages) nb = max_pages;
            int lo = (b == first_b) ? k0 : 0;
            int hi = (b == b1) ? k1 : nb;
            if (hi > nb) hi = nb;
            if (lo > hi) lo = hi;
            ub = b;
            kb0 = lo;
            kb1 = hi;
            ++b;
            return true;
        }
        return false;
    }
    int first_b;
};

__device__ __forceinline__ UnitIter make_iter(const Params& p, int part, bool& ok) {
    const int4 r0 = *reinterpret_cast<const int4*>(p.md + 8 * (int64_t)part);
    UnitIter it;
    it.b = r0.x;
    it.first_b = r0.x;
    it.k0 = r0.y;
    it.b1 = r0.z;
    it.k1 = r0.w;
    it.bs = p.bs;
    it.seqlens = p.cache_seqlens;
    it.max_pages = p.max_pages;
    ok = r0.x >= 0 && r0.x <= r0.z && r0.z <= p.bs && r0.y >= 0 && r0.w >= 0 &&
         !(r0.z == p.bs && r0.w != 0) && !(r0.x == r0.z && r0.y > r0.w);
    if (!ok) it.b = it.b1 + 1;  // no units
    return it;
}

// Descriptor of the K operand of S for k-step kk: columns 288 * rank + 16 * kk of the tile,
// inside the CTA's boxes that start at column 256 * rank.
__device__ __forceinline__ uint64_t k_desc(uint32_t stage_addr, uint32_t rank, int kk) {
    const uint32_t rel = 32u * rank + 16u * kk;
    const uint32_t addr = stage_addr + (rel >> 6) * kBoxBytes + (rel & 63u) * 2u;
    return smem_desc_sw128(addr, 16, 1024);
}

// Descriptor of the V operand for k-step kk (tokens 16kk .. 16kk + 15), N = 256 columns
// spanning boxes 0..3 (MN-major: 64-column groups 8 KB apart, 8-row groups 1 KB apart).
__device__ __forceinline__ uint64_t v_desc(uint32_t stage_addr, int kk) {
    return smem_desc_sw128(stage_addr + kk * 2048u, kBoxBytes, 1024);
}

template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t xbuf = sbase + kStages * kStageBytes;
    const uint32_t bars = xbuf + kXbufBytes;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kStages * kStageBytes + kXbufBytes +
                                                      kNumBars * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t peer = rank ^ 1u;
    const int part = blockIdx.x >> 1;
    const int mtile = blockIdx.y;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(kBarKvFull + s), 1);
            mbar_init(bar(kBarKvEmpty + s), 1);
        }
        mbar_init(bar(kBarQFull), 4);
        mbar_init(bar(kBarQEmpty), 1);
        mbar_init(bar(kBarSFull), 1);
        mbar_init(bar(kBarSFree), 4);
        mbar_init(bar(kBarPFull), 4);
        mbar_init(bar(kBarPvDone), 1);
        mbar_init(bar(kBarOFull), 1);
        mbar_init(bar(kBarOEmpty), 4);
        mbar_init(bar(kBarXFull), 4);
        mbar_init(bar(kBarXEmpty), 4);
        *abort_flag = 0;
        fence_mbarrier_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) prefetch_tensormap(&kv_map);
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool md_ok = true;
    UnitIter iter = make_iter(p, part, md_ok);
    if (!md_ok && threadIdx.x == 0) raise_error(8 /* MLA_DEVERR_BAD_METADATA */);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        uint32_t g = 0;
        int last_parity[kStages];
#pragma unroll
        for (int s = 0; s < kStages; ++s) last_parity[s] = -1;
        bool alive = true;
        int ub, kb0, kb1;
        const int32_t col0 = 256 * (int32_t)rank;
        while (alive && iter.next(ub, kb0, kb1)) {
            const int32_t* bt_row = p.block_table + (int64_t)ub * p.bt_stride;
            for (int base = kb0; alive && base < kb1; base += 32) {
                const int idx = base + lane;
                int pg = idx < kb1 ? __ldg(bt_row + idx) : 0;
                const bool bad = idx < kb1 && (pg < 0 || (int64_t)pg >= p.num_pages);
                if (__any_sync(0xffffffffu, bad) && lane == 0) raise_error(1);
                // An out-of-range page becomes a coordinate past the tensor: TMA fills zeros.
                const int32_t row_coord = bad ? (int32_t)(p.num_pages * kBlock) : pg * kBlock;
                const int cnt = min(32, kb1 - base);
                for (int j = 0; j < cnt; ++j) {
                    const int32_t rc = __shfl_sync(0xffffffffu, row_coord, j);
                    int ok = 1;
                    if (lane == 0) {
                        const int s = g % kStages;
                        const uint32_t ph = (g / kStages) & 1u;
                        ok = mbar_wait_bounded<false>(bar(kBarKvEmpty + s), ph ^ 1u, abort_flag);
                        if (ok) {
                            const uint32_t dst = sbase + s * kStageBytes;
                            mbar_arrive_expect_tx(bar(kBarKvFull + s), kStageBytes);
#pragma unroll
                            for (int bx = 0; bx < kBoxes; ++bx)
                                tma_load_2d(dst + bx * kBoxBytes, &kv_map, bar(kBarKvFull + s),
                                            col0 + bx * kBoxCols, rc);
                            last_parity[s] = (int)ph;
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) {
                        alive = false;
                        break;
                    }
                    ++g;
                }
            }
        }
        if (lane == 0 && *abort_flag) {
            // Let every copy this CTA issued land before shared memory goes away.
            for (int s = 0; s < kStages; ++s) {
                if (last_parity[s] < 0) continue;
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(bar(kBarKvFull + s), (uint32_t)last_parity[s]) &&
                       global_timer_ns() - t0 < 100000000ull) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t g = 0, uq = 0;
            int ub, kb0, kb1;
            bool alive = true;
            auto issue_pv = [&](uint32_t gg, bool first) -> bool {
                if (!mbar_wait_bounded<false>(bar(kBarPFull), gg & 1u, abort_flag)) return false;
                if (first && uq > 0 &&
                    !mbar_wait_bounded<false>(bar(kBarOEmpty), (uq - 1) & 1u, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t stage_addr = sbase + (gg % kStages) * kStageBytes;
#pragma unroll
                for (int kk = 0; kk < kPvSteps; ++kk)
                    mma_ts(tmem + kTmemO, tmem + kTmemP + 8u * kk, v_desc(stage_addr, kk),
                           kIdescPV, (first && kk == 0) ? 0u : 1u);
                tc_commit(bar(kBarKvEmpty + gg % kStages));
                tc_commit(bar(kBarPvDone));
                return true;
            };
            while (alive && iter.next(ub, kb0, kb1)) {
                const int n = kb1 - kb0;
                if (n <= 0) continue;
                if (!mbar_wait_bounded<false>(bar(kBarQFull), uq & 1u, abort_flag)) break;
                for (int t = 0; t < n; ++t) {
                    const int s = g % kStages;
                    if (!mbar_wait_bounded<false>(bar(kBarKvFull + s), (g / kStages) & 1u,
                                                  abort_flag) ||
                        (g > 0 && !mbar_wait_bounded<false>(bar(kBarSFree), (g - 1) & 1u,
                                                            abort_flag))) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t stage_addr = sbase + s * kStageBytes;
#pragma unroll
                    for (int kk = 0; kk < kQkSteps; ++kk)
                        mma_ts(tmem + kTmemS, tmem + kTmemQ + 8u * kk, k_desc(stage_addr, rank, kk),
                               kIdescQK, kk > 0 ? 1u : 0u);
                    tc_commit(bar(kBarSFull));
                    if (t == n - 1) tc_commit(bar(kBarQEmpty));
                    if (t > 0 && !issue_pv(g - 1, t == 1)) {
                        alive = false;
                        break;
                    }
                    ++g;
                }
                if (!alive || !issue_pv(g - 1, n == 1)) break;
                tc_commit(bar(kBarOFull));
                ++uq;
            }
        }
    } else if (warp >= kSoftmaxWarp0) {
        // ------------------------------------------------------------ softmax / epilogue
        const int r = threadIdx.x - kSoftmaxWarp0 * 32;           // query row in the tile
        const uint32_t lane_off = (uint32_t)((warp - kSoftmaxWarp0) * 32) << 16;
        const int rowg = mtile * kRows + r;
        const bool row_valid = rowg < p.rows;
        const int iq = row_valid ? rowg / p.h_q : 0;
        const float dq = p.descale_q ? *p.descale_q : 1.0f;
        const float dk = p.descale_k ? *p.descale_k : 1.0f;
        const float sl2 = p.scale_log2 * dq * dk;
        const uint32_t peer_xbuf = map_to_cta(xbuf, peer);
        const uint32_t peer_xfull = map_to_cta(bar(kBarXFull), peer);
        const uint32_t peer_xempty = map_to_cta(bar(kBarXEmpty), peer);
        const uint32_t my_row = xbuf + (uint32_t)r * 256u;
        const uint32_t peer_row = peer_xbuf + (uint32_t)r * 256u;
        const uint32_t swz = (uint32_t)(r & 7);

        auto load_q = [&](int b) {
            const uint4* src = reinterpret_cast<const uint4*>(
                p.q + ((int64_t)b * p.rows + (row_valid ? rowg : 0)) * kDqk + kHalfK * rank);
#pragma unroll
            for (int grp = 0; grp < 3; ++grp) {
                uint4 v[12];
#pragma unroll
                for (int k = 0; k < 12; ++k)
                    v[k] = row_valid ? __ldg(src + grp * 12 + k) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int c = 0; c < 3; ++c) {
                    uint32_t w[16];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        w[4 * k + 0] = v[4 * c + k].x;
                        w[4 * k + 1] = v[4 * c + k].y;
                        w[4 * k + 2] = v[4 * c + k].z;
                        w[4 * k + 3] = v[4 * c + k].w;
                    }
                    tmem_st16(tmem + lane_off + kTmemQ + 16u * (3 * grp + c), w);
                }
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarQFull));
        };

        auto write_empty = [&](int b) {
            // A request with no key: o = 0, lse = -inf (always a single, direct piece).
            if (!row_valid) return;
            uint4* dst = reinterpret_cast<uint4*>(p.out + ((int64_t)b * p.rows + rowg) * kDv +
                                                  kHalfV * rank);
            for (int c = 0; c < kHalfV / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
            if (rank == 0) p.lse[(int64_t)b * p.rows + rowg] = -INFINITY;
        };

        uint32_t g = 0, uq = 0;
        bool alive = true;
        int cb, ckb0, ckb1;  // current unit
        bool have = false;
        // first non-empty unit
        while (iter.next(cb, ckb0, ckb1)) {
            if (ckb1 > ckb0) {
                have = true;
                break;
            }
            write_empty(cb);
        }
        if (have) load_q(cb);
        while (have && alive) {
            const int L = p.cache_seqlens[cb];
            int lim = p.causal ? L - p.q_len + iq + 1 : L;
            if (lim > L) lim = L;
            float m_run = -INFINITY, l_run = 0.f;
            const int n = ckb1 - ckb0;
            for (int t = 0; t < n; ++t, ++g) {
                if (!mbar_wait_bounded<false>(bar(kBarSFull), g & 1u, abort_flag)) {
                    alive = false;
                    break;
                }
                tc_fence_after();
                float s[64];
                {
                    uint32_t raw[16];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        tmem_ld16(tmem + lane_off + kTmemS + 16u * c, raw);
                        tc_wait_ld();
#pragma unroll
                        for (int k = 0; k < 16; ++k) s[16 * c + k] = __uint_as_float(raw[k]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarSFree));
                // exchange partial S with the peer CTA
                if (!mbar_wait_bounded<false>(bar(kBarXEmpty), (g & 1u) ^ 1u, abort_flag)) {
                    alive = false;
                    break;
                }
#pragma unroll
                for (int v = 0; v < 16; ++v)
                    st_cluster_v4(peer_row + ((v ^ swz) << 4), s[4 * v], s[4 * v + 1], s[4 * v + 2],
                                  s[4 * v + 3]);
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(peer_xfull);
                if (!mbar_wait_bounded<true>(bar(kBarXFull), g & 1u, abort_flag)) {
                    alive = false;
                    break;
                }
#pragma unroll
                for (int v = 0; v < 16; ++v) {
                    const float4 o4 = ld_shared_v4(my_row + ((v ^ swz) << 4));
                    s[4 * v] += o4.x;
                    s[4 * v + 1] += o4.y;
                    s[4 * v + 2] += o4.z;
                    s[4 * v + 3] += o4.w;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(peer_xempty);
                // scale to log2 units, mask, running max
                const int kbase = (ckb0 + t) * kBlock;
                float tmax = -INFINITY;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    float x = s[j] * sl2;
                    if (kbase + j >= lim) x = -INFINITY;
                    s[j] = x;
                    tmax = fmaxf(tmax, x);
                }
                const float m_new = fmaxf(m_run, tmax);
                const bool rescale = m_new > m_run + kRescaleThreshold;
                float factor = 1.f;
                if (rescale) {
                    factor = fast_exp2(m_run - m_new);  // 0 when m_run = -inf
                    l_run *= factor;
                    m_run = m_new;
                }
                // P buffer reuse and O rescale both need the previous PV to have finished.
                if (g > 0 && !mbar_wait_bounded<false>(bar(kBarPvDone), (g - 1) & 1u, abort_flag)) {
                    alive = false;
                    break;
                }
                tc_fence_after();
                if (t > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                    for (int c = 0; c < kHalfV / 16; ++c) {
                        uint32_t raw[16];
                        tmem_ld16(tmem + lane_off + kTmemO + 16u * c, raw);
                        tc_wait_ld();
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            raw[k] = __float_as_uint(__uint_as_float(raw[k]) * factor);
                        tmem_st16(tmem + lane_off + kTmemO + 16u * c, raw);
                    }
                }
                const bool live = m_run != -INFINITY;
                float psum = 0.f;
                uint32_t pk[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float p0 = live ? fast_exp2(s[2 * j] - m_run) : 0.f;
                    const float p1 = live ? fast_exp2(s[2 * j + 1] - m_run) : 0.f;
                    psum += p0 + p1;
                    pk[j] = pack_bf16x2(p0, p1);
                }
                l_run += psum;
                {
                    uint32_t w[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) w[k] = pk[k];
                    tmem_st16(tmem + lane_off + kTmemP, w);
#pragma unroll
                    for (int k = 0; k < 16; ++k) w[k] = pk[16 + k];
                    tmem_st16(tmem + lane_off + kTmemP + 16u, w);
                }
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarPFull));
            }
            if (!alive) break;
            // next unit: load its Q as soon as this unit's last QK^T has completed
            int nb_, nkb0, nkb1;
            bool have_next = false;
            while (iter.next(nb_, nkb0, nkb1)) {
                if (nkb1 > nkb0) {
                    have_next = true;
                    break;
                }
                write_empty(nb_);
            }
            if (have_next) {
                if (!mbar_wait_bounded<false>(bar(kBarQEmpty), uq & 1u, abort_flag)) break;
                tc_fence_after();
                load_q(nb_);
            }
            // epilogue of the current unit
            if (!mbar_wait_bounded<false>(bar(kBarOFull), uq & 1u, abort_flag)) break;
            tc_fence_after();
            const int pieces = p.num_splits[cb + 1] - p.num_splits[cb];
            const bool direct = pieces == 1;
            const int split = p.num_splits[cb] + (cb == iter.first_b ? p.md[8 * part + 4] : 0);
            const float inv = l_run > 0.f ? dk / l_run : 0.f;
            const float lse_val = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f
                                              : -INFINITY;
#pragma unroll 1
            for (int c = 0; c < kHalfV / 16; ++c) {
                uint32_t raw[16];
                tmem_ld16(tmem + lane_off + kTmemO + 16u * c, raw);
                tc_wait_ld();
                if (row_valid) {
                    if (direct) {
                        uint4* dst = reinterpret_cast<uint4*>(
                            p.out + ((int64_t)cb * p.rows + rowg) * kDv + kHalfV * rank + 16 * c);
                        uint32_t w[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            w[k] = pack_bf16x2(__uint_as_float(raw[2 * k]) * inv,
                                               __uint_as_float(raw[2 * k + 1]) * inv);
                        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    } else {
                        float4* dst = reinterpret_cast<float4*>(
                            p.part_o + ((int64_t)split * p.rows + rowg) * kDv + kHalfV * rank + 16 * c);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            dst[k] = make_float4(__uint_as_float(raw[4 * k]) * inv,
                                                 __uint_as_float(raw[4 * k + 1]) * inv,
                                                 __uint_as_float(raw[4 * k + 2]) * inv,
                                                 __uint_as_float(raw[4 * k + 3]) * inv);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarOEmpty));
            if (row_valid && rank == 0) {
                if (direct)
                    p.lse[(int64_t)cb * p.rows + rowg] = lse_val;
                else
                    p.part_lse[(int64_t)split * p.rows + rowg] = lse_val;
            }
            ++uq;
            if (!have_next) break;
            cb = nb_;
            ckb0 = nkb0;
            ckb1 = nkb1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    cluster_sync();
}

}  // namespace decode
}  // namespace mla
