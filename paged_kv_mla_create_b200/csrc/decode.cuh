// Paged MLA decode attention for sm_100a, in the role of flash_mla_with_kvcache as the
// SGLang FlashMLA backend page (flashmla_backend.py, forward_decode / forward_extend)
// calls it: q [bs, q_len, h_q, 576] against the latent cache viewed [-1, 64, 1, 576],
// head_dim_v = kv_lora_rank = 512, softmax_scale, causal, fp8 descales; output o and lse.
//
// Design: one 2-CTA cluster per (scheduler part, 128-row query tile), computing with
// pair MMAs (tcgen05 cta_group::2) issued by the leader CTA.
//   * The 128 query rows of a tile (q_len * h_q flattened, heads fastest) share every KV
//     row, so S = Q K^T and O = P V are dense tensor-core contractions.  In a pair MMA of
//     M = 128 each CTA holds 64 rows: CTA r owns query rows [64r, 64r + 64).  Its half of
//     an accumulator D[64 rows, N] lies in its tensor memory as 128 lanes x N/2 columns:
//     lane l < 64 is row l for columns [0, N/2), lane 64 + l is row l for [N/2, N).
//   * S tiles are 128 tokens = two pages.  For S the B operand is split along N, so CTA r
//     loads page r of the tile (all 576 columns, in 64-column chunks); for O += P V the
//     B operand (V, the first 512 columns of the same rows) is split along N = output
//     columns: two N = 256 MMAs cover the 512 outputs and CTA r loads both pages'
//     columns {256n + 128r + [0, 128)}, n = 0, 1 (a second, L2-served read of those
//     bytes).  No data crosses distributed shared memory: the pair's tensor cores share
//     their operands.  (Pair MMAs keep the tensor pipe busy only with N = 256: at N = 128
//     each SM's half is 64 columns wide and runs at about half rate.)
//   * Tensor memory per CTA: S double buffer 2 x 64 columns, O 256 columns (64 rows x 512
//     outputs).  Q (own 64 rows x 576, 72 KB) and P (64 rows x 128 tokens) live in shared
//     memory; K streams through a 3-slot ring of 24 KB loads (three 64-column chunks of
//     the CTA's page, warp 0) and V through a 4-slot ring of 16 KB loads (this CTA's 128
//     columns of one 256-output block of one page, warp 2).  Loads are few and large because the TMA unit's cost is per
//     load: 64 x 64 boxes stream at about 60% of HBM bandwidth, 24 KB loads at full rate.
//   * Roles per CTA: warps 0 / 3 (Q, K) and 2 / 8 (V) TMA producers (page ids from the block
//     table), warp 9 idle;
//     warp 1 lane 0 of the leader issues every MMA; warps 4..7 (thread t = TMEM lane t:
//     row t % 64, token half t / 64) run the online softmax: partner threads t and t ^ 64
//     agree on each row's maximum through shared memory (an mbarrier orders the exchange,
//     so a timed-out wait can never strand the others), P goes to shared memory for the
//     PV MMA, O is rescaled in tensor memory only when the running maximum grows by more
//     than 2^8, and the epilogue normalises and writes o and lse.
//   * A unit whose block range is a whole request writes bf16 o and lse directly; a split
//     piece writes fp32 partials that combine_splits_kernel merges.
//   * Every wait is bounded (mbar_wait_bounded); out-of-range page ids never fault: TMA
//     reads zeros for out-of-range coordinates and the error word records the event.
#pragma once
#include "ptx.cuh"

namespace mla {
namespace decode {

// Optional pipeline trace (compiled only with -DMLA_TRACE): SM clock at each pipeline
// event of the first kTraceTiles tiles of cluster 0, query tile 0.
#ifdef MLA_TRACE
constexpr int kTraceTiles = 64, kTraceEvents = 32;
__device__ long long g_trace[2][kTraceTiles][kTraceEvents];
#define MLA_TRACE_EVENT(tile, ev)                                                         \
    do {                                                                                  \
        if (blockIdx.x < 2 && blockIdx.y == 0 && (tile) < (uint32_t)kTraceTiles)          \
            g_trace[blockIdx.x][(tile)][(ev)] = clock64();                                \
    } while (0)
#else
#define MLA_TRACE_EVENT(tile, ev) \
    do {                          \
    } while (0)
#endif

constexpr int kRows = 128;                 // query rows per tile (both CTAs)
constexpr int kCtaRows = 64;               // query rows per CTA
constexpr int kPage = 64;                  // tokens per page
constexpr int kTileTokens = 128;           // tokens per S tile (two pages)
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kChunks = kDqk / 64;         // 64-column chunks of the 576 reduction columns
constexpr int kBox = 64 * 128;             // one 64-row x 64-column bf16 box, 128-byte swizzle
constexpr int kQBytes = kChunks * kBox;    // 72 KB: own 64 query rows
constexpr int kKOpChunks = 3;             // one K load = 3 column chunks of the CTA's page (24 KB)
constexpr int kKOps = kChunks / kKOpChunks;
constexpr int kKSlots = 3;                 // K ring: one tile of K in flight per CTA
constexpr int kKSlotBytes = kKOpChunks * kBox;
constexpr int kVOps = 4;                   // per tile: (outputs 0-255, page 0), (0-255, page 1), (256-511, 0), (256-511, 1)
constexpr int kVSlots = 4;                 // V ring: one tile of V
constexpr int kVSlotBytes = 2 * kBox;      // one page x this CTA's 128 columns of a 256-output block
constexpr int kPBytes = 2 * kBox;          // P: 64 rows x 128 tokens bf16 (single buffer)
constexpr int kThreads = 320;              // 10 warps (roles below)
constexpr int kSoftmaxWarp0 = 4;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may reach 2^8 before O is rescaled

// Tensor-memory column map (512 columns allocated for the pair).
constexpr uint32_t kTmemS = 0;             // 2 x 64 columns
constexpr uint32_t kTmemO = 128;           // 256 columns: block n (128 columns) holds outputs
                                           // 256n + [0, 128) in lanes < 64, 256n + 128 + [0, 128) above
constexpr uint32_t kTmemCols = 512;

// Shared-memory map (offsets from the 1024-aligned base).
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffV = kOffK + kKSlots * kKSlotBytes;
constexpr int kOffP = kOffV + kVSlots * kVSlotBytes;
constexpr int kOffX = kOffP + kPBytes;          // row-max exchange: 2 x 128 floats, row sums 128
constexpr int kOffBar = kOffX + 3 * 128 * 4;

enum : int {
    kBarKFull = 0,                      // leader: both CTAs' K op landed (tx bytes)
    kBarKEmpty = kBarKFull + kKSlots,   // both: pair MMAs finished reading a K slot
    kBarVFull = kBarKEmpty + kKSlots,
    kBarVEmpty = kBarVFull + kVSlots,
    kBarQFull = kBarVEmpty + kVSlots,   // leader: both Q halves landed
    kBarQEmpty,                         // both: the unit's last S MMA finished (Q reusable)
    kBarSFull,                          // both (x2): S tile in tensor memory
    kBarSFree = kBarSFull + 2,          // leader (x2): 8 softmax warps have read S
    kBarPFull = kBarSFree + 2,          // leader: 8 softmax warps wrote P
    kBarPvDone,                         // both: the PV MMAs of a tile finished (P reusable)
    kBarOFull,                          // both: the unit's last PV finished
    kBarOEmpty,                         // leader: 8 softmax warps read O out
    kBarXchg,                           // local (x2): the 128 softmax threads posted row maxima
    kBarLx = kBarXchg + 2,              // local: the 128 softmax threads posted row sums
    kNumBars
};

constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, false, true);

struct Params {
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
    int b, b1, k0, k1, bs, first_b;
    const int32_t* seqlens;
    int max_pages;
    __device__ bool next(int& ub, int& kb0, int& kb1) {
        while (b <= b1 && b < bs) {
            if (b == b1 && k1 == 0) return false;
            const int L = seqlens[b];
            int nb = L > 0 ? (L + kPage - 1) / kPage : 0;
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

__device__ __forceinline__ int tiles_of(int kb0, int kb1) { return (kb1 - kb0 + 1) >> 1; }

template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap v_map,
                  const __grid_constant__ CUtensorMap q_map, const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + kNumBars * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int part = blockIdx.x >> 1;
    const int mtile = blockIdx.y;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kKSlots; ++s) {
            mbar_init(bar(kBarKFull + s), 1);
            mbar_init(bar(kBarKEmpty + s), 1);
        }
        for (int s = 0; s < kVSlots; ++s) {
            mbar_init(bar(kBarVFull + s), 1);
            mbar_init(bar(kBarVEmpty + s), 1);
        }
        mbar_init(bar(kBarQFull), 1);
        mbar_init(bar(kBarQEmpty), 1);
        for (int j = 0; j < 2; ++j) {
            mbar_init(bar(kBarSFull + j), 1);
            mbar_init(bar(kBarSFree + j), 8);
        }
        mbar_init(bar(kBarPFull), 8);
        mbar_init(bar(kBarPvDone), 1);
        mbar_init(bar(kBarOFull), 1);
        mbar_init(bar(kBarOEmpty), 8);
        mbar_init(bar(kBarXchg), 128);
        mbar_init(bar(kBarXchg + 1), 128);
        mbar_init(bar(kBarLx), 128);
        *abort_flag = 0;
        fence_mbarrier_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&k_map);
        prefetch_tensormap(&v_map);
        prefetch_tensormap(&q_map);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool md_ok = true;
    UnitIter iter = make_iter(p, part, md_ok);
    if (!md_ok && threadIdx.x == 0) raise_error(8 /* MLA_DEVERR_BAD_METADATA */);

    if (warp == 0 || warp == 2 || warp == 3 || warp == 8) {
        // ------------------------------------------------------------ TMA producers
        // A thread's TMA loads complete one after another (about 500 cycles plus 11 per KB
        // each), so each stream has two issuing warps taking alternate loads: warps 0 / 3
        // load Q (warp 0, once per unit) and K, three 24 KB loads per tile (three 64-column
        // chunks of the CTA's page); warps 2 / 8 load V, four 16 KB loads per tile (this
        // CTA's 128 columns 256n + 128r + [0, 128) of one page, in the order (n, page) =
        // (0,0), (0,1), (1,0), (1,1) the PV MMAs consume).
        const bool is_k = warp == 0 || warp == 3;
        const uint32_t parity = (warp == 3 || warp == 8) ? 1u : 0u;
        uint32_t oc = 0, uq = 0;   // this stream's load counter, unit counter
        bool alive = true;
        int ub, kb0, kb1;
        while (alive && iter.next(ub, kb0, kb1)) {
            const int n = tiles_of(kb0, kb1);
            if (n <= 0) continue;
            const int32_t* bt_row = p.block_table + (int64_t)ub * p.bt_stride;
            if (is_k && parity == 0) {
                int ok = 1;
                if (lane == 0) {
                    if (uq > 0)
                        ok = mbar_wait_bounded<false>(bar(kBarQEmpty), (uq - 1) & 1u, abort_flag);
                    if (ok) {
                        if (leader) mbar_arrive_expect_tx(bar(kBarQFull), 2 * kQBytes);
                        // own 64 query rows, all 9 column chunks, one load
                        tma_load_4d_pair(sbase + kOffQ, &q_map, map_to_cta(bar(kBarQFull), 0), 0,
                                         mtile * kRows + kCtaRows * (int32_t)rank, 0, ub);
                    }
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            }
            // Page ids of blocks [pg_base, pg_base + 32) across the warp, slid forward as the
            // tiles advance.  Block j -> TMA row coordinate page * 64; a bad or missing page
            // -> the first row past the pool, read as zeros (and reported).
            int pg_base = kb0;
            auto fetch_pg = [&](int idx) -> int {
                const int pg = idx < kb1 ? __ldg(bt_row + idx) : -1;
                const bool bad = idx < kb1 && (pg < 0 || (int64_t)pg >= p.num_pages);
                if (__any_sync(0xffffffffu, bad) && lane == 0 && is_k && parity == 0) raise_error(1);
                return (idx < kb1 && !bad) ? pg : -1;
            };
            int pg_lane = fetch_pg(kb0 + lane);
            auto page_row = [&](int blk) -> int32_t {
                if (blk >= kb1) return (int32_t)(p.num_pages * kPage);
                while (blk >= pg_base + 32) {
                    pg_base += 32;
                    pg_lane = fetch_pg(pg_base + lane);
                }
                const int pg = __shfl_sync(0xffffffffu, pg_lane, blk - pg_base);
                return pg >= 0 ? pg * kPage : (int32_t)(p.num_pages * kPage);
            };
            const int per_tile = is_k ? kKOps : kVOps;
            for (int i = 0; alive && i < n; ++i) {
                const int blk0 = kb0 + 2 * i;
                const int32_t row0 = page_row(blk0), row1 = page_row(blk0 + 1);
                for (int op = 0; op < per_tile; ++op, ++oc) {
                    if ((oc & 1u) != parity) continue;
                    int ok = 1;
                    if (lane == 0) {
                        if (is_k) {
                            const int s = oc % kKSlots;
                            ok = mbar_wait_bounded<false>(bar(kBarKEmpty + s), ((oc / kKSlots) & 1u) ^ 1u,
                                                          abort_flag);
                            if (ok) {
                                if (leader) mbar_arrive_expect_tx(bar(kBarKFull + s), 2 * kKSlotBytes);
                                tma_load_3d_pair(sbase + kOffK + s * kKSlotBytes, &k_map,
                                                 map_to_cta(bar(kBarKFull + s), 0), 0, rank ? row1 : row0,
                                                 kKOpChunks * op);
                                MLA_TRACE_EVENT(i, 12 + op);
                            }
                        } else {
                            const int s = oc % kVSlots;
                            ok = mbar_wait_bounded<false>(bar(kBarVEmpty + s), ((oc / kVSlots) & 1u) ^ 1u,
                                                          abort_flag);
                            if (ok) {
                                if (leader) mbar_arrive_expect_tx(bar(kBarVFull + s), 2 * kVSlotBytes);
                                tma_load_4d_pair(sbase + kOffV + s * kVSlotBytes, &v_map,
                                                 map_to_cta(bar(kBarVFull + s), 0), 0, (op & 1) ? row1 : row0, 0,
                                                 2 * (op >> 1) + (int32_t)rank);
                                MLA_TRACE_EVENT(i, 18 + op);
                            }
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, ok, 0)) {
                        alive = false;
                        break;
                    }
                }
            }
            ++uq;
        }
        if (lane == 0 && *abort_flag) {
            // let copies already issued land before shared memory can go away
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 200000ull) {
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        // Per unit: QK(0), QK(1), PV(0), QK(2), PV(1), ..., PV(last): S runs one tile ahead
        // of PV so the tensor pipe computes S(t+1) while the softmax works on tile t.
        if (leader && lane == 0) {
            uint32_t g = 0, uq = 0, kc = 0, vc = 0;
            bool alive = true;
            int ub, kb0, kb1;
            auto issue_pv = [&](uint32_t gg, bool first) -> bool {
                if (!mbar_wait_bounded<true>(bar(kBarPFull), gg & 1u, abort_flag)) return false;
                if (first && uq > 0 &&
                    !mbar_wait_bounded<true>(bar(kBarOEmpty), (uq - 1) & 1u, abort_flag))
                    return false;
                tc_fence_after();
                MLA_TRACE_EVENT(gg, 2);
                const uint32_t pbuf = sbase + kOffP;
#pragma unroll 1
                for (int vop = 0; vop < kVOps; ++vop) {
                    const int pp = vop & 1;
                    const int s = vc % kVSlots;
                    if (!mbar_wait_bounded<true>(bar(kBarVFull + s), (vc / kVSlots) & 1u, abort_flag))
                        return false;
                    MLA_TRACE_EVENT(gg, 22 + vop);
                    tc_fence_after();
                    const uint32_t vslot = sbase + kOffV + s * kVSlotBytes;
                    const int nn = vop >> 1;   // output block: TMEM columns 128nn..
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_pair_ss(tmem + kTmemO + 128u * nn,
                                    smem_desc_sw128(pbuf + pp * kBox + 32u * kk, 16, 1024),
                                    smem_desc_sw128(vslot + 2048u * kk, kBox, 1024), kIdescPV,
                                    (first && pp == 0 && kk == 0) ? 0u : 1u);
                    tc_commit_pair(bar(kBarVEmpty + s));
                    ++vc;
                }
                tc_commit_pair(bar(kBarPvDone));
                return true;
            };
            while (alive && iter.next(ub, kb0, kb1)) {
                const int n = tiles_of(kb0, kb1);
                if (n <= 0) continue;
                if (!mbar_wait_bounded<true>(bar(kBarQFull), uq & 1u, abort_flag)) break;
                const uint32_t g0 = g;
                for (int i = 0; alive && i < n; ++i) {
                    const uint32_t sb = g & 1u;
                    if (g >= 2 &&
                        !mbar_wait_bounded<true>(bar(kBarSFree + sb), ((g >> 1) & 1u) ^ 1u, abort_flag)) {
                        alive = false;
                        break;
                    }
                    MLA_TRACE_EVENT(g, 1);
#pragma unroll 1
                    for (int j = 0; j < kKOps; ++j) {
                        const int s = kc % kKSlots;
                        if (!mbar_wait_bounded<true>(bar(kBarKFull + s), (kc / kKSlots) & 1u, abort_flag)) {
                            alive = false;
                            break;
                        }
                        MLA_TRACE_EVENT(g, 15 + j);
                        tc_fence_after();
                        const uint32_t kslot = sbase + kOffK + s * kKSlotBytes;
#pragma unroll
                        for (int c = 0; c < kKOpChunks; ++c) {
                            const uint32_t qa = sbase + kOffQ + (kKOpChunks * j + c) * kBox;
                            const uint32_t kb = kslot + c * kBox;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_pair_ss(tmem + kTmemS + 64u * sb, smem_desc_sw128(qa + 32u * kk, 16, 1024),
                                            smem_desc_sw128(kb + 32u * kk, 16, 1024), kIdescQK,
                                            (j | c | kk) ? 1u : 0u);
                        }
                        tc_commit_pair(bar(kBarKEmpty + s));
                        ++kc;
                    }
                    if (!alive) break;
                    tc_commit_pair(bar(kBarSFull + sb));
                    if (i == n - 1) tc_commit_pair(bar(kBarQEmpty));
                    if (i >= 1 && !issue_pv(g - 1, i == 1)) {
                        alive = false;
                        break;
                    }
                    ++g;
                }
                if (!alive || !issue_pv(g - 1, g - 1 == g0)) break;
                tc_commit_pair(bar(kBarOFull));
                ++uq;
            }
        }
    } else if (warp >= kSoftmaxWarp0 && warp < kSoftmaxWarp0 + 4) {
        // ------------------------------------------------------------ softmax / epilogue
        const int t = threadIdx.x - kSoftmaxWarp0 * 32;       // TMEM lane
        const int rloc = t & 63;                              // row within this CTA's 64
        const int half = t >> 6;                              // token half of each tile
        const uint32_t lane_off = (uint32_t)((warp - kSoftmaxWarp0) * 32) << 16;
        const int rowg = mtile * kRows + kCtaRows * (int)rank + rloc;
        const bool row_valid = rowg < p.rows;
        const int iq = row_valid ? rowg / p.h_q : 0;
        const float dq = p.descale_q ? *p.descale_q : 1.0f;
        const float dk = p.descale_k ? *p.descale_k : 1.0f;
        const float sl2 = p.scale_log2 * dq * dk;
        float* xmax = reinterpret_cast<float*>(smem + kOffX);  // [2][128] row maxima, [128] sums
        const uint32_t swz = (uint32_t)(rloc & 7);
        // Signals to the leader's barriers: the leader's own warps arrive locally; the peer's
        // warps arrive remotely, releasing at cluster scope only when they publish data.
        auto arrive_leader = [&](int b_idx) {
            __syncwarp();
            if (lane == 0) {
                if (leader)
                    mbar_arrive(bar(b_idx));
                else
                    mbar_arrive_remote(map_to_cta(bar(b_idx), 0));
            }
        };
        auto arrive_leader_done_reading = [&](int b_idx) {
            __syncwarp();
            if (lane == 0) {
                if (leader)
                    mbar_arrive(bar(b_idx));
                else
                    mbar_arrive_remote_relaxed(map_to_cta(bar(b_idx), 0));
            }
        };

        auto write_empty = [&](int b) {
            // A request with no key: o = 0, lse = -inf (always a single, direct piece).
            if (!row_valid) return;
            __nv_bfloat16* row_out = p.out + ((int64_t)b * p.rows + rowg) * kDv;
#pragma unroll 1
            for (int nn = 0; nn < 2; ++nn) {
                uint4* dst = reinterpret_cast<uint4*>(row_out + 256 * nn + 128 * half);
                for (int c = 0; c < 16; ++c) dst[c] = make_uint4(0, 0, 0, 0);
            }
            if (half == 0) p.lse[(int64_t)b * p.rows + rowg] = -INFINITY;
        };

        uint32_t g = 0, uq = 0;
        bool alive = true;
        int ub, kb0, kb1;
        while (alive && iter.next(ub, kb0, kb1)) {
            const int n = tiles_of(kb0, kb1);
            if (n <= 0) {
                write_empty(ub);
                continue;
            }
            const int L = p.cache_seqlens[ub];
            int lim = p.causal ? L - p.q_len + iq + 1 : L;
            if (lim > L) lim = L;
            if (lim > kb1 * kPage) lim = kb1 * kPage;   // keys of this unit only
            float m_run = -INFINITY, l_half = 0.f;
            for (int i = 0; i < n; ++i, ++g) {
                const uint32_t sb = g & 1u;
                if (t == 0) MLA_TRACE_EVENT(g, 3);
                if (!mbar_wait_bounded<false>(bar(kBarSFull + sb), (g >> 1) & 1u, abort_flag)) {
                    alive = false;
                    break;
                }
                if (t == 0) MLA_TRACE_EVENT(g, 4);
                tc_fence_after();
                float s[64];
                {
                    uint32_t raw[4][16];
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        tmem_ld16(tmem + lane_off + kTmemS + 64u * sb + 16u * c, raw[c]);
                    tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int k = 0; k < 16; ++k) s[16 * c + k] = __uint_as_float(raw[c][k]);
                }
                if (t == 0) MLA_TRACE_EVENT(g, 11);
                tc_fence_before();
                arrive_leader_done_reading(kBarSFree + sb);
                if (t == 0) MLA_TRACE_EVENT(g, 7);
                // scale to log2 units, mask, this half's maximum
                const int kbase = (kb0 + 2 * i) * kPage + kPage * half;
                float hmax = -INFINITY;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    float x = s[j] * sl2;
                    if (kbase + j >= lim) x = -INFINITY;
                    s[j] = x;
                    hmax = fmaxf(hmax, x);
                }
                // partner thread t ^ 64 holds the other 64 tokens of this row
                xmax[sb * 128 + t] = hmax;
                if (t == 0) MLA_TRACE_EVENT(g, 8);
                mbar_arrive(bar(kBarXchg + sb));
                if (!mbar_wait_bounded<false>(bar(kBarXchg + sb), (g >> 1) & 1u, abort_flag)) {
                    alive = false;
                    break;
                }
                if (t == 0) MLA_TRACE_EVENT(g, 9);
                const float tmax = fmaxf(hmax, xmax[sb * 128 + (t ^ 64)]);
                const float m_new = fmaxf(m_run, tmax);
                const bool rescale = m_new > m_run + kRescaleThreshold;
                float factor = 1.f;
                if (rescale) {
                    factor = fast_exp2(m_run - m_new);  // 0 when m_run = -inf
                    l_half *= factor;
                    m_run = m_new;
                }
                const bool live = m_run != -INFINITY;
                float psum = 0.f;
                // P packed as bf16 pairs into s[0..31] (s[2j], s[2j+1] are read before s[j]
                // is overwritten, since 2j >= j).
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float p0 = live ? fast_exp2(s[2 * j] - m_run) : 0.f;
                    const float p1 = live ? fast_exp2(s[2 * j + 1] - m_run) : 0.f;
                    psum += p0 + p1;
                    s[j] = __uint_as_float(pack_bf16x2(p0, p1));
                }
                l_half += psum;
                if (t == 0) MLA_TRACE_EVENT(g, 5);
                // the P buffer is free, and O holds every PV up to tile g - 1, once PV(g - 1)
                // has finished
                if (t == 0) MLA_TRACE_EVENT(g, 10);
                if (g >= 1 && !mbar_wait_bounded<false>(bar(kBarPvDone), (g - 1) & 1u, abort_flag)) {
                    alive = false;
                    break;
                }
                if (i > 0 && __any_sync(0xffffffffu, rescale)) {
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 16; ++c) {
                        uint32_t raw[16];
                        tmem_ld16(tmem + lane_off + kTmemO + 16u * c, raw);
                        tc_wait_ld();
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            raw[k] = __float_as_uint(__uint_as_float(raw[k]) * factor);
                        tmem_st16(tmem + lane_off + kTmemO + 16u * c, raw);
                    }
                    tc_wait_st();
                    tc_fence_before();
                }
                // P -> shared memory, K-major with 128-byte swizzle: 16-byte chunk c of row
                // rloc at chunk position c ^ (rloc & 7)
                {
                    const uint32_t prow = sbase + kOffP + half * kBox + rloc * 128u;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        st_shared_v4u(prow + ((c ^ swz) << 4), __float_as_uint(s[4 * c]),
                                      __float_as_uint(s[4 * c + 1]), __float_as_uint(s[4 * c + 2]),
                                      __float_as_uint(s[4 * c + 3]));
                }
                fence_proxy_async_smem();
                arrive_leader(kBarPFull);
                if (t == 0) MLA_TRACE_EVENT(g, 6);
            }
            if (!alive) break;
            // epilogue of the unit
            if (!mbar_wait_bounded<false>(bar(kBarOFull), uq & 1u, abort_flag)) break;
            tc_fence_after();
            xmax[256 + t] = l_half;
            mbar_arrive(bar(kBarLx));
            if (!mbar_wait_bounded<false>(bar(kBarLx), uq & 1u, abort_flag)) break;
            const float l_run = l_half + xmax[256 + (t ^ 64)];
            const int pieces = p.num_splits[ub + 1] - p.num_splits[ub];
            const bool direct = pieces == 1;
            const int split = p.num_splits[ub] + (ub == iter.first_b ? p.md[8 * part + 4] : 0);
            const float inv = l_run > 0.f ? dk / l_run : 0.f;
            const float lse_val = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f
                                              : -INFINITY;
#pragma unroll 1
            for (int c = 0; c < 8; ++c) {
                // TMEM columns [128 + 32c, +32): output columns 256 * (c / 4) + 128 * half + 32 * (c % 4)
                uint32_t raw[32];
                tmem_ld16(tmem + lane_off + kTmemO + 32u * c, *reinterpret_cast<uint32_t(*)[16]>(raw));
                tmem_ld16(tmem + lane_off + kTmemO + 32u * c + 16u,
                          *reinterpret_cast<uint32_t(*)[16]>(raw + 16));
                tc_wait_ld();
                const int col = 256 * (c >> 2) + 128 * half + 32 * (c & 3);
                if (row_valid) {
                    if (direct) {
                        uint4* dst = reinterpret_cast<uint4*>(p.out + ((int64_t)ub * p.rows + rowg) * kDv + col);
                        uint32_t w[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            w[k] = pack_bf16x2(__uint_as_float(raw[2 * k]) * inv,
                                               __uint_as_float(raw[2 * k + 1]) * inv);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                    } else {
                        float4* dst = reinterpret_cast<float4*>(
                            p.part_o + ((int64_t)split * p.rows + rowg) * kDv + col);
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            dst[k] = make_float4(__uint_as_float(raw[4 * k]) * inv,
                                                 __uint_as_float(raw[4 * k + 1]) * inv,
                                                 __uint_as_float(raw[4 * k + 2]) * inv,
                                                 __uint_as_float(raw[4 * k + 3]) * inv);
                    }
                }
            }
            tc_fence_before();
            arrive_leader_done_reading(kBarOEmpty);
            if (row_valid && half == 0) {
                if (direct)
                    p.lse[(int64_t)ub * p.rows + rowg] = lse_val;
                else
                    p.part_lse[(int64_t)split * p.rows + rowg] = lse_val;
            }
            ++uq;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace decode
}  // namespace mla
