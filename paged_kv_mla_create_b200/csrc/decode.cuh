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
//     lane l < 64 is row l for columns [0, N/2), lane 64 + l is row l for [N/2, N).  An A
//     operand read from tensor memory is read the same way: row l from lane l for D's
//     columns [0, N/2) and from lane 64 + l for [N/2, N), two bf16 of consecutive k per
//     32-bit column.
//   * S tiles are 128 tokens = two pages.  For S the B operand is split along N (tokens):
//     CTA r loads page r of the tile, all 576 columns, into a 72 KB slot (nine 64-column
//     chunks; chunk c at 8 KB * c).  For O += P V the B operand (V, the first 512 columns)
//     is split along N = output columns: in the MMA for output block n (256 columns) and
//     page p, CTA 0 supplies columns 256n + [0, 128) (chunks 4n, 4n + 1) and CTA 1
//     columns 256n + [128, 256) (chunks 4n + 2, 4n + 3) of page p, both at slot offset
//     8 KB * (4n + 2p).  CTA p has its own page's chunks there already; the other CTA's
//     chunks at that offset belong to its own page and are dead once S is computed, so
//     after the S MMAs it loads the partner page's four chunks it needs (32 KB, an L2 hit:
//     the partner CTA loads that page) into exactly those positions.  Each KV byte crosses
//     HBM once; each CTA takes in 72 + 32 KB per tile.
//   * Tensor memory per CTA: S double buffer 2 x 64 columns, O 256 columns (64 rows x 512
//     outputs), and Q columns [0, 256) of the CTA's 64 rows (128 columns; row r in lanes r
//     and 64 + r) as the A operand of the first four chunks of S; Q columns [256, 576) (40 KB) and P (64
//     rows x 128 tokens, 16 KB) live in shared memory, with a 2-slot K ring (144 KB).
//   * Roles per CTA: warps 0 / 3 load K (alternate tiles, one 72 KB load each); warps 8..11
//     load Q once per unit (columns [256, 576) by TMA into shared memory, columns [0, 256)
//     into tensor memory), and warp 11 loads the partner V of every tile by TMA once the
//     tile's S is done (an e4m3 cache: all four warps, through registers, widening to f16),
//     and prefetch the later units' query rows into L2; warp 1 of the leader walks the MMA
//     schedule and an elected lane issues every MMA; warps 4..7 (thread t = TMEM lane t: row t % 64, token half
//     t / 64) run the online softmax: partner threads t and t ^ 64 agree on each row's
//     maximum through shared memory (an mbarrier orders the exchange, so a timed-out wait
//     can never strand the others), P goes to shared memory for the PV MMA, O is rescaled
//     in tensor memory only when the running maximum grows by more than 2^8, and the
//     epilogue normalises o (or keeps fp32 partials) and writes it as TMA stores of
//     32-row boxes staged in shared memory, and writes lse.
//   * A unit whose block range is a whole request writes bf16 o and lse directly.  A piece of a
//     request of at most kFusedMergeMaxPieces pieces claims a place on a per-(request, query
//     tile, CTA) word of the workspace during its last tile; the last to claim merges the
//     request's rows (log-sum-exp), the others store fp32 partials and count them stored on
//     the same word.  The last claimer, if in its part's last unit (Q, K ring and P idle) and
//     the request has at most kFoldMaxPieces pieces, folds the others' stored rows into its own
//     tensor-memory O in the epilogue (waiting for their stores if need be); otherwise it stores
//     its partial too and merges all of them once its part is done.  Both ways sum the pieces
//     in split-slot order with the same weights, so the result has the same bits whichever
//     piece merges.  The merging CTA resets the word to zero; combine_splits_kernel merges
//     requests of more pieces.
//   * e4m3 queries with an e4m3 cache (the backend page's fp8 recipe: q quantised with the
//     cache's scale, descale_q and descale_k passed along): S runs as kind::f8f6f4 MMAs (K = 32
//     per instruction, 18 per tile) straight from the raw page and the e4m3 query rows, both in a
//     64-byte-swizzled layout (a 64-value row is one swizzle span); only the V chunks each CTA
//     supplies to PV are widened to f16, after S, by warps 8..11.
//   * Every wait is bounded (mbar_wait_bounded); out-of-range page ids never fault: TMA
//     reads zeros for out-of-range coordinates and the error word records the event.
#pragma once
#include "combine.cuh"
#include "ptx.cuh"

namespace mla {
namespace decode {

constexpr int kRows = 128;                 // query rows per tile (both CTAs)
constexpr int kCtaRows = 64;               // query rows per CTA
constexpr int kPage = 64;                  // tokens per page
constexpr int kTileTokens = 128;           // tokens per S tile (two pages)
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kChunks = kDqk / 64;         // 64-column chunks of the 576 reduction columns
constexpr int kBox = 64 * 128;             // one 64-row x 64-column bf16 box, 128-byte swizzle
constexpr int kQLoChunks = 4;              // Q columns [0, 256): tensor memory
constexpr int kQHiChunks = kChunks - kQLoChunks;   // Q columns [256, 576): shared memory
constexpr int kQHiBytes = kQHiChunks * kBox;       // 40 KB
constexpr int kKSlots = 2;                 // K ring: two tiles
constexpr int kKSlotBytes = kChunks * kBox;        // 72 KB: one page, all 576 columns
constexpr int kPBytes = 2 * kBox;          // P: 64 rows x 128 tokens bf16
constexpr int kThreads = 384;              // 12 warps (roles above)
constexpr int kSoftmaxWarp0 = 4;
constexpr int kQWarp0 = 8;                 // warps 8..11: Q loaders (TMEM lane quarters 0..3)
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may reach 2^8 before O is rescaled

// Tensor-memory column map (512 columns allocated for the pair).
constexpr uint32_t kTmemS = 0;             // 2 x 64 columns
constexpr uint32_t kTmemO = 128;           // 256 columns: block n (128 columns) holds outputs
                                           // 256n + [0, 128) in lanes < 64, 256n + 128 + [0, 128) above
constexpr uint32_t kTmemQ = 384;           // 128 columns, lanes 0..63: Q columns 2j, 2j + 1 in column j
constexpr uint32_t kTmemCols = 512;

// Shared-memory map (offsets from the 1024-aligned base).
constexpr int kOffQ = 0;                            // Q chunks 4..8
constexpr int kOffK = kOffQ + kQHiBytes;
constexpr int kOffP = kOffK + kKSlots * kKSlotBytes;
constexpr int kOffX = kOffP + kPBytes;              // row-max exchange: 2 x 128 floats, row sums 128
constexpr int kOffStage = kOffX + 3 * 1024;         // epilogue staging: 4 warps x 32 rows x 128 B
                                                    // (1 KB aligned: boxes of TMA stores, 128-byte swizzle)
constexpr int kOffPSig = kOffStage + 4 * 32 * 128;  // leader: landing words of the peer's P signals
constexpr int kOffBar = kOffPSig + 128;   // landing words: P 0..3, V 4..7, K 8, Q 9..12,
                                            // S read 16..19, O read 20..23

enum : int {
    kBarKFull = 0,                      // leader (x slots): both CTAs' pages of the tile landed
    kBarKEmpty = kBarKFull + kKSlots,   // both: the tile's PV finished (slot reusable)
    kBarQKDone = kBarKEmpty + kKSlots,  // both: the tile's S MMAs finished reading the slot
    kBarVFull = kBarQKDone + kKSlots,   // leader: the pair's partner V landed
    kBarQFull = kBarVFull + kKSlots,    // leader: Q columns [256, 576) landed (tx) + eight
                                        // warps wrote Q columns [0, 256) to tensor memory
    kBarQEmpty,                         // both: the unit's last S MMA finished (Q reusable)
    kBarSFull,                          // both (x2): S tile in tensor memory
    kBarSFree = kBarSFull + 2,          // leader (x2): 8 softmax warps have read S
    kBarPFull = kBarSFree + 2,          // leader: 8 softmax warps wrote P
    kBarPvDone,                         // both: the PV MMAs of a tile finished (P reusable)
    kBarOFull,                          // both: the unit's last PV finished
    kBarOEmpty,                         // leader: 8 softmax warps read O out
    kBarXchg,                           // local (x2): the 128 softmax threads posted row maxima
    kBarLx = kBarXchg + 2,              // local: the 128 softmax threads posted row sums
    kBarPartial,                        // local: the 128 softmax threads stored a split piece
    kBarVWiden,                         // local, e4m3 q: warps 8..11 read their raw V chunks
    kBarFold,                           // local: the other pieces' partial rows landed (fold-in merge)
    kBarFoldRd,                         // local: the 128 softmax threads read the first fold-in round
    kBarFoldL,                          // local: the other pieces' lse values landed (fold-in merge)
    kBarMerge,                          // local: a tail merge's pass of partial rows landed
    kBarKRaw,                           // local (x2), e4m3 cache: this CTA's page landed
    kNumBars = kBarKRaw + kKSlots
};

// After the barriers: tensor-memory base, abort flag, pending-merge count, up to two pending
// merges (request, first split slot, pieces): only a part's first and last units can be pieces
// of split requests, and the fold decision of the current epilogue.
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kMiscFold = 8;          // int index into the misc area: the fold-in decision
// Fold-in merge: the other pieces' 64 partial rows land in the idle Q, K ring and P areas
// (contiguous from the base, 200 KB) as 2-D TMA boxes of 32 fp32 columns x 64 rows (8 KB each,
// 128-byte swizzle: 16-byte unit u of row r at u ^ (r & 7), so that the row-per-lane reads are
// conflict-free); a TMA operation costs ~70 cycles of the SM's TMA unit whatever its size, so
// boxes, not rows.  One other piece: all sixteen boxes at once, box c at 8 KB * c.  Two or three:
// the eight boxes of columns [0, 256) of every other piece j at 8 KB * (8 j + c), then, once those
// are read, the eight of columns [256, 512) in the same places.
constexpr int kFoldBoxCols = 32;
constexpr int kFoldBoxBytes = kCtaRows * kFoldBoxCols * 4;   // 8 KB
constexpr int kFoldBoxes = kDv / kFoldBoxCols;               // 16
// Requests of up to this many pieces fold in (four-piece requests merge at the end of the part:
// the fold's unrolled sums over four pieces exceed the register budget).
constexpr int kFoldMaxPieces = 3;
static_assert(kOffQ == 0 && kOffK == kOffQ + kQHiBytes && kOffP == kOffK + kKSlots * kKSlotBytes,
              "the fold-in staging is contiguous");
static_assert(kFoldBoxes * kFoldBoxBytes <= kOffX - kOffQ &&
                  (kFoldMaxPieces - 1) * (kFoldBoxes / 2) * kFoldBoxBytes <= kOffX - kOffQ &&
                  kFoldMaxPieces <= kFusedMergeMaxPieces,
              "fold-in rows fit the idle areas");
constexpr int kMaxPendingMerges = 2;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffK % 1024 == 0 && kOffP % 1024 == 0 && kOffStage % 1024 == 0,
              "128-byte swizzle atoms need 1 KB alignment");
static_assert(kOffStage >= kOffX + 3 * 128 * 4, "the exchange area fits before the staging");

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, false, true);
constexpr uint32_t kIdescQK16 = idesc_bf16_f32(128, 128, false, false, true);
constexpr uint32_t kIdescPV16 = idesc_bf16_f32(128, 256, false, true, true);
constexpr uint32_t kIdescQK8 = idesc_e4m3_f32(128, 128);

// e4m3 cache: a page (64 rows x 576 one-byte values, 36 KB) lands in the back half of its
// slot as nine 64 x 64-byte chunks and is widened in place, chunk by chunk from the front,
// to the f16 layout of the bf16 path (chunk c at 8 KB * c): chunk c's output never reaches
// the input of a chunk after c, and each chunk is read whole before it is written.
constexpr int kPage8Bytes = kPage * kDqk;              // 36 KB
constexpr int kRaw8Off = kKSlotBytes - kPage8Bytes;    // 36 KB into the slot
constexpr int kChunk8 = 64 * 64;                       // one 64-row x 64-byte e4m3 chunk

// Widen one 8-bit chunk (64 rows x 64 bytes at src; e5m2 when kE5M2, else e4m3) to f16
// (64 rows x 128 bytes at dst, 128-byte swizzle: 16-byte unit u of row t at u ^ (t & 7)).
// One warp; the whole chunk is read before any of it is written.
template <bool kE5M2>
__device__ __forceinline__ void widen_chunk_fp8(uint32_t src, uint32_t dst, int lane) {
    uint4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = ld_shared_v4u(src + 16u * (uint32_t)(lane + 32 * j));
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int x = lane + 32 * j;        // row x / 4, 16-value quarter x % 4
        const uint32_t t = (uint32_t)(x >> 2), q = (uint32_t)(x & 3);
        const uint32_t row = dst + 128u * t;
        st_shared_v4u(row + 16u * ((2u * q) ^ (t & 7u)), fp8x2_to_f16x2<kE5M2>(v[j].x), fp8x2_to_f16x2<kE5M2>(v[j].x >> 16),
                      fp8x2_to_f16x2<kE5M2>(v[j].y), fp8x2_to_f16x2<kE5M2>(v[j].y >> 16));
        st_shared_v4u(row + 16u * ((2u * q + 1u) ^ (t & 7u)), fp8x2_to_f16x2<kE5M2>(v[j].z),
                      fp8x2_to_f16x2<kE5M2>(v[j].z >> 16), fp8x2_to_f16x2<kE5M2>(v[j].w), fp8x2_to_f16x2<kE5M2>(v[j].w >> 16));
    }
    __syncwarp();
}

// e4m3 queries: Q (64 rows x 576 codes) in shared memory as nine 64 x 64-byte chunks with
// 64-byte swizzle, and the raw page in the back half of its slot in the same layout.
constexpr int kQ8Bytes = kChunks * 64 * 64;            // 36 KB
static_assert(kQ8Bytes <= kQHiBytes, "e4m3 Q fits the Q region");

// Read one raw e4m3 chunk (64 rows x 64 bytes, 64-byte swizzle: 16-byte unit u of row t at
// u ^ ((t >> 1) & 3)) into registers: lane holds units x = lane + 32 j (row x / 4, unit x % 4).
__device__ __forceinline__ void load_chunk_sw64(uint32_t src, int lane, uint4 (&v)[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t x = (uint32_t)(lane + 32 * j), row = x >> 2, u = x & 3u;
        v[j] = ld_shared_v4u(src + 64u * row + 16u * (u ^ ((row >> 1) & 3u)));
    }
}

// Store the chunk read by load_chunk_sw64 widened to f16 (64 rows x 128 bytes, 128-byte
// swizzle: unit k of row t at k ^ (t & 7)); e4m3 -> f16 is exact.
__device__ __forceinline__ void store_chunk_f16(uint32_t dst, int lane, const uint4 (&v)[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t x = (uint32_t)(lane + 32 * j), t = x >> 2, u = x & 3u;
        const uint32_t row = dst + 128u * t;
        st_shared_v4u(row + 16u * ((2u * u) ^ (t & 7u)), e4m3x2_to_f16x2(v[j].x), e4m3x2_to_f16x2(v[j].x >> 16),
                      e4m3x2_to_f16x2(v[j].y), e4m3x2_to_f16x2(v[j].y >> 16));
        st_shared_v4u(row + 16u * ((2u * u + 1u) ^ (t & 7u)), e4m3x2_to_f16x2(v[j].z),
                      e4m3x2_to_f16x2(v[j].z >> 16), e4m3x2_to_f16x2(v[j].w), e4m3x2_to_f16x2(v[j].w >> 16));
    }
}

// bf16 pair -> f16 pair (the e4m3 path computes in f16); flags values beyond f16's range.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, bool& out_of_range) {
    const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
    out_of_range |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
    return pack_f16x2(lo, hi);
}

struct Params {
    const __nv_bfloat16* q;        // [bs, rows, 576]
    const uint8_t* kv;             // [num_pages * 64, 576] bf16 or e4m3
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
    int32_t* arrivals;             // [bs, query tiles, 2]: split pieces arrived (zero between calls)
    uint64_t wait_budget_ns;       // budget of one pipeline wait
    int32_t withhold_tile;         // test hook: the leader's K load of this tile is not issued (-1: none)
    int32_t fold_ok;               // po_map / pl_map cover part_o / part_lse (else no fold-in merge)
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

// A split request's arrival word (per query tile and CTA): its low 16 bits count the pieces that
// claimed a place (the last to claim merges), its high bits the pieces that stored their partial
// rows.  Bounded wait until `target` pieces have stored theirs.  Only pieces that have already
// claimed are waited for, and a piece stores right after it claims without waiting on any other
// CTA, so the wait ends unless a piece gave up (abort).
__device__ __forceinline__ bool wait_stored(const int32_t* word, int target, const AbortCtl& a) {
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if ((ld_acquire_gpu(word) >> 16) >= target) return true;
        if (*a.flag) return false;
        if (global_timer_ns() - t0 > a.budget_ns) {
            raise_abort(a);
            return false;
        }
        __nanosleep(64);
    }
}

// One 64-column step of the fold-in merge for one row (NP pieces, this one in slot OWN): for each
// 16-byte group of 4 columns, the
// pieces' rows in split-slot order, weighted and summed (acc += w_i * v_i from zero, exactly as
// the merge of stored partials computes it), then packed to bf16.  This piece's own row is its
// tensor-memory O times inv (its stored partial's value), the others' (NP - 1 of them) come from
// the staged boxes at base_j + off(group).  Branch-free, so that the shared-memory loads of four
// groups can be issued ahead of their sums.
template <int NP, int OWN>
__device__ __forceinline__ void fold_step(const uint32_t (&raw)[64], uint32_t (&w)[32], float inv, const float* wts,
                                          uint32_t base0, uint32_t base1, int rloc) {
    const uint32_t row = (uint32_t)rloc * 128u, sw = (uint32_t)rloc & 7u;
#pragma unroll
    for (int f4 = 0; f4 < 16; ++f4) {
        const uint32_t off = (uint32_t)(f4 >> 3) * (uint32_t)kFoldBoxBytes + row + ((((uint32_t)f4 & 7u) ^ sw) << 4);
        float4 o[NP - 1];
        o[0] = ld_shared_v4f(base0 + off);
        if constexpr (NP > 2) o[NP - 2] = ld_shared_v4f(base1 + off);
        const float4 mine = make_float4(__uint_as_float(raw[4 * f4]) * inv, __uint_as_float(raw[4 * f4 + 1]) * inv,
                                        __uint_as_float(raw[4 * f4 + 2]) * inv, __uint_as_float(raw[4 * f4 + 3]) * inv);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            // slot i: this piece, or the other piece j = i - 1 (i > OWN) / j = i (i < OWN)
            const float4 v = i == OWN ? mine : o[i > OWN ? (i > 0 ? i - 1 : 0) : (i < NP - 1 ? i : NP - 2)];
            acc.x += wts[i] * v.x;
            acc.y += wts[i] * v.y;
            acc.z += wts[i] * v.z;
            acc.w += wts[i] * v.w;
        }
        w[2 * f4] = pack_bf16x2(acc.x, acc.y);
        w[2 * f4 + 1] = pack_bf16x2(acc.z, acc.w);
        if ((f4 & 3) == 3) __syncwarp();   // loads hoisted four groups ahead at most (registers)
    }
}

// Page ids of one unit's blocks for a whole warp: lanes hold blocks [base, base + 32), slid
// forward as the tiles advance.  row(blk) is the TMA row coordinate page * 64, or the first
// row past the pool (read as zeros) for a block past the unit or a bad page id.
struct PageWindow {
    const int32_t* bt_row;
    int kb1, base, lane, pg;
    int64_t num_pages;
    bool report;
    __device__ int fetch(int idx) {
        const int v = idx < kb1 ? __ldg(bt_row + idx) : -1;
        const bool bad = idx < kb1 && (v < 0 || (int64_t)v >= num_pages);
        if (__any_sync(0xffffffffu, bad) && lane == 0 && report) raise_error(1 /* MLA_DEVERR_PAGE_OUT_OF_RANGE */);
        return (idx < kb1 && !bad) ? v : -1;
    }
    __device__ void init(const int32_t* row, int kb0_, int kb1_, int lane_, int64_t np, bool rep) {
        bt_row = row;
        kb1 = kb1_;
        base = kb0_;
        lane = lane_;
        num_pages = np;
        report = rep;
        pg = fetch(base + lane);
    }
    __device__ int32_t row(int blk) {
        const int32_t past = (int32_t)(num_pages * kPage);
        if (blk >= kb1) return past;
        while (blk >= base + 32) {
            base += 32;
            pg = fetch(base + lane);
        }
        const int v = __shfl_sync(0xffffffffu, pg, blk - base);
        return v >= 0 ? v * kPage : past;
    }
};

// kKv: the cache's element type, 0 bf16, 1 e4m3, 2 e5m2 (both 8-bit caches are widened to f16
// for the MMAs); kFp8Q: e4m3 queries (requires an e4m3 cache).
template <int kKv, bool kFp8Q>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap v_map,
                  const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap po_map,
                  const __grid_constant__ CUtensorMap pl_map, const __grid_constant__ CUtensorMap o_map,
                  const __grid_constant__ CUtensorMap ps_map, const __grid_constant__ Params p) {
    constexpr bool kFp8 = kKv != 0;
    constexpr bool kE5M2 = kKv == 2;
    static_assert(kKv == 1 || !kFp8Q, "e4m3 queries need an e4m3 cache");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* pending = reinterpret_cast<int*>(smem + kOffMisc + 8);   // count, then (ub, s0, n) x 2

    const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);   // warp-uniform to the compiler
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int part = blockIdx.x >> 1;
    const int mtile = blockIdx.y;
    // Launched as a programmatic dependent of the metadata step, this grid is scheduled while
    // that step still runs: the set-up below (barriers, tensor memory, descriptors) reads
    // nothing another grid writes, and overlaps it.

    if (threadIdx.x == 0) {
        for (int s = 0; s < kKSlots; ++s) {
            // bf16: one arrival + the pair's TMA bytes; e4m3: the leader's widening warp
            // arrives, the peer's signal by st.async
            mbar_init(bar(kBarKFull + s), 1);
            mbar_init(bar(kBarKEmpty + s), 1);
            mbar_init(bar(kBarQKDone + s), 1);
            mbar_init(bar(kBarVFull + s), kFp8 ? 4 : 1);
            mbar_init(bar(kBarKRaw + s), 1);
        }
        // the eight Q warps of the pair, plus the Q TMA's arrival in the bf16 path
        // bf16: the Q TMA + 4 warps' tensor-memory stores; e4m3 cache: the 4 warps; e4m3 q: the TMA
        mbar_init(bar(kBarQFull), kFp8Q ? 1 : (kFp8 ? 0 : 1) + 4);
        mbar_init(bar(kBarVWiden), 128);
        mbar_init(bar(kBarFold), 1);
        mbar_init(bar(kBarFoldRd), 128);
        mbar_init(bar(kBarFoldL), 1);
        mbar_init(bar(kBarMerge), 1);
        mbar_init(bar(kBarQEmpty), 1);
        for (int j = 0; j < 2; ++j) {
            mbar_init(bar(kBarSFull + j), 1);
            mbar_init(bar(kBarSFree + j), 4);
        }
        mbar_init(bar(kBarPFull), 4);
        mbar_init(bar(kBarPvDone), 1);
        mbar_init(bar(kBarOFull), 1);
        mbar_init(bar(kBarOEmpty), 4);
        mbar_init(bar(kBarXchg), 128);
        mbar_init(bar(kBarXchg + 1), 128);
        mbar_init(bar(kBarLx), 128);
        mbar_init(bar(kBarPartial), 128);
        *abort_flag = 0;
        pending[0] = 0;
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
        prefetch_tensormap(&po_map);
        prefetch_tensormap(&pl_map);
        prefetch_tensormap(&o_map);
        prefetch_tensormap(&ps_map);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    // Everything from here on may read what the preceding grids wrote (plan, page table,
    // lengths, queries, cache, the workspace's arrival words): wait for them to complete.
    // Without a programmatic launch this returns at once.  Only then is the merge kernel that
    // follows let in, since it reads num_splits before it waits for this grid.
    pdl_wait_prerequisites();
    pdl_launch_dependents();
    bool md_ok = true;
    UnitIter iter = make_iter(p, part, md_ok);
    const uint32_t tmem = *tmem_slot;
    // (the partner's flag was zeroed before the cluster barrier above)
    const AbortCtl actl{abort_flag, map_to_cta(smem_u32(tmem_slot + 1), rank ^ 1u), p.wait_budget_ns};

    const uint64_t kv_pol = l2_policy_evict_first();
    const uint64_t part_pol = l2_policy_evict_last();
    if (!md_ok && threadIdx.x == 0) raise_error(8 /* MLA_DEVERR_BAD_METADATA */);

    // A warp publishing shared-memory data (written with st.shared, then fence.proxy.async by
    // every writing thread) or reporting a finished tensor-memory access to the leader's MMA
    // issuer: the leader's warp arrives with expect_tx of 4 bytes, the peer's warp sends a
    // 4-byte st.async whose complete_tx lands on the leader's barrier (word: a landing slot of
    // its own in the leader).  A remote release arrive took ~1000 cycles longer to reach the
    // leader.
    auto signal_leader = [&](int b_idx, int word) {
        __syncwarp();
        if (lane == 0) {
            if (leader)
                mbar_arrive_expect_tx(bar(b_idx), 4);
            else
                st_async_b32(map_to_cta(sbase + kOffPSig + 4u * (uint32_t)word, 0), 0u,
                             map_to_cta(bar(b_idx), 0));
        }
    };

    if (warp == 0 || warp == 3) {
        // ------------------------------------------------------------ K producers
        // Each tile's page (this CTA's page, all 576 columns) is one load, warps 0 / 3 taking
        // alternate tiles: 72 KB of bf16 completing the leader's barrier, or 36 KB of e4m3 that
        // the loading warp widens in place before it signals the leader.
        const uint32_t mine = warp == 3 ? 1u : 0u;
        uint32_t g = 0;
        bool alive = true;
        int ub, kb0, kb1;
        while (alive && iter.next(ub, kb0, kb1)) {
            const int n = tiles_of(kb0, kb1);
            if (n <= 0) continue;
            PageWindow pw;
            pw.init(p.block_table + (int64_t)ub * p.bt_stride, kb0, kb1, lane, p.num_pages, warp == 0);
            for (int i = 0; i < n; ++i, ++g) {
                const int32_t row = pw.row(kb0 + 2 * i + (int)rank);
                if ((g & 1u) != mine) continue;
                int ok = 1;
                const int s = (int)(g & 1u);
                const uint32_t slot = sbase + kOffK + s * kKSlotBytes;
                // test hook: the leader withholds one tile's page, so a wait runs out
                const bool withhold = leader && (int)g == p.withhold_tile;
                if (lane == 0) {
                    ok = mbar_wait_bounded(bar(kBarKEmpty + s), ((g >> 1) & 1u) ^ 1u, actl);
                    if (ok && !withhold) {
                        if constexpr (kFp8 && !kFp8Q) {
                            mbar_arrive_expect_tx(bar(kBarKRaw + s), kPage8Bytes);
                            tma_load_3d_hint(slot + kRaw8Off, &k_map, bar(kBarKRaw + s), 0, row, 0, kv_pol);
                        } else {
                            // the pair's pages complete the leader's barrier: bf16 pages, or raw
                            // e4m3 pages that S reads as they are (e4m3 queries)
                            const uint32_t kf = bar(kBarKFull + s);
                            if (leader) mbar_arrive_expect_tx(kf, kFp8Q ? 2 * kPage8Bytes : 2 * kChunks * kBox);
                            tma_load_3d_pair_hint(kFp8Q ? slot + kRaw8Off : slot, &k_map, map_to_cta(kf, 0), 0, row,
                                                  0, kv_pol);
                        }
                    }
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    alive = false;
                    break;
                }
                if constexpr (kFp8 && !kFp8Q) {
                    // the whole warp widens the page in place, then signals the leader
                    const bool landed = mbar_wait_bounded(bar(kBarKRaw + s), (g >> 1) & 1u, actl);
                    if (!__all_sync(0xffffffffu, landed)) {
                        alive = false;
                        break;
                    }
#pragma unroll 1
                    for (int c = 0; c < kChunks; ++c)
                        widen_chunk_fp8<kE5M2>(slot + kRaw8Off + c * kChunk8, slot + c * kBox, lane);
                    fence_proxy_async_smem();
                    signal_leader(kBarKFull + s, 8);
                }
            }
        }
        if (lane == 0 && *abort_flag) {
            // let copies already issued land before shared memory can go away
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 200000ull) {
            }
        }
    } else if (warp >= kQWarp0) {
        // ------------------------------------------------------------ Q and partner V
        // Per unit, once the previous unit's last S MMA has finished: warp kQWarp0 + 3
        // (lane 0) loads Q columns [256, 576) of the CTA's 64 rows by TMA (bf16 cache), and
        // the four warps write Q columns [0, 256) into tensor memory, thread = lane.  A pair
        // MMA reads an A operand from tensor memory for output columns [0, N/2) in lanes
        // 0..63 and for [N/2, N) in lanes 64..127, so each row lies twice: lane r and 64 + r.
        // Per tile, the 128 threads load the four chunks of the partner page this CTA
        // supplies to the PV MMAs (columns 256n + 128r + [0, 128), n = 0, 1; an L2 hit, the
        // partner CTA loads that page) into registers ahead of time, and once the tile's S
        // MMAs are done store them (widened to f16 from an e4m3 cache) into the slot
        // positions 4n + 2(1 - r), + 1, which held this CTA's own, now dead, chunks.
        // Warp kQWarp0 + 2 (lane 0) first prefetches the query rows of the part's later
        // units into L2.
        const int quarter = warp & 3;
        const int qt = threadIdx.x - kQWarp0 * 32;          // 0..127
        const int rloc = (32 * quarter + lane) & 63;
        const int rowg = mtile * kRows + kCtaRows * (int)rank + rloc;
        const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
        if (quarter == 2 && lane == 0) {
            UnitIter pk = iter;
            int nb, a0, a1;
            bool first = true;
            while (pk.next(nb, a0, a1)) {
                if (tiles_of(a0, a1) <= 0) continue;
                if (!first) {
                    tma_prefetch_4d(&q_map, 0, mtile * kRows + kCtaRows * (int32_t)rank, 0, nb);
                    if (!kFp8Q)   // the bf16 view's box is five chunks: two prefetches cover a row
                        tma_prefetch_4d(&q_map, 0, mtile * kRows + kCtaRows * (int32_t)rank, kQLoChunks, nb);
                }
                first = false;
            }
        }
        uint32_t uq = 0, g = 0;
        bool q_range = false, alive = true;
        int ub, kb0, kb1;
        while (alive && iter.next(ub, kb0, kb1)) {
            const int n = tiles_of(kb0, kb1);
            if (n <= 0) continue;
            // ---- Q of the unit
            if (uq > 0 && !mbar_wait_bounded(bar(kBarQEmpty), (uq - 1) & 1u, actl)) break;
            tc_fence_after();
            if constexpr (kFp8Q) {
                // e4m3 codes of the CTA's 64 rows, all 576 columns: one 36 KB TMA (64-byte swizzle)
                if (quarter == 3 && lane == 0) {
                    if (leader) mbar_arrive_expect_tx(bar(kBarQFull), 2 * kQ8Bytes);
                    tma_load_4d_pair(sbase + kOffQ, &q_map, map_to_cta(bar(kBarQFull), 0), 0,
                                     mtile * kRows + kCtaRows * (int32_t)rank, 0, ub);
                }
            } else {
                if (!kFp8 && quarter == 3 && lane == 0) {
                    if (leader) mbar_arrive_expect_tx(bar(kBarQFull), 2 * kQHiBytes);
                    tma_load_4d_pair(sbase + kOffQ, &q_map, map_to_cta(bar(kBarQFull), 0), 0,
                                     mtile * kRows + kCtaRows * (int32_t)rank, kQLoChunks, ub);
                }
                const uint4* src = reinterpret_cast<const uint4*>(p.q + ((int64_t)ub * p.rows + rowg) * kDqk);
                {
                    uint4 v[32];   // the row's columns [0, 256): all loads in flight at once
    #pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] = rowg < p.rows ? __ldg(src + k) : make_uint4(0, 0, 0, 0);
    #pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t w[16];
    #pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            w[4 * k] = v[4 * c + k].x;
                            w[4 * k + 1] = v[4 * c + k].y;
                            w[4 * k + 2] = v[4 * c + k].z;
                            w[4 * k + 3] = v[4 * c + k].w;
                        }
                        if constexpr (kFp8) {
    #pragma unroll
                            for (int k = 0; k < 16; ++k) w[k] = bf16x2_to_f16x2(w[k], q_range);
                        }
                        tmem_st16(tmem + lane_off + kTmemQ + 16u * c, w);
                    }
                }
                if constexpr (kFp8) {
                    // Q columns [256, 576) as f16 into shared memory (128-byte swizzle): lane
                    // quarters 0 / 1 take chunks 0..2 of them, quarters 2 / 3 chunks 3..4
                    const int c0 = quarter < 2 ? 0 : 3, c1 = quarter < 2 ? 3 : kQHiChunks;
    #pragma unroll 1
                    for (int cc = c0; cc < c1; ++cc) {
                        const uint32_t qrow = sbase + kOffQ + cc * kBox + (uint32_t)rloc * 128u;
                        uint4 v[8];
    #pragma unroll
                        for (int u = 0; u < 8; ++u) v[u] = rowg < p.rows ? __ldg(src + 32 + 8 * cc + u) : make_uint4(0, 0, 0, 0);
    #pragma unroll
                        for (int u = 0; u < 8; ++u)
                            st_shared_v4u(qrow + 16u * ((uint32_t)u ^ ((uint32_t)rloc & 7u)),
                                          bf16x2_to_f16x2(v[u].x, q_range), bf16x2_to_f16x2(v[u].y, q_range),
                                          bf16x2_to_f16x2(v[u].z, q_range), bf16x2_to_f16x2(v[u].w, q_range));
                    }
                    fence_proxy_async_smem();
                    if (__any_sync(0xffffffffu, q_range) && lane == 0) raise_error(32 /* MLA_DEVERR_Q_RANGE */);
                }
                tc_wait_st();
                tc_fence_before();
                signal_leader(kBarQFull, 9 + quarter);
            }
            ++uq;
            // ---- partner V of each tile of the unit
            const int32_t* bt_row = p.block_table + (int64_t)ub * p.bt_stride;
            for (int i = 0; i < n; ++i, ++g) {
                const int blk = kb0 + 2 * i + 1 - (int)rank;
                int pg = blk < kb1 ? __ldg(bt_row + blk) : -1;
                if (pg < 0 || (int64_t)pg >= p.num_pages) pg = -1;   // reported by the K loads
                const int s = (int)(g & 1u);
                const uint32_t slot = sbase + kOffK + s * kKSlotBytes;
                if constexpr (!kFp8) {
                    // by TMA, after the tile's S MMAs: two 16 KB loads, lane 0 of the last warp
                    if (quarter == 3) {
                        int ok = 1;
                        if (lane == 0) {
                            ok = mbar_wait_bounded(bar(kBarQKDone + s), (g >> 1) & 1u, actl);
                            if (ok) {
                                if (leader) mbar_arrive_expect_tx(bar(kBarVFull + s), 2 * 2 * 2 * kBox);
                                const int32_t row = pg >= 0 ? pg * kPage : (int32_t)(p.num_pages * kPage);
#pragma unroll
                                for (int nn = 0; nn < 2; ++nn)
                                    tma_load_3d_pair_hint(slot + (4 * nn + 2 * (1 - (int)rank)) * kBox, &v_map,
                                                          map_to_cta(bar(kBarVFull + s), 0), 0, row,
                                                          4 * nn + 2 * (int)rank, kv_pol);
                            }
                        }
                        if (!__shfl_sync(0xffffffffu, ok, 0)) {
                            alive = false;
                            break;
                        }
                    }
                } else {
                    // 4 chunks x 64 rows x 4 sixteen-byte units of e4m3: 8 per thread, widened to
                    // f16 on the way into the slot
                    uint4 v[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int x = qt + 128 * j, h = x >> 8, row = (x >> 2) & 63, q4 = x & 3;
                        const int chunk = 4 * (h >> 1) + 2 * (int)rank + (h & 1);
                        v[j] = pg >= 0 ? __ldg(reinterpret_cast<const uint4*>(
                                             p.kv + ((int64_t)pg * kPage + row) * kDqk + chunk * 64 + q4 * 16))
                                       : make_uint4(0, 0, 0, 0);
                    }
                    const bool done = mbar_wait_bounded(bar(kBarQKDone + s), (g >> 1) & 1u, actl);
                    if (!__all_sync(0xffffffffu, done)) {
                        alive = false;
                        break;
                    }
                    if constexpr (kFp8Q) {
                        // S read the raw page; now this CTA's own V chunks (4n + 2 rank + h, one per
                        // warp) are widened to f16 into the positions of the same index.  A widened
                        // chunk (8 KB) can cover raw chunks (4 KB, in the slot's back half) that other
                        // warps read, and so can the partner chunks stored below: every warp reads its
                        // raw chunk before any warp writes.
                        const int oc = 4 * (quarter >> 1) + 2 * (int)rank + (quarter & 1);
                        uint4 w[8];
                        load_chunk_sw64(slot + kRaw8Off + oc * kChunk8, lane, w);
                        mbar_arrive(bar(kBarVWiden));
                        const bool read_all = mbar_wait_bounded(bar(kBarVWiden), g & 1u, actl);
                        if (!__all_sync(0xffffffffu, read_all)) {
                            alive = false;
                            break;
                        }
                        store_chunk_f16(slot + oc * kBox, lane, w);
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int x = qt + 128 * j, h = x >> 8, row = (x >> 2) & 63, q4 = x & 3;
                        const int pos = 4 * (h >> 1) + 2 * (1 - (int)rank) + (h & 1);
                        const uint32_t r = slot + pos * kBox + row * 128;
                        const uint32_t sw = (uint32_t)row & 7u;
                        st_shared_v4u(r + 16u * ((2u * q4) ^ sw), fp8x2_to_f16x2<kE5M2>(v[j].x),
                                      fp8x2_to_f16x2<kE5M2>(v[j].x >> 16), fp8x2_to_f16x2<kE5M2>(v[j].y),
                                      fp8x2_to_f16x2<kE5M2>(v[j].y >> 16));
                        st_shared_v4u(r + 16u * ((2u * q4 + 1u) ^ sw), fp8x2_to_f16x2<kE5M2>(v[j].z),
                                      fp8x2_to_f16x2<kE5M2>(v[j].z >> 16), fp8x2_to_f16x2<kE5M2>(v[j].w),
                                      fp8x2_to_f16x2<kE5M2>(v[j].w >> 16));
                    }
                    fence_proxy_async_smem();
                    signal_leader(kBarVFull + s, 4 + quarter);
                }
            }
        }
        if ((!kFp8 || kFp8Q) && quarter == 3 && lane == 0 && *abort_flag) {
            // let copies already issued land before shared memory can go away
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 200000ull) {
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        // Two cursors walk the same tiles: S(t) = Q K^T and O += P(t) V(t).  Whichever is
        // ready goes first, PV before S: a slot is only refilled after its tile's PV, so a
        // PV that waits behind an S whose page is still in flight would stall the ring.
        // S(t) waits for its page, its S buffer (the softmax read S(t - 2)) and, first in a
        // unit, the unit's Q; PV(t) waits for P(t), the partner V of tile t and, first in a
        // unit, the epilogue of the previous unit having read O.
        if (leader) {
            // The whole warp walks the schedule (an elected lane issues each MMA, see
            // mma_pair_ss).  Non-blocking barrier tests at CTA scope: the data behind a barrier
            // the peer completes is ordered by the peer's fence.proxy.async and the st.async /
            // TMA complete_tx itself (measured ~1% faster than cluster-scope acquire); the vote
            // keeps every decision warp-uniform.
            auto poll = [](uint32_t b, uint32_t parity) -> bool {
                return __all_sync(0xffffffffu, mbar_test_wait(b, parity));
            };
            struct Cursor {
                UnitIter it;
                int n, i;
                uint32_t g, uq;
                bool valid;
                __device__ void next_unit() {
                    int ub_, a_, b_;
                    valid = false;
                    while (it.next(ub_, a_, b_)) {
                        n = tiles_of(a_, b_);
                        if (n > 0) {
                            i = 0;
                            valid = true;
                            return;
                        }
                    }
                }
                __device__ void step() {
                    ++g;
                    if (++i == n) {
                        ++uq;
                        next_unit();
                    }
                }
            };
            Cursor cq, cp;
            cq.it = iter;
            cq.g = 0;
            cq.uq = 0;
            cq.next_unit();
            cp = cq;
            uint64_t t_idle = global_timer_ns();
            while (cq.valid || cp.valid) {
                bool did = false;
                if (cp.valid && cp.g < cq.g) {
                    const int s = (int)(cp.g & 1u);
                    const bool first = cp.i == 0;
                    if (poll(bar(kBarPFull), cp.g & 1u) && poll(bar(kBarVFull + s), (cp.g >> 1) & 1u) &&
                        (!first || cp.uq == 0 || poll(bar(kBarOEmpty), (cp.uq - 1) & 1u))) {
                        tc_fence_after();
                        const uint32_t pbuf = sbase + kOffP;
                        const uint32_t slot = sbase + kOffK + s * kKSlotBytes;
#pragma unroll
                        for (int nn = 0; nn < 2; ++nn)
#pragma unroll
                            for (int pp = 0; pp < 2; ++pp)
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    mma_pair_ss(tmem + kTmemO + 128u * nn,
                                                smem_desc_sw128(pbuf + pp * kBox + 32u * kk, 16, 1024),
                                                smem_desc_sw128(slot + (4 * nn + 2 * pp) * kBox + 2048u * kk, kBox, 1024),
                                                kFp8 ? kIdescPV16 : kIdescPV, (first && pp == 0 && kk == 0) ? 0u : 1u);
                        tc_commit_pair(bar(kBarKEmpty + s));
                        tc_commit_pair(bar(kBarPvDone));
                        if (cp.i == cp.n - 1) tc_commit_pair(bar(kBarOFull));
                        cp.step();
                        did = true;
                    }
                }
                if (!did && cq.valid) {
                    const int s = (int)(cq.g & 1u);
                    const uint32_t sb = cq.g & 1u;
                    if ((cq.i != 0 || poll(bar(kBarQFull), cq.uq & 1u)) &&
                        (cq.g < 2 || poll(bar(kBarSFree + sb), ((cq.g >> 1) & 1u) ^ 1u)) &&
                        poll(bar(kBarKFull + s), (cq.g >> 1) & 1u)) {
                        tc_fence_after();
                        const uint32_t slot = sbase + kOffK + s * kKSlotBytes;
                        const uint32_t d = tmem + kTmemS + 64u * sb;
                        if constexpr (kFp8Q) {
                            // e4m3 x e4m3, K = 32: two MMAs per 64-byte chunk
#pragma unroll
                            for (int c = 0; c < kChunks; ++c)
#pragma unroll
                                for (int kk = 0; kk < 2; ++kk)
                                    mma_pair_ss_f8(d, smem_desc_sw64(sbase + kOffQ + c * kChunk8 + 32u * kk),
                                                   smem_desc_sw64(slot + kRaw8Off + c * kChunk8 + 32u * kk),
                                                   kIdescQK8, (c | kk) ? 1u : 0u);
                        } else {
#pragma unroll
                            for (int c = 0; c < kChunks; ++c) {
                                if (c < kQLoChunks) {
#pragma unroll
                                    for (int kk = 0; kk < 4; ++kk)
                                        mma_pair_ts(d, tmem + kTmemQ + 32u * c + 8u * kk,
                                                    smem_desc_sw128(slot + c * kBox + 32u * kk, 16, 1024),
                                                    kFp8 ? kIdescQK16 : kIdescQK, (c | kk) ? 1u : 0u);
                                } else {
#pragma unroll
                                    for (int kk = 0; kk < 4; ++kk)
                                        mma_pair_ss(d, smem_desc_sw128(sbase + kOffQ + (c - kQLoChunks) * kBox + 32u * kk, 16, 1024),
                                                    smem_desc_sw128(slot + c * kBox + 32u * kk, 16, 1024),
                                                    kFp8 ? kIdescQK16 : kIdescQK, 1u);
                                }
                            }
                        }
                        tc_commit_pair(bar(kBarQKDone + s));
                        tc_commit_pair(bar(kBarSFull + sb));
                        if (cq.i == cq.n - 1) tc_commit_pair(bar(kBarQEmpty));
                        cq.step();
                        did = true;
                    }
                }
                if (did) {
                    t_idle = global_timer_ns();
                } else {
                    if (*abort_flag) break;
                    if (global_timer_ns() - t_idle > actl.budget_ns) {
                        if (lane == 0) raise_abort(actl);
                        break;
                    }
                }
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

        uint32_t g = 0, uq = 0, npartial = 0;
        bool alive = true;
        int ub, kb0, kb1;
        while (alive && iter.next(ub, kb0, kb1)) {
            const int n = tiles_of(kb0, kb1);
            if (n <= 0) {
                write_empty(ub);
                continue;
            }
            const int L = p.cache_seqlens[ub];
            // where the unit's result goes, read now so that the epilogue does not wait for it
            bool last_unit;
            {
                UnitIter rest = iter;
                int b_, a_, c_;
                last_unit = !rest.next(b_, a_, c_);
            }
            const int pieces = p.num_splits[ub + 1] - p.num_splits[ub];
            const bool direct = pieces == 1;
            const int split = p.num_splits[ub] + (ub == iter.first_b ? p.md[8 * part + 4] : 0);
            int lim = p.causal ? L - p.q_len + iq + 1 : L;
            if (lim > L) lim = L;
            if (lim > kb1 * kPage) lim = kb1 * kPage;   // keys of this unit only
            float m_run = -INFINITY, l_half = 0.f;
            // A piece of a request merged in this kernel claims its place once the last tile's P is
            // written, so that the atomic's round trip overlaps the last PV (acquire: a claim that
            // finds every other piece stored also sees their rows).
            int32_t* const arrival = p.arrivals + ((int64_t)ub * gridDim.y + mtile) * 2 + rank;
            const bool merged_here = !direct && pieces <= kFusedMergeMaxPieces;
            int claim_old = 0;
            for (int i = 0; i < n; ++i, ++g) {
                const uint32_t sb = g & 1u;
                if (!mbar_wait_bounded(bar(kBarSFull + sb), (g >> 1) & 1u, actl)) {
                    alive = false;
                    break;
                }
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
                tc_fence_before();
                signal_leader(kBarSFree + sb, 16 + (warp - kSoftmaxWarp0));
                // scale to log2 units, mask the keys at or past the limit (only a tile that
                // reaches it has any), this half's maximum
                const int kbase = (kb0 + 2 * i) * kPage + kPage * half;
#pragma unroll
                for (int j = 0; j < 64; j += 2) mul2(s[j], s[j + 1], sl2);
                if (kbase + 64 > lim) {
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        if (kbase + j >= lim) s[j] = -INFINITY;
                }
                float hmax;
                {
                    float m0 = fmaxf(s[0], s[1]), m1 = fmaxf(s[2], s[3]);
#pragma unroll
                    for (int j = 4; j < 64; j += 4) {
                        m0 = fmax3(m0, s[j], s[j + 1]);
                        m1 = fmax3(m1, s[j + 2], s[j + 3]);
                    }
                    hmax = fmaxf(m0, m1);
                }
                // partner thread t ^ 64 holds the other 64 tokens of this row
                xmax[sb * 128 + t] = hmax;
                mbar_arrive(bar(kBarXchg + sb));
                if (!mbar_wait_bounded(bar(kBarXchg + sb), (g >> 1) & 1u, actl)) {
                    alive = false;
                    break;
                }
                const float tmax = fmaxf(hmax, xmax[sb * 128 + (t ^ 64)]);
                const float m_new = fmaxf(m_run, tmax);
                const bool rescale = m_new > m_run + kRescaleThreshold;
                float factor = 1.f;
                if (rescale) {
                    factor = fast_exp2(m_run - m_new);  // 0 when m_run = -inf
                    l_half *= factor;
                    m_run = m_new;
                }
                // P packed as bf16 pairs into s[0..31] (s[2j], s[2j+1] are read before s[j]
                // is overwritten, since 2j >= j); nothing but zeros while every key so far is masked.
                if (m_run != -INFINITY) {
                    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        float p0 = s[2 * j], p1 = s[2 * j + 1];
                        sub2(p0, p1, m_run);
                        p0 = fast_exp2(p0);
                        p1 = fast_exp2(p1);
                        add2(ps0, ps1, p0, p1);
                        s[j] = __uint_as_float(kFp8 ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1));
                    }
                    l_half += ps0 + ps1;
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) s[j] = 0.f;
                }
                // the P buffer is free, and O holds every PV up to tile g - 1, once PV(g - 1)
                // has finished
                if (g >= 1 && !mbar_wait_bounded(bar(kBarPvDone), (g - 1) & 1u, actl)) {
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
                __syncwarp();
                if (lane == 0) {
                    if (leader)
                        mbar_arrive_expect_tx(bar(kBarPFull), 4);
                    else
                        st_async_b32(map_to_cta(sbase + kOffPSig + 4u * (uint32_t)(warp - kSoftmaxWarp0), 0), g,
                                     map_to_cta(bar(kBarPFull), 0));
                }
                if (t == 0 && merged_here && i == n - 1) claim_old = atom_add_acquire_gpu(arrival, 1);
            }
            if (!alive) break;
            // epilogue of the unit
            if (!mbar_wait_bounded(bar(kBarOFull), uq & 1u, actl)) break;
            tc_fence_after();
            // How this piece ends (t == 0 decides from its claim): 0 whole request (or a piece of
            // one merged by the merge kernel), 1 store the partial rows and count them, 2 the last
            // claimer in its part's last unit (Q, K ring and P idle): fold the other pieces' rows
            // into its own O and write the final o, 3 the last claimer elsewhere: store, then merge
            // at the end of the part.
            if (t == 0) {
                int mode = 0;
                if (merged_here) {
                    const int claimed = claim_old & 0xFFFF, stored = (claim_old >> 16) & 0x7FFF;
                    mode = 1;
                    if (claim_old < 0 || claimed >= pieces || stored > claimed)
                        raise_error(128 /* MLA_DEVERR_WORKSPACE_STATE */);
                    else if (claimed == pieces - 1)
                        mode = (p.fold_ok && last_unit && pieces <= kFoldMaxPieces) ? 2 : 3;
                }
                pending[kMiscFold] = mode;
            }
            xmax[256 + t] = l_half;
            mbar_arrive(bar(kBarLx));
            if (!mbar_wait_bounded(bar(kBarLx), uq & 1u, actl)) break;
            const int mode = pending[kMiscFold];
            const bool fold = mode == 2;
            const float l_run = l_half + xmax[256 + (t ^ 64)];
            // the partial state in the stored form (also the fold's own piece)
            const float inv = l_run > 0.f ? dk / l_run : 0.f;
            float lse_val = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
            // fold-in: the pieces' weights in split-slot order, as the merge of stored partials
            // computes them (so that the result does not depend on which piece merges)
            float wts[kFoldMaxPieces];
            // this piece's index in the request (nonzero only for a part's first unit) and the
            // request's first split slot, read only where a merge needs them
            const int own = (mode >= 2 && ub == iter.first_b) ? p.md[8 * part + 4] : 0;
            const int s0 = split - own;
            const int row_base = mtile * kRows + kCtaRows * (int)rank;
            // rows past this CTA's last (a partial query tile) load the next piece's rows, or
            // zeros past the workspace: loaded, never used
            // (one TMA operation brings eight boxes; in the first round the other pieces' 64 lse
            // values come too, into the row-max exchange area, idle now: piece j at 256 j bytes)
            auto fold_issue = [&](int round) {
                const int nbox = pieces == 2 ? kFoldBoxes : kFoldBoxes / 2;
                if (round == 0) mbar_arrive_expect_tx(bar(kBarFoldL), (uint32_t)((pieces - 1) * kCtaRows * 4));
                mbar_arrive_expect_tx(bar(kBarFold), (uint32_t)((pieces - 1) * nbox * kFoldBoxBytes));
#pragma unroll 1
                for (int j = 0; j < pieces - 1; ++j) {
                    const int slot = s0 + j + (j >= own ? 1 : 0);
                    if (round == 0)
                        tma_load_2d(sbase + kOffX + 256u * (uint32_t)j, &pl_map, bar(kBarFoldL), row_base, slot);
#pragma unroll 1
                    for (int c = 0; c < nbox; c += 8)
                        tma_load_3d(sbase + kOffQ + (uint32_t)((pieces == 2 ? c : 8 * j + c) * kFoldBoxBytes), &po_map,
                                    bar(kBarFold), 0, slot * p.rows + row_base, 8 * round + c);
                }
            };
            if (fold) {
                if (t == 0) {
                    // the others have claimed before this piece: unless the claim found them all
                    // stored, wait until they have
                    if (((claim_old >> 16) & 0x7FFF) >= pieces - 1 || wait_stored(arrival, pieces - 1, actl)) {
                        *arrival = 0;   // every piece is done with the word: ready for the next call
                        fence_proxy_async_global();   // the acquired partial rows, read by the async proxy
                        fence_proxy_async_smem();     // the exchange area, written by the async proxy
                        fold_issue(0);
                    }
                }
                // the weights while the rows are in flight (one fold per CTA at most: phase 0)
                if (!mbar_wait_bounded(bar(kBarFoldL), 0u, actl)) break;
                float m = -INFINITY;
#pragma unroll
                for (int i = 0; i < kFoldMaxPieces; ++i) {
                    wts[i] = -INFINITY;
                    if (i < pieces)
                        wts[i] = i == own ? lse_val : (row_valid ? xmax[64 * (i - (i > own ? 1 : 0)) + rloc] : -INFINITY);
                    m = fmaxf(m, wts[i]);
                }
                if (m == -INFINITY) {
#pragma unroll
                    for (int i = 0; i < kFoldMaxPieces; ++i) wts[i] = 0.f;   // no key in any piece: o = 0
                    lse_val = -INFINITY;
                } else {
                    float sum = 0.f;
#pragma unroll
                    for (int i = 0; i < kFoldMaxPieces; ++i)
                        if (i < pieces) sum += expf(wts[i] - m);
                    lse_val = m + logf(sum);
#pragma unroll
                    for (int i = 0; i < kFoldMaxPieces; ++i) wts[i] = i < pieces ? expf(wts[i] - lse_val) : 0.f;
                }
                if (!mbar_wait_bounded(bar(kBarFold), 0u, actl)) break;
            }
            const bool write_final = direct || fold;
            bool ep_ok = true;
            // Each warp holds 32 rows.  A step reads 64 tensor-memory columns of its rows (one
            // wait) and moves them, 128 bytes of each row at a time (64 bf16 outputs, or 32 fp32
            // partial columns: two passes), through a per-warp staging area, so that every global
            // store writes whole 128-byte lines (8 lanes per row).  TMEM columns [128 + 64 st, +64)
            // hold outputs 256 (st / 2) + 128 half + 64 (st % 2) + [0, 64).
            {
                // staging: the warp's own 4 KB and its 4 KB of the P buffer (idle until this
                // warp writes the next unit's first P)
                const uint32_t stage_a = sbase + kOffStage + (uint32_t)(warp - kSoftmaxWarp0) * 4096u;
                const uint32_t stage_b = sbase + kOffP + (uint32_t)(warp - kSoftmaxWarp0) * 4096u;
                uint32_t npass = 0;
                const int row0 = mtile * kRows + kCtaRows * (int)rank + 32 * ((warp - kSoftmaxWarp0) & 1);
#pragma unroll 1
                for (int st = 0; st < 4; ++st) {
                    if (fold && pieces > 2 && st == 2) {
                        // second fold-in round: columns [256, 512) of the other pieces, once every
                        // thread has read the first round
                        mbar_arrive(bar(kBarFoldRd));
                        if (!mbar_wait_bounded(bar(kBarFoldRd), 0u, actl)) {
                            ep_ok = false;
                            break;
                        }
                        if (t == 0) fold_issue(1);
                        if (!mbar_wait_bounded(bar(kBarFold), 1u, actl)) {
                            ep_ok = false;
                            break;
                        }
                    }
                    uint32_t raw[64];
                    tmem_ld16(tmem + lane_off + kTmemO + 64u * st, *reinterpret_cast<uint32_t(*)[16]>(raw));
                    tmem_ld16(tmem + lane_off + kTmemO + 64u * st + 16u, *reinterpret_cast<uint32_t(*)[16]>(raw + 16));
                    tmem_ld16(tmem + lane_off + kTmemO + 64u * st + 32u, *reinterpret_cast<uint32_t(*)[16]>(raw + 32));
                    tmem_ld16(tmem + lane_off + kTmemO + 64u * st + 48u, *reinterpret_cast<uint32_t(*)[16]>(raw + 48));
                    tc_wait_ld();
                    if (st == 3) {
                        tc_fence_before();
                        signal_leader(kBarOEmpty, 20 + (warp - kSoftmaxWarp0));   // O is free for the next unit
                    }
#pragma unroll
                    for (int pass = 0; pass < 2; ++pass) {
                        if (write_final && pass == 1) break;
                        uint32_t w[32];
                        int col;
                        if (fold) {
                            // sum over the pieces in slot order of weight x normalised partial row,
                            // this piece's own from tensor memory (rounded as its stored partial
                            // would be), the others' from the staged boxes: columns col .. col + 63
                            // are boxes cb0 and cb0 + 1 of each other piece
                            col = 256 * (st >> 1) + 128 * half + 64 * (st & 1);
                            const int cb0 = col / kFoldBoxCols;
                            const uint32_t stg = sbase + kOffQ;
                            const uint32_t b2 = stg + (uint32_t)cb0 * kFoldBoxBytes;
                            const uint32_t b30 = stg + (uint32_t)(cb0 & 7) * kFoldBoxBytes;
                            const uint32_t b31 = stg + (uint32_t)(8 + (cb0 & 7)) * kFoldBoxBytes;
                            switch (3 * (pieces - 2) + own) {   // uniform over the CTA
                            case 0: fold_step<2, 0>(raw, w, inv, wts, b2, 0u, rloc); break;
                            case 1: fold_step<2, 1>(raw, w, inv, wts, b2, 0u, rloc); break;
                            case 3: fold_step<3, 0>(raw, w, inv, wts, b30, b31, rloc); break;
                            case 4: fold_step<3, 1>(raw, w, inv, wts, b30, b31, rloc); break;
                            default: fold_step<3, 2>(raw, w, inv, wts, b30, b31, rloc); break;
                            }
                        } else if (direct) {
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                w[k] = pack_bf16x2(__uint_as_float(raw[2 * k]) * inv, __uint_as_float(raw[2 * k + 1]) * inv);
                            col = 256 * (st >> 1) + 128 * half + 64 * (st & 1);
                        } else {
#pragma unroll
                            for (int k = 0; k < 32; ++k) w[k] = __float_as_uint(__uint_as_float(raw[32 * pass + k]) * inv);
                            col = 256 * (st >> 1) + 128 * half + 64 * (st & 1) + 32 * pass;
                        }
                        // this thread's 128 bytes -> staging row `lane` (16-byte unit k at k ^ (lane & 7), the
                        // 128-byte swizzle of a 32-row x 128-byte box), then one TMA store of the box
                        // (rows past the request's last are clipped).  Two staging buffers alternate;
                        // a buffer is rewritten once the store that used it has read it.
                        const uint32_t stage = (npass & 1u) ? stage_b : stage_a;
                        if (lane == 0 && npass >= 2) bulk_wait_read<1>();
                        __syncwarp();
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            st_shared_v4u(stage + (uint32_t)lane * 128u + 16u * ((uint32_t)k ^ ((uint32_t)lane & 7u)),
                                          w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0 && row0 < p.rows) {   // (a warp past the request's rows stores nothing)
                            if (write_final)
                                tma_store_3d(&o_map, stage, col, row0, ub);
                            else
                                tma_store_3d_hint(&ps_map, stage, col, row0, split, part_pol);
                            bulk_commit();
                        }
                        ++npass;
                        __syncwarp();
                    }
                }
            }
            // the staging (and the P buffer) free again; a stored piece's rows also complete (their
            // count below makes them visible to other CTAs, whose loads go through the async proxy)
            if (lane == 0) {
                if (write_final) {
                    bulk_wait_read<0>();
                } else {
                    bulk_wait<0>();
                    fence_proxy_async_global();
                }
            }
            __syncwarp();
            if (!ep_ok) break;
            if (row_valid && half == 0) {
                if (write_final)
                    p.lse[(int64_t)ub * p.rows + rowg] = lse_val;
                else
                    st_global_f32_hint(p.part_lse + (int64_t)split * p.rows + rowg, lse_val, part_pol);
            }
            if (mode == 1 || mode == 3) {
                // This piece's partial rows are written: make them visible device-wide, then
                // count them stored (high half of the word); the last claimer merges once all the
                // others have.  (An mbarrier, not bar.sync, gathers the 128 threads: a bounded
                // wait can never strand them if another role gave up.)
                __threadfence();
                mbar_arrive(bar(kBarPartial));
                if (!mbar_wait_bounded(bar(kBarPartial), npartial & 1u, actl)) break;
                ++npartial;
                if (t == 0) {
                    if (mode == 1) {
                        atomicAdd(arrival, 1 << 16);
                    } else {
                        const int k = pending[0];
                        if (k < kMaxPendingMerges) {
                            pending[1 + 3 * k] = ub;
                            pending[2 + 3 * k] = s0;
                            pending[3 + 3 * k] = pieces;
                            pending[0] = k + 1;
                        } else {
                            raise_error(8 /* MLA_DEVERR_BAD_METADATA */);
                        }
                    }
                }
            }
            ++uq;
        }
    }

    if (warp >= kSoftmaxWarp0 && warp < kSoftmaxWarp0 + 4 && lane == 0) bulk_wait<0>();   // the epilogues' stores
    tc_fence_before();
    __syncthreads();
    // Merges of the requests whose last piece arrived here, by the whole CTA: the pieces' rows
    // come in by bulk copies into the now idle Q, K ring and P areas (200 KB, as many rows per
    // pass as fit); the row-max exchange area holds the weights.
    const int npending = pending[0];
    if (npending > 0 && !*abort_flag) {
        __threadfence();   // the other pieces' partials: their fences preceded their arrivals
        const int row_base = mtile * kRows + kCtaRows * (int)rank;
        const int nrows = min(kCtaRows, p.rows - row_base);
        uint32_t phase = 0;
        auto wait = [&](uint32_t b, uint32_t parity) { return mbar_wait_bounded(b, parity, actl); };
        for (int k = 0; k < npending; ++k) {
            const int mb = pending[1 + 3 * k], s0 = pending[2 + 3 * k], n = pending[3 + 3 * k];
            if (threadIdx.x == 0) {
                // the other pieces claimed before this one: wait until they have stored
                int32_t* const word = p.arrivals + ((int64_t)mb * gridDim.y + mtile) * 2 + rank;
                const bool ok = wait_stored(word, n - 1, actl);
                if (ok) *word = 0;   // every piece is done with the word: ready for the next call
                pending[kMiscFold] = ok ? 1 : 0;
            }
            __syncthreads();
            const bool stored_all = pending[kMiscFold] != 0;
            __syncthreads();   // read before thread 0 can write the flag again
            if (!stored_all) break;
            if (nrows <= 0) continue;   // a CTA past the query rows: nothing to write
            __threadfence();
            if (!merge_rows_cta_bulk<kThreads>(p.part_o, p.part_lse, s0, n, p.rows, row_base, nrows,
                                               p.out + ((int64_t)mb * p.rows + row_base) * kDv,
                                               p.lse + (int64_t)mb * p.rows + row_base,
                                               reinterpret_cast<float*>(smem + kOffX), sbase + kOffQ,
                                               (uint32_t)(kOffX - kOffQ), bar(kBarMerge), phase, wait, threadIdx.x))
                break;
        }
    }
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace decode
}  // namespace mla
