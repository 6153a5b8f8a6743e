/*
 * mla_b200.h — C ABI of the B200 (sm_100a) paged MLA decode library.
 *
 * Three operations, in the order a decode step calls them, each in the role the
 * SGLang FlashMLA attention backend page (flashmla_backend.py) gives it:
 *
 *   mla_build_block_table  the per-request page table of
 *                          FlashMLABackend.init_forward_metadata (decode and
 *                          target-verify branches, create_flashmla_kv_indices_triton);
 *   mla_get_mla_metadata   the split-KV scheduler of get_mla_metadata
 *                          (tile_scheduler_metadata [num_sm_parts, 8], num_splits [bs+1]);
 *   mla_decode_paged       the attention of flash_mla_with_kvcache as called by
 *                          forward_decode / forward_extend (target-verify), with the
 *                          log-sum-exp merge of KV splits.
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is a DEVICE pointer owned by the caller (for example a
 *     torch tensor's data_ptr()), unless its comment says "host".  The library keeps
 *     no state between calls and allocates no device memory: scratch space is the
 *     caller's `workspace`.  Every call is asynchronous on `stream` (NULL = the legacy
 *     default stream), makes no host synchronisation and no allocation, and may
 *     therefore be captured in a CUDA graph.
 *   - Stream order holds as for ordinary launches.  mla_decode_paged's kernel is a
 *     programmatic dependent launch, and the metadata kernels let their dependent in at
 *     their start.  Placed right after one of them, the attention kernel therefore sets
 *     itself up while the metadata kernel still runs, and reads nothing before that
 *     kernel has completed.  After any other kernel, copy or event it starts as an
 *     ordinary launch would.
 *   - Arguments are validated on the host before any launch; a violation returns
 *     MLA_ERR_INVALID_ARG (or MLA_ERR_UNSUPPORTED for a valid but unimplemented
 *     combination) and launches nothing.  A CUDA launch error returns MLA_ERR_CUDA.
 *   - Facts only the device can see (a page id outside the pool, a request-pool row
 *     outside req_to_token, a length beyond the page table, a malformed scheduler row,
 *     a pipeline wait that timed out) never fault: the kernel skips or clamps the
 *     access and ORs a bit into a sticky device error word, which
 *     mla_read_device_error returns and clears.
 *   - bs == 0 (the idle batch) returns MLA_OK and launches nothing.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,   /* an argument is out of its documented range     */
    MLA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (dtype, head dims)    */
    MLA_ERR_CUDA = 3,          /* a CUDA runtime / driver call failed             */
    MLA_ERR_DEVICE_CHECK = 4,  /* mla_read_device_error found a device-side error */
    MLA_ERR_WORKSPACE = 5      /* workspace missing or smaller than required      */
} mla_status_t;

/* Element / index types. */
enum {
    MLA_DTYPE_BF16 = 0,
    MLA_DTYPE_FP8_E4M3 = 1,    /* OCP e4m3 "fn": no infinities, S.1111.111 = NaN */
    MLA_DTYPE_INT32 = 2,
    MLA_DTYPE_INT64 = 3,
    MLA_DTYPE_FP8_E5M2 = 4     /* OCP e5m2: exponent 31 holds infinities and NaNs   */
};

/* Bits of the sticky device error word (mla_read_device_error). */
enum {
    MLA_DEVERR_PAGE_OUT_OF_RANGE = 1,  /* block-table page id not in [0, num_pages): tile read as zeros */
    MLA_DEVERR_ROW_OUT_OF_RANGE = 2,   /* req_pool_indices[b] not a row of req_to_token: row skipped   */
    MLA_DEVERR_LEN_OUT_OF_RANGE = 4,   /* a length exceeds the table / req_to_token width: clamped     */
    MLA_DEVERR_BAD_METADATA = 8,       /* a scheduler row is not a valid cursor range: part skipped    */
    MLA_DEVERR_WAIT_TIMEOUT = 16,      /* a pipeline wait exceeded its bound: the CTA gave up          */
    MLA_DEVERR_Q_RANGE = 32,           /* 8-bit cache, bf16 q: a q value beyond f16's range (> 65504)  */
    MLA_DEVERR_SLOT_INVALID = 64,      /* page table: a req_to_token slot read for page p is negative    */
                                       /* (entry -1) or not the first slot of a page (slot % 64 != 0)  */
    MLA_DEVERR_WORKSPACE_STATE = 128,  /* decode: a workspace arrival word was not zero at the call's  */
                                       /* start (workspace not zero-filled before its first use)       */
    MLA_DEVERR_SLOT_OUT_OF_RANGE = 256 /* KV write: cache_loc[i] not a pool row: that token skipped    */
};

typedef struct CUstream_st* mla_stream_t;  /* identical to cudaStream_t */

/* Human-readable name of a status code (static storage, never NULL). */
MLA_API const char* mla_status_string(mla_status_t status);

/* Version of this ABI; bumped whenever a signature or layout below changes. */
MLA_API int32_t mla_abi_version(void);

/*
 * Page table (flashmla_backend.py, init_forward_metadata: block_kv_indices of shape
 * [bs, cdiv(max L, 64)], int32, pre-filled with -1, filled from req_to_token,
 * req_pool_indices and seq_lens; the target-verify branch first adds
 * num_draft_tokens to every length).
 *
 * For request b with L_b = seq_lens[b] + seq_len_add and every page p < cdiv(L_b, page_size):
 *     block_table[b * block_table_stride + p] =
 *         req_to_token[req_pool_indices[b] * req_to_token_stride + p * page_size] / page_size
 * (the pool viewed [-1, page_size, 1, 576] puts slots page_size*P .. page_size*P+page_size-1
 * in page P, so slots must be page-aligned and in order inside a page).
 * Entries p in [cdiv(L_b, page_size), max_pages) are written with -1 when fill_tail != 0
 * and left untouched otherwise (the caller's pre-fill, as in the graph-capture path, which
 * fills its table with 1); columns from max_pages to block_table_stride are never touched.
 *
 *   req_to_token         int32 [req_to_token_rows, req_to_token_stride] (row-major)
 *   req_pool_indices     [bs], int32 or int64 (rpi_dtype)
 *   seq_lens             [bs], int32 or int64 (seq_lens_dtype)
 *   block_table          int32 [bs, block_table_stride], written for p < max_pages
 *   page_size            must be 64
 * Device checks: a row index outside [0, req_to_token_rows) leaves the row at -1 and
 * sets MLA_DEVERR_ROW_OUT_OF_RANGE; L_b beyond max_pages pages or beyond
 * req_to_token_stride positions is clamped and sets MLA_DEVERR_LEN_OUT_OF_RANGE; a slot
 * read for page p that is not page-aligned (slot % 64 != 0: the request's slots are not
 * whole pages in order) still gives slot / 64 but sets MLA_DEVERR_SLOT_INVALID, and a
 * negative slot gives -1 and sets the same bit.
 */
MLA_API mla_status_t mla_build_block_table(const int32_t* req_to_token, int64_t req_to_token_rows,
                                   int64_t req_to_token_stride, const void* req_pool_indices,
                                   int32_t rpi_dtype, const void* seq_lens, int32_t seq_lens_dtype,
                                   int32_t seq_len_add, int32_t bs, int32_t* block_table,
                                   int64_t block_table_stride, int32_t max_pages,
                                   int32_t page_size, int32_t fill_tail, mla_stream_t stream);

/*
 * Number of scheduler parts (the first dimension of tile_scheduler_metadata) for
 * get_mla_metadata(cache_seqlens, num_heads_per_head_k, num_heads_k): every part is
 * served by a pair of SMs per 128-row query tile, so
 *     num_sm_parts = max(1, sm_count / (2 * cdiv(num_heads_per_head_k, 128) * num_heads_k)).
 * num_heads_per_head_k is q_len * h_q (num_draft_tokens * h_q in target-verify, as the
 * backend passes it); num_heads_k is 1 for MLA.  Returns -1 on a non-positive argument.
 * Pure host function.
 */
MLA_API int32_t mla_num_sm_parts(int32_t sm_count, int32_t num_heads_per_head_k, int32_t num_heads_k);

/*
 * Split-KV scheduler (flashmla_backend.py, get_mla_metadata(cache_seqlens,
 * num_heads_per_head_k, num_heads_k, is_fp8_kvcache) returning tile_scheduler_metadata
 * int32 [num_sm_parts, 8], num_sm_parts <= the SM count, and num_splits int32 [bs+1]).
 * The part count is num_sm_parts = mla_num_sm_parts(sm_count, num_heads_per_head_k,
 * num_heads_k); the caller sizes tile_scheduler_metadata with the same call.
 * The pages fix only these shapes; the contents are defined here:
 *   blocks_b = cdiv(cache_seqlens[b], 64); each piece of a request costs its blocks plus
 *   a fixed overhead of 5 blocks; total = sum_b (blocks_b + 5); every part has the budget
 *   cdiv(total, num_sm_parts) + 5 and is filled greedily in request order: a request that
 *   fits in what is left is taken whole, otherwise the part takes (budget - 5) blocks of it
 *   when that is positive, and ends.
 *   Row i = [begin_req, begin_block, end_req, end_block, begin_split, 0, 0, 0], where
 *   (end_req, end_block) is the exclusive cursor after the part and begin_split the index
 *   of the part's first piece within its request; num_splits[0] = 0 and
 *   num_splits[b+1] - num_splits[b] = number of pieces of request b.
 * Every block of every request is covered exactly once within num_sm_parts parts, and
 * num_splits[bs] <= bs + num_sm_parts - 1.
 *   cache_seqlens          int32 [bs] (negative lengths count as 0)
 *   num_heads_per_head_k   q_len * h_q (num_draft_tokens * h_q in target-verify), > 0
 *   num_heads_k            1 for MLA, > 0
 *   is_fp8_kvcache         accepted; it does not change the plan
 *   sm_count               SMs of the device the attention runs on, > 0
 *   tile_scheduler_metadata int32 [num_sm_parts, 8] (written), 16-byte aligned
 *   num_splits             int32 [bs + 1] (written)
 * One single-CTA launch; bs must be <= 1,048,576.
 */
MLA_API mla_status_t mla_get_mla_metadata(const int32_t* cache_seqlens, int32_t bs,
                                  int32_t num_heads_per_head_k, int32_t num_heads_k,
                                  int32_t is_fp8_kvcache, int32_t sm_count,
                                  int32_t* tile_scheduler_metadata, int32_t* num_splits,
                                  mla_stream_t stream);

/*
 * The whole per-batch metadata step in one launch: mla_build_block_table,
 * the int32 cache_seqlens the attention call takes (flashmla_backend.py,
 * init_forward_metadata: seq_lens.to(torch.int32), plus num_draft_tokens in the
 * target-verify branch) and mla_get_mla_metadata over those lengths.
 *
 * Arguments are those of mla_build_block_table followed by those of
 * mla_get_mla_metadata; the lengths the plan uses are seq_lens[b] + seq_len_add.
 *   cache_seqlens          int32 [bs], written with seq_lens[b] + seq_len_add; may be NULL
 * block_table, tile_scheduler_metadata and num_splits are bit-identical to what the two
 * separate calls write (one CTA plans while the others fill the table).  Errors and
 * device checks are those of the two calls.
 */
MLA_API mla_status_t mla_build_decode_metadata(
    const int32_t* req_to_token, int64_t req_to_token_rows, int64_t req_to_token_stride,
    const void* req_pool_indices, int32_t rpi_dtype, const void* seq_lens, int32_t seq_lens_dtype,
    int32_t seq_len_add, int32_t bs, int32_t* block_table, int64_t block_table_stride,
    int32_t max_pages, int32_t page_size, int32_t fill_tail, int32_t num_heads_per_head_k,
    int32_t num_heads_k, int32_t is_fp8_kvcache, int32_t sm_count, int32_t* cache_seqlens,
    int32_t* tile_scheduler_metadata, int32_t* num_splits, mla_stream_t stream);

/*
 * Bytes of workspace mla_decode_paged needs, 256-byte aligned parts in this order:
 *   arrival words  int32 [bs, cdiv(q_len * h_q, 128), 2]: split pieces of a request claim a
 *                  place and count their stored partials here, and the last to claim merges
 *                  the request's rows
 *                  (requests of up to 4 pieces); every completed call leaves them zero;
 *   partial outputs fp32 [(bs + num_sm_parts) * q_len * h_q, 512] and their log-sum-exps.
 * Pure host function; returns 0 on a non-positive argument.
 */
MLA_API size_t mla_decode_workspace_bytes(int32_t bs, int32_t q_len, int32_t h_q, int32_t num_sm_parts);

/*
 * Paged MLA attention (flashmla_backend.py, forward_decode / forward_extend:
 * flash_mla_with_kvcache(q, k_cache.view(-1, 64, 1, 576), block_table, cache_seqlens,
 * head_dim_v = kv_lora_rank, tile_scheduler_metadata, num_splits, softmax_scale,
 * causal, descale_q, descale_k)).
 *
 * For every request b, query position i < q_len and head h (row r = i * h_q + h):
 *   L = cache_seqlens[b]; keys j < lim with lim = L - q_len + i + 1 when causal
 *   (the draft tokens are the last q_len positions of the cache) and lim = L otherwise;
 *   k_j = KV row of position j (through block_table, page j / 64, row j % 64) * descale_k;
 *   v_j = k_j[0:512];  s_j = softmax_scale * descale_q * <q[b,i,h,:], k_j>;
 *   lse = ln sum_j exp(s_j);  o = sum_j exp(s_j - lse) v_j.
 *   A row with no allowed key gets o = 0 and lse = -inf.
 *   Arithmetic: S in fp32 from bf16 products (bf16 cache) or f16 products (8-bit cache with
 *   bf16 q: every e4m3 and e5m2 value is exact in f16; a bf16 q value is exact in f16 when its magnitude
 *   lies in [2^-14, 65504] or it is zero, while magnitudes in [2^-24, 2^-14) keep only
 *   the bits of an f16 subnormal and smaller ones round to zero, an error far below the
 *   attention tolerance; |q| > 65504 records MLA_DEVERR_Q_RANGE and o is undefined); P
 *   rounded to bf16 (f16 with an 8-bit cache) for the P V product; O accumulated in fp32.
 *   With e4m3 q, S is fp32 from exact e4m3 x e4m3 products.
 *
 *   q                 bf16 [bs, q_len, h_q, head_dim], contiguous; q_len * h_q must not
 *                     exceed 65535 * 128 (MLA_ERR_UNSUPPORTED)
 *   q_dtype           MLA_DTYPE_BF16, or MLA_DTYPE_FP8_E4M3 with an e4m3 cache (the backend
 *                     page's fp8 branch: q quantised with scaled_fp8_quant(q, k_scale),
 *                     descale_q = descale_k = k_scale); S then runs on e4m3 x e4m3 tensor
 *                     cores, PV on f16.  e4m3 q with another cache: MLA_ERR_UNSUPPORTED
 *   head_dim          576 (kv_lora_rank 512 + qk_rope_head_dim 64); head_dim_v 512
 *   k_cache           [num_pages, page_size, head_dim] bf16, e4m3 or e5m2 (kv_dtype), contiguous;
 *                     every value must be finite (tail rows of a page are read and masked)
 *   page_size         64
 *   block_table       int32 [bs, block_table_stride]; entries p < cdiv(L, 64) are read
 *   max_pages         usable columns of block_table (L must be <= 64 * max_pages)
 *   cache_seqlens     int32 [bs]
 *   tile_scheduler_metadata, num_splits  from mla_get_mla_metadata for the same
 *                     cache_seqlens and num_sm_parts, with num_sm_parts from
 *                     mla_num_sm_parts(sm_count, q_len * h_q, 1)
 *   softmax_scale     host float (1/sqrt(192) for DeepSeek-V3)
 *   causal            0 or 1
 *   descale_q, descale_k  device fp32 [1]; NULL means 1.0.  descale_k scales the 8-bit
 *                     cache values and must be NULL with a bf16 cache (the backend passes
 *                     the descales only with an fp8 cache), else MLA_ERR_INVALID_ARG;
 *                     descale_q scales q.
 *   out               bf16 [bs, q_len, h_q, 512] (written)
 *   lse               fp32 [bs, q_len, h_q] natural-log log-sum-exp (written)
 *   workspace         at least mla_decode_workspace_bytes(bs, q_len, h_q, num_sm_parts)
 *                     bytes, 256-byte aligned, zero-filled before its first use: its leading
 *                     arrival words must be zero when a call starts, and every completed call
 *                     leaves them zero again, so a workspace is zero-filled once and then
 *                     reused (after a call that recorded MLA_DEVERR_WAIT_TIMEOUT or
 *                     MLA_DEVERR_WORKSPACE_STATE, zero-fill it again).  The partial-output
 *                     part needs no initialisation and is undefined after the call (the merge
 *                     may drop its L2 lines without writing them back)
 * Calls on the same workspace that overlap on the GPU race; use one workspace per stream.
 * The first call on a device also sets the kernel's shared-memory limit (a host-side
 * attribute; no allocation).
 */
MLA_API mla_status_t mla_decode_paged(const void* q, int32_t q_dtype, int32_t bs, int32_t q_len,
                              int32_t h_q, int32_t head_dim, int32_t head_dim_v,
                              const void* k_cache, int32_t kv_dtype, int64_t num_pages,
                              int32_t page_size, const int32_t* block_table,
                              int64_t block_table_stride, int32_t max_pages,
                              const int32_t* cache_seqlens, const int32_t* tile_scheduler_metadata,
                              int32_t num_sm_parts, const int32_t* num_splits, float softmax_scale,
                              int32_t causal, const float* descale_q, const float* descale_k,
                              void* out, float* lse, void* workspace, size_t workspace_bytes,
                              mla_stream_t stream);

/*
 * KV-cache write (flashmla_backend.py, forward_decode / forward_extend:
 * token_to_kv_pool.set_kv_buffer(layer, cache_loc, k, v) before attention).  For every new
 * token i, pool row cache_loc[i] receives k[i, 0:576], the latent row (kv_lora_rank 512 +
 * qk_rope_head_dim 64); in MLA the value is the first 512 columns of that row, so v is not
 * passed.  A bf16 pool stores the row bit for bit; an fp8 pool (MLA_DTYPE_FP8_E4M3 or
 * MLA_DTYPE_FP8_E5M2, the two fp8 types the backend's __init__ accepts) stores
 * x = k / k_scale, one correctly rounded single-precision division (x = k when k_scale is
 * NULL), rounded to the nearest code, ties to even, magnitudes beyond the largest finite
 * value saturating to it.
 *
 *   kv_cache      the pool [num_slots, 576] of kv_dtype, contiguous; 16-byte aligned (bf16)
 *                 or 8-byte aligned (fp8)
 *   cache_loc     [n_tokens] int32 or int64 (loc_dtype): each token's pool row
 *   k             bf16 [n_tokens, k_row_stride] (elements), 16-byte aligned;
 *                 k_row_stride >= 576 and a multiple of 8
 *   k_scale       device fp32 [1] or NULL; must be NULL for a bf16 pool
 * Rows not listed are untouched.  A cache_loc outside [0, num_slots) skips that token and
 * sets MLA_DEVERR_SLOT_OUT_OF_RANGE.  Two tokens with the same slot race (one wins).
 * n_tokens == 0 returns MLA_OK and launches nothing.
 */
MLA_API mla_status_t mla_set_kv_buffer(void* kv_cache, int32_t kv_dtype, int64_t num_slots,
                                       const void* cache_loc, int32_t loc_dtype, int32_t n_tokens,
                                       const void* k, int64_t k_row_stride, const float* k_scale,
                                       mla_stream_t stream);

/*
 * merge_state (flashinfer_backend.py, forward_extend: o, _ = merge_state(o1, s1, o2, s2)): the
 * exact log-sum-exp merge of two partial attention results of the same rows,
 *     lse = ln(exp(lse_a) + exp(lse_b)),   o = exp(lse_a - lse) o_a + exp(lse_b - lse) o_b.
 *   o_a, o_b      bf16 [rows, head_dim_v], 16-byte aligned; lse_a, lse_b fp32 [rows], natural
 *                 log, -inf for a part that saw no key
 *   head_dim_v    512 (else MLA_ERR_UNSUPPORTED)
 *   o, lse        bf16 [rows, head_dim_v] (16-byte aligned) and fp32 [rows], written; a row with
 *                 no key in either part gets o = 0 and lse = -inf.
 * The weights are computed in fp32 from the max-shifted lse values; one warp per row.
 */
MLA_API mla_status_t mla_merge_state(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                                     int64_t rows, int32_t head_dim_v, void* o, float* lse, mla_stream_t stream);

/*
 * Bytes of workspace mla_extend_paged_prefix needs (256-byte aligned parts: a padded copy of the
 * new rows when e is not a multiple of 64, the page tables, lengths and plans of both parts,
 * two mla_decode_paged workspaces and the two partial results).  Pure host function; returns 0
 * on a non-positive bs, e, h_q or sm_count or a negative max_prefix_pages.
 */
MLA_API size_t mla_extend_workspace_bytes(int32_t bs, int32_t e, int32_t h_q, int32_t max_prefix_pages,
                                          int32_t sm_count);

/*
 * Extend with a cached prefix (flashinfer_backend.py, forward_extend, the ragged-plus-paged
 * branch), in MLA form: each request has prefix_lens[b] latent rows already in the paged pool
 * and e new tokens; the new tokens' queries attend
 *   (1) the new tokens' own latent rows k_new, causally (new token i sees new tokens 0 .. i):
 *       the ragged part, o1 / s1;
 *   (2) the whole cached prefix, non-causally: the paged part, o2 / s2;
 * and the result is merge_state(o1, s1, o2, s2) -- exactly attention over the prefix followed
 * by the new rows with the new tokens causal.  Both parts run on the paged attention kernel
 * (mla_decode_paged): the new rows are presented to it as a pool of their own (copied to a
 * 64-row-aligned layout in the workspace unless e is a multiple of 64), the prefix through a
 * page table built from req_to_token.  The caller writes the new rows into the pool afterwards
 * (mla_set_kv_buffer), as the page writes them after the two attention calls.
 *   q                 bf16 [bs, e, h_q, 576]; e new tokens per request (uniform), h_q heads;
 *                     e * h_q <= 65535 * 128
 *   k_new             bf16 [bs, e, 576], 16-byte aligned: the new tokens' latent rows
 *   kv_cache, kv_dtype, num_pages   the pool holding the prefix (bf16, e4m3 or e5m2, pages of
 *                     64 rows), as for mla_decode_paged; descale_k with an fp8 pool
 *   req_to_token .. rpi_dtype       the request-to-slot map, as for mla_build_block_table
 *   prefix_lens       int32 [bs]: cached rows per request (0: no prefix; then o = o1)
 *   max_prefix_pages  >= max cdiv(prefix_lens[b], 64) (longer prefixes are clamped and reported
 *                     as by mla_build_block_table)
 *   softmax_scale     applied to q . k
 *   sm_count          SMs of the device (sizes the two split plans)
 *   out, lse          bf16 [bs, e, h_q, 512] and fp32 [bs, e, h_q], written
 *   workspace         at least mla_extend_workspace_bytes(bs, e, h_q, max_prefix_pages,
 *                     sm_count) bytes, 256-byte aligned, zero-filled before its first use (the
 *                     two attention calls' arrival words; every completed call leaves them zero)
 * Errors: those of the calls it makes; MLA_ERR_WORKSPACE for a missing or short workspace.
 */
MLA_API mla_status_t mla_extend_paged_prefix(const void* q, int32_t bs, int32_t e, int32_t h_q, const void* k_new,
                                             const void* kv_cache, int32_t kv_dtype, int64_t num_pages,
                                             const int32_t* req_to_token, int64_t req_to_token_rows,
                                             int64_t req_to_token_stride, const void* req_pool_indices,
                                             int32_t rpi_dtype, const int32_t* prefix_lens, int32_t max_prefix_pages,
                                             float softmax_scale, const float* descale_k, int32_t sm_count,
                                             void* out, float* lse, void* workspace, size_t workspace_bytes,
                                             mla_stream_t stream);

/*
 * Test hooks for the failure path of mla_decode_paged; not for production use.  They set
 * process-wide values that every later mla_decode_paged launch (from any thread) takes:
 *   wait_budget_ns  the budget of one pipeline wait (0 restores the default of 2 s);
 *   withhold_tile   the index (within a scheduler part, counting from 0) of a tile whose page
 *                   load the leader CTA of every pair does not issue, so that the wait for it
 *                   runs out (-1 restores normal operation);
 *   no_fold_in      nonzero: the last piece of a split request never folds the other pieces
 *                   into its own result but stores its partial and merges at the end of its
 *                   part (the two ways give identical bits; 0 restores normal operation).
 * When a wait runs out the CTA records MLA_DEVERR_WAIT_TIMEOUT, both CTAs of the pair stop at
 * their next wait, let their issued copies land, release their tensor memory and return; the
 * call's outputs are then undefined and its workspace must be zero-filled again.  Host-only,
 * no synchronisation.  Returns MLA_ERR_INVALID_ARG for withhold_tile < -1.
 */
MLA_API mla_status_t mla_set_test_hooks(uint64_t wait_budget_ns, int32_t withhold_tile, int32_t no_fold_in);

/*
 * Read and clear the sticky device error word of the current device (a bitwise OR of
 * MLA_DEVERR_* since the last read).  Synchronises `stream`, so it is not for use inside
 * graph capture.  *code_out (host) receives the word; returns MLA_ERR_DEVICE_CHECK when it
 * is non-zero, MLA_OK when it is zero.
 */
MLA_API mla_status_t mla_read_device_error(int32_t* code_out, mla_stream_t stream);

/*
 * mla_decode_paged without a caller-supplied workspace.
 *
 * The pages have no counterpart to this call; it exists for callers that cannot
 * allocate device memory at the point where they run attention: an engine that plans
 * every byte of device memory ahead of time and forbids allocation afterwards, a plugin
 * whose host framework owns all device memory and rejects cudaMalloc inside its
 * execute hook, or code running where cudaMalloc would block on the device or fail under
 * memory pressure.  Such callers still pass every input and output buffer; only the
 * split-KV scratch comes from the library.
 *
 * That scratch is one fixed array of MLA_NOALLOC_SCRATCH_BYTES (64 MiB) in the library's
 * device memory.  Every GPU on which the library's kernels are loaded holds it until the
 * process exits.  A problem whose workspace (mla_decode_workspace_bytes) exceeds it is
 * rejected with MLA_ERR_WORKSPACE before anything is launched; the five DeepSeek-V3-shaped
 * workloads of this project (up to bs 128 x 128 heads, or bs 32 x 4 x 128 rows) fit.
 *
 * All calls share the one array and it keeps whatever the last call left in it: each call
 * first clears the array's leading arrival words (the only scratch that must start at zero;
 * an asynchronous memset on `stream`, no allocation), and its kernels write every other
 * scratch value before reading it.  Calls
 * whose execution overlaps on the GPU (on different streams, or from different threads)
 * race on the array and corrupt each other's results: serialise them.
 *
 * The first call on a device looks up the array's device address there (a host-side
 * query, once per device, with that device current); make that first call before any
 * stream capture.  This call allocates nothing: no cudaMalloc, no cudaFree.
 * Arguments, results and errors are otherwise those of mla_decode_paged.
 */
#define MLA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

MLA_API mla_status_t mla_decode_paged_noalloc(
    const void* q, int32_t q_dtype, int32_t bs, int32_t q_len, int32_t h_q, int32_t head_dim,
    int32_t head_dim_v, const void* k_cache, int32_t kv_dtype, int64_t num_pages,
    int32_t page_size, const int32_t* block_table, int64_t block_table_stride, int32_t max_pages,
    const int32_t* cache_seqlens, const int32_t* tile_scheduler_metadata, int32_t num_sm_parts,
    const int32_t* num_splits, float softmax_scale, int32_t causal, const float* descale_q,
    const float* descale_k, void* out, float* lse, mla_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H */
