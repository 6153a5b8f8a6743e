// C ABI of the paged MLA decode library (declared in include/mla_b200.h): host-side
// argument validation, TMA tensor-map encoding and kernel launches.  The kernels live in
// the headers included below; this file is the library's only translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "../../include/mla_b200.h"
#include "block_table.cuh"
#include "combine.cuh"
#include "decode.cuh"
#include "extend.cuh"
#include "kv_write.cuh"
#include "planner.cuh"

namespace {

constexpr int kMaxDevices = 64;

bool is_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

mla_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// An NVTX range around each entry point, named after it, for timeline tools (header-only NVTX:
// without an attached tool a range costs a few nanoseconds).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

// cuTensorMapEncodeTiled through the runtime's driver entry point, so that the library
// links against no driver library at build time and loads on hosts without a GPU.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Per-device one-time setting of the decode kernels' shared-memory limit.
mla_status_t prepare_decode_kernels() {
    static std::once_flag flags[kMaxDevices];
    static cudaError_t results[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return MLA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
    std::call_once(flags[dev], [dev] {
        const void* kernels[] = {
            reinterpret_cast<const void*>(mla::decode::mla_decode_kernel<0, false>),
            reinterpret_cast<const void*>(mla::decode::mla_decode_kernel<1, false>),
            reinterpret_cast<const void*>(mla::decode::mla_decode_kernel<1, true>),
            reinterpret_cast<const void*>(mla::decode::mla_decode_kernel<2, false>)};
        results[dev] = cudaSuccess;
        for (const void* k : kernels)
            if (results[dev] == cudaSuccess)
                results[dev] = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    mla::decode::kSmemBytes);
    });
    return from_cuda(results[dev]);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Test hooks (mla_set_test_hooks): the wait budget, the withheld tile and the fold-in switch of
// later launches.
std::atomic<uint64_t> g_hook_wait_budget_ns{0};
std::atomic<int32_t> g_hook_withhold_tile{-1};
std::atomic<int32_t> g_hook_no_fold_in{0};

// Workspace layout: arrival words int32 [bs, query tiles, 2], then the split partials
// fp32 [splits, rows, 512] and their lse fp32 [splits, rows], each 256-byte aligned.
size_t arrival_bytes(int32_t bs, int32_t q_len, int32_t h_q) {
    const size_t tiles = ((size_t)q_len * (size_t)h_q + 127) / 128;
    return align256((size_t)bs * tiles * 2 * sizeof(int32_t));
}

}  // namespace

extern "C" {

const char* mla_status_string(mla_status_t s) {
    switch (s) {
        case MLA_OK: return "MLA_OK";
        case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
        case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
        case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
        case MLA_ERR_DEVICE_CHECK: return "MLA_ERR_DEVICE_CHECK";
        case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    }
    return "MLA_ERR_UNKNOWN";
}

int32_t mla_abi_version(void) { return 2; }

mla_status_t mla_build_block_table(const int32_t* req_to_token, int64_t req_to_token_rows,
                                   int64_t req_to_token_stride, const void* req_pool_indices,
                                   int32_t rpi_dtype, const void* seq_lens, int32_t seq_lens_dtype,
                                   int32_t seq_len_add, int32_t bs, int32_t* block_table,
                                   int64_t block_table_stride, int32_t max_pages,
                                   int32_t page_size, int32_t fill_tail, mla_stream_t stream) {
    const NvtxRange nvtx_range("mla_build_block_table");
    if (bs < 0 || max_pages < 0 || page_size != 64) return MLA_ERR_INVALID_ARG;
    if (rpi_dtype != MLA_DTYPE_INT32 && rpi_dtype != MLA_DTYPE_INT64) return MLA_ERR_INVALID_ARG;
    if (seq_lens_dtype != MLA_DTYPE_INT32 && seq_lens_dtype != MLA_DTYPE_INT64)
        return MLA_ERR_INVALID_ARG;
    if (bs == 0 || max_pages == 0) return MLA_OK;
    if (!req_to_token || !req_pool_indices || !seq_lens || !block_table) return MLA_ERR_INVALID_ARG;
    if (req_to_token_rows <= 0 || req_to_token_stride <= 0 || block_table_stride < max_pages)
        return MLA_ERR_INVALID_ARG;
    if (bs > 65535) return MLA_ERR_UNSUPPORTED;
    const dim3 grid(bs, (max_pages + 255) / 256);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define MLA_BT_LAUNCH(IT, LT)                                                                     \
    mla::build_block_table_kernel<IT, LT><<<grid, 256, 0, st>>>(                                 \
        req_to_token, req_to_token_rows, req_to_token_stride,                                     \
        static_cast<const IT*>(req_pool_indices), static_cast<const LT*>(seq_lens), seq_len_add, \
        block_table, block_table_stride, max_pages, fill_tail)
    if (rpi_dtype == MLA_DTYPE_INT64 && seq_lens_dtype == MLA_DTYPE_INT64) MLA_BT_LAUNCH(int64_t, int64_t);
    else if (rpi_dtype == MLA_DTYPE_INT64) MLA_BT_LAUNCH(int64_t, int32_t);
    else if (seq_lens_dtype == MLA_DTYPE_INT64) MLA_BT_LAUNCH(int32_t, int64_t);
    else MLA_BT_LAUNCH(int32_t, int32_t);
#undef MLA_BT_LAUNCH
    return from_cuda(cudaGetLastError());
}

int32_t mla_num_sm_parts(int32_t sm_count, int32_t num_heads_per_head_k, int32_t num_heads_k) {
    if (sm_count <= 0 || num_heads_per_head_k <= 0 || num_heads_k <= 0) return -1;
    const int32_t m_tiles = (num_heads_per_head_k + 127) / 128;
    const int32_t parts = sm_count / (2 * m_tiles * num_heads_k);
    return parts < 1 ? 1 : parts;
}

mla_status_t mla_get_mla_metadata(const int32_t* cache_seqlens, int32_t bs,
                                  int32_t num_heads_per_head_k, int32_t num_heads_k,
                                  int32_t is_fp8_kvcache, int32_t sm_count,
                                  int32_t* tile_scheduler_metadata, int32_t* num_splits,
                                  mla_stream_t stream) {
    const NvtxRange nvtx_range("mla_get_mla_metadata");
    (void)is_fp8_kvcache;  // accepted for call compatibility; the plan does not depend on it
    const int32_t num_sm_parts = mla_num_sm_parts(sm_count, num_heads_per_head_k, num_heads_k);
    if (bs < 0 || num_sm_parts < 1 || bs > (1 << 20)) return MLA_ERR_INVALID_ARG;
    if (!tile_scheduler_metadata || !num_splits || (bs > 0 && !cache_seqlens))
        return MLA_ERR_INVALID_ARG;
    if (!is_aligned(tile_scheduler_metadata, 16)) return MLA_ERR_INVALID_ARG;
    mla::get_mla_metadata_kernel<<<1, mla::kPlannerThreads, 0,
                                   reinterpret_cast<cudaStream_t>(stream)>>>(
        cache_seqlens, bs, num_sm_parts, tile_scheduler_metadata, num_splits);
    return from_cuda(cudaGetLastError());
}

mla_status_t mla_build_decode_metadata(
    const int32_t* req_to_token, int64_t req_to_token_rows, int64_t req_to_token_stride,
    const void* req_pool_indices, int32_t rpi_dtype, const void* seq_lens, int32_t seq_lens_dtype,
    int32_t seq_len_add, int32_t bs, int32_t* block_table, int64_t block_table_stride,
    int32_t max_pages, int32_t page_size, int32_t fill_tail, int32_t num_heads_per_head_k,
    int32_t num_heads_k, int32_t is_fp8_kvcache, int32_t sm_count, int32_t* cache_seqlens,
    int32_t* tile_scheduler_metadata, int32_t* num_splits, mla_stream_t stream) {
    const NvtxRange nvtx_range("mla_build_decode_metadata");
    (void)is_fp8_kvcache;  // accepted for call compatibility; the plan does not depend on it
    const int32_t parts = mla_num_sm_parts(sm_count, num_heads_per_head_k, num_heads_k);
    if (bs < 0 || max_pages < 0 || page_size != 64 || parts < 1 || bs > (1 << 20))
        return MLA_ERR_INVALID_ARG;
    if (rpi_dtype != MLA_DTYPE_INT32 && rpi_dtype != MLA_DTYPE_INT64) return MLA_ERR_INVALID_ARG;
    if (seq_lens_dtype != MLA_DTYPE_INT32 && seq_lens_dtype != MLA_DTYPE_INT64)
        return MLA_ERR_INVALID_ARG;
    if (!tile_scheduler_metadata || !num_splits || !is_aligned(tile_scheduler_metadata, 16))
        return MLA_ERR_INVALID_ARG;
    if (bs > 0 && (!req_to_token || !req_pool_indices || !seq_lens || !block_table))
        return MLA_ERR_INVALID_ARG;
    if (bs > 0 && (req_to_token_rows <= 0 || req_to_token_stride <= 0 || block_table_stride < max_pages))
        return MLA_ERR_INVALID_ARG;
    const int64_t entries = (int64_t)bs * max_pages;
    const int64_t table_ctas = (entries + mla::kPlannerThreads - 1) / mla::kPlannerThreads;
    if (table_ctas + 1 > INT32_MAX) return MLA_ERR_UNSUPPORTED;
    const dim3 grid((unsigned)(1 + table_ctas));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define MLA_MD_LAUNCH(IT, LT)                                                                      \
    mla::decode_metadata_kernel<IT, LT><<<grid, mla::kPlannerThreads, 0, st>>>(                   \
        req_to_token, req_to_token_rows, req_to_token_stride,                                      \
        static_cast<const IT*>(req_pool_indices), static_cast<const LT*>(seq_lens), seq_len_add,  \
        bs, block_table, block_table_stride, max_pages, fill_tail, parts, cache_seqlens,           \
        tile_scheduler_metadata, num_splits)
    if (rpi_dtype == MLA_DTYPE_INT64 && seq_lens_dtype == MLA_DTYPE_INT64) MLA_MD_LAUNCH(int64_t, int64_t);
    else if (rpi_dtype == MLA_DTYPE_INT64) MLA_MD_LAUNCH(int64_t, int32_t);
    else if (seq_lens_dtype == MLA_DTYPE_INT64) MLA_MD_LAUNCH(int32_t, int64_t);
    else MLA_MD_LAUNCH(int32_t, int32_t);
#undef MLA_MD_LAUNCH
    return from_cuda(cudaGetLastError());
}

size_t mla_decode_workspace_bytes(int32_t bs, int32_t q_len, int32_t h_q, int32_t num_sm_parts) {
    if (bs <= 0 || q_len <= 0 || h_q <= 0 || num_sm_parts <= 0) return 0;
    const size_t splits = (size_t)bs + (size_t)num_sm_parts;
    const size_t rows = (size_t)q_len * (size_t)h_q;
    return arrival_bytes(bs, q_len, h_q) + align256(splits * rows * 512 * sizeof(float)) +
           align256(splits * rows * sizeof(float));
}

mla_status_t mla_decode_paged(const void* q, int32_t q_dtype, int32_t bs, int32_t q_len,
                              int32_t h_q, int32_t head_dim, int32_t head_dim_v,
                              const void* k_cache, int32_t kv_dtype, int64_t num_pages,
                              int32_t page_size, const int32_t* block_table,
                              int64_t block_table_stride, int32_t max_pages,
                              const int32_t* cache_seqlens, const int32_t* tile_scheduler_metadata,
                              int32_t num_sm_parts, const int32_t* num_splits, float softmax_scale,
                              int32_t causal, const float* descale_q, const float* descale_k,
                              void* out, float* lse, void* workspace, size_t workspace_bytes,
                              mla_stream_t stream) {
    const NvtxRange nvtx_range("mla_decode_paged");
    if (bs < 0 || q_len <= 0 || h_q <= 0 || num_sm_parts < 1) return MLA_ERR_INVALID_ARG;
    if (head_dim != 576 || head_dim_v != 512 || page_size != 64) return MLA_ERR_UNSUPPORTED;
    if (q_dtype != MLA_DTYPE_BF16 && q_dtype != MLA_DTYPE_FP8_E4M3) return MLA_ERR_INVALID_ARG;
    if (kv_dtype != MLA_DTYPE_BF16 && kv_dtype != MLA_DTYPE_FP8_E4M3 && kv_dtype != MLA_DTYPE_FP8_E5M2)
        return MLA_ERR_INVALID_ARG;
    // e4m3 queries run e4m3 x e4m3 MMAs: only with an e4m3 cache (the backend's fp8 branch)
    if (q_dtype == MLA_DTYPE_FP8_E4M3 && kv_dtype != MLA_DTYPE_FP8_E4M3) return MLA_ERR_UNSUPPORTED;
    if (kv_dtype == MLA_DTYPE_BF16 && descale_k) return MLA_ERR_INVALID_ARG;  // fp8 caches only
    if (causal != 0 && causal != 1) return MLA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
    if (bs == 0) return MLA_OK;
    if (!q || !k_cache || !block_table || !cache_seqlens || !tile_scheduler_metadata ||
        !num_splits || !out || !lse)
        return MLA_ERR_INVALID_ARG;
    if (num_pages <= 0 || num_pages * 64 >= (int64_t(1) << 31)) return MLA_ERR_INVALID_ARG;
    if (max_pages <= 0 || block_table_stride < max_pages) return MLA_ERR_INVALID_ARG;
    // grid.y = cdiv(q_len * h_q, 128) query tiles, at most 65535
    if ((int64_t)q_len * h_q > int64_t(65535) * 128 || bs > 65535) return MLA_ERR_UNSUPPORTED;
    if (!is_aligned(q, 16) || !is_aligned(k_cache, 16) || !is_aligned(out, 16) ||
        !is_aligned(tile_scheduler_metadata, 16))
        return MLA_ERR_INVALID_ARG;
    const size_t need = mla_decode_workspace_bytes(bs, q_len, h_q, num_sm_parts);
    if (!workspace || workspace_bytes < need || !is_aligned(workspace, 256)) return MLA_ERR_WORKSPACE;

    mla_status_t st = prepare_decode_kernels();
    if (st != MLA_OK) return st;
    EncodeTiledFn encode = encode_tiled();
    if (!encode) return MLA_ERR_CUDA;

    // Tensor maps (bf16, 128-byte swizzle; coordinates past an extent read as zeros).  Each
    // view orders its dimensions so that one load lands as consecutive 64-row x 64-column
    // boxes (8 KB each), the layout the MMAs read:
    //   K: (64 columns, pool rows [1152 B], 9 column chunks [128 B]); a load = all nine
    //      column chunks of one page (72 KB).
    //   V: the same view with a box of two column chunks (16 KB): a partner page's V chunks.
    //   Q: (64 columns, rows of a request [1152 B], 9 column chunks [128 B], requests); a load
    //      = 64 query rows x columns [256, 576) (40 KB).
    const int32_t rows = q_len * h_q;
    CUtensorMap k_map, v_map, q_map;
    std::memset(&k_map, 0, sizeof k_map);
    std::memset(&v_map, 0, sizeof v_map);
    std::memset(&q_map, 0, sizeof q_map);
    const cuuint64_t pool_rows = (cuuint64_t)num_pages * 64;
    const bool fp8 = kv_dtype != MLA_DTYPE_BF16;
    if (!fp8) {
        const cuuint64_t gdim[3] = {64, pool_rows, 9};
        const cuuint64_t gstride[2] = {1152, 128};
        const cuuint32_t kbox[3] = {64, 64, (cuuint32_t)mla::decode::kChunks};
        const cuuint32_t vbox[3] = {64, 64, 2};
        const cuuint32_t estride[3] = {1, 1, 1};
        if (encode(&k_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(k_cache), gdim, gstride,
                   kbox, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MLA_ERR_CUDA;
        if (encode(&v_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(k_cache), gdim, gstride,
                   vbox, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MLA_ERR_CUDA;
    } else {
        // 8-bit: (64 one-byte columns, pool rows [576 B], 9 column chunks [64 B]); a K load = one
        // page as 9 chunks of 64 rows x 64 bytes (36 KB).  Unswizzled for bf16 queries (the page
        // is widened to f16 before S); 64-byte swizzle for e4m3 queries (S reads it as it is).
        const bool q8 = q_dtype == MLA_DTYPE_FP8_E4M3;
        const cuuint64_t gdim[3] = {64, pool_rows, 9};
        const cuuint64_t gstride[2] = {576, 64};
        const cuuint32_t kbox[3] = {64, 64, 9};
        const cuuint32_t estride[3] = {1, 1, 1};
        if (encode(&k_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(k_cache), gdim, gstride,
                   kbox, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   q8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MLA_ERR_CUDA;
        v_map = k_map;   // the e4m3 path reads partner V through registers
    }
    if (q_dtype == MLA_DTYPE_FP8_E4M3) {
        // e4m3 q: (64 one-byte columns, rows of a request [576 B], 9 column chunks [64 B],
        // requests); a load = 64 query rows x all 576 columns (36 KB), 64-byte swizzle
        const cuuint64_t gdim[4] = {64, (cuuint64_t)rows, 9, (cuuint64_t)bs};
        const cuuint64_t gstride[3] = {576, 64, (cuuint64_t)rows * 576};
        const cuuint32_t box[4] = {64, 64, 9, 1};
        const cuuint32_t estride[4] = {1, 1, 1, 1};
        if (encode(&q_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(q), gdim, gstride, box,
                   estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MLA_ERR_CUDA;
    } else {
        const cuuint64_t gdim[4] = {64, (cuuint64_t)rows, 9, (cuuint64_t)bs};
        const cuuint64_t gstride[3] = {1152, 128, (cuuint64_t)rows * 1152};
        const cuuint32_t box[4] = {64, 64, 5, 1};
        const cuuint32_t estride[4] = {1, 1, 1, 1};
        if (encode(&q_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(q), gdim, gstride, box,
                   estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MLA_ERR_CUDA;
    }

    const size_t splits = (size_t)bs + (size_t)num_sm_parts;
    mla::decode::Params p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.kv = static_cast<const uint8_t*>(k_cache);
    p.block_table = block_table;
    p.bt_stride = block_table_stride;
    p.max_pages = max_pages;
    p.cache_seqlens = cache_seqlens;
    p.md = tile_scheduler_metadata;
    p.num_splits = num_splits;
    p.bs = bs;
    p.q_len = q_len;
    p.h_q = h_q;
    p.rows = rows;
    p.num_pages = num_pages;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.descale_q = descale_q;
    p.descale_k = descale_k;
    p.causal = causal;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.arrivals = reinterpret_cast<int32_t*>(ws);
    const uint64_t budget = g_hook_wait_budget_ns.load(std::memory_order_relaxed);
    p.wait_budget_ns = budget ? budget : mla::kWaitBudgetNs;
    p.withhold_tile = g_hook_withhold_tile.load(std::memory_order_relaxed);
    p.part_o = reinterpret_cast<float*>(ws + arrival_bytes(bs, q_len, h_q));
    p.part_lse = reinterpret_cast<float*>(ws + arrival_bytes(bs, q_len, h_q) +
                                          align256(splits * rows * 512 * sizeof(float)));
    // For the fold-in merge's loads: part_o viewed as fp32 [column group (16, 128 B apart)][row
    // (splits * rows, 2048 B apart)][32 columns], boxes of 8 groups x 64 rows x 32 columns (64 KB,
    // landing as eight 64-row x 128-byte blocks, 128-byte swizzle); part_lse as [splits][rows],
    // boxes of 64 rows of one piece (rows a multiple of 4, so that its stride is a multiple of 16
    // bytes; otherwise no fold-in).
    CUtensorMap po_map, pl_map;
    std::memset(&po_map, 0, sizeof po_map);
    std::memset(&pl_map, 0, sizeof pl_map);
    p.fold_ok = 0;
    if ((uint64_t)splits * (uint64_t)rows <= (uint64_t)INT32_MAX && rows % 4 == 0) {
        const cuuint64_t gdim[3] = {(cuuint64_t)mla::decode::kFoldBoxCols, (cuuint64_t)splits * (cuuint64_t)rows,
                                    512 / (cuuint64_t)mla::decode::kFoldBoxCols};
        const cuuint64_t gstride[2] = {512 * sizeof(float), mla::decode::kFoldBoxCols * sizeof(float)};
        const cuuint32_t box[3] = {(cuuint32_t)mla::decode::kFoldBoxCols, (cuuint32_t)mla::decode::kCtaRows, 8};
        const cuuint32_t estride[3] = {1, 1, 1};
        const cuuint64_t ldim[2] = {(cuuint64_t)rows, (cuuint64_t)splits};
        const cuuint64_t lstride[1] = {(cuuint64_t)rows * sizeof(float)};
        const cuuint32_t lbox[2] = {(cuuint32_t)mla::decode::kCtaRows, 1};
        if (encode(&po_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p.part_o, gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS &&
            encode(&pl_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, p.part_lse, ldim, lstride, lbox, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            p.fold_ok = g_hook_no_fold_in.load(std::memory_order_relaxed) ? 0 : 1;
    }
    // The epilogue's stores: o bf16 viewed as [bs][rows][512] in boxes of 32 rows x 64 columns, the
    // partials fp32 [splits][rows][512] in boxes of 32 rows x 32 columns (128 bytes a row, 128-byte
    // swizzle); rows past a request's last are clipped by the view.
    CUtensorMap o_map, ps_map;
    std::memset(&o_map, 0, sizeof o_map);
    std::memset(&ps_map, 0, sizeof ps_map);
    {
        const cuuint64_t odim[3] = {512, (cuuint64_t)rows, (cuuint64_t)bs};
        const cuuint64_t ostride[2] = {512 * 2, (cuuint64_t)rows * 512 * 2};
        const cuuint32_t obox[3] = {64, 32, 1};
        const cuuint64_t sdim[3] = {512, (cuuint64_t)rows, (cuuint64_t)splits};
        const cuuint64_t sstride[2] = {512 * 4, (cuuint64_t)rows * 512 * 4};
        const cuuint32_t sbox[3] = {32, 32, 1};
        const cuuint32_t estride[3] = {1, 1, 1};
        if (encode(&o_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, out, odim, ostride, obox, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
            encode(&ps_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p.part_o, sdim, sstride, sbox, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MLA_ERR_CUDA;
    }

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid(2 * num_sm_parts, (rows + 127) / 128);
    using mla::decode::kSmemBytes;
    using mla::decode::kThreads;
    // A programmatic dependent launch (the pair size comes from the kernel's cluster
    // dimensions): when the grid before it in the stream lets it in early, as the metadata
    // kernels do, its set-up overlaps that grid; it waits for that grid to complete before it
    // reads anything (with any other predecessor it starts once that one has completed).
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t dcfg = {};
    dcfg.gridDim = grid;
    dcfg.blockDim = dim3(kThreads);
    dcfg.dynamicSmemBytes = kSmemBytes;
    dcfg.stream = s;
    dcfg.attrs = pdl;
    dcfg.numAttrs = 1;
    cudaError_t e;
    if (q_dtype == MLA_DTYPE_FP8_E4M3)
        e = cudaLaunchKernelEx(&dcfg, mla::decode::mla_decode_kernel<1, true>, k_map, v_map, q_map, po_map, pl_map, o_map, ps_map, p);
    else if (kv_dtype == MLA_DTYPE_FP8_E4M3)
        e = cudaLaunchKernelEx(&dcfg, mla::decode::mla_decode_kernel<1, false>, k_map, v_map, q_map, po_map, pl_map, o_map, ps_map, p);
    else if (kv_dtype == MLA_DTYPE_FP8_E5M2)
        e = cudaLaunchKernelEx(&dcfg, mla::decode::mla_decode_kernel<2, false>, k_map, v_map, q_map, po_map, pl_map, o_map, ps_map, p);
    else
        e = cudaLaunchKernelEx(&dcfg, mla::decode::mla_decode_kernel<0, false>, k_map, v_map, q_map, po_map, pl_map, o_map, ps_map, p);
    if (e != cudaSuccess) return MLA_ERR_CUDA;
    // The merge of requests of many pieces, as a programmatic dependent launch: scheduled while
    // the attention kernel runs, it waits on the device for that grid to complete.
    cudaLaunchConfig_t cfg = {};
    {
        const int64_t need = ((int64_t)bs * rows * mla::kMergeSlices + mla::kCombineWarps - 1) / mla::kCombineWarps;
        // a warp per (request, row, column slice), at most as many CTAs as the attention grid (one per SM)
        cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(need, (int64_t)grid.x * grid.y)));
    }
    cfg.blockDim = dim3(mla::kCombineWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, mla::combine_splits_kernel, (const float*)p.part_o, (const float*)p.part_lse,
                           num_splits, rows, bs, p.out, lse);
    return from_cuda(e);
}

mla_status_t mla_set_kv_buffer(void* kv_cache, int32_t kv_dtype, int64_t num_slots, const void* cache_loc,
                               int32_t loc_dtype, int32_t n_tokens, const void* k, int64_t k_row_stride,
                               const float* k_scale, mla_stream_t stream) {
    const NvtxRange nvtx_range("mla_set_kv_buffer");
    if (n_tokens < 0 || num_slots < 0) return MLA_ERR_INVALID_ARG;
    if (kv_dtype != MLA_DTYPE_BF16 && kv_dtype != MLA_DTYPE_FP8_E4M3 && kv_dtype != MLA_DTYPE_FP8_E5M2)
        return MLA_ERR_INVALID_ARG;
    if (loc_dtype != MLA_DTYPE_INT32 && loc_dtype != MLA_DTYPE_INT64) return MLA_ERR_INVALID_ARG;
    if (kv_dtype == MLA_DTYPE_BF16 && k_scale) return MLA_ERR_INVALID_ARG;   // a scale is for fp8 pools
    if (n_tokens == 0) return MLA_OK;
    if (!kv_cache || !cache_loc || !k) return MLA_ERR_INVALID_ARG;
    if (k_row_stride < 576 || k_row_stride % 8 != 0 || !is_aligned(k, 16)) return MLA_ERR_INVALID_ARG;
    if (!is_aligned(kv_cache, kv_dtype == MLA_DTYPE_BF16 ? 16 : 8)) return MLA_ERR_INVALID_ARG;
    const dim3 grid((unsigned)((n_tokens + mla::kKvWriteWarps - 1) / mla::kKvWriteWarps));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* pool = static_cast<uint8_t*>(kv_cache);
    const __nv_bfloat16* kk = static_cast<const __nv_bfloat16*>(k);
#define MLA_KV_LAUNCH(FMT, LT)                                                                     \
    mla::set_kv_buffer_kernel<FMT, LT><<<grid, mla::kKvWriteWarps * 32, 0, st>>>(                  \
        pool, num_slots, static_cast<const LT*>(cache_loc), n_tokens, kk, k_row_stride, k_scale)
    const bool l64 = loc_dtype == MLA_DTYPE_INT64;
    if (kv_dtype == MLA_DTYPE_BF16) {
        if (l64) MLA_KV_LAUNCH(0, int64_t); else MLA_KV_LAUNCH(0, int32_t);
    } else if (kv_dtype == MLA_DTYPE_FP8_E4M3) {
        if (l64) MLA_KV_LAUNCH(1, int64_t); else MLA_KV_LAUNCH(1, int32_t);
    } else {
        if (l64) MLA_KV_LAUNCH(2, int64_t); else MLA_KV_LAUNCH(2, int32_t);
    }
#undef MLA_KV_LAUNCH
    return from_cuda(cudaGetLastError());
}

mla_status_t mla_merge_state(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                             int64_t rows, int32_t head_dim_v, void* o, float* lse, mla_stream_t stream) {
    const NvtxRange nvtx_range("mla_merge_state");
    if (rows < 0 || head_dim_v != 512) return rows < 0 ? MLA_ERR_INVALID_ARG : MLA_ERR_UNSUPPORTED;
    if (rows == 0) return MLA_OK;
    if (!o_a || !lse_a || !o_b || !lse_b || !o || !lse) return MLA_ERR_INVALID_ARG;
    if (!is_aligned(o_a, 16) || !is_aligned(o_b, 16) || !is_aligned(o, 16)) return MLA_ERR_INVALID_ARG;
    const int64_t blocks = (rows + mla::kMergeStateWarps - 1) / mla::kMergeStateWarps;
    if (blocks > INT32_MAX) return MLA_ERR_UNSUPPORTED;
    mla::merge_state_kernel<<<(unsigned)blocks, mla::kMergeStateWarps * 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16*>(o_a), lse_a, static_cast<const __nv_bfloat16*>(o_b), lse_b, rows,
        static_cast<__nv_bfloat16*>(o), lse);
    return from_cuda(cudaGetLastError());
}

namespace {
// The extend workspace, 256-byte aligned parts in this order (sizes in bytes).
struct ExtendLayout {
    size_t pool, bt_r, cl_r, md_r, ns_r, ws_r, o1, lse1, bt_p, cl_p, md_p, ns_p, ws_p, o2, lse2, total;
    int32_t parts, e_pad;
    bool copy;
};
bool extend_layout(int32_t bs, int32_t e, int32_t h_q, int32_t max_prefix_pages, int32_t sm_count, ExtendLayout& L) {
    if (bs <= 0 || e <= 0 || h_q <= 0 || max_prefix_pages < 0 || sm_count <= 0) return false;
    L.parts = mla_num_sm_parts(sm_count, e * h_q, 1);
    if (L.parts < 1) return false;
    L.e_pad = (int32_t)(((int64_t)e + 63) / 64 * 64);
    L.copy = L.e_pad != e;
    const size_t rows = (size_t)bs * (size_t)e * (size_t)h_q;
    const size_t ws = mla_decode_workspace_bytes(bs, e, h_q, L.parts);
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t at = off; off += align256(bytes); return at; };
    L.pool = take(L.copy ? (size_t)bs * L.e_pad * 576 * 2 : 0);
    L.bt_r = take((size_t)bs * (L.e_pad / 64) * 4);
    L.cl_r = take((size_t)bs * 4);
    L.md_r = take((size_t)L.parts * 8 * 4);
    L.ns_r = take(((size_t)bs + 1) * 4);
    L.ws_r = take(ws);
    L.o1 = take(rows * 512 * 2);
    L.lse1 = take(rows * 4);
    L.bt_p = take((size_t)bs * std::max(max_prefix_pages, 1) * 4);
    L.cl_p = take((size_t)bs * 4);
    L.md_p = take((size_t)L.parts * 8 * 4);
    L.ns_p = take(((size_t)bs + 1) * 4);
    L.ws_p = take(ws);
    L.o2 = take(rows * 512 * 2);
    L.lse2 = take(rows * 4);
    L.total = off;
    return true;
}
}  // namespace

size_t mla_extend_workspace_bytes(int32_t bs, int32_t e, int32_t h_q, int32_t max_prefix_pages, int32_t sm_count) {
    ExtendLayout L;
    return extend_layout(bs, e, h_q, max_prefix_pages, sm_count, L) ? L.total : 0;
}

mla_status_t mla_extend_paged_prefix(const void* q, int32_t bs, int32_t e, int32_t h_q, const void* k_new,
                                     const void* kv_cache, int32_t kv_dtype, int64_t num_pages,
                                     const int32_t* req_to_token, int64_t req_to_token_rows,
                                     int64_t req_to_token_stride, const void* req_pool_indices,
                                     int32_t rpi_dtype, const int32_t* prefix_lens, int32_t max_prefix_pages,
                                     float softmax_scale, const float* descale_k, int32_t sm_count, void* out,
                                     float* lse, void* workspace, size_t workspace_bytes, mla_stream_t stream) {
    const NvtxRange nvtx_range("mla_extend_paged_prefix");
    if (bs == 0) return MLA_OK;
    ExtendLayout L;
    if (!extend_layout(bs, e, h_q, max_prefix_pages, sm_count, L)) return MLA_ERR_INVALID_ARG;
    if ((int64_t)e * h_q > 65535LL * 128) return MLA_ERR_UNSUPPORTED;
    if (!q || !k_new || !kv_cache || !prefix_lens || !out || !lse) return MLA_ERR_INVALID_ARG;
    if (!is_aligned(k_new, 16)) return MLA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < L.total || !is_aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
    const int64_t ragged_pages = (int64_t)bs * (L.e_pad / 64);
    if (ragged_pages * 64 > INT32_MAX) return MLA_ERR_UNSUPPORTED;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    auto at = [&](size_t off) { return static_cast<void*>(w + off); };
    auto i32 = [&](size_t off) { return reinterpret_cast<int32_t*>(w + off); };
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t rows = (size_t)bs * e * h_q;
    mla_status_t r;
    // (1) the new tokens among themselves, causal: their rows as a paged pool of their own
    {
        const int64_t units = L.copy ? (int64_t)bs * e * 72 : (int64_t)bs * (L.e_pad / 64);
        const int64_t blocks = std::min<int64_t>((units + mla::kExtendThreads - 1) / mla::kExtendThreads, 4096);
        mla::extend_ragged_view_kernel<<<(unsigned)std::max<int64_t>(blocks, 1), mla::kExtendThreads, 0, st>>>(
            static_cast<const uint4*>(k_new), bs, e, L.e_pad, L.copy ? static_cast<uint4*>(at(L.pool)) : nullptr,
            i32(L.bt_r), i32(L.cl_r));
        if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    }
    r = mla_get_mla_metadata(i32(L.cl_r), bs, e * h_q, 1, 0, sm_count, i32(L.md_r), i32(L.ns_r), stream);
    if (r != MLA_OK) return r;
    r = mla_decode_paged(q, MLA_DTYPE_BF16, bs, e, h_q, 576, 512, L.copy ? at(L.pool) : k_new, MLA_DTYPE_BF16,
                         ragged_pages, 64, i32(L.bt_r), L.e_pad / 64, L.e_pad / 64, i32(L.cl_r), i32(L.md_r), L.parts,
                         i32(L.ns_r), softmax_scale, 1, nullptr, nullptr, at(L.o1),
                         reinterpret_cast<float*>(at(L.lse1)), at(L.ws_r), L.o1 - L.ws_r, stream);
    if (r != MLA_OK) return r;
    // (2) the cached prefix, all of it
    const int32_t mpp = std::max(max_prefix_pages, 1);
    r = mla_build_decode_metadata(req_to_token, req_to_token_rows, req_to_token_stride, req_pool_indices, rpi_dtype,
                                  prefix_lens, MLA_DTYPE_INT32, 0, bs, i32(L.bt_p), mpp, mpp, 64, 1, e * h_q, 1,
                                  kv_dtype != MLA_DTYPE_BF16, sm_count, i32(L.cl_p), i32(L.md_p), i32(L.ns_p), stream);
    if (r != MLA_OK) return r;
    r = mla_decode_paged(q, MLA_DTYPE_BF16, bs, e, h_q, 576, 512, kv_cache, kv_dtype, num_pages, 64, i32(L.bt_p), mpp,
                         mpp, i32(L.cl_p), i32(L.md_p), L.parts, i32(L.ns_p), softmax_scale, 0, nullptr, descale_k,
                         at(L.o2), reinterpret_cast<float*>(at(L.lse2)), at(L.ws_p), L.o2 - L.ws_p, stream);
    if (r != MLA_OK) return r;
    // (3) merge_state
    return mla_merge_state(at(L.o1), reinterpret_cast<const float*>(at(L.lse1)), at(L.o2),
                           reinterpret_cast<const float*>(at(L.lse2)), (int64_t)rows, 512, out, lse, stream);
}

mla_status_t mla_set_test_hooks(uint64_t wait_budget_ns, int32_t withhold_tile, int32_t no_fold_in) {
    if (withhold_tile < -1) return MLA_ERR_INVALID_ARG;
    g_hook_wait_budget_ns.store(wait_budget_ns, std::memory_order_relaxed);
    g_hook_withhold_tile.store(withhold_tile, std::memory_order_relaxed);
    g_hook_no_fold_in.store(no_fold_in != 0, std::memory_order_relaxed);
    return MLA_OK;
}

mla_status_t mla_read_device_error(int32_t* code_out, mla_stream_t stream) {
    if (!code_out) return MLA_ERR_INVALID_ARG;
    int value = 0;
    const int zero = 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyFromSymbolAsync(&value, mla::g_device_error, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(mla::g_device_error, &zero, sizeof(int), 0,
                                    cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return MLA_ERR_CUDA;
    *code_out = value;
    return value ? MLA_ERR_DEVICE_CHECK : MLA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Workspace-free variant of mla_decode_paged for callers that cannot allocate device
// memory (see the header).  Its split-KV scratch is this fixed array, which every GPU
// that loads the library holds until exit.
namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

// The array's name is only a host-side stand-in; the device address must be looked up on
// each device, with that device current.  Done once per device, on its first call.
mla_status_t noalloc_scratch_address(void** out) {
    static std::once_flag flags[kMaxDevices];
    static void* addrs[kMaxDevices];
    static cudaError_t results[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
    std::call_once(flags[dev], [dev] {
        void* p = nullptr;
        results[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        addrs[dev] = p;
    });
    if (results[dev] != cudaSuccess || addrs[dev] == nullptr) return MLA_ERR_CUDA;
    *out = addrs[dev];
    return MLA_OK;
}

}  // namespace

extern "C" mla_status_t mla_decode_paged_noalloc(
    const void* q, int32_t q_dtype, int32_t bs, int32_t q_len, int32_t h_q, int32_t head_dim,
    int32_t head_dim_v, const void* k_cache, int32_t kv_dtype, int64_t num_pages,
    int32_t page_size, const int32_t* block_table, int64_t block_table_stride, int32_t max_pages,
    const int32_t* cache_seqlens, const int32_t* tile_scheduler_metadata, int32_t num_sm_parts,
    const int32_t* num_splits, float softmax_scale, int32_t causal, const float* descale_q,
    const float* descale_k, void* out, float* lse, mla_stream_t stream) {
    if (bs > 0 && q_len > 0 && h_q > 0 && num_sm_parts > 0 &&
        mla_decode_workspace_bytes(bs, q_len, h_q, num_sm_parts) > MLA_NOALLOC_SCRATCH_BYTES)
        return MLA_ERR_WORKSPACE;  // the problem needs more scratch than the fixed array holds
    void* scratch = nullptr;
    if (bs > 0) {
        const mla_status_t st = noalloc_scratch_address(&scratch);
        if (st != MLA_OK) return st;
        // The array keeps whatever the last call left; its leading arrival words must be zero
        // when the attention starts (a completed call leaves them zero, an aborted one may not).
        if (q_len > 0 && h_q > 0 &&
            cudaMemsetAsync(scratch, 0, arrival_bytes(bs, q_len, h_q), reinterpret_cast<cudaStream_t>(stream)) !=
                cudaSuccess)
            return MLA_ERR_CUDA;
    }
    return mla_decode_paged(q, q_dtype, bs, q_len, h_q, head_dim, head_dim_v, k_cache, kv_dtype,
                            num_pages, page_size, block_table, block_table_stride, max_pages,
                            cache_seqlens, tile_scheduler_metadata, num_sm_parts, num_splits,
                            softmax_scale, causal, descale_q, descale_k, out, lse, scratch,
                            MLA_NOALLOC_SCRATCH_BYTES, stream);
}
