/*
 * Plain CPU fp64 oracle for paged MLA decode — TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
 * load this library.  It shares no code, header, table or constant with the CUDA
 * path: every routine below is written from the definitions of the operations as
 * the SGLang FlashMLA attention backend page (flashmla_backend.py) calls them,
 * in the most direct loop form, with no blocking, fusion or reordering.
 *
 * Functions and the passages they follow:
 *   oracle_build_block_table  flashmla_backend.py, FlashMLABackend.init_forward_metadata
 *                             (decode and target-verify branches: a [bs, cdiv(max L,64)]
 *                             int32 table pre-filled with -1, filled from req_to_token /
 *                             req_pool_indices / seq_lens by the kv-indices kernel).
 *   oracle_num_sm_parts,      flashmla_backend.py, init_forward_metadata and
 *   oracle_get_mla_metadata   _apply_decode_target_verify_metadata (get_mla_metadata:
 *                             [num_sm_parts, 8] int32 scheduler rows, num_splits [bs+1]).
 *                             The pages fix only the shapes; the field contents are this
 *                             project's stated reading (a greedy balanced partition of
 *                             64-token blocks with a fixed per-piece overhead).
 *   oracle_mla_decode_rows    flashmla_backend.py, forward_decode / forward_extend
 *                             (flash_mla_with_kvcache: q [bs, q_len, h, 576] over the latent
 *                             cache viewed [-1, 64, 1, 576], head_dim_v = kv_lora_rank = 512,
 *                             softmax_scale, causal, descale_q / descale_k for fp8).
 *                             Keys are gathered token by token through req_to_token, never
 *                             through the page table.
 *   oracle_merge_states       the log-sum-exp merge of partial attention states
 *                             (flashinfer_backend.py, forward_extend: merge_state of a
 *                             ragged and a paged partial result).
 *   oracle_set_kv_buffer      flashmla_backend.py, forward_decode / forward_extend
 *                             (token_to_kv_pool.set_kv_buffer(layer, cache_loc, k, v): the
 *                             new tokens' 576-wide latent rows written at their pool slots
 *                             before attention; an fp8 pool, float8_e4m3fn or float8_e5m2 as
 *                             __init__ lists them, stores k / k_scale rounded to its format).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 is the upper half of an IEEE binary32; widening to double is exact. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP float8 e4m3 ("fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits,
 * subnormals when the exponent field is 0, S.1111.111 is NaN, no infinities. */
static double e4m3_bits_to_double(uint8_t bits) {
    int sign = bits >> 7;
    int e = (bits >> 3) & 0xF;
    int m = bits & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);            /* m/8 * 2^(1-7) */
    else
        v = ldexp((double)(8 + m), e - 10);  /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* OCP float8 e5m2: 1 sign, 5 exponent (bias 15), 2 mantissa bits, subnormals when the
 * exponent field is 0; exponent field 31 holds infinities (mantissa 0) and NaNs. */
static double e5m2_bits_to_double(uint8_t bits) {
    int sign = bits >> 7;
    int e = (bits >> 2) & 0x1F;
    int m = bits & 0x3;
    double v;
    if (e == 0x1F) v = m == 0 ? INFINITY : NAN;
    else if (e == 0)
        v = ldexp((double)m, -16);           /* m/4 * 2^(1-15) */
    else
        v = ldexp((double)(4 + m), e - 17);  /* (1 + m/4) * 2^(e-15) */
    return sign ? -v : v;
}

/* Element of an 8-bit cache: format 1 = e4m3, 2 = e5m2. */
static double fp8_bits_to_double(uint8_t bits, int format) {
    return format == 2 ? e5m2_bits_to_double(bits) : e4m3_bits_to_double(bits);
}

/*
 * Round x to the 8-bit format (1 = e4m3, 2 = e5m2) by brute force: among the codes of x's
 * sign, the one whose value is nearest to x, ties to the code with an even mantissa (even
 * code); magnitudes beyond the largest finite value give that value (saturation); NaN gives
 * the format's NaN code.
 */
static uint8_t quantize_fp8(double x, int format) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    int best = -1, top = 0;
    double best_err = INFINITY;
    for (int code = 0; code < 0x80; ++code)   /* the largest finite code of the format */
        if (isfinite(fp8_bits_to_double((uint8_t)code, format))) top = code;
    if (a >= fp8_bits_to_double((uint8_t)top, format)) return (uint8_t)(sign | top);
    for (int code = 0; code < 0x80; ++code) {
        double v = fp8_bits_to_double((uint8_t)code, format);
        if (!isfinite(v)) continue;
        double err = fabs(v - a);
        if (err < best_err || (err == best_err && (code & 1) == 0)) {
            best = code;
            best_err = err;
        }
    }
    return (uint8_t)(sign | best);
}

/* Threads the OpenMP loops use (the host's cores unless OMP_NUM_THREADS says otherwise). */
int oracle_num_threads(void) { return omp_get_max_threads(); }

double oracle_e4m3_to_double(uint8_t bits) { return e4m3_bits_to_double(bits); }
double oracle_e5m2_to_double(uint8_t bits) { return e5m2_bits_to_double(bits); }
uint8_t oracle_quantize_fp8(double x, int format) { return quantize_fp8(x, format); }
double oracle_bf16_to_double(uint16_t bits) { return bf16_bits_to_double(bits); }

static int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }

/*
 * Page table.  For request b with total KV length L_b = seq_lens[b] + seq_len_add
 * (seq_len_add is the number of draft tokens in target-verify, 0 in decode), and
 * for every page p < cdiv(L_b, page_size):
 *     block_table[b, p] = req_to_token[req_pool_indices[b], p * page_size] / page_size
 * Every other entry of the row (up to max_pages) is -1.  The slot -> page division
 * follows from the kernel viewing the token-slot pool as [-1, 64, 1, 576]: page P
 * holds slots 64P .. 64P+63.
 */
void oracle_build_block_table(const int32_t* req_to_token, int64_t r2t_stride,
                              const int64_t* req_pool_indices, const int64_t* seq_lens,
                              int64_t seq_len_add, int64_t bs, int32_t* block_table,
                              int64_t bt_stride, int64_t max_pages, int64_t page_size) {
    for (int64_t b = 0; b < bs; ++b) {
        int64_t L = seq_lens[b] + seq_len_add;
        int64_t npages = L > 0 ? cdiv64(L, page_size) : 0;
        for (int64_t p = 0; p < max_pages; ++p) {
            int32_t v = -1;
            if (p < npages) {
                int64_t slot = req_to_token[req_pool_indices[b] * r2t_stride + p * page_size];
                v = (int32_t)(slot / page_size);
            }
            block_table[b * bt_stride + p] = v;
        }
    }
}

/* Number of scheduler parts: one part per pair of SMs per 128-row query tile,
 * divided among the KV heads (this project's reading of get_mla_metadata's
 * num_sm_parts; it must not exceed the SM count, which the pages assert). */
int64_t oracle_num_sm_parts(int64_t sm_count, int64_t num_heads_per_head_k, int64_t num_heads_k) {
    int64_t m_tiles = cdiv64(num_heads_per_head_k, 128);
    int64_t parts = sm_count / (2 * m_tiles * num_heads_k);
    return parts < 1 ? 1 : parts;
}

/*
 * Split-KV plan (this project's reading of get_mla_metadata; the pages show only
 * its shapes).  blocks_b = cdiv(L_b, 64); every piece of a request costs its blocks
 * plus a fixed overhead F; total = sum_b (blocks_b + F); each of the P parts gets a
 * budget payload = cdiv(total, P) + F and is filled greedily, earliest request first:
 * a request that fits in what is left of the budget is taken whole; otherwise the
 * part takes (budget - F) blocks of it when that is positive, and ends.
 *
 * Row i of tile_scheduler_metadata is
 *     [begin_req, begin_block, end_req, end_block, begin_split, 0, 0, 0]
 * with (end_req, end_block) the exclusive cursor after the part, and begin_split the
 * index of the part's first piece within its request.  num_splits[0] = 0 and
 * num_splits[b+1] = num_splits[b] + (number of pieces of request b).
 */
void oracle_get_mla_metadata(const int32_t* cache_seqlens, int64_t bs, int64_t num_parts,
                             int64_t fixed_overhead, int32_t* md, int32_t* num_splits) {
    int64_t total = 0;
    for (int64_t b = 0; b < bs; ++b) {
        int64_t L = cache_seqlens[b] > 0 ? cache_seqlens[b] : 0;
        total += cdiv64(L, 64) + fixed_overhead;
    }
    int64_t payload = cdiv64(total, num_parts) + fixed_overhead;
    int64_t b = 0, k = 0, s = 0, cum = 0;
    num_splits[0] = 0;
    for (int64_t i = 0; i < num_parts; ++i) {
        int64_t begin_b = b, begin_k = k, begin_s = s;
        int64_t budget = payload;
        while (b < bs) {
            int64_t L = cache_seqlens[b] > 0 ? cache_seqlens[b] : 0;
            int64_t rem = cdiv64(L, 64) - k;
            if (budget >= rem + fixed_overhead) {
                cum += s + 1;
                num_splits[b + 1] = (int32_t)cum;
                budget -= rem + fixed_overhead;
                ++b;
                k = 0;
                s = 0;
            } else {
                if (budget - fixed_overhead > 0) {
                    k += budget - fixed_overhead;
                    ++s;
                }
                break;
            }
        }
        int32_t* row = md + 8 * i;
        row[0] = (int32_t)begin_b;
        row[1] = (int32_t)begin_k;
        row[2] = (int32_t)b;
        row[3] = (int32_t)k;
        row[4] = (int32_t)begin_s;
        row[5] = row[6] = row[7] = 0;
    }
}

/*
 * One attention row: query (b, i, h) against keys j in [j_begin, j_end) of request b,
 * restricted to the causally allowed keys.  The allowed keys are j < lim with
 * lim = L - q_len + i + 1 under causal (the draft tokens' own KV is the last q_len
 * positions of the cache, written before attention), lim = L otherwise.
 *   k_j = KV[req_to_token[rpi[b], j], 0:dq] (* descale_k for an fp8 cache)   (fp64, exact)
 *   v_j = k_j[0:dv]
 *   s_j = softmax_scale * descale_q * sum_d q[d] * k_j[d]
 *   lse = m + ln(sum_j exp(s_j - m)),  m = max_j s_j
 *   o   = sum_j exp(s_j - lse) * v_j
 * With no allowed key: o = 0 and lse = -inf.
 */
static void attend_row(const void* q_row, int q_is_fp8, const uint8_t* kv, int kv_format,
                       double descale_q, double descale_k, const int32_t* r2t_row, int64_t j_begin,
                       int64_t j_end, int64_t dq, int64_t dv, double softmax_scale, double* o,
                       double* lse, double* s_buf) {
    double qd[1024];
    for (int64_t d = 0; d < dq; ++d)
        qd[d] = q_is_fp8 ? e4m3_bits_to_double(((const uint8_t*)q_row)[d])
                         : bf16_bits_to_double(((const uint16_t*)q_row)[d]);
    int64_t n = j_end - j_begin;
    if (n <= 0) {
        for (int64_t d = 0; d < dv; ++d) o[d] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int64_t t = 0; t < n; ++t) {
        int64_t slot = r2t_row[j_begin + t];
        double acc = 0.0;
        for (int64_t d = 0; d < dq; ++d) {
            double kd = kv_format ? fp8_bits_to_double(kv[slot * dq + d], kv_format) * descale_k
                                  : bf16_bits_to_double(((const uint16_t*)kv)[slot * dq + d]);
            acc += qd[d] * kd;
        }
        s_buf[t] = softmax_scale * descale_q * acc;
        if (s_buf[t] > m) m = s_buf[t];
    }
    double sum = 0.0;
    for (int64_t t = 0; t < n; ++t) sum += exp(s_buf[t] - m);
    double l = m + log(sum);
    for (int64_t d = 0; d < dv; ++d) o[d] = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        int64_t slot = r2t_row[j_begin + t];
        double w = exp(s_buf[t] - l);
        for (int64_t d = 0; d < dv; ++d) {
            double vd = kv_format ? fp8_bits_to_double(kv[slot * dq + d], kv_format) * descale_k
                                  : bf16_bits_to_double(((const uint16_t*)kv)[slot * dq + d]);
            o[d] += w * vd;
        }
    }
    *lse = l;
}

/*
 * Attention for a list of rows.  row_ids[r] is the flat index (b * q_len + i) * h + hh
 * into the [bs, q_len, h] grid; o_out is [n_rows, dv] and lse_out [n_rows].
 * key_begin / key_end (nullable, indexed by b) restrict request b's keys to a range
 * before the causal limit is applied; null means the whole [0, L).
 * kv is the flat token-slot pool [num_slots, dq] of bf16 bits (kv_format = 0), e4m3
 * bytes (kv_format = 1) or e5m2 bytes (kv_format = 2); q is [bs, q_len, h, dq] of bf16 bits (q_is_fp8 = 0) or e4m3
 * bytes (q_is_fp8 = 1: the flash_mla_with_kvcache call of the FlashMLA backend page, with q
 * quantised by scaled_fp8_quant and descale_q its scale).  Returns 0, or -1 when the query
 * width exceeds 1024.
 */
int oracle_mla_decode_rows(const void* q, int q_is_fp8, const void* kv, int kv_format, double descale_q,
                           double descale_k, const int32_t* req_to_token, int64_t r2t_stride,
                           const int64_t* req_pool_indices, const int32_t* cache_seqlens,
                           const int64_t* key_begin, const int64_t* key_end, int64_t bs,
                           int64_t q_len, int64_t h, int64_t dq, int64_t dv, double softmax_scale,
                           int causal, int64_t n_rows, const int64_t* row_ids, double* o_out,
                           double* lse_out) {
    if (dq > 1024) return -1;
    (void)bs;
    int64_t max_len = 0;
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t b = row_ids[r] / (q_len * h);
        if (cache_seqlens[b] > max_len) max_len = cache_seqlens[b];
    }
#pragma omp parallel
    {
        double* s_buf = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t flat = row_ids[r];
            int64_t b = flat / (q_len * h);
            int64_t i = (flat / h) % q_len;
            int64_t L = cache_seqlens[b];
            int64_t lim = causal ? L - q_len + i + 1 : L;
            if (lim > L) lim = L;
            int64_t j0 = key_begin ? key_begin[b] : 0;
            int64_t j1 = key_end ? key_end[b] : L;
            if (j0 < 0) j0 = 0;
            if (j1 > lim) j1 = lim;
            const void* q_row = q_is_fp8 ? (const void*)((const uint8_t*)q + flat * dq)
                                         : (const void*)((const uint16_t*)q + flat * dq);
            attend_row(q_row, q_is_fp8, (const uint8_t*)kv, kv_format, descale_q, descale_k,
                       req_to_token + req_pool_indices[b] * r2t_stride, j0, j1, dq, dv,
                       softmax_scale, o_out + r * dv, lse_out + r, s_buf);
        }
        free(s_buf);
    }
    return 0;
}

/*
 * Log-sum-exp merge of n partial states (o_k, lse_k) of one row:
 *     lse = ln(sum_k exp(lse_k)),  o = sum_k exp(lse_k - lse) * o_k
 * Partials with lse_k = -inf carry no weight; if all are -inf, o = 0, lse = -inf.
 */
void oracle_merge_states(int64_t n, int64_t dv, const double* o_parts, const double* lse_parts,
                         double* o, double* lse) {
    double m = -INFINITY;
    for (int64_t k = 0; k < n; ++k)
        if (lse_parts[k] > m) m = lse_parts[k];
    for (int64_t d = 0; d < dv; ++d) o[d] = 0.0;
    if (m == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double sum = 0.0;
    for (int64_t k = 0; k < n; ++k) sum += exp(lse_parts[k] - m);
    double l = m + log(sum);
    for (int64_t k = 0; k < n; ++k) {
        double w = exp(lse_parts[k] - l);
        for (int64_t d = 0; d < dv; ++d) o[d] += w * o_parts[k * dv + d];
    }
    *lse = l;
}

/*
 * KV-cache write: for every new token i, row cache_loc[i] of the pool [num_slots, dim]
 * receives k[i, 0:dim] (k is bf16 bits with row stride k_stride).  A bf16 pool (format 0)
 * stores the bits as they are.  An fp8 pool (format 1 = e4m3, 2 = e5m2) stores
 * quantize_fp8(x), with x = k / k_scale evaluated in float32 (one correctly rounded
 * division) when has_scale, else k itself.  Slots outside [0, num_slots) are skipped.
 */
void oracle_set_kv_buffer(void* pool, int format, int64_t num_slots, int64_t dim,
                          const int64_t* cache_loc, int64_t n_tokens, const uint16_t* k,
                          int64_t k_stride, int has_scale, float k_scale) {
    for (int64_t i = 0; i < n_tokens; ++i) {
        int64_t slot = cache_loc[i];
        if (slot < 0 || slot >= num_slots) continue;
        for (int64_t d = 0; d < dim; ++d) {
            uint16_t bits = k[i * k_stride + d];
            if (format == 0) {
                ((uint16_t*)pool)[slot * dim + d] = bits;
            } else {
                float x = (float)bf16_bits_to_double(bits);
                if (has_scale) x = x / k_scale;
                ((uint8_t*)pool)[slot * dim + d] = quantize_fp8((double)x, format);
            }
        }
    }
}
