/*
 * kvqref.h -- CPU oracle for the KV-cache format conversions.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the plain, slow, single-threaded,
 * obviously-correct restatement of what the KV-cache conversions compute,
 * used to check the CUDA library bit for bit.  Only the tests, the smoke
 * check and the benchmark's CPU-baseline leg may load it.  It shares no code,
 * header, table or constant with the CUDA library, and it never calls it.
 *
 * Source being restated: the web page "Implementation: Turboderp org
 * Exllamav2 Ext Cache" (sections Description, Signature and I/O Contract),
 * which defines fp16_to_fp8, fp8_to_fp16, fp16_to_q_kv and q_to_fp16_kv on
 * FP16 caches of shape [batch, seq, kv_heads, head_dim] over a position
 * window [offset, offset + width), contiguous or paged.  The page names the
 * operations but not their numerics; the numerics below are the readings
 * fixed for this project:
 *
 *   FP8      = E5M2, i.e. binary16 rounded to 2 mantissa bits, round to
 *              nearest, ties to even, IEEE overflow to +-Inf (no
 *              saturation), NaN -> quiet NaN (sign | 0x7E).  Decoding is
 *              exact (every E5M2 value is a binary16 value).
 *   Q4/Q6/Q8 = symmetric absmax over 32-element blocks along head_dim
 *              (wbits 4, 6 or 8).
 *              maxq = 2^(b-1) - 1, zero point z = 2^(b-1).
 *              s    = RN16( fl32( absmax / maxq ) )      (stored as FP16)
 *              code = clamp( rint( fl32( x / s ) ) + z, 0, 2^b - 1 ),
 *                     every code = z and s = +0 when s == +0.
 *              dequantized value = RN16( (code - z) * s ).
 *              Codes of one head row are a little-endian bit stream:
 *              code j occupies bits [b*j, b*j + b) of the row's bytes.
 *   Paged    = sequence i covers logical positions
 *              [max(0, seqlens[i] + offset), seqlens[i] + offset + width);
 *              position p lives in page block_table[i][p / page_size] at
 *              row p % page_size.
 *
 * Layouts (row-major, all host memory, caller-owned):
 *   FP16 cache      [dim0, dim1, heads, head_dim]            uint16 bits
 *   FP8 cache       [dim0, dim1, heads, head_dim]            uint8
 *   Q codes         [dim0, dim1, heads, head_dim * wbits / 8] uint8
 *   Q scales        [dim0, dim1, heads, head_dim / 32]        uint16 bits
 * Contiguous mode: dim0 = allocated sequences, dim1 = max positions.
 * Paged mode:      dim0 = pages in the pool, dim1 = page_size.
 *
 * Return value of the cache functions: KVQREF_OK, KVQREF_BAD_ARG (nothing
 * written) or KVQREF_BAD_PAGE (a block-table entry or a logical page index
 * was out of range; that position was skipped, the rest was written).
 */
#ifndef KVQREF_H
#define KVQREF_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { KVQREF_OK = 0, KVQREF_BAD_ARG = 1, KVQREF_BAD_PAGE = 2 };

/* ---- scalar primitives (exposed so the tests can pin each one) ---------- */

/* binary16 bits -> exact value as a double (NaN and Inf preserved). */
double   kvqref_half_to_double(uint16_t h);
/* Round a double to the nearest binary16, ties to even, overflow to Inf. */
uint16_t kvqref_double_to_half(double v);
/* binary16 -> E5M2 byte (round to nearest even, no saturation). */
uint8_t  kvqref_e5m2_encode(uint16_t h);
/* E5M2 byte -> binary16 bits (exact; a NaN keeps its sign and payload). */
uint16_t kvqref_e5m2_decode(uint8_t b);
/* FP16 scale for one block whose absmax is the binary16 'absmax_bits'. */
uint16_t kvqref_block_scale(uint16_t absmax_bits, int wbits);
/* Quantize n (a multiple of 32) binary16 values: one unpacked code per
 * element in codes[n], one scale per 32 elements in scales[n / 32].
 * Returns KVQREF_BAD_ARG for bad n or wbits. */
int kvqref_quantize_row(const uint16_t* x, int n, int wbits,
                        uint8_t* codes, uint16_t* scales);
/* Dequantize n unpacked codes with their per-32 scales. */
int kvqref_dequantize_row(const uint8_t* codes, const uint16_t* scales, int n,
                          int wbits, uint16_t* y);
/* Pack n codes into n * wbits / 8 bytes (little-endian bit stream). */
int kvqref_pack_row(const uint8_t* codes, int n, int wbits, uint8_t* packed);
/* Inverse of kvqref_pack_row. */
int kvqref_unpack_row(const uint8_t* packed, int n, int wbits, uint8_t* codes);

/* ---- the four cache conversions ------------------------------------------ */

int kvqref_fp16_to_fp8(const uint16_t* in, uint8_t* out,
                       int dim0, int dim1, int heads, int head_dim,
                       int batch_size, int offset, int width);

int kvqref_fp8_to_fp16(const uint8_t* in, uint16_t* out,
                       int dim0, int dim1, int heads, int head_dim,
                       int batch_size, int offset, int width);

/* FP8 for K and V together, contiguous (page_size == 0) or paged (page_size
 * > 0, same window and page rules as the Q functions below). */
int kvqref_fp16_to_fp8_kv(const uint16_t* k_in, uint8_t* k_out, const uint16_t* v_in, uint8_t* v_out,
                          int dim0, int dim1, int heads, int head_dim,
                          int batch_size, int offset, int width,
                          int page_size, const int32_t* cache_seqlens,
                          const int32_t* block_table, int bt_stride);

int kvqref_fp8_to_fp16_kv(const uint8_t* k_in, uint16_t* k_out, const uint8_t* v_in, uint16_t* v_out,
                          int dim0, int dim1, int heads, int head_dim,
                          int batch_size, int offset, int width,
                          int page_size, const int32_t* cache_seqlens,
                          const int32_t* block_table, int bt_stride);

/* page_size == 0: contiguous (cache_seqlens / block_table ignored).
 * page_size  > 0: paged; dim1 must equal page_size and block_table is
 *                 [batch_size, bt_stride] int32. */
int kvqref_fp16_to_q_kv(const uint16_t* k_in, uint8_t* k_out, uint16_t* k_scales,
                        const uint16_t* v_in, uint8_t* v_out, uint16_t* v_scales,
                        int dim0, int dim1, int heads, int head_dim,
                        int batch_size, int offset, int width,
                        int page_size, const int32_t* cache_seqlens,
                        const int32_t* block_table, int bt_stride, int wbits);

int kvqref_q_to_fp16_kv(const uint8_t* k_in, uint16_t* k_out, const uint16_t* k_scales,
                        const uint8_t* v_in, uint16_t* v_out, const uint16_t* v_scales,
                        int dim0, int dim1, int heads, int head_dim,
                        int batch_size, int offset, int width,
                        int page_size, const int32_t* cache_seqlens,
                        const int32_t* block_table, int bt_stride, int wbits);

/* Decode attention over a quantized cache: for every sequence i < batch_size
 * and query head h < n_heads (GQA: kv head h / (n_heads / heads)), attend the
 * single query q[i, h, :] to logical positions [0, cache_seqlens[i]) of the
 * cache, whose keys and values are the dequantized codes (exactly what
 * kvqref_q_to_fp16_kv produces).  In double precision:
 *   s_p = softmax_scale * sum_d q_d * k_{p,d};  w_p = exp(s_p - max_p s_p);
 *   o = sum_p w_p * v_p / sum_p w_p;   out = RN16(o)   (0 when the window is empty).
 * q, out: [batch_size, n_heads, head_dim] binary16.  out_exact (optional,
 * may be NULL) receives o before rounding.  Paged / contiguous addressing as
 * in kvqref_q_to_fp16_kv.  Returns KVQREF_BAD_ARG / KVQREF_BAD_PAGE like it. */
int kvqref_decode_attention_q(const uint16_t* q, const uint8_t* k_codes, const uint16_t* k_scales,
                              const uint8_t* v_codes, const uint16_t* v_scales, uint16_t* out,
                              double* out_exact, int dim0, int dim1, int heads, int head_dim,
                              int batch_size, int n_heads, int page_size, const int32_t* cache_seqlens,
                              const int32_t* block_table, int bt_stride, int wbits, double softmax_scale);

/* Decode attention over an FP8 (E5M2) cache: as kvqref_decode_attention_q,
 * with keys and values the E5M2 bytes decoded exactly as kvqref_fp8_to_fp16
 * does.  k_fp8, v_fp8: [dim0, dim1, heads, head_dim] bytes. */
int kvqref_decode_attention_fp8(const uint16_t* q, const uint8_t* k_fp8, const uint8_t* v_fp8, uint16_t* out,
                                double* out_exact, int dim0, int dim1, int heads, int head_dim, int batch_size,
                                int n_heads, int page_size, const int32_t* cache_seqlens, const int32_t* block_table,
                                int bt_stride, double softmax_scale);

/* count_match (Description; I/O Contract): length of the common prefix of two
 * 64-bit element sequences, looking at no more than max_a elements. */
long long kvqref_count_match(const int64_t* a, long long a_len, const int64_t* b, long long b_len,
                             long long max_a);

#ifdef __cplusplus
}
#endif

#endif /* KVQREF_H */
