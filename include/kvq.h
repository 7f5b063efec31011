/*
 * kvq.h -- C ABI of the B200 (sm_100a) KV-cache format conversion library,
 * libkvq.so.
 *
 * The four conversions are the ones the page "Implementation: Turboderp org
 * Exllamav2 Ext Cache" defines (sections Description, Signature and I/O
 * Contract): fp16_to_fp8, fp8_to_fp16, fp16_to_q_kv and q_to_fp16_kv.  Each
 * entry point keeps the page's argument order (in / out / scales pointers,
 * batch_size, offset, width, page_size, cache_seqlens, block_table, wbits),
 * replaces each torch tensor by a raw device pointer plus the shape the tensor
 * carried (kvq_cache_desc), and takes the CUDA stream explicitly instead of
 * using "the current stream".
 *
 * Numerics (fixed by this library, since the page leaves them open):
 *   FP8   E5M2 = the upper byte of binary16 after rounding to 2 fraction bits,
 *         round to nearest, ties to even; no saturation (|x| >= 61440 -> Inf);
 *         any NaN -> sign | 0x7E.  Decoding is exact: half bits = byte << 8.
 *   Q4/Q6/Q8 symmetric absmax over 32 consecutive head_dim elements
 *         (wbits 4 or 6 as the page's I/O Contract gives; 8 as its Usage
 *         section's Q8 cache class implies, same rules).
 *         maxq = 2^(wbits-1) - 1, z = 2^(wbits-1).
 *         scale s = RN16(fl32(absmax / maxq)) stored as FP16;
 *         code    = clamp(rint(fl32(x / s)) + z, 0, 2^wbits - 1), ties to even,
 *                   and every code = z with s = +0 when s rounds to +0;
 *         dequant = RN16((code - z) * s).
 *         The codes of one head row form a little-endian bit stream: code j
 *         occupies bits [wbits*j, wbits*j + wbits) of the row's bytes (Q4: two
 *         codes per byte, even element in the low nibble; Q6: 16 codes per
 *         three 32-bit little-endian words; Q8: one byte per code).
 *   Results are bit-exact with these definitions; there is no tolerance.
 *
 * Layouts (row-major; all pointers are device memory on the current device):
 *   FP16 cache   [dim0, dim1, kv_heads, head_dim]                 binary16
 *   FP8 cache    [dim0, dim1, kv_heads, head_dim]                 uint8
 *   Q codes      [dim0, dim1, kv_heads, head_dim * wbits / 8]     uint8
 *   Q scales     [dim0, dim1, kv_heads, head_dim / 32]            binary16
 *   Contiguous:  dim0 = allocated sequences, dim1 = max positions (seq).
 *   Paged:       dim0 = pages in the pool, dim1 = page_size positions.
 *   cache_seqlens [batch_size] int32; block_table [batch_size,
 *   block_table_stride] int32 (entries that no window reaches may be -1).
 *
 * Windows:
 *   Contiguous: for every sequence b < batch_size, positions
 *               [offset, offset + width).
 *   Paged:      for every sequence i < batch_size, logical positions
 *               [max(0, cache_seqlens[i] + offset), cache_seqlens[i] + offset + width);
 *               logical position p is row p % page_size of physical page
 *               block_table[i][p / page_size].  FP16 and Q tensors share the
 *               same page geometry and block table.
 *   Nothing outside the window is read or written.
 *
 * Ownership: every buffer belongs to the caller and must stay valid until the
 *   work enqueued on `stream` has finished.  The library allocates nothing.
 *   Inputs and outputs must not overlap.  All calls are asynchronous: they
 *   validate the arguments on the host, enqueue kernels on `stream` (a
 *   cudaStream_t; NULL = the legacy default stream) and return.
 *
 * Errors: arguments are checked on the host before anything is enqueued; a
 *   failed check returns a kvq_status and enqueues nothing.  Launch failures
 *   return KVQ_ERR_CUDA.  Problems only the device can see (a block_table entry
 *   outside [0, dim0), or a logical page index >= block_table_stride) skip the
 *   affected positions and record a code in a per-device error word that
 *   kvq_poll_device_error() reads.  No kernel traps and no exception crosses
 *   the ABI.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvq_status {
  KVQ_OK = 0,
  KVQ_ERR_NULL = 1,    /* a required pointer is NULL */
  KVQ_ERR_SHAPE = 2,   /* bad dims: negative, head_dim not a multiple of 8 (FP8) or 32 (Q) */
  KVQ_ERR_WBITS = 3,   /* wbits is not 4, 6 or 8 */
  KVQ_ERR_RANGE = 4,   /* window or batch outside the cache, page_size != dim1 */
  KVQ_ERR_ALIGN = 5,   /* a buffer is not 16-byte aligned */
  KVQ_ERR_CUDA = 6,    /* the CUDA runtime reported an error */
  KVQ_ERR_DEVICE = 7   /* the device recorded bad paging metadata (kvq_poll_device_error) */
} kvq_status;

/* Device-side error codes stored in the error word. */
enum {
  KVQ_DEV_OK = 0,
  KVQ_DEV_BAD_PAGE = 1,       /* block_table entry outside [0, dim0) */
  KVQ_DEV_BAD_PAGE_INDEX = 2, /* logical page index >= block_table_stride */
  KVQ_DEV_TIMEOUT = 3         /* a bulk-engine pipeline wait ran past its limit (1 s) */
};

/* Load engines and work decompositions (kvq_set_engine).  All give
 * bit-identical results. */
enum {
  KVQ_ENGINE_AUTO = 0, /* per operation, the engine measured faster on B200 (default) */
  KVQ_ENGINE_LDG = 1,  /* 16-byte global loads issued up front; contiguous mode: one tile
                          per CTA; paged mode: one wave of CTAs taking equal shares of the
                          flattened windows of all sequences, walked in interleaved rounds
                          (batches of up to 1024 sequences whose windows total under 2^31
                          positions; otherwise per-sequence tiles as in
                          KVQ_ENGINE_LDG_TILED).  Measured slower than the tiles on B200 */
  KVQ_ENGINE_BULK = 2, /* persistent CTAs, TMA bulk copies (cp.async.bulk, no multicast)
                          into a 4-stage shared-memory ring, one producer warp and eight
                          consumer warps; used when one position of the input stream is a
                          multiple of 16 bytes, otherwise the LDG engine runs */
  KVQ_ENGINE_LDG_TILED = 3 /* the LDG engine with per-sequence tiles in paged mode too
                              (one tile of a sequence's window per CTA): what AUTO runs */
};

/* The shape the torch tensor carried in the original extension. */
typedef struct kvq_cache_desc {
  int32_t dim0;               /* contiguous: allocated sequences; paged: pages in the pool */
  int32_t dim1;               /* contiguous: max positions per sequence; paged: page_size */
  int32_t kv_heads;           /* H */
  int32_t head_dim;           /* D */
  int32_t block_table_stride; /* paged: columns of block_table; contiguous: ignored */
} kvq_cache_desc;

/* fp16_to_fp8 (Description; Signature): encode the FP16 cache `in` into the
 * E5M2 cache `out` (same shape) over the contiguous window.  head_dim must be
 * a multiple of 8.  `in` and `out` 16-byte aligned. */
KVQ_API kvq_status kvq_fp16_to_fp8(const void* in, void* out, const kvq_cache_desc* desc,
                           int batch_size, int offset, int width, void* stream);

/* fp8_to_fp16 (Description; Signature): decode the E5M2 cache `in` into the
 * FP16 cache `out` over the same kind of window. */
KVQ_API kvq_status kvq_fp8_to_fp16(const void* in, void* out, const kvq_cache_desc* desc,
                           int batch_size, int offset, int width, void* stream);

/* FP8 for K and V in one launch, contiguous or paged.  No counterpart on the
 * page: it extends fp16_to_fp8 (Description; Signature) to both caches and to
 * the paged layout, with exactly the window, page, alignment and error rules
 * of kvq_fp16_to_q_kv (page_size == 0: contiguous, cache_seqlens /
 * block_table ignored; page_size > 0: paged, page_size == desc->dim1).
 * head_dim must be a multiple of 8.  All four cache pointers 16-byte
 * aligned. */
KVQ_API kvq_status kvq_fp16_to_fp8_kv(const void* k_in, void* k_out, const void* v_in, void* v_out,
                                      const kvq_cache_desc* desc, int batch_size, int offset, int width,
                                      int page_size, const int32_t* cache_seqlens,
                                      const int32_t* block_table, void* stream);

/* The reverse of kvq_fp16_to_fp8_kv (extends fp8_to_fp16 the same way). */
KVQ_API kvq_status kvq_fp8_to_fp16_kv(const void* k_in, void* k_out, const void* v_in, void* v_out,
                                      const kvq_cache_desc* desc, int batch_size, int offset, int width,
                                      int page_size, const int32_t* cache_seqlens,
                                      const int32_t* block_table, void* stream);

/* fp16_to_q_kv (Description; Signature; I/O Contract): quantize the FP16 K
 * and V caches to wbits-bit codes and FP16 scales in one launch.  page_size
 * == 0 selects contiguous mode (cache_seqlens, block_table ignored and may be
 * NULL); page_size > 0 selects paged mode (page_size == desc->dim1,
 * cache_seqlens and block_table required).  head_dim must be a multiple of
 * 32 (the scale block, the page's Q_CACHE_BLOCKSIZE_Q alignment).  wbits is
 * 4, 6 or 8.  All six cache pointers 16-byte aligned. */
KVQ_API kvq_status kvq_fp16_to_q_kv(const void* k_in, void* k_out, void* k_scales,
                            const void* v_in, void* v_out, void* v_scales,
                            const kvq_cache_desc* desc, int batch_size, int offset, int width,
                            int page_size, const int32_t* cache_seqlens,
                            const int32_t* block_table, int wbits, void* stream);

/* q_to_fp16_kv (Description; Signature): dequantize K and V codes + scales
 * back into the FP16 caches, same modes and checks as kvq_fp16_to_q_kv. */
KVQ_API kvq_status kvq_q_to_fp16_kv(const void* k_in, void* k_out, const void* k_scales,
                            const void* v_in, void* v_out, const void* v_scales,
                            const kvq_cache_desc* desc, int batch_size, int offset, int width,
                            int page_size, const int32_t* cache_seqlens,
                            const int32_t* block_table, int wbits, void* stream);

/* Decode attention over a quantized KV cache (the conversions' consumer: the
 * page's Usage section converts the cache "during the attention forward
 * pass"; this reads the Q4/Q6/Q8 codes directly, so no FP16 cache is written).
 * For every sequence i < batch_size and query head h < n_heads (GQA: kv head
 * h / (n_heads / kv_heads)), the query q[i, h, :] attends to logical
 * positions [0, cache_seqlens[i]) of the cache, keys and values being
 * exactly what kvq_q_to_fp16_kv would produce:
 *   out[i, h, :] = sum_p softmax_p(softmax_scale * q . k_p) * v_p   (binary16),
 * 0 for an empty window.  Arithmetic: fp16 products with fp32 accumulation
 * (tensor cores), base-2 online softmax in fp32; the tests hold every output
 * to an error bound derived from that arithmetic against the exact result.
 *   q, out     [batch_size, n_heads, head_dim] binary16, 16-byte aligned
 *   k/v codes  [dim0, dim1, kv_heads, head_dim * wbits / 8] uint8
 *   k/v scales [dim0, dim1, kv_heads, head_dim / 32] binary16
 *   page_size == 0: contiguous (dim1 = max positions, cache_seqlens[i] <=
 *   dim1); page_size > 0: paged as in kvq_fp16_to_q_kv.  head_dim is 64, 128
 *   or 256; n_heads / kv_heads <= 8; wbits 4, 6 or 8.
 *   workspace: caller-owned device memory of at least
 *   kvq_decode_attention_workspace_size(...) bytes (partial results: 2 +
 *   head_dim floats per sequence, query head and 128-position chunk the
 *   cache geometry allows), 16-byte aligned; its contents on entry do not
 *   matter.
 * Two kernels are enqueued on `stream`.  A window longer than the cache, or
 * paging metadata pointing outside it, skips those positions and sets the
 * device error word. */
KVQ_API kvq_status kvq_decode_attention_q(const void* q, const void* k_codes, const void* k_scales,
                                          const void* v_codes, const void* v_scales, void* out,
                                          const kvq_cache_desc* desc, int batch_size, int n_heads, int page_size,
                                          const int32_t* cache_seqlens, const int32_t* block_table, int wbits,
                                          float softmax_scale, void* workspace, size_t workspace_bytes,
                                          void* stream);

/* Decode attention over an FP8 (E5M2) KV cache: kvq_decode_attention_q with
 * keys and values the E5M2 bytes decoded exactly as kvq_fp8_to_fp16 does (the
 * page's Usage section converts the FP8 cache during the attention forward
 * pass as it does the Q cache).  There are no scales.
 *   k_fp8, v_fp8  [dim0, dim1, kv_heads, head_dim] uint8 (E5M2), 16-byte aligned
 *   Everything else (q, out, paging, workspace, softmax_scale, stream, errors,
 *   two kernels enqueued) as for kvq_decode_attention_q; head_dim 64, 128 or 256.
 *   A stored Inf or NaN byte propagates into the outputs that attend to it. */
KVQ_API kvq_status kvq_decode_attention_fp8(const void* q, const void* k_fp8, const void* v_fp8, void* out,
                                            const kvq_cache_desc* desc, int batch_size, int n_heads, int page_size,
                                            const int32_t* cache_seqlens, const int32_t* block_table,
                                            float softmax_scale, void* workspace, size_t workspace_bytes,
                                            void* stream);

/* Workspace bytes kvq_decode_attention_q and kvq_decode_attention_fp8 need for
 * this geometry (0 for bad arguments, SIZE_MAX when the size overflows size_t,
 * which the attention calls reject with KVQ_ERR_RANGE).  Host-only. */
KVQ_API size_t kvq_decode_attention_workspace_size(const kvq_cache_desc* desc, int batch_size, int n_heads,
                                                   int page_size);

/* Size of the scratch array kvq_decode_attention_q_noalloc uses (32 MiB per
 * device). */
#define KVQ_ATTENTION_SCRATCH_BYTES ((size_t)32 << 20)

/* kvq_decode_attention_q without a caller workspace.  The pages have no
 * counterpart: this is a convenience of this library for callers that cannot
 * allocate device memory at the call site (a serving loop whose HBM belongs
 * to its own KV-page pool, or a decode step that cannot afford the device
 * synchronization cudaMalloc / cudaFree may cause).  The split-K workspace is
 * a fixed array of KVQ_ATTENTION_SCRATCH_BYTES inside the library (one per
 * device), so the call allocates nothing.
 *   Arguments, layouts, results and errors are those of
 *   kvq_decode_attention_q.  A geometry whose
 *   kvq_decode_attention_workspace_size(...) exceeds
 *   KVQ_ATTENTION_SCRATCH_BYTES returns KVQ_ERR_RANGE and enqueues nothing
 *   (for example, batch 8 x 32 query heads x head_dim 128 with up to 16384
 *   positions needs 17 MB and fits; batch 16 with up to 16384 positions
 *   needs 34 MB and does not).
 *   Every call looks up the device address of the current device's copy of
 *   the array (a host-side query that enqueues nothing), so a reset and
 *   re-created device context is picked up; the first call on a device may
 *   also load the library's device code there, so make it before any stream
 *   capture.  KVQ_ERR_CUDA if the lookup fails.
 *   Every call on a device shares the one array and leaves its partial
 *   results there; nothing in it has to start at zero, because each call
 *   writes every entry it later reads.  Calls whose kernels overlap on the
 *   GPU (other streams, other host threads) race on the array and must be
 *   serialized by the caller. */
KVQ_API kvq_status kvq_decode_attention_q_noalloc(const void* q, const void* k_codes, const void* k_scales,
                                                  const void* v_codes, const void* v_scales, void* out,
                                                  const kvq_cache_desc* desc, int batch_size, int n_heads,
                                                  int page_size, const int32_t* cache_seqlens,
                                                  const int32_t* block_table, int wbits, float softmax_scale,
                                                  void* stream);

/* count_match (Description; I/O Contract): the number of leading elements on
 * which the 64-bit sequences a[0..a_len) and b[0..b_len) agree, comparing no
 * more than max_a elements (max_a <= 0 gives 0).  Host function: a and b are
 * host pointers, read only; nothing is enqueued on any device.  Returns -1
 * when a pointer is NULL and there is something to compare. */
KVQ_API long long kvq_count_match(const int64_t* a, long long a_len, const int64_t* b, long long b_len,
                                  long long max_a);

/* Human-readable name of a status (static storage; never NULL). */
KVQ_API const char* kvq_status_string(kvq_status status);

/* Waits for `stream`, then reads and clears the current device's error word.
 * *code_out receives the KVQ_DEV_* code (0 when none).  Returns KVQ_ERR_DEVICE
 * when the word was set, KVQ_OK when not, KVQ_ERR_CUDA on a runtime error. */
KVQ_API kvq_status kvq_poll_device_error(int32_t* code_out, void* stream);

/* Select the load engine for all later calls in this process (any thread).
 * Returns KVQ_ERR_RANGE for an unknown value.  Host-only; no device work. */
KVQ_API kvq_status kvq_set_engine(int engine);

/* The engine currently selected (a KVQ_ENGINE_* value). */
KVQ_API int kvq_get_engine(void);

/* Decode-attention kernels (kvq_set_attention_path).  Both compute the same
 * attention within the error bound stated at kvq_decode_attention_q. */
enum {
  KVQ_ATTENTION_AUTO = 0,    /* the kernel measured faster on B200: mma.sync (default) */
  KVQ_ATTENTION_MMA = 1,     /* warp-level mma.sync tiles for every geometry */
  KVQ_ATTENTION_TCGEN05 = 2  /* tcgen05.mma with tensor-memory accumulators for head_dim 128
                                and batches of up to 256 sequences; other geometries run
                                the mma.sync kernel.  Measured slower than mma.sync on B200 */
};

/* Select the decode-attention kernel for all later calls in this process (any
 * thread).  Returns KVQ_ERR_RANGE for an unknown value.  Host-only. */
KVQ_API kvq_status kvq_set_attention_path(int path);

/* The decode-attention kernel currently selected (a KVQ_ATTENTION_* value). */
KVQ_API int kvq_get_attention_path(void);

/* Self-check (no counterpart on the page): compares, on the device, the
 * kernels' fast code rounding (reciprocal, one FMA correction step, rounding
 * by magic-number addition) with IEEE binary32 division followed by rint and
 * the clamp, for every finite binary16 x and every binary16 scale s in
 * [+0, 65504] (about 2^31 pairs).  `mismatches` is a caller-owned device pointer to one
 * unsigned 64-bit counter; it is zeroed and then receives the number of
 * pairs whose codes differ (0 expected).  Asynchronous on `stream`. */
KVQ_API kvq_status kvq_selfcheck_code_rounding(int wbits, unsigned long long* mismatches, void* stream);

/* Self-check (no counterpart on the page): measures, on the device, the
 * arithmetic constants the decode-attention error bound is built from.
 * `results` is a caller-owned device pointer to three doubles (8-byte
 * aligned), zeroed and then filled with:
 *   [0] the largest relative error of the hardware 2^x approximation the
 *       softmax uses (ex2.approx.ftz.f32), over every binary32 x in [-126, 8];
 *   [1] the largest relative error of exp2f over every binary32 x in
 *       [-126, 0] (the chunk merge factors);
 *   [2] the largest error of one mma.sync m16n8k16 step (binary16 products,
 *       binary32 accumulator) over 310 M adversarial random accumulations,
 *       in units of 2^-23 times the largest magnitude among the step's 16
 *       products and its accumulator (the bound assumes at most 18).
 * Asynchronous on `stream`; a few hundred milliseconds of device time. */
KVQ_API kvq_status kvq_selfcheck_attention_numerics(double* results, void* stream);

/* Self-check of the bulk engine's bounded waits (no counterpart on the page):
 * one CTA waits, with the same bounded wait the bulk engine's pipeline uses,
 * on a shared-memory mbarrier that nothing ever arrives on.  After the wait's
 * limit (1 s) it gives up, writes 1 to *waited_out (a caller-owned device
 * int32, written 0 first) and records KVQ_DEV_TIMEOUT in the device error
 * word, and the kernel ends; no fault, no hang, and the context stays usable.
 * Asynchronous on `stream`. */
KVQ_API kvq_status kvq_selfcheck_wait_timeout(int32_t* waited_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
