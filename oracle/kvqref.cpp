// kvqref.cpp -- CPU oracle for the KV-cache format conversions.
//
// TEST INFRASTRUCTURE ONLY: loaded by the tests, the smoke check and the
// benchmark's CPU-baseline leg, never by the CUDA library.  Plain,
// single-threaded, one element at a time, in the order the definitions give.
// The numerics and layouts it restates are listed in kvqref.h; every
// function below names the part of the page "Implementation: Turboderp org
// Exllamav2 Ext Cache" it follows.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math (x86-64 SSE
// arithmetic, so float operations are IEEE binary32 with round to nearest
// even and no excess precision).

#include "kvqref.h"

#include <cmath>
#include <cstdint>
#include <cstring>

namespace {

// ---------------------------------------------------------------------------
// binary16 <-> real, written from the IEEE 754 binary16 definition:
// 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits; exponent field 0
// holds the subnormals (fraction * 2^-24), field 31 holds Inf and NaN.
// ---------------------------------------------------------------------------

double half_to_double(uint16_t h) {
  const int sign = h >> 15;
  const int e = (h >> 10) & 0x1F;
  const int f = h & 0x3FF;
  double v;
  if (e == 0) {
    v = std::ldexp(static_cast<double>(f), -24);
  } else if (e == 31) {
    v = f ? NAN : INFINITY;
  } else {
    v = std::ldexp(static_cast<double>(1024 + f), e - 25);
  }
  return sign ? -v : v;
}

// Round v to the nearest binary16 value, ties to the even significand,
// values that round past the largest finite one become Inf.
uint16_t double_to_half(double v) {
  const uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  if (std::isnan(v)) return sign | 0x7E00;
  double a = std::fabs(v);
  if (std::isinf(a)) return sign | 0x7C00;
  if (a < std::ldexp(1.0, -14)) {
    // subnormal range: a multiple of 2^-24; rint rounds ties to even
    double q = std::rint(std::ldexp(a, 24));  // exact scaling, q in [0, 1024]
    return sign | static_cast<uint16_t>(q);    // q == 1024 is the smallest normal
  }
  int k;
  std::frexp(a, &k);  // a = m * 2^k, m in [0.5, 1)
  int E = k - 1;      // a in [2^E, 2^(E+1))
  double q = std::rint(std::ldexp(a, 10 - E));  // significand in [1024, 2048]
  if (q == 2048.0) {
    q = 1024.0;
    E += 1;
  }
  if (E > 15) return sign | 0x7C00;
  return sign | static_cast<uint16_t>(((E + 15) << 10) | (static_cast<int>(q) - 1024));
}

float half_to_float(uint16_t h) { return static_cast<float>(half_to_double(h)); }

// ---------------------------------------------------------------------------
// FP8 E5M2 (1 sign, 5 exponent bits with bias 15, 2 fraction bits).  The
// page's Description calls the target "FP8 (unsigned 8-bit)"; the format is
// read as E5M2 with round to nearest, ties to even, and IEEE overflow.
// Largest finite value 1.75 * 2^15 = 57344; smallest normal 2^-14;
// subnormal step 2^-16.
// ---------------------------------------------------------------------------

uint8_t e5m2_encode(uint16_t h) {
  const uint8_t sign = (h >> 15) ? 0x80 : 0;
  const double v = half_to_double(h);
  if (std::isnan(v)) return sign | 0x7E;
  const double a = std::fabs(v);
  if (std::isinf(a)) return sign | 0x7C;
  if (a < std::ldexp(1.0, -14)) {
    double q = std::rint(std::ldexp(a, 16));  // q in [0, 4]; 4 = smallest normal
    return sign | static_cast<uint8_t>(q);
  }
  int k;
  std::frexp(a, &k);
  int E = k - 1;
  double q = std::rint(std::ldexp(a, 2 - E));  // significand in [4, 8]
  if (q == 8.0) {
    q = 4.0;
    E += 1;
  }
  if (E > 15) return sign | 0x7C;
  return sign | static_cast<uint8_t>(((E + 15) << 2) | (static_cast<int>(q) - 4));
}

uint16_t e5m2_decode(uint8_t b) {
  const uint16_t sign = (b & 0x80) ? 0x8000 : 0;
  const int e = (b >> 2) & 0x1F;
  const int f = b & 3;
  if (e == 31) {
    // Inf, or a NaN whose 2-bit payload becomes the top of the binary16
    // payload (E5M2 is the upper byte of the binary16 encoding).
    return sign | 0x7C00 | static_cast<uint16_t>(f << 8);
  }
  double v = (e == 0) ? std::ldexp(static_cast<double>(f), -16)
                      : std::ldexp(static_cast<double>(4 + f), e - 17);
  if (sign) v = -v;
  return double_to_half(v);  // exact: every finite E5M2 value is a binary16 value
}

// ---------------------------------------------------------------------------
// Q4 / Q6 / Q8 codec (I/O Contract: k_scales / v_scales are "per-block
// quantization scale factors", kHalf; wbits is 4 or 6 there, and the page's
// Usage section also names a Q8 cache class, so 8 is accepted with the same
// rules: maxq 127, zero point 128, one byte per code).
// ---------------------------------------------------------------------------

constexpr int kBlock = 32;  // elements per scale block along head_dim

bool valid_wbits(int wbits) { return wbits == 4 || wbits == 6 || wbits == 8; }
int maxq_of(int wbits) { return (1 << (wbits - 1)) - 1; }
int zero_of(int wbits) { return 1 << (wbits - 1); }

uint16_t block_scale(float absmax, int wbits) {
  const float q = absmax / static_cast<float>(maxq_of(wbits));  // IEEE binary32 division
  return double_to_half(static_cast<double>(q));                // then RN16
}

int quantize_value(float x, float s, int wbits) {
  const int z = zero_of(wbits);
  if (s == 0.0f) return z;
  const float r = x / s;           // IEEE binary32 division
  const float ri = std::rint(r);   // ties to even in the default rounding mode
  long c = static_cast<long>(ri) + z;
  const long top = (1L << wbits) - 1;
  if (c < 0) c = 0;
  if (c > top) c = top;
  return static_cast<int>(c);
}

uint16_t dequantize_value(int code, uint16_t s_bits, int wbits) {
  const float s = half_to_float(s_bits);
  const float p = static_cast<float>(code - zero_of(wbits)) * s;  // exact in binary32
  return double_to_half(static_cast<double>(p));
}

void quantize_row(const uint16_t* x, int n, int wbits, uint8_t* codes, uint16_t* scales) {
  for (int b0 = 0; b0 < n; b0 += kBlock) {
    float absmax = 0.0f;
    for (int j = 0; j < kBlock; ++j) {
      const float a = std::fabs(half_to_float(x[b0 + j]));
      if (a > absmax) absmax = a;
    }
    const uint16_t s_bits = block_scale(absmax, wbits);
    const float s = half_to_float(s_bits);
    scales[b0 / kBlock] = s_bits;
    for (int j = 0; j < kBlock; ++j) {
      codes[b0 + j] = static_cast<uint8_t>(quantize_value(half_to_float(x[b0 + j]), s, wbits));
    }
  }
}

void dequantize_row(const uint8_t* codes, const uint16_t* scales, int n, int wbits, uint16_t* y) {
  for (int j = 0; j < n; ++j) y[j] = dequantize_value(codes[j], scales[j / kBlock], wbits);
}

// Little-endian bit stream: bit t of code j goes to stream bit wbits*j + t,
// stream bit k is bit (k % 8) of byte k / 8.
void pack_row(const uint8_t* codes, int n, int wbits, uint8_t* packed) {
  std::memset(packed, 0, static_cast<size_t>(n) * wbits / 8);
  for (int j = 0; j < n; ++j) {
    for (int t = 0; t < wbits; ++t) {
      if ((codes[j] >> t) & 1) {
        const long k = static_cast<long>(wbits) * j + t;
        packed[k / 8] |= static_cast<uint8_t>(1u << (k % 8));
      }
    }
  }
}

void unpack_row(const uint8_t* packed, int n, int wbits, uint8_t* codes) {
  for (int j = 0; j < n; ++j) {
    int c = 0;
    for (int t = 0; t < wbits; ++t) {
      const long k = static_cast<long>(wbits) * j + t;
      c |= ((packed[k / 8] >> (k % 8)) & 1) << t;
    }
    codes[j] = static_cast<uint8_t>(c);
  }
}

// ---------------------------------------------------------------------------
// Window resolution (Description: "batch_size, offset, and width for partial
// cache updates"; paged mode "uses block_table and cache_seqlens").
// For each (sequence i, window position p) the callback gets the physical
// row index into the [dim0 * dim1] rows of the cache, or a negative value
// when the paging metadata points outside the pool (the position is skipped
// and KVQREF_BAD_PAGE is returned).
// ---------------------------------------------------------------------------

struct Window {
  int dim0, dim1, batch_size, offset, width, page_size, bt_stride;
  const int32_t* seqlens;
  const int32_t* block_table;
};

bool window_args_ok(const Window& w) {
  if (w.dim0 < 0 || w.dim1 < 0 || w.batch_size < 0 || w.width < 0) return false;
  if (w.page_size == 0) {
    if (w.batch_size > w.dim0) return false;
    if (w.offset < 0 || static_cast<long>(w.offset) + w.width > w.dim1) return false;
    return true;
  }
  if (w.page_size < 0 || w.dim1 != w.page_size) return false;
  if (w.batch_size > 0 && (w.seqlens == nullptr || w.block_table == nullptr)) return false;
  if (w.bt_stride < 0) return false;
  return true;
}

template <class F>
int for_each_row(const Window& w, F&& fn) {
  int status = KVQREF_OK;
  for (int i = 0; i < w.batch_size; ++i) {
    if (w.page_size == 0) {
      for (int s = w.offset; s < w.offset + w.width; ++s) {
        fn(static_cast<long>(i) * w.dim1 + s);
      }
      continue;
    }
    const long start = static_cast<long>(w.seqlens[i]) + w.offset;
    const long lo = start < 0 ? 0 : start;
    const long hi = start + w.width;
    for (long p = lo; p < hi; ++p) {
      const long logical_page = p / w.page_size;
      if (logical_page >= w.bt_stride) {
        status = KVQREF_BAD_PAGE;
        continue;
      }
      const int32_t page = w.block_table[static_cast<long>(i) * w.bt_stride + logical_page];
      if (page < 0 || page >= w.dim0) {
        status = KVQREF_BAD_PAGE;
        continue;
      }
      fn(static_cast<long>(page) * w.page_size + p % w.page_size);
    }
  }
  return status;
}

}  // namespace

// ---------------------------------------------------------------------------
// extern "C" surface
// ---------------------------------------------------------------------------

extern "C" {

double kvqref_half_to_double(uint16_t h) { return half_to_double(h); }
uint16_t kvqref_double_to_half(double v) { return double_to_half(v); }
uint8_t kvqref_e5m2_encode(uint16_t h) { return e5m2_encode(h); }
uint16_t kvqref_e5m2_decode(uint8_t b) { return e5m2_decode(b); }

uint16_t kvqref_block_scale(uint16_t absmax_bits, int wbits) {
  if (!valid_wbits(wbits)) return 0xFFFF;
  return block_scale(std::fabs(half_to_float(absmax_bits)), wbits);
}

int kvqref_quantize_row(const uint16_t* x, int n, int wbits, uint8_t* codes, uint16_t* scales) {
  if (!valid_wbits(wbits) || n < 0 || n % kBlock) return KVQREF_BAD_ARG;
  quantize_row(x, n, wbits, codes, scales);
  return KVQREF_OK;
}

int kvqref_dequantize_row(const uint8_t* codes, const uint16_t* scales, int n, int wbits,
                          uint16_t* y) {
  if (!valid_wbits(wbits) || n < 0 || n % kBlock) return KVQREF_BAD_ARG;
  dequantize_row(codes, scales, n, wbits, y);
  return KVQREF_OK;
}

int kvqref_pack_row(const uint8_t* codes, int n, int wbits, uint8_t* packed) {
  if (!valid_wbits(wbits) || n < 0 || (static_cast<long>(n) * wbits) % 8) return KVQREF_BAD_ARG;
  pack_row(codes, n, wbits, packed);
  return KVQREF_OK;
}

int kvqref_unpack_row(const uint8_t* packed, int n, int wbits, uint8_t* codes) {
  if (!valid_wbits(wbits) || n < 0 || (static_cast<long>(n) * wbits) % 8) return KVQREF_BAD_ARG;
  unpack_row(packed, n, wbits, codes);
  return KVQREF_OK;
}

// Description, fp16_to_fp8: every element of every window row is encoded.
int kvqref_fp16_to_fp8(const uint16_t* in, uint8_t* out, int dim0, int dim1, int heads,
                       int head_dim, int batch_size, int offset, int width) {
  if (heads < 0 || head_dim < 0) return KVQREF_BAD_ARG;
  const Window w{dim0, dim1, batch_size, offset, width, 0, 0, nullptr, nullptr};
  if (!window_args_ok(w)) return KVQREF_BAD_ARG;
  const long row_elems = static_cast<long>(heads) * head_dim;
  return for_each_row(w, [&](long row) {
    for (long e = 0; e < row_elems; ++e) out[row * row_elems + e] = e5m2_encode(in[row * row_elems + e]);
  });
}

// Description, fp8_to_fp16: the reverse, same window.
int kvqref_fp8_to_fp16(const uint8_t* in, uint16_t* out, int dim0, int dim1, int heads,
                       int head_dim, int batch_size, int offset, int width) {
  if (heads < 0 || head_dim < 0) return KVQREF_BAD_ARG;
  const Window w{dim0, dim1, batch_size, offset, width, 0, 0, nullptr, nullptr};
  if (!window_args_ok(w)) return KVQREF_BAD_ARG;
  const long row_elems = static_cast<long>(heads) * head_dim;
  return for_each_row(w, [&](long row) {
    for (long e = 0; e < row_elems; ++e) out[row * row_elems + e] = e5m2_decode(in[row * row_elems + e]);
  });
}

// FP8 applied to K and V over one window description (contiguous or paged);
// the page's fp16_to_fp8 / fp8_to_fp16 per element, with the window and page
// rules of fp16_to_q_kv.
int kvqref_fp16_to_fp8_kv(const uint16_t* k_in, uint8_t* k_out, const uint16_t* v_in, uint8_t* v_out,
                          int dim0, int dim1, int heads, int head_dim,
                          int batch_size, int offset, int width,
                          int page_size, const int32_t* cache_seqlens,
                          const int32_t* block_table, int bt_stride) {
  if (heads < 0 || head_dim < 0) return KVQREF_BAD_ARG;
  const Window w{dim0, dim1, batch_size, offset, width, page_size, bt_stride, cache_seqlens, block_table};
  if (!window_args_ok(w)) return KVQREF_BAD_ARG;
  const long row_elems = static_cast<long>(heads) * head_dim;
  auto one = [&](const uint16_t* in, uint8_t* out, long row) {
    for (long e = 0; e < row_elems; ++e) out[row * row_elems + e] = e5m2_encode(in[row * row_elems + e]);
  };
  const int st_k = for_each_row(w, [&](long row) { one(k_in, k_out, row); });
  const int st_v = for_each_row(w, [&](long row) { one(v_in, v_out, row); });
  return st_k != KVQREF_OK ? st_k : st_v;
}

int kvqref_fp8_to_fp16_kv(const uint8_t* k_in, uint16_t* k_out, const uint8_t* v_in, uint16_t* v_out,
                          int dim0, int dim1, int heads, int head_dim,
                          int batch_size, int offset, int width,
                          int page_size, const int32_t* cache_seqlens,
                          const int32_t* block_table, int bt_stride) {
  if (heads < 0 || head_dim < 0) return KVQREF_BAD_ARG;
  const Window w{dim0, dim1, batch_size, offset, width, page_size, bt_stride, cache_seqlens, block_table};
  if (!window_args_ok(w)) return KVQREF_BAD_ARG;
  const long row_elems = static_cast<long>(heads) * head_dim;
  auto one = [&](const uint8_t* in, uint16_t* out, long row) {
    for (long e = 0; e < row_elems; ++e) out[row * row_elems + e] = e5m2_decode(in[row * row_elems + e]);
  };
  const int st_k = for_each_row(w, [&](long row) { one(k_in, k_out, row); });
  const int st_v = for_each_row(w, [&](long row) { one(v_in, v_out, row); });
  return st_k != KVQREF_OK ? st_k : st_v;
}

// Description, fp16_to_q_kv: K and V are each quantized per head row.
int kvqref_fp16_to_q_kv(const uint16_t* k_in, uint8_t* k_out, uint16_t* k_scales,
                        const uint16_t* v_in, uint8_t* v_out, uint16_t* v_scales,
                        int dim0, int dim1, int heads, int head_dim,
                        int batch_size, int offset, int width,
                        int page_size, const int32_t* cache_seqlens,
                        const int32_t* block_table, int bt_stride, int wbits) {
  if (!valid_wbits(wbits) || heads < 0 || head_dim < 0 || head_dim % kBlock) return KVQREF_BAD_ARG;
  const Window w{dim0, dim1, batch_size, offset, width, page_size, bt_stride, cache_seqlens, block_table};
  if (!window_args_ok(w)) return KVQREF_BAD_ARG;
  const long code_bytes = static_cast<long>(head_dim) * wbits / 8;
  const long nscales = head_dim / kBlock;
  uint8_t codes[65536];
  if (head_dim > 65536) return KVQREF_BAD_ARG;
  auto one = [&](const uint16_t* in, uint8_t* out, uint16_t* scales, long row) {
    for (long h = 0; h < heads; ++h) {
      const long hr = row * heads + h;  // head row index
      quantize_row(in + hr * head_dim, head_dim, wbits, codes, scales + hr * nscales);
      pack_row(codes, head_dim, wbits, out + hr * code_bytes);
    }
  };
  int st_k = for_each_row(w, [&](long row) { one(k_in, k_out, k_scales, row); });
  int st_v = for_each_row(w, [&](long row) { one(v_in, v_out, v_scales, row); });
  return st_k != KVQREF_OK ? st_k : st_v;
}

// Description, q_to_fp16_kv: the mirror of fp16_to_q_kv.
int kvqref_q_to_fp16_kv(const uint8_t* k_in, uint16_t* k_out, const uint16_t* k_scales,
                        const uint8_t* v_in, uint16_t* v_out, const uint16_t* v_scales,
                        int dim0, int dim1, int heads, int head_dim,
                        int batch_size, int offset, int width,
                        int page_size, const int32_t* cache_seqlens,
                        const int32_t* block_table, int bt_stride, int wbits) {
  if (!valid_wbits(wbits) || heads < 0 || head_dim < 0 || head_dim % kBlock) return KVQREF_BAD_ARG;
  const Window w{dim0, dim1, batch_size, offset, width, page_size, bt_stride, cache_seqlens, block_table};
  if (!window_args_ok(w)) return KVQREF_BAD_ARG;
  const long code_bytes = static_cast<long>(head_dim) * wbits / 8;
  const long nscales = head_dim / kBlock;
  uint8_t codes[65536];
  if (head_dim > 65536) return KVQREF_BAD_ARG;
  auto one = [&](const uint8_t* in, uint16_t* out, const uint16_t* scales, long row) {
    for (long h = 0; h < heads; ++h) {
      const long hr = row * heads + h;
      unpack_row(in + hr * code_bytes, head_dim, wbits, codes);
      dequantize_row(codes, scales + hr * nscales, head_dim, wbits, out + hr * head_dim);
    }
  };
  int st_k = for_each_row(w, [&](long row) { one(k_in, k_out, k_scales, row); });
  int st_v = for_each_row(w, [&](long row) { one(v_in, v_out, v_scales, row); });
  return st_k != KVQREF_OK ? st_k : st_v;
}

// Usage ("convert KV tensors during the attention forward pass"): attention of
// one new query per sequence over the dequantized cache, in double precision,
// one position at a time.
}  // extern "C" (the shared attention loop below is C++)

namespace {

// Decode attention for one query over positions [0, seqlen) of sequence i:
// `key_row(hr, out)` / `value_row(hr, out)` write the binary16 key / value of
// cache row hr (row * heads + kv head).  Scores, softmax and the weighted sum
// in double precision, one position at a time, in the order the definition
// states them.
template <class KeyRow, class ValueRow>
int attention_rows(const uint16_t* q, uint16_t* out, double* out_exact, int dim0, int dim1, int heads, int head_dim,
                   int batch_size, int n_heads, int page_size, const int32_t* cache_seqlens,
                   const int32_t* block_table, int bt_stride, double softmax_scale, KeyRow key_row,
                   ValueRow value_row) {
  const int group = n_heads / heads;
  int status = KVQREF_OK;
  uint16_t deq[65536];
  for (int i = 0; i < batch_size; ++i) {
    const long L = cache_seqlens[i] < 0 ? 0 : cache_seqlens[i];
    if (page_size == 0 && L > dim1) return KVQREF_BAD_ARG;
    for (int h = 0; h < n_heads; ++h) {
      const int kvh = h / group;
      const uint16_t* qh = q + (static_cast<long>(i) * n_heads + h) * head_dim;
      // pass 1: scores
      double* s = new double[L > 0 ? L : 1];
      long n_valid = 0;
      long* rows = new long[L > 0 ? L : 1];
      for (long p = 0; p < L; ++p) {
        long row;
        if (page_size == 0) {
          row = static_cast<long>(i) * dim1 + p;
        } else {
          const long lp = p / page_size;
          const int32_t page = lp < bt_stride ? block_table[static_cast<long>(i) * bt_stride + lp] : -1;
          if (lp >= bt_stride || page < 0 || page >= dim0) {
            status = KVQREF_BAD_PAGE;
            continue;
          }
          row = static_cast<long>(page) * page_size + p % page_size;
        }
        const long hr = row * heads + kvh;
        key_row(hr, deq);
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d) dot += half_to_double(qh[d]) * half_to_double(deq[d]);
        s[n_valid] = softmax_scale * dot;
        rows[n_valid] = hr;
        ++n_valid;
      }
      double m = -INFINITY;
      for (long j = 0; j < n_valid; ++j) m = s[j] > m ? s[j] : m;
      double denom = 0.0;
      for (long j = 0; j < n_valid; ++j) denom += std::exp(s[j] - m);
      // pass 2: weighted values
      double* acc = new double[head_dim];
      for (int d = 0; d < head_dim; ++d) acc[d] = 0.0;
      for (long j = 0; j < n_valid; ++j) {
        const double w = std::exp(s[j] - m) / denom;
        value_row(rows[j], deq);
        for (int d = 0; d < head_dim; ++d) acc[d] += w * half_to_double(deq[d]);
      }
      uint16_t* oh = out + (static_cast<long>(i) * n_heads + h) * head_dim;
      for (int d = 0; d < head_dim; ++d) {
        oh[d] = double_to_half(acc[d]);
        if (out_exact) out_exact[(static_cast<long>(i) * n_heads + h) * head_dim + d] = acc[d];
      }
      delete[] acc;
      delete[] rows;
      delete[] s;
    }
  }
  return status;
}

}  // namespace

extern "C" {

int kvqref_decode_attention_q(const uint16_t* q, const uint8_t* k_codes, const uint16_t* k_scales,
                              const uint8_t* v_codes, const uint16_t* v_scales, uint16_t* out,
                              double* out_exact, int dim0, int dim1, int heads, int head_dim,
                              int batch_size, int n_heads, int page_size, const int32_t* cache_seqlens,
                              const int32_t* block_table, int bt_stride, int wbits, double softmax_scale) {
  if (!valid_wbits(wbits) || heads <= 0 || head_dim <= 0 || head_dim % kBlock || head_dim > 65536) return KVQREF_BAD_ARG;
  if (n_heads <= 0 || n_heads % heads || batch_size < 0 || dim0 < 0 || dim1 < 0 || !cache_seqlens) return KVQREF_BAD_ARG;
  if (page_size < 0 || (page_size > 0 && (dim1 != page_size || !block_table))) return KVQREF_BAD_ARG;
  if (page_size == 0 && batch_size > dim0) return KVQREF_BAD_ARG;
  const long code_bytes = static_cast<long>(head_dim) * wbits / 8;
  const long nscales = head_dim / kBlock;
  uint8_t codes[65536];
  // keys and values: the packed codes unpacked and dequantized exactly as kvqref_q_to_fp16_kv does
  auto k_row = [&](long hr, uint16_t* o) {
    unpack_row(k_codes + hr * code_bytes, head_dim, wbits, codes);
    dequantize_row(codes, k_scales + hr * nscales, head_dim, wbits, o);
  };
  auto v_row = [&](long hr, uint16_t* o) {
    unpack_row(v_codes + hr * code_bytes, head_dim, wbits, codes);
    dequantize_row(codes, v_scales + hr * nscales, head_dim, wbits, o);
  };
  return attention_rows(q, out, out_exact, dim0, dim1, heads, head_dim, batch_size, n_heads, page_size, cache_seqlens,
                        block_table, bt_stride, softmax_scale, k_row, v_row);
}

int kvqref_decode_attention_fp8(const uint16_t* q, const uint8_t* k_fp8, const uint8_t* v_fp8, uint16_t* out,
                                double* out_exact, int dim0, int dim1, int heads, int head_dim, int batch_size,
                                int n_heads, int page_size, const int32_t* cache_seqlens, const int32_t* block_table,
                                int bt_stride, double softmax_scale) {
  if (heads <= 0 || head_dim <= 0 || head_dim > 65536) return KVQREF_BAD_ARG;
  if (n_heads <= 0 || n_heads % heads || batch_size < 0 || dim0 < 0 || dim1 < 0 || !cache_seqlens) return KVQREF_BAD_ARG;
  if (page_size < 0 || (page_size > 0 && (dim1 != page_size || !block_table))) return KVQREF_BAD_ARG;
  if (page_size == 0 && batch_size > dim0) return KVQREF_BAD_ARG;
  // keys and values: each E5M2 byte decoded exactly as kvqref_fp8_to_fp16 does
  auto k_row = [&](long hr, uint16_t* o) {
    for (int d = 0; d < head_dim; ++d) o[d] = e5m2_decode(k_fp8[hr * head_dim + d]);
  };
  auto v_row = [&](long hr, uint16_t* o) {
    for (int d = 0; d < head_dim; ++d) o[d] = e5m2_decode(v_fp8[hr * head_dim + d]);
  };
  return attention_rows(q, out, out_exact, dim0, dim1, heads, head_dim, batch_size, n_heads, page_size, cache_seqlens,
                        block_table, bt_stride, softmax_scale, k_row, v_row);
}

// Description, count_match: compare element by element from the start and
// stop at the first difference, at the end of either sequence, or at max_a.
long long kvqref_count_match(const int64_t* a, long long a_len, const int64_t* b, long long b_len,
                             long long max_a) {
  long long n = a_len < b_len ? a_len : b_len;
  if (max_a < n) n = max_a;
  long long i = 0;
  while (i < n && a[i] == b[i]) ++i;
  return i < 0 ? 0 : i;
}

}  // extern "C"
