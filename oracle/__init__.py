"""Python face of the CPU oracle (oracle/libkvqref.so).

TEST INFRASTRUCTURE ONLY.  The oracle is the plain single-threaded C++
restatement of the KV-cache conversions from the page "Implementation:
Turboderp org Exllamav2 Ext Cache" (Description, Signature, I/O Contract);
its numerics are listed in ``kvqref.h``.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this module.  It works on host numpy arrays (FP16 as ``uint16`` bit patterns
or ``float16``) and never touches the CUDA library.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

OK, BAD_ARG, BAD_PAGE = 0, 1, 2

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i32p = ctypes.POINTER(ctypes.c_int32)
        I = ctypes.c_int
        L.kvqref_half_to_double.argtypes = [ctypes.c_uint16]
        L.kvqref_half_to_double.restype = ctypes.c_double
        L.kvqref_double_to_half.argtypes = [ctypes.c_double]
        L.kvqref_double_to_half.restype = ctypes.c_uint16
        L.kvqref_e5m2_encode.argtypes = [ctypes.c_uint16]
        L.kvqref_e5m2_encode.restype = ctypes.c_uint8
        L.kvqref_e5m2_decode.argtypes = [ctypes.c_uint8]
        L.kvqref_e5m2_decode.restype = ctypes.c_uint16
        L.kvqref_block_scale.argtypes = [ctypes.c_uint16, I]
        L.kvqref_block_scale.restype = ctypes.c_uint16
        L.kvqref_quantize_row.argtypes = [u16p, I, I, u8p, u16p]
        L.kvqref_dequantize_row.argtypes = [u8p, u16p, I, I, u16p]
        L.kvqref_pack_row.argtypes = [u8p, I, I, u8p]
        L.kvqref_unpack_row.argtypes = [u8p, I, I, u8p]
        L.kvqref_fp16_to_fp8.argtypes = [u16p, u8p] + [I] * 7
        L.kvqref_fp8_to_fp16.argtypes = [u8p, u16p] + [I] * 7
        L.kvqref_fp16_to_fp8_kv.argtypes = [u16p, u8p, u16p, u8p] + [I] * 8 + [i32p, i32p, I]
        L.kvqref_fp8_to_fp16_kv.argtypes = [u8p, u16p, u8p, u16p] + [I] * 8 + [i32p, i32p, I]
        L.kvqref_fp16_to_q_kv.argtypes = [u16p, u8p, u16p, u16p, u8p, u16p] + [I] * 8 + [i32p, i32p, I, I]
        L.kvqref_q_to_fp16_kv.argtypes = [u8p, u16p, u16p, u8p, u16p, u16p] + [I] * 8 + [i32p, i32p, I, I]
        f64p = ctypes.POINTER(ctypes.c_double)
        L.kvqref_decode_attention_q.argtypes = [u16p, u8p, u16p, u8p, u16p, u16p, f64p] + [I] * 7 + \
            [i32p, i32p, I, I, ctypes.c_double]
        L.kvqref_decode_attention_q.restype = ctypes.c_int
        L.kvqref_decode_attention_fp8.argtypes = [u16p, u8p, u8p, u16p, f64p] + [I] * 7 + \
            [i32p, i32p, I, ctypes.c_double]
        L.kvqref_decode_attention_fp8.restype = ctypes.c_int
        i64p = ctypes.POINTER(ctypes.c_int64)
        LL = ctypes.c_longlong
        L.kvqref_count_match.argtypes = [i64p, LL, i64p, LL, LL]
        L.kvqref_count_match.restype = LL
        for name in ("kvqref_quantize_row", "kvqref_dequantize_row", "kvqref_pack_row",
                     "kvqref_unpack_row", "kvqref_fp16_to_fp8", "kvqref_fp8_to_fp16",
                     "kvqref_fp16_to_q_kv", "kvqref_q_to_fp16_kv", "kvqref_fp16_to_fp8_kv",
                     "kvqref_fp8_to_fp16_kv"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray | None, ctype):
    if a is None:
        return ctypes.POINTER(ctype)()
    assert a.flags["C_CONTIGUOUS"], "oracle buffers must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _bits(a: np.ndarray) -> np.ndarray:
    """View float16 data as its uint16 bit patterns (uint16 passes through)."""
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


# ---- scalar primitives --------------------------------------------------------

def half_to_double(h: int) -> float:
    return lib().kvqref_half_to_double(h)


def double_to_half(v: float) -> int:
    return lib().kvqref_double_to_half(v)


def e5m2_encode(h: int) -> int:
    return lib().kvqref_e5m2_encode(h)


def e5m2_decode(b: int) -> int:
    return lib().kvqref_e5m2_decode(b)


def block_scale(absmax_bits: int, wbits: int) -> int:
    return lib().kvqref_block_scale(absmax_bits, wbits)


def quantize_row(x: np.ndarray, wbits: int):
    """-> (codes uint8[n], scales uint16[n/32]) for one row of FP16 values."""
    x = np.ascontiguousarray(_bits(x))
    n = x.size
    codes = np.zeros(n, np.uint8)
    scales = np.zeros(n // 32, np.uint16)
    st = lib().kvqref_quantize_row(_p(x, ctypes.c_uint16), n, wbits, _p(codes, ctypes.c_uint8),
                                   _p(scales, ctypes.c_uint16))
    assert st == OK, st
    return codes, scales


def dequantize_row(codes: np.ndarray, scales: np.ndarray, wbits: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(_bits(scales))
    y = np.zeros(codes.size, np.uint16)
    st = lib().kvqref_dequantize_row(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint16),
                                     codes.size, wbits, _p(y, ctypes.c_uint16))
    assert st == OK, st
    return y


def pack_row(codes: np.ndarray, wbits: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    out = np.zeros(codes.size * wbits // 8, np.uint8)
    st = lib().kvqref_pack_row(_p(codes, ctypes.c_uint8), codes.size, wbits, _p(out, ctypes.c_uint8))
    assert st == OK, st
    return out


def unpack_row(packed: np.ndarray, n: int, wbits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.uint8)
    assert packed.size == n * wbits // 8
    out = np.zeros(n, np.uint8)
    st = lib().kvqref_unpack_row(_p(packed, ctypes.c_uint8), n, wbits, _p(out, ctypes.c_uint8))
    assert st == OK, st
    return out


# ---- cache conversions (in place on caller-owned numpy arrays) ------------------

def fp16_to_fp8(inp: np.ndarray, out: np.ndarray, batch_size: int, offset: int, width: int) -> int:
    """inp [d0, d1, H, D] float16/uint16 -> out [d0, d1, H, D] uint8 (in place)."""
    d0, d1, H, D = inp.shape
    assert out.shape == inp.shape and out.dtype == np.uint8
    x = np.ascontiguousarray(_bits(inp))
    return lib().kvqref_fp16_to_fp8(_p(x, ctypes.c_uint16), _p(out, ctypes.c_uint8),
                                    d0, d1, H, D, batch_size, offset, width)


def fp8_to_fp16(inp: np.ndarray, out: np.ndarray, batch_size: int, offset: int, width: int) -> int:
    """inp [d0, d1, H, D] uint8 -> out [d0, d1, H, D] float16/uint16 (in place)."""
    d0, d1, H, D = inp.shape
    assert out.shape == inp.shape and inp.dtype == np.uint8
    o = _bits(out)
    assert o.flags["C_CONTIGUOUS"]
    return lib().kvqref_fp8_to_fp16(_p(np.ascontiguousarray(inp), ctypes.c_uint8), _p(o, ctypes.c_uint16),
                                    d0, d1, H, D, batch_size, offset, width)


def _page_args(page_size, cache_seqlens, block_table):
    if page_size and cache_seqlens is not None:
        sl = np.ascontiguousarray(cache_seqlens, np.int32)
        bt = np.ascontiguousarray(block_table, np.int32)
        stride = bt.shape[1] if bt.ndim == 2 else 0
        return sl, bt, stride
    return None, None, 0


def fp16_to_fp8_kv(k_in, k_out, v_in, v_out, batch_size, offset, width, page_size=0, cache_seqlens=None,
                   block_table=None) -> int:
    """E5M2-encode K and V (float16/uint16 [d0, d1, H, D]) into uint8 caches, contiguous or paged."""
    d0, d1, H, D = k_in.shape
    sl, bt, stride = _page_args(page_size, cache_seqlens, block_table)
    for a in (k_out, v_out):
        assert a.flags["C_CONTIGUOUS"] and a.dtype == np.uint8
    return lib().kvqref_fp16_to_fp8_kv(
        _p(np.ascontiguousarray(_bits(k_in)), ctypes.c_uint16), _p(k_out, ctypes.c_uint8),
        _p(np.ascontiguousarray(_bits(v_in)), ctypes.c_uint16), _p(v_out, ctypes.c_uint8),
        d0, d1, H, D, batch_size, offset, width, page_size, _p(sl, ctypes.c_int32), _p(bt, ctypes.c_int32), stride)


def fp8_to_fp16_kv(k_in, k_out, v_in, v_out, batch_size, offset, width, page_size=0, cache_seqlens=None,
                   block_table=None) -> int:
    """Decode K and V E5M2 caches (uint8 [d0, d1, H, D]) into FP16 caches, contiguous or paged."""
    d0, d1, H, D = k_in.shape
    sl, bt, stride = _page_args(page_size, cache_seqlens, block_table)
    ko, vo = _bits(k_out), _bits(v_out)
    for a in (ko, vo):
        assert a.flags["C_CONTIGUOUS"]
    return lib().kvqref_fp8_to_fp16_kv(
        _p(np.ascontiguousarray(k_in, np.uint8), ctypes.c_uint8), _p(ko, ctypes.c_uint16),
        _p(np.ascontiguousarray(v_in, np.uint8), ctypes.c_uint8), _p(vo, ctypes.c_uint16),
        d0, d1, H, D, batch_size, offset, width, page_size, _p(sl, ctypes.c_int32), _p(bt, ctypes.c_int32), stride)


def fp16_to_q_kv(k_in, k_out, k_scales, v_in, v_out, v_scales, batch_size, offset, width,
                 page_size, cache_seqlens, block_table, wbits) -> int:
    """Quantize K and V (float16/uint16 [d0, d1, H, D]) into codes [d0, d1, H, D*wbits/8]
    uint8 and scales [d0, d1, H, D/32] uint16/float16, in place."""
    d0, d1, H, D = k_in.shape
    sl, bt, stride = _page_args(page_size, cache_seqlens, block_table)
    ks, vs = _bits(k_scales), _bits(v_scales)
    for a in (k_out, v_out, ks, vs):
        assert a.flags["C_CONTIGUOUS"]
    return lib().kvqref_fp16_to_q_kv(
        _p(np.ascontiguousarray(_bits(k_in)), ctypes.c_uint16), _p(k_out, ctypes.c_uint8), _p(ks, ctypes.c_uint16),
        _p(np.ascontiguousarray(_bits(v_in)), ctypes.c_uint16), _p(v_out, ctypes.c_uint8), _p(vs, ctypes.c_uint16),
        d0, d1, H, D, batch_size, offset, width, page_size,
        _p(sl, ctypes.c_int32), _p(bt, ctypes.c_int32), stride, wbits)


def q_to_fp16_kv(k_in, k_out, k_scales, v_in, v_out, v_scales, batch_size, offset, width,
                 page_size, cache_seqlens, block_table, wbits) -> int:
    """Dequantize K and V codes/scales into FP16 caches [d0, d1, H, D], in place."""
    d0, d1, H, _ = k_in.shape
    D = k_out.shape[3]
    sl, bt, stride = _page_args(page_size, cache_seqlens, block_table)
    ko, vo = _bits(k_out), _bits(v_out)
    for a in (ko, vo):
        assert a.flags["C_CONTIGUOUS"]
    return lib().kvqref_q_to_fp16_kv(
        _p(np.ascontiguousarray(k_in, np.uint8), ctypes.c_uint8), _p(ko, ctypes.c_uint16),
        _p(np.ascontiguousarray(_bits(k_scales)), ctypes.c_uint16),
        _p(np.ascontiguousarray(v_in, np.uint8), ctypes.c_uint8), _p(vo, ctypes.c_uint16),
        _p(np.ascontiguousarray(_bits(v_scales)), ctypes.c_uint16),
        d0, d1, H, D, batch_size, offset, width, page_size,
        _p(sl, ctypes.c_int32), _p(bt, ctypes.c_int32), stride, wbits)


def count_match(a: np.ndarray, b: np.ndarray, max_a: int) -> int:
    """Common-prefix length of two int64 sequences, capped at max_a."""
    a = np.ascontiguousarray(a, np.int64)
    b = np.ascontiguousarray(b, np.int64)
    return lib().kvqref_count_match(_p(a, ctypes.c_int64), a.size, _p(b, ctypes.c_int64), b.size, int(max_a))


def decode_attention_q(q, k_codes, k_scales, v_codes, v_scales, batch_size, n_heads, page_size,
                       cache_seqlens, block_table, wbits, softmax_scale, head_dim):
    """fp64 decode attention over the dequantized cache.  q: [batch, n_heads, D] float16/uint16;
    codes [d0, d1, H, D*wbits/8] uint8; scales [d0, d1, H, D/32].  Returns (status, out uint16
    [batch, n_heads, D], exact float64 [batch, n_heads, D])."""
    d0, d1, H, _ = k_codes.shape
    qb = np.ascontiguousarray(_bits(q))
    out = np.zeros((batch_size, n_heads, head_dim), np.uint16)
    ex = np.zeros((batch_size, n_heads, head_dim), np.float64)
    sl = np.ascontiguousarray(cache_seqlens, np.int32)
    if page_size:
        bt = np.ascontiguousarray(block_table, np.int32)
        stride = bt.shape[1]
    else:
        bt, stride = None, 0
    st = lib().kvqref_decode_attention_q(
        _p(qb, ctypes.c_uint16), _p(np.ascontiguousarray(k_codes, np.uint8), ctypes.c_uint8),
        _p(np.ascontiguousarray(_bits(k_scales)), ctypes.c_uint16),
        _p(np.ascontiguousarray(v_codes, np.uint8), ctypes.c_uint8),
        _p(np.ascontiguousarray(_bits(v_scales)), ctypes.c_uint16), _p(out, ctypes.c_uint16),
        _p(ex, ctypes.c_double), d0, d1, H, head_dim, batch_size, n_heads, page_size,
        _p(sl, ctypes.c_int32), _p(bt, ctypes.c_int32), stride, wbits, float(softmax_scale))
    return st, out, ex


def decode_attention_fp8(q, k_fp8, v_fp8, batch_size, n_heads, page_size, cache_seqlens, block_table,
                         softmax_scale):
    """fp64 decode attention over an FP8 (E5M2) cache, keys and values decoded exactly.
    q: [batch, n_heads, D] float16/uint16; k_fp8, v_fp8: [d0, d1, H, D] uint8.  Returns
    (status, out uint16 [batch, n_heads, D], exact float64 [batch, n_heads, D])."""
    d0, d1, H, D = k_fp8.shape
    qb = np.ascontiguousarray(_bits(q))
    out = np.zeros((batch_size, n_heads, D), np.uint16)
    ex = np.zeros((batch_size, n_heads, D), np.float64)
    sl = np.ascontiguousarray(cache_seqlens, np.int32)
    if page_size:
        bt = np.ascontiguousarray(block_table, np.int32)
        stride = bt.shape[1]
    else:
        bt, stride = None, 0
    st = lib().kvqref_decode_attention_fp8(
        _p(qb, ctypes.c_uint16), _p(np.ascontiguousarray(k_fp8, np.uint8), ctypes.c_uint8),
        _p(np.ascontiguousarray(v_fp8, np.uint8), ctypes.c_uint8), _p(out, ctypes.c_uint16),
        _p(ex, ctypes.c_double), d0, d1, H, D, batch_size, n_heads, page_size,
        _p(sl, ctypes.c_int32), _p(bt, ctypes.c_int32), stride, float(softmax_scale))
    return st, out, ex
