"""Pins for the CPU oracle: each check ties it to something other than itself.

* binary16 conversions: numpy's IEEE float16 (exhaustive over bit patterns,
  plus every rounding boundary).
* E5M2 encode: brute-force nearest search over all finite E5M2 values
  (exhaustive over 65 536 inputs), numpy/ml_dtypes casts, hand-derived values.
* Scale: exact rational rounding (Fraction) of absmax / maxq, exhaustive over
  every finite binary16 absmax for both bit widths.
* Codes: exact rational round-half-even of x / s on structured and random
  blocks; dequantization: exact rational product rounded to binary16.
* Packing: an independent big-integer bit stream, plus hand-derived blocks.

Source of the operations: page "Implementation: Turboderp org Exllamav2 Ext
Cache", Description and I/O Contract.
"""
from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import exact

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ALL16 = np.arange(65536, dtype=np.uint32).astype(np.uint16)


def _is_nan16(bits):
    bits = np.asarray(bits)
    return (((bits >> 10) & 0x1F) == 31) & ((bits & 0x3FF) != 0)


# ---------------------------------------------------------------- binary16 ----

def test_half_to_double_exhaustive_vs_numpy(oracle_mod):
    ref = ALL16.view(np.float16).astype(np.float64)
    got = np.array([oracle_mod.half_to_double(int(h)) for h in ALL16])
    nan = _is_nan16(ALL16)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # the sign of zero is kept
    assert np.signbit(got[0x8000]) and not np.signbit(got[0])


def test_double_to_half_boundaries_vs_numpy(oracle_mod):
    """Every binary16 value, every midpoint between neighbours and the doubles just
    either side of each midpoint: numpy's float64 -> float16 cast rounds to nearest
    even, so both must agree on all of them."""
    finite = ALL16[~_is_nan16(ALL16) & (((ALL16 >> 10) & 0x1F) != 31)]
    vals = np.sort(np.unique(finite.view(np.float16).astype(np.float64)))
    mids = (vals[:-1] + vals[1:]) / 2  # exact in float64
    # overflow boundary: midpoint of 65504 and 65536
    extra = np.array([65520.0, -65520.0, 65519.99, 1e6, -1e6, 2.0 ** -25, -(2.0 ** -25),
                      2.0 ** -26, 3 * 2.0 ** -26, np.inf, -np.inf, 0.0, -0.0])
    probe = np.concatenate([vals, mids, np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf), extra])
    rng = np.random.default_rng(7)
    probe = np.concatenate([probe, rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 5, 20000)])
    with np.errstate(over="ignore"):
        ref = probe.astype(np.float16).view(np.uint16)
    got = np.array([oracle_mod.double_to_half(float(v)) for v in probe], dtype=np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(probe[i], hex(got[i]), hex(ref[i])) for i in bad[:5]]


def test_double_to_half_nan(oracle_mod):
    assert oracle_mod.double_to_half(float("nan")) & 0x7FFF == 0x7E00


# -------------------------------------------------------------------- E5M2 ----

def test_e5m2_encode_exhaustive_bruteforce(oracle_mod):
    ref = exact.e5m2_nearest_all(ALL16)
    got = np.array([oracle_mod.e5m2_encode(int(h)) for h in ALL16], dtype=np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(hex(int(ALL16[i])), hex(got[i]), hex(ref[i])) for i in bad[:8]]


def test_e5m2_encode_vs_library_casts(oracle_mod):
    """Finite, non-NaN inputs against a library E5M2 cast (ml_dtypes; torch on CPU as
    a second one): both round to nearest even and overflow to Inf."""
    finite = ALL16[~_is_nan16(ALL16)]
    got = np.array([oracle_mod.e5m2_encode(int(h)) for h in finite], dtype=np.uint8)
    try:
        import ml_dtypes

        ref = finite.view(np.float16).astype(ml_dtypes.float8_e5m2).view(np.uint8)
        assert np.array_equal(got, ref)
    except ImportError:
        pass
    import torch

    ref_t = torch.from_numpy(finite.view(np.float16).copy()).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(got, ref_t)


def test_e5m2_decode_exhaustive(oracle_mod):
    table = dict(exact.e5m2_table())
    for b in range(256):
        h = oracle_mod.e5m2_decode(b)
        if b in table:
            assert exact.half_value(h) == table[b], hex(b)
            assert (h >> 15) == (b >> 7)  # sign, including -0
        else:  # Inf / NaN: E5M2 is the top byte of the binary16 encoding
            assert h == b << 8, hex(b)


def test_e5m2_roundtrip_identity(oracle_mod):
    """Every binary16 whose low byte is zero is an E5M2 value: enc then dec is exact."""
    for h in range(0, 65536, 256):
        if _is_nan16(h):
            continue
        assert oracle_mod.e5m2_decode(oracle_mod.e5m2_encode(h)) == h, hex(h)


def _golden_fp8():
    rows = []
    with open(os.path.join(GOLDEN, "fp8_e5m2_worked.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                a, b, c = (int(t, 16) for t in line.split())
                rows.append((a, b, c))
    return rows


@pytest.mark.parametrize("h,byte,dec", _golden_fp8())
def test_e5m2_worked_values(oracle_mod, h, byte, dec):
    assert oracle_mod.e5m2_encode(h) == byte
    assert oracle_mod.e5m2_decode(byte) == dec


# ------------------------------------------------------------------- scale ----

@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_block_scale_exhaustive_exact(oracle_mod, wbits):
    """s = RN16(fl32(a / maxq)) equals the binary16 nearest to the exact quotient for
    every finite absmax a (so the binary32 intermediate never double-rounds)."""
    maxq = (1 << (wbits - 1)) - 1
    for a in range(0, 0x7C00):
        ref = exact.round_to_half_bits(exact.half_value(a) / maxq)
        got = oracle_mod.block_scale(a, wbits)
        assert got == ref, (hex(a), hex(got), hex(ref))


# ------------------------------------------------------------ codes / deq ----

def _codes_exact(x_bits, wbits):
    maxq = (1 << (wbits - 1)) - 1
    z = 1 << (wbits - 1)
    vals = [exact.half_value(int(b)) for b in x_bits]
    a = max(abs(v) for v in vals)
    s_bits = exact.round_to_half_bits(a / maxq)
    s = exact.half_value(s_bits)
    if s == 0:
        return [z] * len(vals), s_bits
    codes = [min(max(exact.round_half_even(v / s) + z, 0), (1 << wbits) - 1) for v in vals]
    return codes, s_bits


def _deq_exact(codes, s_bits, wbits):
    z = 1 << (wbits - 1)
    s = exact.half_value(s_bits)
    return [exact.round_to_half_bits((c - z) * s) for c in codes]


def _test_blocks(seed):
    """Blocks that stress rounding: N(0,1); channel-scaled; outliers; tiny values that
    give subnormal or zero scales; exact ties (small multiples of s/2)."""
    rng = np.random.default_rng(seed)
    blocks = []
    for _ in range(300):
        blocks.append(rng.standard_normal(32).astype(np.float16))
    for _ in range(100):
        blocks.append((rng.standard_normal(32) * np.exp(rng.standard_normal(32))).astype(np.float16))
    for _ in range(100):
        x = rng.standard_normal(32)
        x[rng.integers(0, 32)] = rng.choice([-1, 1]) * rng.uniform(20, 60000)
        blocks.append(x.astype(np.float16))
    for _ in range(200):  # subnormal magnitudes: scale is subnormal or zero
        bits = rng.integers(0, 64, 32).astype(np.uint16) | np.where(rng.random(32) < 0.5, 0x8000, 0).astype(np.uint16)
        blocks.append(bits.view(np.float16))
    for wb in (4, 6, 8):  # exact ties: absmax maxq * 2^k, members (k+0.5) * 2^k
        maxq = (1 << (wb - 1)) - 1
        for _ in range(100):
            e = float(2.0 ** rng.integers(-8, 8))
            half_steps = rng.integers(-2 * maxq, 2 * maxq + 1, 32)
            x = half_steps * 0.5 * e
            x[0] = maxq * e
            blocks.append(x.astype(np.float16))
    blocks.append(np.zeros(32, np.float16))
    return blocks


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_quantize_codes_exact(oracle_mod, wbits):
    for blk in _test_blocks(11 + wbits):
        bits = blk.view(np.uint16)
        codes, scales = oracle_mod.quantize_row(bits, wbits)
        ref_codes, ref_s = _codes_exact(bits, wbits)
        assert int(scales[0]) == ref_s
        assert codes.tolist() == ref_codes, (blk, codes, ref_codes)


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_dequantize_exact(oracle_mod, wbits):
    rng = np.random.default_rng(5 + wbits)
    for blk in _test_blocks(21 + wbits)[:400]:
        codes, scales = oracle_mod.quantize_row(blk.view(np.uint16), wbits)
        y = oracle_mod.dequantize_row(codes, scales, wbits)
        assert y.tolist() == _deq_exact(codes.tolist(), int(scales[0]), wbits)
    # every code against random finite scales, with numpy's binary16 multiply as a
    # second reference (it rounds the exact binary32 product once)
    z = 1 << (wbits - 1)
    for _ in range(200):
        s_bits = int(rng.integers(0, 0x7C00))
        n = max(64, 1 << wbits)
        codes = np.resize(np.arange(1 << wbits, dtype=np.uint8), n)
        scales = np.full(n // 32, s_bits, np.uint16)
        y = oracle_mod.dequantize_row(codes, scales, wbits)
        with np.errstate(over="ignore"):
            ref = (codes.astype(np.float16) - np.float16(z)) * scales.view(np.float16)[0]
        assert np.array_equal(y, ref.astype(np.float16).view(np.uint16))
        assert y.tolist() == _deq_exact(codes.tolist(), s_bits, wbits)


# ----------------------------------------------------------------- packing ----

@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_pack_bitstream(oracle_mod, wbits):
    rng = np.random.default_rng(wbits)
    for n in (32, 64, 128, 256):
        codes = rng.integers(0, 1 << wbits, n).astype(np.uint8)
        packed = oracle_mod.pack_row(codes, wbits)
        stream = 0
        for j, c in enumerate(codes.tolist()):
            stream |= c << (wbits * j)
        ref = stream.to_bytes(n * wbits // 8, "little")
        assert packed.tobytes() == ref
        assert np.array_equal(oracle_mod.unpack_row(packed, n, wbits), codes)


def test_q6_group_words(oracle_mod):
    """Q6: 16 codes per three little-endian 32-bit words, code j at bits 6j..6j+5 of
    the 96-bit group (codes 5 and 10 straddle words)."""
    codes = np.arange(16, dtype=np.uint8) * 4 + 3  # 3, 7, ..., 63
    words = np.frombuffer(oracle_mod.pack_row(np.resize(codes, 32), 6).tobytes(), "<u4")
    for j in range(16):
        bit = 6 * j
        w, off = divmod(bit, 32)
        val = int(words[w]) >> off
        if off > 26:
            val |= int(words[w + 1]) << (32 - off)
        assert val & 63 == codes[j]


# ---------------------------------------------------------- worked blocks ----

def _golden_blocks():
    out = []
    with open(os.path.join(GOLDEN, "q_worked_blocks.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                out.append(json.loads(line))
    return out


@pytest.mark.parametrize("case", _golden_blocks(), ids=lambda c: c["why"][:40])
def test_worked_blocks(oracle_mod, case):
    wb = case["wbits"]
    z = 1 << (wb - 1)
    x = np.zeros(32, np.uint16)
    for i, b in case["x"].items():
        x[int(i)] = int(b, 16)
    codes, scales = oracle_mod.quantize_row(x, wb)
    assert int(scales[0]) == int(case["scale"], 16)
    exp_codes = case["codes"] + [z] * (32 - len(case["codes"]))
    assert codes.tolist() == exp_codes
    assert oracle_mod.pack_row(codes, wb).tobytes().hex() == case["packed"]
    y = oracle_mod.dequantize_row(codes, scales, wb)
    exp_y = np.zeros(32, np.uint16)
    for i, b in case["deq"].items():
        exp_y[int(i)] = int(b, 16)
    assert y.tolist() == exp_y.tolist()
    # and the hand-derived values agree with exact rational arithmetic
    assert _codes_exact(x, wb) == (exp_codes, int(case["scale"], 16))
