"""Cache-level pins for the CPU oracle: invariants that any correct KV-cache
conversion must satisfy, checked on the workload recipes at small sizes.

Operations from page "Implementation: Turboderp org Exllamav2 Ext Cache":
Description (window `batch_size, offset, width`; paged mode via block_table and
cache_seqlens) and I/O Contract (codes, per-block FP16 scales, wbits 4 or 6).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads

SENT8 = 0xA5
SENT16 = 0xA5A5


def _np16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def _q_buffers(shape, wbits, fill=True):
    d0, d1, H, D = shape
    codes = np.full((d0, d1, H, D * wbits // 8), SENT8 if fill else 0, np.uint8)
    scales = np.full((d0, d1, H, D // 32), SENT16 if fill else 0, np.uint16)
    return codes, scales


def _quant_contig(o, k, v, wbits, batch, offset, width):
    kc, ks = _q_buffers(k.shape, wbits)
    vc, vs = _q_buffers(v.shape, wbits)
    st = o.fp16_to_q_kv(k, kc, ks, v, vc, vs, batch, offset, width, 0, None, None, wbits)
    assert st == o.OK
    return kc, ks, vc, vs


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_zero_blocks_error_bound_idempotence(oracle_mod, wbits):
    k, v = workloads.channel_outliers(shape=(2, 64, 8, 128))
    k, v = _np16(k), _np16(v)
    B, S, H, D = k.shape
    kc, ks, vc, vs = _quant_contig(oracle_mod, k, v, wbits, B, 0, S)
    z = 1 << (wbits - 1)
    for x, c, s in ((k, kc, ks), (v, vc, vs)):
        y = np.zeros_like(x)
        y2 = np.zeros_like(x)
        st = oracle_mod.q_to_fp16_kv(c, y, s, c, y2, s, B, 0, S, 0, None, None, wbits)
        assert st == oracle_mod.OK and np.array_equal(y, y2)
        xb = x.reshape(-1, 32)
        zero_blk = (xb & 0x7FFF).max(axis=1) == 0
        assert zero_blk.sum() > 0
        sc = s.reshape(-1)
        # (1) all-zero blocks: scale +0 and every code z (Q4 bytes 0x88, Q6 pattern)
        assert np.all(sc[zero_blk] == 0)
        codes = np.stack([oracle_mod.unpack_row(r, D, wbits) for r in c.reshape(-1, D * wbits // 8)])
        assert np.all(codes.reshape(-1, 32)[zero_blk] == z)
        assert np.all(y.reshape(-1, 32)[zero_blk] == 0)
        # (2) error bound for normal scales: |x - y| <= s/2 + ulp16(y)/2
        xf = x.view(np.float16).astype(np.float64).reshape(-1, 32)
        yf = y.view(np.float16).astype(np.float64).reshape(-1, 32)
        sf = sc.view(np.float16).astype(np.float64)
        normal = sf >= 2.0 ** -14
        ulp = np.spacing(np.abs(yf).astype(np.float16)).astype(np.float64)
        err = np.abs(xf - yf)
        bound = sf[:, None] / 2 + ulp / 2
        assert np.all(err[normal] <= bound[normal])
        # (3) codes are idempotent: Q(D(Q(x))) has the same codes
        c2, s2 = _q_buffers(x.shape, wbits)
        st = oracle_mod.fp16_to_q_kv(y, c2, s2, y, c2.copy(), s2.copy(), B, 0, S, 0, None, None, wbits)
        assert st == oracle_mod.OK
        codes2 = np.stack([oracle_mod.unpack_row(r, D, wbits) for r in c2.reshape(-1, D * wbits // 8)])
        sel = normal
        assert np.array_equal(codes2.reshape(-1, 32)[sel], codes.reshape(-1, 32)[sel])


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_paged_identity_equals_contiguous(oracle_mod, wbits):
    B, S, H, D, ps = 3, 96, 4, 64, 32
    k, v = workloads.small(shape=(B, S, H, D))
    k, v = _np16(k), _np16(v)
    offset, width = 20, 50
    ref = _quant_contig(oracle_mod, k, v, wbits, B, offset, width)
    bt = workloads.identity_block_table(B, S, ps).numpy()
    pages = (B * S // ps, ps, H, D)
    kc, ks = _q_buffers(pages, wbits)
    vc, vs = _q_buffers(pages, wbits)
    seqlens = np.zeros(B, np.int32)
    st = oracle_mod.fp16_to_q_kv(k.reshape(pages), kc, ks, v.reshape(pages), vc, vs, B, offset, width,
                                 ps, seqlens, bt, wbits)
    assert st == oracle_mod.OK
    for a, b in zip(ref, (kc, ks, vc, vs)):
        assert np.array_equal(a.reshape(-1), b.reshape(-1))
    # dequantize both ways too
    y_ref = np.full(k.shape, SENT16, np.uint16)
    y_pg = np.full(pages, SENT16, np.uint16)
    oracle_mod.q_to_fp16_kv(ref[0], y_ref, ref[1], ref[2], y_ref.copy(), ref[3], B, offset, width, 0, None, None, wbits)
    oracle_mod.q_to_fp16_kv(kc, y_pg, ks, vc, y_pg.copy(), vs, B, offset, width, ps, seqlens, bt, wbits)
    assert np.array_equal(y_ref.reshape(-1), y_pg.reshape(-1))


def _expected_rows_paged(seqlens, bt, ps, batch, offset, width):
    rows = set()
    for i in range(batch):
        for p in range(max(0, seqlens[i] + offset), seqlens[i] + offset + width):
            rows.add(int(bt[i][p // ps]) * ps + p % ps)
    return rows


@pytest.mark.parametrize("offset,width", [(0, 1), (-40, 40), (-5, 6), (-1000, 17)])
def test_paged_window_touches_exactly_its_rows(oracle_mod, offset, width):
    ps, H, D, npages, batch = 16, 2, 32, 40, 5
    lens, bt = workloads.paged_tables(3, batch, 60, npages, ps)
    lens, bt = lens.numpy(), bt.numpy()
    k, v = workloads.small(shape=(npages, ps, H, D))
    k, v = _np16(k), _np16(v)
    kc, ks = _q_buffers(k.shape, 4)
    vc, vs = _q_buffers(v.shape, 4)
    st = oracle_mod.fp16_to_q_kv(k, kc, ks, v, vc, vs, batch, offset, width, ps, lens, bt, 4)
    assert st == oracle_mod.OK
    rows = _expected_rows_paged(lens, bt, ps, batch, offset, width)
    touched = {r for r in range(npages * ps) if np.any(kc.reshape(npages * ps, -1)[r] != SENT8)}
    assert touched == rows
    touched_s = {r for r in range(npages * ps) if np.any(vs.reshape(npages * ps, -1)[r] != SENT16)}
    assert touched_s == rows


def test_paged_bad_entries_are_skipped(oracle_mod):
    ps, H, D, npages = 8, 1, 32, 6
    k, v = workloads.small(shape=(npages, ps, H, D))
    k, v = _np16(k), _np16(v)
    kc, ks = _q_buffers(k.shape, 4)
    vc, vs = _q_buffers(v.shape, 4)
    bt = np.array([[0, 7], [1, -1]], np.int32)  # page 7 is outside the pool, -1 unused
    lens = np.array([4, 6], np.int32)
    st = oracle_mod.fp16_to_q_kv(k, kc, ks, v, vc, vs, 2, 0, 8, ps, lens, bt, 4)
    assert st == oracle_mod.BAD_PAGE
    # sequence 0: positions 4..7 in page 0 written, 8..11 (page 7) skipped;
    # sequence 1: positions 6..7 in page 1 written, 8..13 (entry -1) skipped
    flat = kc.reshape(npages * ps, -1)
    written = {r for r in range(npages * ps) if np.any(flat[r] != SENT8)}
    assert written == {4, 5, 6, 7, 8 + 6, 8 + 7}


def test_contiguous_window_untouched_outside(oracle_mod):
    k, v = workloads.fp8_window(shape=(3, 64, 2, 64))
    k = _np16(k)
    out = np.full(k.shape, SENT8, np.uint8)
    assert oracle_mod.fp16_to_fp8(k, out, 2, 10, 30) == oracle_mod.OK
    mask = np.zeros(k.shape, bool)
    mask[:2, 10:40] = True
    assert np.all(out[~mask] == SENT8)
    back = np.full(k.shape, SENT16, np.uint16)
    assert oracle_mod.fp8_to_fp16(out, back, 2, 10, 30) == oracle_mod.OK
    assert np.all(back[~mask] == SENT16)
    # inside the window: each element is the E5M2 rounding of the input
    enc = np.array([oracle_mod.e5m2_encode(int(h)) for h in k[mask][:2000]], np.uint8)
    assert np.array_equal(out[mask][:2000], enc)
    # every E5M2 value decodes to the binary16 with that top byte
    assert np.array_equal(back[mask], out[mask].astype(np.uint16) << 8)


def test_bad_arguments(oracle_mod):
    k = np.zeros((2, 8, 1, 32), np.uint16)
    out = np.zeros(k.shape, np.uint8)
    assert oracle_mod.fp16_to_fp8(k, out, 3, 0, 8) == oracle_mod.BAD_ARG   # batch > dim0
    assert oracle_mod.fp16_to_fp8(k, out, 2, 4, 5) == oracle_mod.BAD_ARG   # window past the end
    assert oracle_mod.fp16_to_fp8(k, out, 2, -1, 2) == oracle_mod.BAD_ARG  # negative offset
    kc, ks = _q_buffers(k.shape, 4)
    assert oracle_mod.fp16_to_q_kv(k, kc, ks, k, kc, ks, 2, 0, 8, 0, None, None, 5) == oracle_mod.BAD_ARG
    assert oracle_mod.fp16_to_q_kv(k, kc, ks, k, kc, ks, 2, 0, 8, 0, None, None, 7) == oracle_mod.BAD_ARG


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_numpy_restatement_agrees(oracle_mod, wbits):
    """A second, vectorised restatement (numpy binary32 division, np.rint ties to
    even, float16 casts) agrees with the oracle on the small and channel-outlier
    recipes."""
    maxq = (1 << (wbits - 1)) - 1
    z = 1 << (wbits - 1)
    for k, _ in (workloads.small(), workloads.channel_outliers(shape=(1, 128, 8, 128))):
        x = _np16(k)
        B, S, H, D = x.shape
        kc, ks, _, _ = _quant_contig(oracle_mod, x, x, wbits, B, 0, S)
        xf = x.view(np.float16).astype(np.float32).reshape(-1, 32)
        a = np.abs(xf).max(axis=1)
        s16 = (a / np.float32(maxq)).astype(np.float16)
        s32 = s16.astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.rint(xf / s32[:, None])
        codes = np.where(s32[:, None] == 0, z, np.clip(q + z, 0, (1 << wbits) - 1)).astype(np.uint8)
        assert np.array_equal(ks.reshape(-1), s16.view(np.uint16))
        got = np.stack([oracle_mod.unpack_row(r, D, wbits) for r in kc.reshape(-1, D * wbits // 8)])
        assert np.array_equal(got.reshape(-1, 32), codes)


def test_fp8_kv_contiguous_matches_single_tensor(oracle_mod):
    k, v = workloads.fp8_window(shape=(3, 64, 2, 64))
    k, v = _np16(k), _np16(v)
    k8, v8 = np.full(k.shape, SENT8, np.uint8), np.full(v.shape, SENT8, np.uint8)
    assert oracle_mod.fp16_to_fp8_kv(k, k8, v, v8, 2, 7, 40) == oracle_mod.OK
    r8 = np.full(k.shape, SENT8, np.uint8)
    assert oracle_mod.fp16_to_fp8(k, r8, 2, 7, 40) == oracle_mod.OK
    assert np.array_equal(k8, r8)
    r8v = np.full(v.shape, SENT8, np.uint8)
    assert oracle_mod.fp16_to_fp8(v, r8v, 2, 7, 40) == oracle_mod.OK
    assert np.array_equal(v8, r8v)
    ky, vy = np.full(k.shape, SENT16, np.uint16), np.full(v.shape, SENT16, np.uint16)
    assert oracle_mod.fp8_to_fp16_kv(k8, ky, v8, vy, 2, 7, 40) == oracle_mod.OK
    ry = np.full(k.shape, SENT16, np.uint16)
    assert oracle_mod.fp8_to_fp16(k8, ry, 2, 7, 40) == oracle_mod.OK
    assert np.array_equal(ky, ry)


@pytest.mark.parametrize("offset,width", [(0, 1), (-40, 40), (-1000, 17)])
def test_fp8_kv_paged_identity_and_rows(oracle_mod, offset, width):
    # identity block table: paged == contiguous
    B, S, H, D, ps = 3, 96, 2, 32, 32
    k, v = workloads.fp8_window(shape=(B, S, H, D))
    k, v = _np16(k), _np16(v)
    bt = workloads.identity_block_table(B, S, ps).numpy()
    pages = (B * S // ps, ps, H, D)
    c_k = np.full(k.shape, SENT8, np.uint8)
    c_v = np.full(v.shape, SENT8, np.uint8)
    assert oracle_mod.fp16_to_fp8_kv(k, c_k, v, c_v, B, 20, 50) == oracle_mod.OK
    p_k = np.full(pages, SENT8, np.uint8)
    p_v = np.full(pages, SENT8, np.uint8)
    assert oracle_mod.fp16_to_fp8_kv(k.reshape(pages), p_k, v.reshape(pages), p_v, B, 20, 50, ps,
                                     np.zeros(B, np.int32), bt) == oracle_mod.OK
    assert np.array_equal(c_k.reshape(-1), p_k.reshape(-1)) and np.array_equal(c_v.reshape(-1), p_v.reshape(-1))
    # shuffled pool: exactly the window rows are written
    ps, npages, batch = 16, 40, 5
    lens, bt = workloads.paged_tables(3, batch, 60, npages, ps)
    lens, bt = lens.numpy(), bt.numpy()
    k, v = workloads.fp8_window(shape=(npages, ps, H, D))
    k, v = _np16(k), _np16(v)
    ko, vo = np.full(k.shape, SENT8, np.uint8), np.full(v.shape, SENT8, np.uint8)
    assert oracle_mod.fp16_to_fp8_kv(k, ko, v, vo, batch, offset, width, ps, lens, bt) == oracle_mod.OK
    rows = _expected_rows_paged(lens, bt, ps, batch, offset, width)
    flat = ko.reshape(npages * ps, -1)
    assert {r for r in range(npages * ps) if np.any(flat[r] != SENT8)} == rows
    for r in rows:  # each written row is the element-wise E5M2 encoding
        src = k.reshape(npages * ps, -1)[r]
        assert np.array_equal(flat[r], [oracle_mod.e5m2_encode(int(h)) for h in src])
