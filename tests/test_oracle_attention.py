"""Pins for the oracle's decode attention over a quantized (Q4/Q6/Q8) or FP8 (E5M2) cache
(the consumer the page's Usage section names: conversions "during the attention forward
pass").

* one position: the output is that position's dequantized value exactly;
* zero query: every score is 0, the output is the mean of the values;
* two positions with scores 0 and ln 3: weights 1/4 and 3/4 (closed form);
* a dominant score: the output is that position's value (one-hot softmax);
* paged == contiguous for the same logical cache, and invariance to the
  physical page order;
* GQA: equal queries in one group give equal outputs;
* agreement with numpy's exp / sum over the cache the pinned q_to_fp16_kv
  dequantizes (library routines for the softmax and the weighted sum).
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import workloads


def _np16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def _quantize(oracle_mod, k, v, wbits):
    d0, d1, H, D = k.shape
    kc = np.zeros((d0, d1, H, D * wbits // 8), np.uint8)
    vc = np.zeros_like(kc)
    ks = np.zeros((d0, d1, H, D // 32), np.uint16)
    vs = np.zeros_like(ks)
    assert oracle_mod.fp16_to_q_kv(k, kc, ks, v, vc, vs, d0, 0, d1, 0, None, None, wbits) == oracle_mod.OK
    return kc, ks, vc, vs


def _dequant(oracle_mod, kc, ks, vc, vs, wbits, D):
    d0, d1, H, _ = kc.shape
    ky = np.zeros((d0, d1, H, D), np.uint16)
    vy = np.zeros_like(ky)
    assert oracle_mod.q_to_fp16_kv(kc, ky, ks, vc, vy, vs, d0, 0, d1, 0, None, None, wbits) == oracle_mod.OK
    return ky.view(np.float16).astype(np.float64), vy.view(np.float16).astype(np.float64)


def _rand_cache(B, S, H, D, seed):
    k, v = workloads.normal_kv((B, S, H, D), seed)
    return _np16(k), _np16(v)


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_single_position_returns_value(oracle_mod, wbits):
    B, S, H, D, NH = 2, 4, 2, 64, 4
    k, v = _rand_cache(B, S, H, D, 1)
    kc, ks, vc, vs = _quantize(oracle_mod, k, v, wbits)
    _, vy = _dequant(oracle_mod, kc, ks, vc, vs, wbits, D)
    q = _np16(torch.randn(B, NH, D, generator=torch.Generator().manual_seed(200)).half())
    st, out, ex = oracle_mod.decode_attention_q(q, kc, ks, vc, vs, B, NH, 0, np.array([1, 1], np.int32), None,
                                                wbits, 0.125, D)
    assert st == oracle_mod.OK
    for i in range(B):
        for h in range(NH):
            assert np.array_equal(ex[i, h], vy[i, 0, h // 2])


def test_zero_query_is_the_mean(oracle_mod):
    B, S, H, D, NH, wbits = 1, 37, 1, 32, 1, 6
    k, v = _rand_cache(B, S, H, D, 2)
    kc, ks, vc, vs = _quantize(oracle_mod, k, v, wbits)
    _, vy = _dequant(oracle_mod, kc, ks, vc, vs, wbits, D)
    q = np.zeros((B, NH, D), np.uint16)
    st, out, ex = oracle_mod.decode_attention_q(q, kc, ks, vc, vs, B, NH, 0, np.array([S], np.int32), None,
                                                wbits, 1.0, D)
    assert st == oracle_mod.OK
    assert np.allclose(ex[0, 0], vy[0, :, 0].mean(axis=0), rtol=1e-13, atol=1e-15)


def test_two_positions_closed_form(oracle_mod):
    """k_0 = 0 (all-zero block -> codes z -> 0), k_1 has k_1[0] = 1 exactly; q = e_0 and
    scale ln 3 give scores 0 and ln 3, so the weights are exactly 1/4 and 3/4."""
    D, wbits = 32, 4
    k = np.zeros((1, 2, 1, D), np.float16)
    k[0, 1, 0, 0] = 7.0  # absmax 7 -> s = 1, code 15 -> 7; scale below divides by 7
    v = _np16(torch.randn(1, 2, 1, D, generator=torch.Generator().manual_seed(201)).half())
    kc, ks, vc, vs = _quantize(oracle_mod, k.view(np.uint16), v, wbits)
    _, vy = _dequant(oracle_mod, kc, ks, vc, vs, wbits, D)
    q = np.zeros((1, 1, D), np.float16)
    q[0, 0, 0] = 1.0
    st, out, ex = oracle_mod.decode_attention_q(q.view(np.uint16), kc, ks, vc, vs, 1, 1, 0, np.array([2], np.int32),
                                                None, wbits, math.log(3.0) / 7.0, D)
    assert st == oracle_mod.OK
    assert np.allclose(ex[0, 0], 0.25 * vy[0, 0, 0] + 0.75 * vy[0, 1, 0], rtol=1e-13, atol=1e-15)


def test_dominant_score_is_one_hot(oracle_mod):
    B, S, H, D, NH, wbits = 1, 20, 1, 64, 1, 8
    k, v = _rand_cache(B, S, H, D, 3)
    kc, ks, vc, vs = _quantize(oracle_mod, k, v, wbits)
    ky, vy = _dequant(oracle_mod, kc, ks, vc, vs, wbits, D)
    j = 13
    q = (ky[0, j, 0] / np.linalg.norm(ky[0, j, 0])).astype(np.float16)[None, None, :]
    st, out, ex = oracle_mod.decode_attention_q(q.view(np.uint16), kc, ks, vc, vs, B, NH, 0,
                                                np.array([S], np.int32), None, wbits, 1e4, D)
    assert st == oracle_mod.OK
    assert np.array_equal(out[0, 0], vy[0, j, 0].astype(np.float16).view(np.uint16))


@pytest.mark.parametrize("wbits", [4, 6])
def test_paged_equals_contiguous_and_page_order(oracle_mod, wbits):
    B, S, H, D, NH, ps = 3, 64, 2, 64, 8, 16
    k, v = _rand_cache(B, S, H, D, 4)
    kc, ks, vc, vs = _quantize(oracle_mod, k, v, wbits)
    lens = np.array([64, 1, 40], np.int32)
    q = _np16(torch.randn(B, NH, D, generator=torch.Generator().manual_seed(202)).half())
    st, out_c, ex_c = oracle_mod.decode_attention_q(q, kc, ks, vc, vs, B, NH, 0, lens, None, wbits, 0.125, D)
    assert st == oracle_mod.OK
    pages = (B * S // ps, ps, H)
    ident = workloads.identity_block_table(B, S, ps).numpy()
    st, out_p, ex_p = oracle_mod.decode_attention_q(q, kc.reshape(*pages, -1), ks.reshape(*pages, -1),
                                                    vc.reshape(*pages, -1), vs.reshape(*pages, -1), B, NH, ps,
                                                    lens, ident, wbits, 0.125, D)
    assert st == oracle_mod.OK and np.array_equal(out_c, out_p) and np.array_equal(ex_c, ex_p)
    # move the pages to other physical slots: same logical cache, same result
    perm = np.random.default_rng(0).permutation(pages[0])
    def mv(a):
        a = a.reshape(*pages, -1)
        b = np.empty_like(a)
        b[perm] = a
        return b
    bt = perm[ident].astype(np.int32)
    st, out_m, ex_m = oracle_mod.decode_attention_q(q, mv(kc), mv(ks), mv(vc), mv(vs), B, NH, ps, lens, bt, wbits,
                                                    0.125, D)
    assert st == oracle_mod.OK and np.array_equal(out_m, out_c)


def test_gqa_groups(oracle_mod):
    B, S, H, D, NH, wbits = 1, 30, 2, 32, 6, 4
    k, v = _rand_cache(B, S, H, D, 5)
    kc, ks, vc, vs = _quantize(oracle_mod, k, v, wbits)
    q = _np16(torch.randn(B, NH, D, generator=torch.Generator().manual_seed(203)).half())
    q[0, 1] = q[0, 0]
    q[0, 3] = q[0, 0]  # head 3 is in the second group (kv head 1)
    st, out, ex = oracle_mod.decode_attention_q(q, kc, ks, vc, vs, B, NH, 0, np.array([S], np.int32), None,
                                                wbits, 0.2, D)
    assert st == oracle_mod.OK
    assert np.array_equal(out[0, 0], out[0, 1])
    assert not np.array_equal(out[0, 0], out[0, 3])


@pytest.mark.parametrize("wbits", [4, 6, 8])
@pytest.mark.parametrize("D,NH", [(64, 2), (128, 4), (256, 16)])
def test_matches_numpy_softmax(oracle_mod, wbits, D, NH):
    B, S, H = 2, 50, 2
    k, v = _rand_cache(B, S, H, D, 6)
    kc, ks, vc, vs = _quantize(oracle_mod, k, v, wbits)
    ky, vy = _dequant(oracle_mod, kc, ks, vc, vs, wbits, D)
    q16 = torch.randn(B, NH, D, generator=torch.Generator().manual_seed(204)).half()
    q = _np16(q16)
    qf = q16.double().numpy()
    lens = np.array([50, 17], np.int32)
    st, out, ex = oracle_mod.decode_attention_q(q, kc, ks, vc, vs, B, NH, 0, lens, None, wbits, 0.0883883, D)
    assert st == oracle_mod.OK
    group = NH // H
    for i in range(B):
        for h in range(NH):
            kk, vv = ky[i, : lens[i], h // group], vy[i, : lens[i], h // group]
            sc = 0.0883883 * kk @ qf[i, h]
            w = np.exp(sc - sc.max())
            ref = (w / w.sum()) @ vv
            assert np.allclose(ex[i, h], ref, rtol=1e-12, atol=1e-14)
    # the binary16 outputs are the exact results rounded to nearest even
    assert np.array_equal(out, ex.astype(np.float16).view(np.uint16))


def test_empty_window_and_bad_args(oracle_mod):
    D = 32
    kc = np.zeros((1, 4, 2, 16), np.uint8)
    ks = np.zeros((1, 4, 2, 1), np.uint16)
    q = np.zeros((1, 2, D), np.uint16)
    st, out, ex = oracle_mod.decode_attention_q(q, kc, ks, kc, ks, 1, 2, 0, np.array([0], np.int32), None, 4, 1.0, D)
    assert st == oracle_mod.OK and not out.any()
    q3 = np.zeros((1, 3, D), np.uint16)
    st, _, _ = oracle_mod.decode_attention_q(q3, kc, ks, kc, ks, 1, 3, 0, np.array([2], np.int32), None, 4, 1.0, D)
    assert st == oracle_mod.BAD_ARG  # 3 query heads do not split over 2 kv heads
    st, _, _ = oracle_mod.decode_attention_q(q, kc, ks, kc, ks, 1, 2, 0, np.array([5], np.int32), None, 4, 1.0, D)
    assert st == oracle_mod.BAD_ARG  # window longer than the cache


# ---- decode attention over an FP8 (E5M2) cache -------------------------------------------

def _e5m2_numpy(b: np.ndarray) -> np.ndarray:
    """E5M2 bytes to float64 without the oracle: the byte is the high byte of a binary16."""
    return (b.astype(np.uint16) << 8).view(np.float16).astype(np.float64)


def _fp8_cache(B, S, H, D, seed):
    """Random E5M2 bytes drawn directly (independent of the oracle's encoder): random sign and
    mantissa bits, exponent field in [9, 17], so magnitudes lie in [2^-6, 7] and no byte is
    Inf or NaN."""
    g = np.random.default_rng(seed)
    def draw():
        b = g.integers(0, 256, (B, S, H, D), dtype=np.uint8)
        e = g.integers(9, 18, (B, S, H, D), dtype=np.uint8)
        return ((b & 0x83) | (e << 2)).astype(np.uint8)
    return draw(), draw()


def test_fp8_single_position_returns_value(oracle_mod):
    B, S, H, D, NH = 2, 3, 2, 64, 4
    k8, v8 = _fp8_cache(B, S, H, D, 11)
    q = _np16(torch.randn(B, NH, D, generator=torch.Generator().manual_seed(205)).half())
    st, out, ex = oracle_mod.decode_attention_fp8(q, k8, v8, B, NH, 0, np.array([1, 1], np.int32), None, 0.125)
    assert st == oracle_mod.OK
    vv = _e5m2_numpy(v8)
    for i in range(B):
        for h in range(NH):
            assert np.array_equal(ex[i, h], vv[i, 0, h // 2])
            assert np.array_equal(out[i, h], (v8[i, 0, h // 2].astype(np.uint16) << 8))


def test_fp8_zero_query_is_the_mean(oracle_mod):
    B, S, H, D, NH = 1, 29, 1, 32, 2
    k8, v8 = _fp8_cache(B, S, H, D, 12)
    q = np.zeros((B, NH, D), np.uint16)
    st, out, ex = oracle_mod.decode_attention_fp8(q, k8, v8, B, NH, 0, np.array([S], np.int32), None, 1.0)
    assert st == oracle_mod.OK
    assert np.allclose(ex[0, 0], _e5m2_numpy(v8)[0, :, 0].mean(axis=0), rtol=1e-13, atol=1e-15)


def test_fp8_two_positions_closed_form(oracle_mod):
    """k_0 = 0 and k_1[0] = 2 (byte 0x40); q = e_0 and scale ln 3 / 2 give scores 0 and ln 3, so
    the weights are exactly 1/4 and 3/4; v_0 = 1 (0x3C), v_1 = 2 (0x40) everywhere makes the
    output exactly 1/4 + 3/2 = 1.75."""
    D = 16
    k8 = np.zeros((1, 2, 1, D), np.uint8)
    k8[0, 1, 0, 0] = 0x40
    v8 = np.zeros((1, 2, 1, D), np.uint8)
    v8[0, 0], v8[0, 1] = 0x3C, 0x40
    q = np.zeros((1, 1, D), np.float16)
    q[0, 0, 0] = 1.0
    st, out, ex = oracle_mod.decode_attention_fp8(q.view(np.uint16), k8, v8, 1, 1, 0, np.array([2], np.int32), None,
                                                  math.log(3.0) / 2.0)
    assert st == oracle_mod.OK
    assert np.allclose(ex[0, 0], 1.75, rtol=1e-14, atol=0)
    assert np.all(out[0, 0] == np.float16(1.75).view(np.uint16))


@pytest.mark.parametrize("D,NH", [(64, 8), (128, 2), (256, 16)])
def test_fp8_paged_equals_contiguous_and_matches_numpy(oracle_mod, D, NH):
    B, S, H, ps = 3, 64, 2, 16
    k8, v8 = _fp8_cache(B, S, H, D, 13)
    lens = np.array([64, 1, 40], np.int32)
    q16 = torch.randn(B, NH, D, generator=torch.Generator().manual_seed(206)).half()
    q = _np16(q16)
    st, out_c, ex_c = oracle_mod.decode_attention_fp8(q, k8, v8, B, NH, 0, lens, None, 0.125)
    assert st == oracle_mod.OK
    pages = (B * S // ps, ps, H, D)
    ident = workloads.identity_block_table(B, S, ps).numpy()
    st, out_p, ex_p = oracle_mod.decode_attention_fp8(q, k8.reshape(pages), v8.reshape(pages), B, NH, ps, lens,
                                                      ident, 0.125)
    assert st == oracle_mod.OK and np.array_equal(out_c, out_p) and np.array_equal(ex_c, ex_p)
    perm = np.random.default_rng(1).permutation(pages[0])
    kp, vp = np.empty_like(k8.reshape(pages)), np.empty_like(v8.reshape(pages))
    kp[perm], vp[perm] = k8.reshape(pages), v8.reshape(pages)
    st, out_m, _ = oracle_mod.decode_attention_fp8(q, kp, vp, B, NH, ps, lens, perm[ident].astype(np.int32), 0.125)
    assert st == oracle_mod.OK and np.array_equal(out_m, out_c)
    # numpy restatement: decode, softmax, weighted sum
    kk, vv, qf = _e5m2_numpy(k8), _e5m2_numpy(v8), q16.double().numpy()
    group = NH // H
    for i in range(B):
        for h in range(NH):
            sc = 0.125 * kk[i, : lens[i], h // group] @ qf[i, h]
            w = np.exp(sc - sc.max())
            assert np.allclose(ex_c[i, h], (w / w.sum()) @ vv[i, : lens[i], h // group], rtol=1e-12, atol=1e-14)
    assert np.array_equal(out_c, ex_c.astype(np.float16).view(np.uint16))


def test_fp8_bad_args(oracle_mod):
    k8 = np.zeros((1, 4, 2, 16), np.uint8)
    q3 = np.zeros((1, 3, 16), np.uint16)
    st, _, _ = oracle_mod.decode_attention_fp8(q3, k8, k8, 1, 3, 0, np.array([2], np.int32), None, 1.0)
    assert st == oracle_mod.BAD_ARG  # 3 query heads do not split over 2 kv heads
    q = np.zeros((1, 2, 16), np.uint16)
    st, _, _ = oracle_mod.decode_attention_fp8(q, k8, k8, 1, 2, 0, np.array([5], np.int32), None, 1.0)
    assert st == oracle_mod.BAD_ARG  # window longer than the cache
