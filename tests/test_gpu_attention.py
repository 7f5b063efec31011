"""Decode attention reading the quantized cache (the conversions' consumer) against
the CPU oracle's fp64 attention over the dequantized cache.

Tolerance, from the arithmetic: products q_d * k_d are exact (binary16 x
binary16 in fp32), dot products and sums accumulate in fp32 (relative error a
few 2^-24 per term), softmax weights carry ~22 bits (binary16 high part +
binary16 residual) and exp2f is within 2 ulp; the fp32 result before the final
RN16 is within ~1e-5 of the largest |v| of the exact value, so the binary16
output is within one binary16 ulp of the exact value plus 2^-14 max|v|
(a margin for cancellation when the result is near 0).
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kv_cache_quantization_fp16_b200 as m

    return m


@pytest.fixture(scope="module")
def dev(kvq):
    return torch.device("cuda:0")


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def quantize_on_gpu(kvq, k, v, wbits, dev):
    cs, ss = kvq.q_shapes(tuple(k.shape), wbits)
    kc = torch.zeros(cs, dtype=torch.uint8, device=dev)
    vc = torch.zeros_like(kc)
    ks = torch.zeros(ss, dtype=torch.float16, device=dev)
    vs = torch.zeros_like(ks)
    d0, d1 = k.shape[:2]
    kvq.fp16_to_q_kv(k.to(dev), kc, ks, v.to(dev), vc, vs, d0, 0, d1, 0, None, None, wbits)
    return kc, ks, vc, vs


def check(kvq, oracle_mod, q, kc, ks, vc, vs, lens, wbits, scale, dev, page_size=0, bt=None, heads_subset=None):
    B, NH, D = q.shape
    out = torch.full((B, NH, D), float("nan"), dtype=torch.float16, device=dev)
    ws = torch.full((kvq.attention_workspace_bytes((*kc.shape[:3], D), B, NH, page_size,
                                                   bt.shape[1] if bt is not None else 0),), 0xFF,
                    dtype=torch.uint8, device=dev)
    kvq.decode_attention_q(q.to(dev), kc, ks, vc, vs, out, B, lens.to(dev), wbits, scale, page_size,
                           bt.to(dev) if bt is not None else None, workspace=ws)
    assert kvq.poll_device_error() == 0
    st, ref, ex = oracle_mod.decode_attention_q(u16(q), kc.cpu().numpy(), u16(ks), vc.cpu().numpy(), u16(vs), B, NH,
                                                page_size, lens.numpy(), bt.numpy() if bt is not None else None,
                                                wbits, scale, D)
    assert st == oracle_mod.OK
    got = out.float().cpu().numpy().astype(np.float64)
    assert not np.isnan(got).any()
    # dequantized |v| bound for the absolute margin
    vmax = float(vs.float().abs().max().cpu()) * ((1 << (wbits - 1)))
    tol = np.spacing(np.maximum(np.abs(ex), 2.0 ** -14).astype(np.float16)).astype(np.float64) + 2.0 ** -14 * vmax
    err = np.abs(got - ex)
    bad = np.nonzero(err > tol)
    assert bad[0].size == 0, f"{bad[0].size} outputs off, worst {err.max():.3g} (tol there {tol[bad][0]:.3g})"
    exact16 = (ref == u16(out))
    return err.max(), float(exact16.mean())


@pytest.mark.parametrize("wbits", [4, 6, 8])
@pytest.mark.parametrize("D,H,NH", [(128, 2, 8), (64, 4, 4), (256, 1, 8), (128, 1, 2)])
def test_contiguous(kvq, oracle_mod, dev, wbits, D, H, NH):
    B, S = 3, 600
    k, v = workloads.channel_outliers(shape=(B, S, H, D))
    kc, ks, vc, vs = quantize_on_gpu(kvq, k, v, wbits, dev)
    q = torch.randn(B, NH, D, generator=torch.Generator().manual_seed(100)).half()
    lens = torch.tensor([600, 37, 257], dtype=torch.int32)
    err, same = check(kvq, oracle_mod, q, kc, ks, vc, vs, lens, wbits, 1.0 / math.sqrt(D), dev)
    assert same > 0.9  # nearly every output is the correctly rounded fp64 result


@pytest.mark.parametrize("wbits", [4, 6, 8])
@pytest.mark.parametrize("ps", [256, 16, 7])
def test_paged(kvq, oracle_mod, dev, wbits, ps):
    pool = workloads.paged_pool(num_pages=4000 // ps + 40, page_size=ps, heads=2, head_dim=128, batch=5,
                                max_len=700)
    kc, ks, vc, vs = quantize_on_gpu(kvq, pool.k, pool.v, wbits, dev)
    q = torch.randn(5, 8, 128, generator=torch.Generator().manual_seed(101)).half()
    lens = pool.cache_seqlens.clone()
    lens[0] = 0
    lens[1] = 1
    check(kvq, oracle_mod, q, kc, ks, vc, vs, lens, wbits, 0.088, dev, page_size=ps, bt=pool.block_table)


def test_sharp_and_flat_softmax(kvq, oracle_mod, dev):
    """Large scores (one-hot) and zero scores (mean) exercise the online max / rescale."""
    B, S, H, D, NH = 2, 900, 1, 128, 4
    k, v = workloads.normal_kv((B, S, H, D), 11)
    kc, ks, vc, vs = quantize_on_gpu(kvq, k, v, 6, dev)
    lens = torch.tensor([900, 513], dtype=torch.int32)
    q = torch.randn(B, NH, D, generator=torch.Generator().manual_seed(102)).half() * 4
    check(kvq, oracle_mod, q, kc, ks, vc, vs, lens, 6, 2.0, dev)
    check(kvq, oracle_mod, torch.zeros(B, NH, D).half(), kc, ks, vc, vs, lens, 6, 1.0, dev)


@pytest.mark.parametrize("wbits", [4, 6])
def test_paged_pool_full_size_sampled(kvq, oracle_mod, dev, wbits):
    """The 2048-page pool (32 sequences, lengths up to 16384, 8 kv heads, 32 query heads),
    checked against the oracle on 6 sequences (all heads)."""
    pool = workloads.paged_pool(device=dev)
    kc, ks, vc, vs = quantize_on_gpu(kvq, pool.k, pool.v, wbits, dev)
    NH, D = 32, 128
    q = torch.randn(32, NH, D, generator=torch.Generator().manual_seed(7)).half()
    out = torch.empty(32, NH, D, dtype=torch.float16, device=dev)
    kvq.decode_attention_q(q.to(dev), kc, ks, vc, vs, out, 32, pool.cache_seqlens, wbits, 1.0 / math.sqrt(D), 256,
                           pool.block_table)
    assert kvq.poll_device_error() == 0
    pick = [0, 5, 11, 17, 23, 31]
    lens = pool.cache_seqlens.cpu()[pick].contiguous()
    bt = pool.block_table.cpu()[pick].contiguous()
    st, ref, ex = oracle_mod.decode_attention_q(u16(q[pick]), kc.cpu().numpy(), u16(ks), vc.cpu().numpy(), u16(vs),
                                                len(pick), NH, 256, lens.numpy(), bt.numpy(), wbits,
                                                1.0 / math.sqrt(D), D)
    assert st == oracle_mod.OK
    got = out[pick].float().cpu().numpy().astype(np.float64)
    vmax = float(vs.float().abs().max().cpu()) * (1 << (wbits - 1))
    tol = np.spacing(np.maximum(np.abs(ex), 2.0 ** -14).astype(np.float16)).astype(np.float64) + 2.0 ** -14 * vmax
    assert np.all(np.abs(got - ex) <= tol)


def test_many_short_sequences(kvq, oracle_mod, dev):
    """More sequences than the kernel stages lengths for in shared memory (its lengths
    then come from global memory), lengths 0..150 so that most work items are empty or
    partial, and two 128-position chunks for the longest ones."""
    B, S, H, D, NH = 300, 150, 2, 64, 4
    k, v = workloads.normal_kv((B, S, H, D), 23)
    kc, ks, vc, vs = quantize_on_gpu(kvq, k, v, 4, dev)
    g = torch.Generator().manual_seed(5)
    lens = torch.randint(0, S + 1, (B,), generator=g, dtype=torch.int32)
    lens[:3] = torch.tensor([0, 1, S], dtype=torch.int32)
    q = torch.randn(B, NH, D, generator=g).half()
    check(kvq, oracle_mod, q, kc, ks, vc, vs, lens, 4, 1.0 / math.sqrt(D), dev)


@pytest.mark.parametrize("wbits", [4, 8])
def test_per_warp_items_with_empty_and_short_sequences(kvq, oracle_mod, dev, wbits):
    """A batch with more work-item slots than the GPU holds CTAs, so that every warp walks
    its own items (not the CTA-shared split used for one or two sequences), with empty,
    one-position and chunk-boundary sequence lengths among random ones."""
    B, S, H, D, NH = 48, 600, 8, 64, 16
    k, v = workloads.normal_kv((B, S, H, D), 61)
    kc, ks, vc, vs = quantize_on_gpu(kvq, k, v, wbits, dev)
    g = torch.Generator().manual_seed(62)
    lens = torch.randint(0, S + 1, (B,), generator=g, dtype=torch.int32)
    lens[:6] = torch.tensor([0, 1, 255, 256, 257, S], dtype=torch.int32)
    q = torch.randn(B, NH, D, generator=g).half()
    check(kvq, oracle_mod, q, kc, ks, vc, vs, lens, wbits, 1.0 / math.sqrt(D), dev)


def test_small_batches_long_sequences(kvq, oracle_mod, dev):
    """Batches far too small to give every resident warp a work item: one sequence of up to
    5000 positions, and 8 sequences of up to 8192, over 8 kv heads and 32 query heads."""
    for (B, S, H, D, NH), seed in [((1, 5000, 8, 128, 32), 51), ((8, 8192, 8, 128, 32), 52)]:
        k, v = workloads.normal_kv((B, S, H, D), seed)
        kc, ks, vc, vs = quantize_on_gpu(kvq, k, v, 4, dev)
        g = torch.Generator().manual_seed(seed)
        lens = torch.randint(S // 2, S + 1, (B,), generator=g, dtype=torch.int32)
        q = torch.randn(B, NH, D, generator=g).half()
        check(kvq, oracle_mod, q, kc, ks, vc, vs, lens, 4, 1.0 / math.sqrt(D), dev)


def test_bad_paging_reported(kvq, dev):
    ps, H, D = 16, 1, 64
    k, v = workloads.small(shape=(4, ps, H, D))
    kc, ks, vc, vs = quantize_on_gpu(kvq, k, v, 4, dev)
    bt = torch.tensor([[0, 9]], dtype=torch.int32, device=dev)  # page 9 is outside the 4-page pool
    lens = torch.tensor([30], dtype=torch.int32, device=dev)
    out = torch.empty(1, 2, D, dtype=torch.float16, device=dev)
    assert kvq.poll_device_error() == 0
    q = torch.randn(1, 2, D, generator=torch.Generator().manual_seed(103)).half().to(dev)
    kvq.decode_attention_q(q, kc, ks, vc, vs, out, 1, lens, 4, 0.1, ps, bt)
    assert kvq.poll_device_error() != 0
    assert not torch.isnan(out.float()).any()


# ---- decode attention over an FP8 (E5M2) cache -------------------------------------------

def fp8_on_gpu(kvq, k, v, dev):
    d0, d1 = k.shape[:2]
    k8 = torch.zeros(k.shape, dtype=torch.uint8, device=dev)
    v8 = torch.zeros_like(k8)
    kvq.fp16_to_fp8_kv(k.to(dev), k8, v.to(dev), v8, d0, 0, d1)
    return k8, v8


def check_fp8(kvq, oracle_mod, q, k8, v8, lens, scale, dev, page_size=0, bt=None, pick=None):
    B, NH, D = q.shape
    out = torch.full((B, NH, D), float("nan"), dtype=torch.float16, device=dev)
    kvq.decode_attention_fp8(q.to(dev), k8, v8, out, B, lens.to(dev), scale, page_size,
                             bt.to(dev) if bt is not None else None)
    assert kvq.poll_device_error() == 0
    rows = list(range(B)) if pick is None else pick
    qs = q[rows].contiguous()
    ls = lens.cpu()[rows].contiguous()
    bts = bt.cpu()[rows].contiguous() if bt is not None else None
    st, ref, ex = oracle_mod.decode_attention_fp8(u16(qs), k8.cpu().numpy(), v8.cpu().numpy(), len(rows), NH,
                                                  page_size, ls.numpy(), bts.numpy() if bts is not None else None,
                                                  scale)
    assert st == oracle_mod.OK
    got = out[rows].float().cpu().numpy().astype(np.float64)
    assert not np.isnan(got).any()
    vals = np.abs((v8.cpu().numpy().astype(np.uint16) << 8).view(np.float16).astype(np.float64))
    vmax = float(vals[np.isfinite(vals)].max())  # finite values only: bytes past a window may hold NaN
    tol = np.spacing(np.maximum(np.abs(ex), 2.0 ** -14).astype(np.float16)).astype(np.float64) + 2.0 ** -14 * vmax
    err = np.abs(got - ex)
    bad = np.nonzero(err > tol)
    assert bad[0].size == 0, f"{bad[0].size} outputs off, worst {err.max():.3g} (tol there {tol[bad][0]:.3g})"
    return float((ref == u16(out[rows])).mean())


@pytest.mark.parametrize("D,H,NH", [(128, 2, 8), (64, 4, 4), (256, 1, 8), (128, 1, 2)])
def test_fp8_contiguous(kvq, oracle_mod, dev, D, H, NH):
    B, S = 3, 600
    k, v = workloads.fp8_window(shape=(B, S, H, D))  # N(0,1) with outliers and subnormals
    k8, v8 = fp8_on_gpu(kvq, k, v, dev)
    q = torch.randn(B, NH, D, generator=torch.Generator().manual_seed(104)).half()
    lens = torch.tensor([600, 37, 257], dtype=torch.int32)
    same = check_fp8(kvq, oracle_mod, q, k8, v8, lens, 1.0 / math.sqrt(D), dev)
    assert same > 0.9


@pytest.mark.parametrize("ps", [256, 16, 7])
def test_fp8_paged(kvq, oracle_mod, dev, ps):
    pool = workloads.paged_pool(num_pages=4000 // ps + 40, page_size=ps, heads=2, head_dim=128, batch=5,
                                max_len=700)
    k8, v8 = fp8_on_gpu(kvq, pool.k, pool.v, dev)
    q = torch.randn(5, 8, 128, generator=torch.Generator().manual_seed(105)).half()
    lens = pool.cache_seqlens.clone()
    lens[0], lens[1] = 0, 1
    check_fp8(kvq, oracle_mod, q, k8, v8, lens, 0.088, dev, page_size=ps, bt=pool.block_table)


def test_fp8_paged_pool_full_size_sampled(kvq, oracle_mod, dev):
    """The 2048-page pool (32 sequences up to 16384 positions, 8 kv heads, 32 query heads) in
    E5M2, checked against the oracle on 6 sequences (all heads)."""
    pool = workloads.paged_pool(device=dev)
    k8, v8 = fp8_on_gpu(kvq, pool.k, pool.v, dev)
    q = torch.randn(32, 32, 128, generator=torch.Generator().manual_seed(8)).half()
    check_fp8(kvq, oracle_mod, q, k8, v8, pool.cache_seqlens.cpu(), 1.0 / math.sqrt(128), dev, page_size=256,
              bt=pool.block_table.cpu(), pick=[0, 5, 11, 17, 23, 31])


def test_fp8_stale_nan_bytes_do_not_leak(kvq, oracle_mod, dev):
    """Positions past a sequence's length whose bytes are NaN patterns get weight 0 and must
    not turn the output into NaN (the kernel zeroes value rows without data)."""
    B, S, H, D, NH = 2, 96, 1, 64, 2
    k, v = workloads.normal_kv((B, S, H, D), 31)
    k8, v8 = fp8_on_gpu(kvq, k, v, dev)
    k8[:, 40:] = 0x7E  # NaN bytes beyond the attended window
    v8[:, 40:] = 0xFF
    q = torch.randn(B, NH, D, generator=torch.Generator().manual_seed(106)).half()
    check_fp8(kvq, oracle_mod, q, k8, v8, torch.tensor([40, 33], dtype=torch.int32), 0.125, dev)
