"""GPU parity: the CUDA path through the C ABI against the CPU oracle, bit for bit.

Every comparison is exact (0 ULP): codes, scales, E5M2 bytes and FP16 outputs.
Output buffers are pre-filled with a sentinel on both sides, so comparing the
whole buffers also checks that nothing outside the window was written.

Workloads follow the KV-cache conversion workloads (seeded recipes in
``workloads``): small Q4 + FP8 round trip, FP8 partial window with outliers
and subnormals, Q4 / Q6 with channel outliers and zero blocks, paged decode +
prefill, and the model-sized paged Q6 layer (sampled at full size).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

SENT8 = 0xA5
SENT16 = 0xA5A5


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kv_cache_quantization_fp16_b200 as m

    return m


@pytest.fixture(scope="module")
def dev(kvq):
    return torch.device("cuda:0")


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy()


def sent_like16(shape, dev):
    return torch.full(shape, SENT16 - 65536, dtype=torch.int16, device=dev).view(torch.float16)


def sent_like8(shape, dev):
    return torch.full(shape, SENT8, dtype=torch.uint8, device=dev)


# ----------------------------------------------------------------- helpers ----

def run_fp8(kvq, oracle_mod, x: torch.Tensor, batch, offset, width, dev):
    """Encode + decode on GPU and in the oracle; assert bitwise equality."""
    xd = x.to(dev)
    f8 = sent_like8(x.shape, dev)
    back = sent_like16(x.shape, dev)
    kvq.fp16_to_fp8(xd, f8, batch, offset, width)
    kvq.fp8_to_fp16(f8, back, batch, offset, width)
    torch.cuda.synchronize()
    xn = u16(x)
    r8 = np.full(x.shape, SENT8, np.uint8)
    rb = np.full(x.shape, SENT16, np.uint16)
    assert oracle_mod.fp16_to_fp8(xn, r8, batch, offset, width) == oracle_mod.OK
    assert oracle_mod.fp8_to_fp16(r8, rb, batch, offset, width) == oracle_mod.OK
    g8 = u8(f8)
    bad = np.nonzero(g8 != r8)
    assert bad[0].size == 0, f"{bad[0].size} E5M2 bytes differ, first at {tuple(a[0] for a in bad)}"
    assert np.array_equal(u16(back), rb)


def run_q(kvq, oracle_mod, k, v, wbits, batch, offset, width, dev, page_size=0, seqlens=None, bt=None,
          check_oracle=True):
    """Quantize + dequantize K and V on the GPU (fused launch) and in the oracle."""
    cs, ss = kvq.q_shapes(tuple(k.shape), wbits)
    kd, vd = k.to(dev), v.to(dev)
    kc, vc = sent_like8(cs, dev), sent_like8(cs, dev)
    ks, vs = sent_like16(ss, dev), sent_like16(ss, dev)
    sl = seqlens.to(dev) if seqlens is not None else None
    btd = bt.to(dev) if bt is not None else None
    kvq.fp16_to_q_kv(kd, kc, ks, vd, vc, vs, batch, offset, width, page_size, sl, btd, wbits)
    ky, vy = sent_like16(k.shape, dev), sent_like16(k.shape, dev)
    kvq.q_to_fp16_kv(kc, ky, ks, vc, vy, vs, batch, offset, width, page_size, sl, btd, wbits)
    assert kvq.poll_device_error() == 0
    if not check_oracle:
        return kc, ks, ky
    kn, vn = u16(k), u16(v)
    rkc, rvc = np.full(cs, SENT8, np.uint8), np.full(cs, SENT8, np.uint8)
    rks, rvs = np.full(ss, SENT16, np.uint16), np.full(ss, SENT16, np.uint16)
    sln = seqlens.numpy() if seqlens is not None else None
    btn = bt.numpy() if bt is not None else None
    assert oracle_mod.fp16_to_q_kv(kn, rkc, rks, vn, rvc, rvs, batch, offset, width, page_size, sln, btn,
                                   wbits) == oracle_mod.OK
    rky, rvy = np.full(k.shape, SENT16, np.uint16), np.full(k.shape, SENT16, np.uint16)
    assert oracle_mod.q_to_fp16_kv(rkc, rky, rks, rvc, rvy, rvs, batch, offset, width, page_size, sln, btn,
                                   wbits) == oracle_mod.OK
    for name, g, r in (("K codes", u8(kc), rkc), ("V codes", u8(vc), rvc), ("K scales", u16(ks), rks),
                       ("V scales", u16(vs), rvs), ("K deq", u16(ky), rky), ("V deq", u16(vy), rvy)):
        bad = np.nonzero(g != r)
        assert bad[0].size == 0, f"{name}: {bad[0].size} differ, first at {tuple(a[0] for a in bad)}"
    return kc, ks, ky


# ------------------------------------------------------------ exhaustive ----

def test_fp8_encode_every_fp16(kvq, oracle_mod, dev):
    x = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.float16).reshape(1, 64, 1, 1024)
    run_fp8(kvq, oracle_mod, x, 1, 0, 64, dev)


def test_fp8_decode_every_byte(kvq, oracle_mod, dev):
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8).reshape(1, 4, 8, 8).to(dev)
    out = sent_like16((1, 4, 8, 8), dev)
    kvq.fp8_to_fp16(b, out, 1, 0, 4)
    torch.cuda.synchronize()
    ref = np.array([oracle_mod.e5m2_decode(i) for i in range(256)], np.uint16).reshape(1, 4, 8, 8)
    assert np.array_equal(u16(out), ref)


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_scale_every_absmax(kvq, oracle_mod, dev, wbits):
    """One block per finite binary16 absmax a (block = [a, -a/3, 0, ...] shuffled)."""
    n = 0x7C00
    a = torch.arange(n, dtype=torch.int32).to(torch.int16).view(torch.float16)
    x = torch.zeros(n, 32, dtype=torch.float16)
    x[:, 5] = a
    x[:, 17] = -(a.float() / 3).half()
    x[:, 30] = (a.float() * 0.7).half()
    x = x.reshape(1, n, 1, 32)
    run_q(kvq, oracle_mod, x, x.flip(1).contiguous(), wbits, 1, 0, n, dev)


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_code_rounding_selfcheck(kvq, dev, wbits):
    """The fast code rounding equals IEEE division + rint + clamp for all 2^31 (x, s) pairs."""
    assert kvq.selfcheck_code_rounding(wbits) == 0


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_ties_and_subnormal_scales(kvq, oracle_mod, dev, wbits):
    rng = np.random.default_rng(100 + wbits)
    maxq = (1 << (wbits - 1)) - 1
    blocks = []
    for _ in range(2048):  # exact half-integer multiples of the scale
        e = float(2.0 ** rng.integers(-20, 10))
        x = rng.integers(-2 * maxq, 2 * maxq + 1, 32) * 0.5 * e
        x[rng.integers(0, 32)] = maxq * e * rng.choice([-1, 1])
        blocks.append(x)
    for _ in range(2048):  # subnormal magnitudes
        bits = rng.integers(0, 96, 32) | np.where(rng.random(32) < 0.5, 0x8000, 0)
        blocks.append(bits.astype(np.uint16).view(np.float16).astype(np.float64))
    x = torch.from_numpy(np.array(blocks, np.float64).astype(np.float16)).reshape(1, len(blocks) // 4, 4, 32)
    run_q(kvq, oracle_mod, x, x.roll(7).contiguous(), wbits, 1, 0, x.shape[1], dev)


# ---------------------------------------------------------------- configs ----

def test_small_q4_and_fp8_roundtrip(kvq, oracle_mod, dev):
    """[1, 256, 8, 128] N(0,1): Q4 quantize then dequantize, FP8 E5M2 encode then decode."""
    k, v = workloads.small()
    run_q(kvq, oracle_mod, k, v, 4, 1, 0, 256, dev)
    run_fp8(kvq, oracle_mod, k, 1, 0, 256, dev)
    run_fp8(kvq, oracle_mod, v, 1, 0, 256, dev)


def test_fp8_partial_window_full_size(kvq, oracle_mod, dev):
    """[4, 4096, 8, 128] with 1% outliers and 0.1% subnormals, window 1024..3072."""
    k, v = workloads.fp8_window()
    run_fp8(kvq, oracle_mod, k, 4, 1024, 2048, dev)
    run_fp8(kvq, oracle_mod, v, 4, 1024, 2048, dev)


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_channel_outliers_reduced(kvq, oracle_mod, dev, wbits):
    """Channel-outlier K, N(0, 0.5) V, 2% zero blocks, at [2, 512, 8, 128] (every tile
    boundary and a ragged window), full comparison."""
    k, v = workloads.channel_outliers(shape=(2, 512, 8, 128))
    run_q(kvq, oracle_mod, k, v, wbits, 2, 0, 512, dev)
    run_q(kvq, oracle_mod, k, v, wbits, 2, 37, 301, dev)


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_channel_outliers_full_size_sampled(kvq, oracle_mod, dev, wbits):
    """[16, 8192, 8, 128] on the device; 3000 sampled positions checked against the oracle
    one position at a time."""
    k, v = workloads.channel_outliers(device=dev)
    B, S, H, D = k.shape
    kc, ks, ky = run_q(kvq, oracle_mod, k, v, wbits, B, 0, S, dev, check_oracle=False)
    rng = np.random.default_rng(wbits)
    bs = rng.integers(0, B, 3000)
    ss = rng.integers(0, S, 3000)
    bs[:2], ss[:2] = [0, B - 1], [0, S - 1]
    kn = u16(k[bs, ss])              # [n, H, D]
    gc, gs, gy = u8(kc[bs, ss]), u16(ks[bs, ss]), u16(ky[bs, ss])
    n = len(bs)
    cs, sshape = kvq.q_shapes((n, 1, H, D), wbits)
    rc, rs = np.full(cs, SENT8, np.uint8), np.full(sshape, SENT16, np.uint16)
    x = kn.reshape(n, 1, H, D).copy()
    assert oracle_mod.fp16_to_q_kv(x, rc, rs, x, rc.copy(), rs.copy(), n, 0, 1, 0, None, None, wbits) == 0
    ry = np.full(x.shape, SENT16, np.uint16)
    assert oracle_mod.q_to_fp16_kv(rc, ry, rs, rc, ry.copy(), rs, n, 0, 1, 0, None, None, wbits) == 0
    assert np.array_equal(gc.reshape(rc.shape), rc)
    assert np.array_equal(gs.reshape(rs.shape), rs)
    assert np.array_equal(gy.reshape(ry.shape), ry)
    # property at full size: every all-zero block has scale 0 and dequantizes to +0
    zero = (k.view(torch.int16) & 0x7FFF).reshape(B, S, H, D // 32, 32).amax(-1) == 0
    assert bool((ks.view(torch.int16)[zero] == 0).all())
    assert int(zero.sum()) > 0


@pytest.mark.parametrize("phase", ["decode", "prefill"])
def test_paged_decode_prefill_full_pool(kvq, oracle_mod, dev, phase):
    """2048 pages x 256 x 8 x 128 pools, 32 sequences, shuffled block table; Q4."""
    pool = workloads.paged_pool()
    offset, width = (0, 1) if phase == "decode" else (-512, 512)
    run_q(kvq, oracle_mod, pool.k, pool.v, 4, 32, offset, width, dev, page_size=256,
          seqlens=pool.cache_seqlens, bt=pool.block_table)


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_model_layer_paged_q6_sampled(kvq, oracle_mod, dev, wbits):
    """One 8 x 32768-position layer (1024 pages), full-window dequantize then quantize,
    sampled rows against the oracle; the round trip of a quantized cache is a fixed point."""
    pool = workloads.model_layer(0, device=dev)
    P, ps, H, D = pool.k.shape
    seqs, S = 8, 32768
    kc, ks, ky = run_q(kvq, oracle_mod, pool.k, pool.v, wbits, seqs, -S, S, dev, page_size=ps,
                       seqlens=pool.cache_seqlens, bt=pool.block_table, check_oracle=False)
    # paged full window over a permutation covers every row of the pool exactly once
    assert not bool((ky.view(torch.int16) == SENT16 - 65536).all(-1).any())
    rng = np.random.default_rng(50 + wbits)
    rows = rng.integers(0, P * ps, 2000)
    x = u16(pool.k.reshape(P * ps, H, D)[rows]).reshape(len(rows), 1, H, D).copy()
    cs, sshape = kvq.q_shapes(x.shape, wbits)
    rc, rs = np.zeros(cs, np.uint8), np.zeros(sshape, np.uint16)
    assert oracle_mod.fp16_to_q_kv(x, rc, rs, x, rc.copy(), rs.copy(), len(rows), 0, 1, 0, None, None,
                                   wbits) == 0
    ry = np.zeros(x.shape, np.uint16)
    assert oracle_mod.q_to_fp16_kv(rc, ry, rs, rc, ry.copy(), rs, len(rows), 0, 1, 0, None, None, wbits) == 0
    assert np.array_equal(u8(kc.reshape(P * ps, H, -1)[rows]).reshape(rc.shape), rc)
    assert np.array_equal(u16(ks.reshape(P * ps, H, -1)[rows]).reshape(rs.shape), rs)
    assert np.array_equal(u16(ky.reshape(P * ps, H, D)[rows]).reshape(ry.shape), ry)


# -------------------------------------------------------------- edge cases ----

@pytest.mark.parametrize("shape", [(2, 40, 1, 32), (3, 17, 3, 96), (1, 9, 5, 64), (2, 5, 32, 512)])
@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_ragged_shapes(kvq, oracle_mod, dev, shape, wbits):
    k, v = workloads.channel_outliers(shape=shape)
    B, S = shape[0], shape[1]
    run_q(kvq, oracle_mod, k, v, wbits, B, 1, S - 2, dev)
    run_q(kvq, oracle_mod, k, v, wbits, B - 1 if B > 1 else 1, S - 1, 1, dev)


@pytest.mark.parametrize("shape", [(2, 33, 1, 8), (1, 7, 5, 24), (3, 300, 8, 128)])
def test_fp8_ragged_shapes(kvq, oracle_mod, dev, shape):
    k, _ = workloads.fp8_window(shape=shape)
    run_fp8(kvq, oracle_mod, k, shape[0], 0, shape[1], dev)
    run_fp8(kvq, oracle_mod, k, shape[0], shape[1] - 3, 3, dev)


def test_empty_windows_write_nothing(kvq, dev):
    k, v = workloads.small(shape=(2, 16, 2, 64))
    kd = k.to(dev)
    f8 = sent_like8(k.shape, dev)
    kvq.fp16_to_fp8(kd, f8, 2, 5, 0)
    kvq.fp16_to_fp8(kd, f8, 0, 0, 16)
    cs, ss = kvq.q_shapes(tuple(k.shape), 4)
    kc, ks = sent_like8(cs, dev), sent_like16(ss, dev)
    kvq.fp16_to_q_kv(kd, kc, ks, kd, kc, ks, 2, 3, 0, 0, None, None, 4)
    torch.cuda.synchronize()
    assert bool((f8 == SENT8).all()) and bool((kc == SENT8).all())


@pytest.mark.parametrize("ps", [16, 24, 7, 256])
@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_paged_identity_equals_contiguous(kvq, oracle_mod, dev, ps, wbits):
    B, H, D = 3, 2, 64
    S = ps * 6
    k, v = workloads.small(shape=(B, S, H, D))
    bt = workloads.identity_block_table(B, S, ps)
    offset, width = 5, S - 9
    kc1, ks1, ky1 = run_q(kvq, oracle_mod, k, v, wbits, B, offset, width, dev)
    pages = (B * S // ps, ps, H, D)
    kc2, ks2, ky2 = run_q(kvq, oracle_mod, k.reshape(pages), v.reshape(pages), wbits, B, offset, width, dev,
                          page_size=ps, seqlens=torch.zeros(B, dtype=torch.int32), bt=bt)
    assert torch.equal(kc1.reshape(-1), kc2.reshape(-1))
    assert torch.equal(ks1.view(torch.int16).reshape(-1), ks2.view(torch.int16).reshape(-1))
    assert torch.equal(ky1.view(torch.int16).reshape(-1), ky2.view(torch.int16).reshape(-1))


@pytest.mark.parametrize("offset,width", [(0, 1), (-40, 40), (-5, 6), (-1000, 17), (-3, 3)])
def test_paged_windows_small_pool(kvq, oracle_mod, dev, offset, width):
    ps, H, D, npages, batch = 16, 2, 32, 40, 5
    lens, bt = workloads.paged_tables(3, batch, 60, npages, ps)
    k, v = workloads.small(shape=(npages, ps, H, D))
    for wbits in (4, 6, 8):
        run_q(kvq, oracle_mod, k, v, wbits, batch, offset, width, dev, page_size=ps, seqlens=lens, bt=bt)


def test_bad_block_table_sets_device_error(kvq, oracle_mod, dev):
    ps, H, D, npages = 8, 1, 32, 6
    k, v = workloads.small(shape=(npages, ps, H, D))
    bt = torch.tensor([[0, 7], [1, -1]], dtype=torch.int32)
    lens = torch.tensor([4, 6], dtype=torch.int32)
    cs, ss = kvq.q_shapes(tuple(k.shape), 4)
    kd, vd = k.to(dev), v.to(dev)
    kc, vc = sent_like8(cs, dev), sent_like8(cs, dev)
    ks, vs = sent_like16(ss, dev), sent_like16(ss, dev)
    assert kvq.poll_device_error() == 0
    kvq.fp16_to_q_kv(kd, kc, ks, vd, vc, vs, 2, 0, 8, ps, lens.to(dev), bt.to(dev), 4)
    assert kvq.poll_device_error() in (1, 2)
    assert kvq.poll_device_error() == 0  # cleared by the read
    # the valid positions were written exactly as the oracle writes them
    rc, rs = np.full(cs, SENT8, np.uint8), np.full(ss, SENT16, np.uint16)
    st = oracle_mod.fp16_to_q_kv(u16(k), rc, rs, u16(v), rc.copy(), rs.copy(), 2, 0, 8, ps, lens.numpy(),
                                 bt.numpy(), 4)
    assert st == oracle_mod.BAD_PAGE
    assert np.array_equal(u8(kc), rc) and np.array_equal(u16(ks), rs)
    # a logical page index past the table's width
    kvq.fp16_to_q_kv(kd, kc, ks, vd, vc, vs, 1, 4, 30, ps, lens.to(dev), bt.to(dev), 4)
    assert kvq.poll_device_error() in (1, 2)


def test_runs_on_a_side_stream(kvq, oracle_mod, dev):
    k, v = workloads.small(shape=(2, 64, 4, 128))
    s = torch.cuda.Stream(dev)
    with torch.cuda.stream(s):
        run_q(kvq, oracle_mod, k, v, 6, 2, 0, 64, dev)


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_paged_wide_block_table(kvq, oracle_mod, dev, wbits):
    """A block table wider than a CTA (300 pages per sequence) takes the unstaged lookup."""
    ps, H, D, batch = 2, 1, 32, 2
    lens = torch.tensor([599, 433], dtype=torch.int32)
    lens, bt = workloads.paged_tables(9, batch, 599, 610, ps, lens=lens)
    assert bt.shape[1] == 300
    k, v = workloads.small(shape=(610, ps, H, D))
    run_q(kvq, oracle_mod, k, v, wbits, batch, -500, 501, dev, page_size=ps, seqlens=lens, bt=bt)
