"""The load engines (plain loads on the balanced paged grid, plain loads on per-sequence
tiles, and TMA bulk copies) against the CPU oracle, and
against each other, bit for bit: contiguous and paged windows, FP8 and Q4/Q6,
ragged tails, shapes where the bulk engine is not applicable (it then runs the
plain-load engine), and the empty-window no-op."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads
from test_gpu_parity import run_fp8, run_q, u8, u16

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


@pytest.fixture(params=["ldg", "ldg_tiled", "bulk"])
def eng(request, kvq):
    with kvq.engine(request.param):
        yield request.param


def test_engine_switch(kvq):
    assert kvq.get_engine() == "auto"
    with kvq.engine("bulk"):
        assert kvq.get_engine() == "bulk"
    assert kvq.get_engine() == "auto"
    assert kvq.library().kvq_set_engine(7) == 4  # KVQ_ERR_RANGE
    assert kvq.get_engine() == "auto"


def test_fp8_window(kvq, oracle_mod, dev, eng):
    k, _ = workloads.fp8_window(shape=(4, 1024, 8, 128))
    run_fp8(kvq, oracle_mod, k, 4, 100, 801, dev)


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_q_contiguous(kvq, oracle_mod, dev, eng, wbits):
    k, v = workloads.channel_outliers(shape=(2, 512, 8, 128))
    run_q(kvq, oracle_mod, k, v, wbits, 2, 3, 500, dev)


@pytest.mark.parametrize("wbits", [4, 6, 8])
def test_q_paged(kvq, oracle_mod, dev, eng, wbits):
    pool = workloads.paged_pool(num_pages=160, batch=6, max_len=1500, heads=4, head_dim=64)
    for offset, width in ((0, 1), (-300, 300), (-1500, 1501)):
        run_q(kvq, oracle_mod, pool.k, pool.v, wbits, 6, offset, width, dev, page_size=256,
              seqlens=pool.cache_seqlens, bt=pool.block_table)


@pytest.mark.parametrize("shape", [(2, 40, 1, 32), (3, 17, 3, 96), (2, 5, 32, 512)])
def test_ragged_and_fallback_shapes(kvq, oracle_mod, dev, eng, shape):
    """H*D = 32 or 288 make one position of the Q6 / FP8 streams not a multiple of 16 bytes
    (the bulk engine falls back); H*D = 16384 exceeds a bulk stage (falls back too)."""
    k, v = workloads.channel_outliers(shape=shape)
    for wbits in (4, 6, 8):
        run_q(kvq, oracle_mod, k, v, wbits, shape[0], 1, shape[1] - 2, dev)
    run_fp8(kvq, oracle_mod, k, shape[0], 0, shape[1], dev)


def test_engines_agree_at_scale(kvq, dev):
    """Full-size channel-outlier Q4/Q6 both directions: both engines write identical bytes."""
    k, v = workloads.channel_outliers(shape=(4, 8192, 8, 128), device=dev)
    B, S = k.shape[:2]
    for wbits in (4, 6, 8):
        outs = []
        for name in ("ldg", "bulk"):
            with kvq.engine(name):
                cs, ss = kvq.q_shapes(tuple(k.shape), wbits)
                kc = torch.zeros(cs, dtype=torch.uint8, device=dev)
                vc = torch.zeros_like(kc)
                ks = torch.zeros(ss, dtype=torch.float16, device=dev)
                vs = torch.zeros_like(ks)
                kvq.fp16_to_q_kv(k, kc, ks, v, vc, vs, B, 0, S, 0, None, None, wbits)
                ky, vy = torch.zeros_like(k), torch.zeros_like(v)
                kvq.q_to_fp16_kv(kc, ky, ks, vc, vy, vs, B, 0, S, 0, None, None, wbits)
                f8 = torch.zeros(k.shape, dtype=torch.uint8, device=dev)
                kvq.fp16_to_fp8(k, f8, B, 0, S)
                fy = torch.zeros_like(k)
                kvq.fp8_to_fp16(f8, fy, B, 0, S)
                torch.cuda.synchronize()
                outs.append((kc, vc, ks.view(torch.int16), vs.view(torch.int16), ky.view(torch.int16),
                             vy.view(torch.int16), f8, fy.view(torch.int16)))
        for a, b in zip(*outs):
            assert torch.equal(a, b)
    assert kvq.poll_device_error() == 0


def test_balanced_grid_edge_windows(kvq, oracle_mod, dev):
    """The balanced paged grid on windows that are empty, one position long, end exactly
    at page boundaries, or cross several pages, with more sequences than CTAs would take
    one each, and a batch above its shared-memory staging (1100 sequences: the tiled grid
    runs instead); bytes outside the windows stay untouched."""
    for batch, max_len in ((40, 700), (1100, 60)):
        g = torch.Generator().manual_seed(workloads.SEED_BASE + 300 + batch)
        lens = torch.randint(0, max_len + 1, (batch,), generator=g, dtype=torch.int32)
        lens[:6] = torch.tensor([0, 1, 15, 16, 17, max_len], dtype=torch.int32)
        num_pages = batch * ((max_len + 1 + 15) // 16)
        lens, bt = workloads.paged_tables(workloads.SEED_BASE + 301 + batch, batch, max_len, num_pages, 16, lens=lens)
        k, v = workloads.normal_kv((num_pages, 16, 2, 64), workloads.SEED_BASE + 302 + batch)
        for offset, width in ((-64, 64), (-33, 32), (0, 1), (-max_len, max_len)):
            for wbits in (4, 6):
                run_q(kvq, oracle_mod, k, v, wbits, batch, offset, width, dev, page_size=16, seqlens=lens, bt=bt)
            run_fp8_kv(kvq, oracle_mod, k, v, batch, offset, width, dev, page_size=16, seqlens=lens, bt=bt)


def test_balanced_and_tiled_agree_model_layer(kvq, dev):
    """One model-sized paged layer (1024 pages x 256 x 8 x 128, shuffled block table), Q6
    and Q4 both directions and FP8 both directions, on the balanced and the per-sequence
    tiled grids: identical bytes."""
    pool = workloads.model_layer(3, device=dev)
    P, ps, H, D = pool.k.shape
    args = (8, -32768, 32768, ps, pool.cache_seqlens, pool.block_table)
    for wbits in (6, 4):
        outs = []
        for name in ("ldg", "ldg_tiled"):
            with kvq.engine(name):
                cs, ss = kvq.q_shapes(tuple(pool.k.shape), wbits)
                kc, vc = torch.zeros(cs, dtype=torch.uint8, device=dev), torch.zeros(cs, dtype=torch.uint8, device=dev)
                ks = torch.zeros(ss, dtype=torch.float16, device=dev)
                vs = torch.zeros_like(ks)
                kvq.fp16_to_q_kv(pool.k, kc, ks, pool.v, vc, vs, *args, wbits)
                ky, vy = torch.zeros_like(pool.k), torch.zeros_like(pool.v)
                kvq.q_to_fp16_kv(kc, ky, ks, vc, vy, vs, *args, wbits)
                torch.cuda.synchronize()
                outs.append((kc, vc, ks.view(torch.int16), vs.view(torch.int16), ky.view(torch.int16),
                             vy.view(torch.int16)))
        for a, b in zip(*outs):
            assert torch.equal(a, b)
        del outs
    outs = []
    for name in ("ldg", "ldg_tiled"):
        with kvq.engine(name):
            k8, v8 = (torch.zeros(pool.k.shape, dtype=torch.uint8, device=dev) for _ in range(2))
            kvq.fp16_to_fp8_kv(pool.k, k8, pool.v, v8, *args)
            ky, vy = torch.zeros_like(pool.k), torch.zeros_like(pool.v)
            kvq.fp8_to_fp16_kv(k8, ky, v8, vy, *args)
            torch.cuda.synchronize()
            outs.append((k8, v8, ky.view(torch.int16), vy.view(torch.int16)))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    assert kvq.poll_device_error() == 0


def test_bulk_bad_block_table_reports(kvq, oracle_mod, dev):
    ps, H, D, npages = 8, 2, 64, 6
    k, v = workloads.small(shape=(npages, ps, H, D))
    bt = torch.tensor([[0, 7], [1, -1]], dtype=torch.int32)
    lens = torch.tensor([4, 6], dtype=torch.int32)
    cs, ss = kvq.q_shapes(tuple(k.shape), 4)
    kd, vd = k.to(dev), v.to(dev)
    kc, vc = torch.full(cs, 0xA5, dtype=torch.uint8, device=dev), torch.full(cs, 0xA5, dtype=torch.uint8,
                                                                              device=dev)
    ks, vs = torch.zeros(ss, dtype=torch.float16, device=dev), torch.zeros(ss, dtype=torch.float16, device=dev)
    assert kvq.poll_device_error() == 0
    with kvq.engine("bulk"):
        kvq.fp16_to_q_kv(kd, kc, ks, vd, vc, vs, 2, 0, 8, ps, lens.to(dev), bt.to(dev), 4)
    assert kvq.poll_device_error() in (1, 2)
    rc = np.full(cs, 0xA5, np.uint8)
    rs = np.zeros(ss, np.uint16)
    oracle_mod.fp16_to_q_kv(u16(k), rc, rs, u16(v), rc.copy(), rs.copy(), 2, 0, 8, ps, lens.numpy(), bt.numpy(), 4)
    assert np.array_equal(u8(kc), rc)


def run_fp8_kv(kvq, oracle_mod, k, v, batch, offset, width, dev, page_size=0, seqlens=None, bt=None):
    """Fused K+V FP8 encode then decode on the GPU and in the oracle, sentinel-filled buffers."""
    kd, vd = k.to(dev), v.to(dev)
    k8 = torch.full(k.shape, 0xA5, dtype=torch.uint8, device=dev)
    v8 = torch.full(k.shape, 0xA5, dtype=torch.uint8, device=dev)
    sl = seqlens.to(dev) if seqlens is not None else None
    btd = bt.to(dev) if bt is not None else None
    kvq.fp16_to_fp8_kv(kd, k8, vd, v8, batch, offset, width, page_size, sl, btd)
    ky = torch.full(k.shape, 0xA5A5 - 65536, dtype=torch.int16, device=dev).view(torch.float16)
    vy = ky.clone()
    kvq.fp8_to_fp16_kv(k8, ky, v8, vy, batch, offset, width, page_size, sl, btd)
    assert kvq.poll_device_error() == 0
    rk8, rv8 = np.full(k.shape, 0xA5, np.uint8), np.full(k.shape, 0xA5, np.uint8)
    sln = seqlens.numpy() if seqlens is not None else None
    btn = bt.numpy() if bt is not None else None
    assert oracle_mod.fp16_to_fp8_kv(u16(k), rk8, u16(v), rv8, batch, offset, width, page_size, sln, btn) == 0
    rky, rvy = np.full(k.shape, 0xA5A5, np.uint16), np.full(k.shape, 0xA5A5, np.uint16)
    assert oracle_mod.fp8_to_fp16_kv(rk8, rky, rv8, rvy, batch, offset, width, page_size, sln, btn) == 0
    assert np.array_equal(u8(k8), rk8) and np.array_equal(u8(v8), rv8)
    assert np.array_equal(u16(ky), rky) and np.array_equal(u16(vy), rvy)


def test_fp8_kv_contiguous_window(kvq, oracle_mod, dev, eng):
    k, v = workloads.fp8_window(shape=(4, 1024, 8, 128))
    run_fp8_kv(kvq, oracle_mod, k, v, 4, 100, 801, dev)


def test_fp8_kv_paged(kvq, oracle_mod, dev, eng):
    pool = workloads.paged_pool(num_pages=160, batch=6, max_len=1500, heads=4, head_dim=64)
    for offset, width in ((0, 1), (-300, 300), (-1500, 1501)):
        run_fp8_kv(kvq, oracle_mod, pool.k, pool.v, 6, offset, width, dev, page_size=256,
                   seqlens=pool.cache_seqlens, bt=pool.block_table)


@pytest.mark.parametrize("ps", [16, 7])
def test_fp8_kv_paged_identity_equals_contiguous(kvq, oracle_mod, dev, eng, ps):
    B, H, D = 3, 2, 24
    S = ps * 6
    k, v = workloads.fp8_window(shape=(B, S, H, D))
    bt = workloads.identity_block_table(B, S, ps)
    run_fp8_kv(kvq, oracle_mod, k, v, B, 5, S - 9, dev)
    pages = (B * S // ps, ps, H, D)
    run_fp8_kv(kvq, oracle_mod, k.reshape(pages), v.reshape(pages), B, 5, S - 9, dev, page_size=ps,
               seqlens=torch.zeros(B, dtype=torch.int32), bt=bt)


def test_fp8_kv_bad_block_table(kvq, dev, eng):
    ps, H, D, npages = 8, 1, 32, 6
    k, v = workloads.small(shape=(npages, ps, H, D))
    bt = torch.tensor([[0, 7], [1, -1]], dtype=torch.int32, device=dev)
    lens = torch.tensor([4, 6], dtype=torch.int32, device=dev)
    kd, vd = k.to(dev), v.to(dev)
    k8, v8 = torch.zeros(k.shape, dtype=torch.uint8, device=dev), torch.zeros(k.shape, dtype=torch.uint8, device=dev)
    assert kvq.poll_device_error() == 0
    kvq.fp16_to_fp8_kv(kd, k8, vd, v8, 2, 0, 8, ps, lens, bt)
    assert kvq.poll_device_error() in (1, 2)


def test_bounded_wait_gives_up_and_context_stays_usable(kvq, oracle_mod, dev):
    """The bulk engine's bounded pipeline wait, run against an mbarrier that nothing
    arrives on, gives up after its 1 s limit and records KVQ_DEV_TIMEOUT (no fault, no
    hang); the bulk engine then still converts bit-exactly."""
    import time

    assert kvq.poll_device_error() == 0
    t0 = time.perf_counter()
    assert kvq.selfcheck_wait_timeout() == 1
    assert time.perf_counter() - t0 >= 0.9
    assert kvq.poll_device_error() == 3  # KVQ_DEV_TIMEOUT
    assert kvq.poll_device_error() == 0  # read and cleared
    with kvq.engine("bulk"):
        k, v = workloads.channel_outliers(shape=(2, 512, 8, 128))
        run_q(kvq, oracle_mod, k, v, 4, 2, 3, 500, dev)
