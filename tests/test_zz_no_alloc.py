"""kvq_decode_attention_q_noalloc, the decode attention entry point that takes its
workspace from the library's own scratch array, against kvq_decode_attention_q with a
caller workspace: two calls in a row (different queries, lengths and paging, so a
stale partial result left in the shared array would show).  Both entry points run the
same deterministic kernels (a fixed enumeration of work items and a fixed merge order)
over the same inputs, so their outputs must be identical bit for bit; a difference
would mean a stale or raced workspace entry.  The file sorts last so that it also runs
after every other GPU test; it passes on its own as well."""
from __future__ import annotations

import ctypes

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


def _case(kvq, dev, seed, wbits, page_size):
    B, S, H, D, NH = 4, 1024, 2, 128, 8
    k, v = workloads.normal_kv((B, S, H, D), seed)
    cs, ss = kvq.q_shapes((B, S, H, D), wbits)
    kc, vc = (torch.zeros(cs, dtype=torch.uint8, device=dev) for _ in range(2))
    ks, vs = (torch.zeros(ss, dtype=torch.float16, device=dev) for _ in range(2))
    kvq.fp16_to_q_kv(k.to(dev), kc, ks, v.to(dev), vc, vs, B, 0, S, 0, None, None, wbits)
    g = torch.Generator().manual_seed(workloads.SEED_BASE + seed)
    q = torch.randn(B, NH, D, generator=g).half().to(dev)
    lens = torch.randint(1, S + 1, (B,), generator=g, dtype=torch.int32)
    bt = None
    if page_size:
        pages = (B * S // page_size, page_size, H)
        kc, vc = kc.view(*pages, -1), vc.view(*pages, -1)
        ks, vs = ks.view(*pages, -1), vs.view(*pages, -1)
        bt = workloads.identity_block_table(B, S, page_size).to(dev)
    return q, kc, ks, vc, vs, lens.to(dev), bt


def _noalloc_via_abi(kvq, q, kc, ks, vc, vs, out, lens, wbits, scale, page_size, bt):
    lib = kvq.library()
    B, NH, D = q.shape
    d0, d1, H, _ = kc.shape
    desc = kvq._Desc(d0, d1, H, D, bt.shape[1] if bt is not None else 0)
    return lib.kvq_decode_attention_q_noalloc(q.data_ptr(), kc.data_ptr(), ks.data_ptr(), vc.data_ptr(),
                                              vs.data_ptr(), out.data_ptr(), ctypes.byref(desc), B, NH, page_size,
                                              lens.data_ptr(), bt.data_ptr() if bt is not None else None, wbits,
                                              ctypes.c_float(scale), torch.cuda.current_stream(q.device).cuda_stream)


def test_noalloc_matches_workspace_entry_point(kvq):
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    scale = 128 ** -0.5
    for call, (seed, wbits, page_size) in enumerate(((11, 4, 0), (12, 6, 16))):
        q, kc, ks, vc, vs, lens, bt = _case(kvq, dev, seed, wbits, page_size)
        ref = torch.empty_like(q)
        kvq.decode_attention_q(q, kc, ks, vc, vs, ref, q.shape[0], lens, wbits, scale, page_size, bt)
        out = torch.full_like(q, float("nan"))
        st = _noalloc_via_abi(kvq, q, kc, ks, vc, vs, out, lens, wbits, scale, page_size, bt)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        assert kvq.poll_device_error() == 0
        assert not torch.isnan(out.float()).any()
        same = out.view(torch.int16) == ref.view(torch.int16)
        assert bool(same.all()), (f"call {call}: {int((~same).sum())} of {same.numel()} outputs differ from the "
                                  f"workspace entry point's, worst by {float((out.float() - ref.float()).abs().max()):.3g}")


def test_noalloc_rejects_geometry_beyond_the_scratch(kvq):
    dev = torch.device("cuda:0")
    q, kc, ks, vc, vs, lens, bt = _case(kvq, dev, 13, 4, 0)
    B, NH, D = q.shape
    # 64 sequences x 64 query heads x 1M positions need far more than 32 MiB of workspace
    desc = kvq._Desc(64, 1 << 20, 8, D, 0)
    assert kvq.library().kvq_decode_attention_workspace_size(ctypes.byref(desc), 64, 64, 0) > \
        kvq.ATTENTION_SCRATCH_BYTES
    lib = kvq.library()
    st = lib.kvq_decode_attention_q_noalloc(q.data_ptr(), kc.data_ptr(), ks.data_ptr(), vc.data_ptr(), vs.data_ptr(),
                                            q.data_ptr(), ctypes.byref(desc), 64, 64, 0, lens.data_ptr(), None, 4,
                                            ctypes.c_float(1.0), None)
    assert st == 4  # KVQ_ERR_RANGE, nothing enqueued
    # 64 sequences x 128 query heads x eight 128-position chunk slots x 130 floats: 34.1 MB
    big_q = torch.zeros(64, 128, D, dtype=torch.float16, device=dev)
    with pytest.raises(ValueError, match="scratch"):
        kvq.decode_attention_q_noalloc(big_q, kc, ks, vc, vs, torch.empty_like(big_q), 64,
                                       torch.ones(64, dtype=torch.int32, device=dev), 4, 1.0)
