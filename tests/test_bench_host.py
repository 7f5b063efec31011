"""Host logic of the benchmark's multi-GPU path, run as two gloo ranks on the CPU:
the shard split (weak scaling, every rank converts its own sequences, no
collective on the data path) and the max-over-ranks reduction of step times."""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


@pytest.mark.parametrize("total,world", [(4, 1), (4, 2), (7, 2), (32, 3), (5, 8), (0, 2)])
def test_shard_range_partitions(total, world):
    seen = []
    for r in range(world):
        lo, hi = bench.shard_range(total, r, world)
        assert 0 <= lo <= hi <= total
        seen.extend(range(lo, hi))
    assert seen == list(range(total))
    sizes = [bench.shard_range(total, r, world)[1] - bench.shard_range(total, r, world)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.5 + 2.0 * rank)
        lo, hi = bench.shard_range(8, rank, world)
        q.put((rank, got, lo, hi))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [3.5, 3.5]
    assert [(r[2], r[3]) for r in res] == [(0, 4), (4, 8)]


def test_max_over_ranks_without_group():
    assert bench.max_over_ranks(2.25) == 2.25


def test_algorithmic_bytes_per_element():
    """The roofline numerators: FP16 in (2 B) plus the format's bytes out (or the reverse),
    scales at 2 B per 32 elements."""
    assert bench.BYTES_PER_ELEM["fp8"] == 3.0
    assert bench.BYTES_PER_ELEM[4] == 2.5625 and bench.BYTES_PER_ELEM[6] == 2.8125
    assert bench.BYTES_PER_ELEM[8] == 3.0625
    m = bench.MODEL32
    assert (m["layers"], m["seqs"], m["seq_len"], m["kv_heads"], m["head_dim"], m["wbits"]) == \
        (32, 8, 32768, 8, 128, 6)
    # one fused K+V launch of a model layer: 2.8125 B x 2 x 8 x 32768 x 8 x 128
    assert bench.step_launch_bytes() == 1509949440
    # the FP8 window per-op row: one fused K+V encode launch is 3 B x 2 x 4 x 2048 x 8 x 128
    B, S, H, D = bench.FP8_WINDOW["shape"]
    assert (B, S, H, D) == (4, 4096, 8, 128) and bench.FP8_WINDOW["width"] == 2048
    assert 3 * 2 * B * bench.FP8_WINDOW["width"] * H * D == 50331648


def test_position_tasks_cover_exactly_the_first_positions():
    lens = [1000, 700, 5]
    for n in (0, 1, 999, 1000, 1001, 1700, 1705, 5000):
        tasks = bench.position_tasks(lens, n, 256)
        covered = [(i, p) for i, a, b in tasks for p in range(a, b)]
        want = [(i, p) for i, L in enumerate(lens) for p in range(L)][:n]
        assert covered == want
        assert all(0 < b - a <= 256 for _, a, b in tasks)


def test_oracle_harness_split_gives_the_single_call_result(oracle_mod):
    """The CPU baseline's split of a layer into position ranges over several threads computes
    exactly what one oracle call over the whole window computes."""
    import numpy as np
    import torch

    import workloads

    pool = workloads.model_layer(0, seqs=2, seq_len=1024, page_size=256, heads=2, head_dim=64)
    kb = pool.k.view(torch.int16).numpy().view(np.uint16)
    vb = pool.v.view(torch.int16).numpy().view(np.uint16)
    P, ps, H, D = kb.shape
    lens = pool.cache_seqlens.numpy().astype(np.int32)
    bt = pool.block_table.numpy().astype(np.int32)

    def fresh():
        kc = np.zeros((P, ps, H, D * 6 // 8), np.uint8)
        ks = np.zeros((P, ps, H, D // 32), np.uint16)
        assert oracle_mod.fp16_to_q_kv(kb, kc, ks, vb, kc.copy(), ks.copy(), 2, -1024, 1024, ps, lens, bt, 6) == 0
        vc, vs = kc.copy(), ks.copy()
        assert oracle_mod.fp16_to_q_kv(kb, kc, ks, vb, vc, vs, 2, -1024, 1024, ps, lens, bt, 6) == 0
        return dict(kc=kc, vc=vc, ks=ks, vs=vs, lens=lens, bt=bt, ps=ps, ky=np.zeros_like(kb), vy=np.zeros_like(vb))

    one, split = fresh(), fresh()
    assert oracle_mod.q_to_fp16_kv(one["kc"], one["ky"], one["ks"], one["vc"], one["vy"], one["vs"], 2, -1024, 1024,
                                   ps, lens, bt, 6) == 0
    assert oracle_mod.fp16_to_q_kv(one["ky"], one["kc"], one["ks"], one["vy"], one["vc"], one["vs"], 2, -1024, 1024,
                                   ps, lens, bt, 6) == 0
    sec, n = bench.oracle_model_tasks(split, bench.position_tasks(lens, 2048, 100), 3)
    assert n == 2048 and sec > 0
    for name in ("kc", "vc", "ks", "vs", "ky", "vy"):
        assert np.array_equal(one[name], split[name]), name


def test_attention_bytes():
    # Q4, D = 128: per position and kv head 64 B of codes + 8 B of scales, for K and V;
    # plus the queries read and the outputs written (2 B each)
    assert bench.attention_bytes([10, 0], 8, 128, 4, 32) == 2 * 10 * 8 * 72 + 2 * 2 * 2 * 32 * 128
    assert bench.attention_bytes([16384], 8, 128, 4, 32) == 18890752


def test_recorded_traffic_follows_the_source_digest(tmp_path, monkeypatch):
    f = tmp_path / "traffic.txt"
    f.write_text(f"# comment\nfp16_to_fp8_kv 1234 {bench.kernel_source_digest()}\nother 5 0000000000000000\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.recorded_traffic("fp16_to_fp8_kv") == 1234
    assert bench.recorded_traffic("other") is None           # stale digest
    assert bench.recorded_traffic("missing") is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "absent.txt"))
    assert bench.recorded_traffic("fp16_to_fp8_kv") is None
