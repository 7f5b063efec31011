"""Seeded synthetic inputs for the KV-cache conversion workloads.

This module holds only random-number generation and shape bookkeeping; it
contains none of the conversion arithmetic, so both the CPU oracle's tests and
the CUDA path draw identical inputs from it without sharing any of the method.

Every generator takes a seed and an optional ``device``.  On ``"cpu"`` the
values come from ``torch.Generator("cpu")``; on a CUDA device they come from
that device's generator (same recipe, different bits), which is used for the
model-sized workloads that are too large to draw on the host.  FP16 values are
produced as ``float32`` draws rounded with ``.half()``.

Workload recipes (shapes follow the KV cache layout
[batch, seq, kv_heads, head_dim]):

1. ``small``: K, V [1, 256, 8, 128] ~ N(0, 1).
2. ``fp8_window``: K, V [4, 4096, 8, 128] ~ N(0, 1); each element is
   independently replaced with probability 1% by a +-U(20, 60000) outlier
   (fair sign) and with probability 0.1% by a random nonzero FP16 subnormal
   (bits 0x001..0x3FF, fair sign).
3. ``channel_outliers``: K [16, 8192, 8, 128] = N(0, 1) * c[h, d] with
   c = exp(N(0, 1)) drawn once per (head, channel); V = 0.5 * N(0, 1);
   each 32-element block along head_dim is zeroed with probability 2%,
   independently for K and V.
4. ``paged_pool``: 2048 pages x 256 positions x 8 heads x 128 FP16 pools for
   K and V ~ N(0, 1); 32 sequences with cache_seqlens ~ U{1..16384}; sequence
   i owns ceil((seqlens[i] + 1) / 256) pages taken in order from a seeded
   permutation of the pool; block_table [32, 65] int32 padded with -1.
5. ``model_layer``: one layer of a 32-layer model, K and V pools of
   1024 pages x 256 x 8 x 128 FP16 holding 8 sequences x 32768 positions;
   block_table [8, 128] a seeded permutation of the pool; K = N(0, 1) * c[h, d]
   with c = exp(N(0, 1)), V = N(0, 1).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

SEED_BASE = 1000


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _rand(shape, g, device) -> torch.Tensor:
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32)


def normal_kv(shape, seed: int, device="cpu"):
    """K, V ~ N(0, 1) FP16 of the given 4-D shape."""
    g = _gen(seed, device)
    k = _randn(shape, g, device).half()
    v = _randn(shape, g, device).half()
    return k, v


def small(seed: int = SEED_BASE + 1, shape=(1, 256, 8, 128), device="cpu"):
    return normal_kv(shape, seed, device)


def with_outliers_and_subnormals(x32: torch.Tensor, g, device, p_out=0.01, p_sub=0.001) -> torch.Tensor:
    """Replace elements of an fp32 draw: outliers +-U(20, 60000), subnormals; returns FP16."""
    u = _rand(x32.shape, g, device)
    mag = 20.0 + (60000.0 - 20.0) * _rand(x32.shape, g, device)
    sgn = torch.where(_rand(x32.shape, g, device) < 0.5, -1.0, 1.0)
    h = torch.where(u < p_out, sgn * mag, x32).half()
    sub_bits = torch.randint(1, 0x400, x32.shape, generator=g, device=device, dtype=torch.int32)
    sub_bits = sub_bits | torch.where(_rand(x32.shape, g, device) < 0.5, 0x8000, 0).to(torch.int32)
    sub_bits = torch.where(sub_bits >= 0x8000, sub_bits - 0x10000, sub_bits)  # as signed 16-bit
    sub = sub_bits.to(torch.int16).view(torch.float16)  # reinterpret the bit pattern
    is_sub = (u >= p_out) & (u < p_out + p_sub)
    return torch.where(is_sub, sub, h)


def channel_outlier_keys(shape, seed: int, lo: float, hi: float, device="cpu"):
    """K ~ N(0, 1) FP16 with channel 0 of every (position, head) replaced by +-U(lo, hi)
    (fair sign), so that query-key scores are dominated by one channel; V drawn by the
    fp8_window recipe with the next seed."""
    g = _gen(seed, device)
    k = _randn(shape, g, device)
    mag = lo + (hi - lo) * _rand(shape[:-1], g, device)
    sign = torch.where(_rand(shape[:-1], g, device) < 0.5, -1.0, 1.0)
    k[..., 0] = sign * mag
    _, v = fp8_window(seed=seed + 1, shape=shape, device=device)
    return k.half(), v


def fp8_window(seed: int = SEED_BASE + 2, shape=(4, 4096, 8, 128), device="cpu"):
    g = _gen(seed, device)
    k = with_outliers_and_subnormals(_randn(shape, g, device), g, device)
    v = with_outliers_and_subnormals(_randn(shape, g, device), g, device)
    return k, v


def zero_blocks(x: torch.Tensor, p: float, g, device) -> torch.Tensor:
    """Zero each 32-element block along the last dim with probability p."""
    *lead, D = x.shape
    keep = (_rand((*lead, D // 32, 1), g, device) >= p).to(x.dtype)
    return (x.reshape(*lead, D // 32, 32) * keep).reshape(x.shape)


def channel_outliers(seed: int = SEED_BASE + 3, shape=(16, 8192, 8, 128), device="cpu",
                     p_zero_block=0.02):
    g = _gen(seed, device)
    B, S, H, D = shape
    c = torch.exp(_randn((H, D), g, device))
    k = zero_blocks(_randn(shape, g, device) * c, p_zero_block, g, device).half()
    v = zero_blocks(_randn(shape, g, device) * 0.5, p_zero_block, g, device).half()
    return k, v


@dataclass
class PagedPool:
    k: torch.Tensor            # [pages, page_size, H, D] fp16
    v: torch.Tensor
    cache_seqlens: torch.Tensor  # [batch] int32
    block_table: torch.Tensor    # [batch, max_pages] int32, -1 padded
    page_size: int


def paged_tables(seed: int, batch: int, max_len: int, num_pages: int, page_size: int,
                 extra_positions: int = 1, lens=None):
    """Seeded cache_seqlens ~ U{1..max_len} (or the given lens) and a block table that
    gives sequence i ceil((len_i + extra_positions) / page_size) pages drawn in order
    from a random permutation of the pool.  Returns (seqlens, block_table) on CPU."""
    g = _gen(seed, "cpu")
    if lens is None:
        lens = torch.randint(1, max_len + 1, (batch,), generator=g, dtype=torch.int32)
    else:
        lens = torch.as_tensor(lens, dtype=torch.int32)
    max_pages = (max_len + extra_positions + page_size - 1) // page_size
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    bt = torch.full((batch, max_pages), -1, dtype=torch.int32)
    cursor = 0
    for i in range(batch):
        n = (int(lens[i]) + extra_positions + page_size - 1) // page_size
        if cursor + n > num_pages:
            raise ValueError("page pool too small for the drawn sequence lengths")
        bt[i, :n] = perm[cursor:cursor + n]
        cursor += n
    return lens, bt


def paged_pool(seed: int = SEED_BASE + 4, num_pages=2048, page_size=256, heads=8, head_dim=128,
               batch=32, max_len=16384, device="cpu") -> PagedPool:
    lens, bt = paged_tables(seed, batch, max_len, num_pages, page_size)
    k, v = normal_kv((num_pages, page_size, heads, head_dim), seed + 100, device)
    return PagedPool(k, v, lens.to(device), bt.to(device), page_size)


def model_layer(layer: int, seed: int = SEED_BASE + 5, seqs=8, seq_len=32768, page_size=256,
                heads=8, head_dim=128, device="cpu") -> PagedPool:
    num_pages = seqs * seq_len // page_size
    g = _gen(seed * 1000 + layer, "cpu")
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    bt = perm.reshape(seqs, seq_len // page_size).contiguous()
    lens = torch.full((seqs,), seq_len, dtype=torch.int32)
    gd = _gen(seed * 1000 + layer, device)
    shape = (num_pages, page_size, heads, head_dim)
    c = torch.exp(_randn((heads, head_dim), gd, device))
    k = (_randn(shape, gd, device) * c).half()
    v = _randn(shape, gd, device).half()
    return PagedPool(k, v, lens.to(device), bt.to(device), page_size)


def identity_block_table(batch: int, seq: int, page_size: int) -> torch.Tensor:
    """block_table[i][j] = i * seq / page_size + j: paged view of a contiguous cache."""
    ppseq = seq // page_size
    return (torch.arange(batch, dtype=torch.int32)[:, None] * ppseq
            + torch.arange(ppseq, dtype=torch.int32)[None, :]).contiguous()
