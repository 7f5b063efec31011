"""The decode-attention error bound (tests/attn_bound.py) on the CPU: its exact output is
the oracle's, a binary32 restatement of the kernels' arithmetic stays inside it on
typical and adversarial inputs, and it is tight enough that plausible mistakes of an
attention kernel (a dropped position, another head's values, a wrong softmax scale)
land outside it."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import attn_bound
import workloads


def _fp8_case(seed, B=2, S=300, H=1, D=128, NH=4, outliers=False):
    if outliers:
        k, v = workloads.channel_outlier_keys((B, S, H, D), workloads.SEED_BASE + 710 + seed, 2000.0, 57344.0)
    else:
        k, v = workloads.fp8_window(seed=workloads.SEED_BASE + 720 + seed, shape=(B, S, H, D))
    q = torch.randn(B, NH, D, generator=torch.Generator().manual_seed(workloads.SEED_BASE + 730 + seed)).half()
    return q, k, v


def _encode_fp8(oracle_mod, k, v):
    kb = k.view(torch.int16).numpy().view(np.uint16)
    vb = v.view(torch.int16).numpy().view(np.uint16)
    k8, v8 = np.zeros(kb.shape, np.uint8), np.zeros(vb.shape, np.uint8)
    B, S = kb.shape[:2]
    assert oracle_mod.fp16_to_fp8_kv(kb, k8, vb, v8, B, 0, S) == oracle_mod.OK
    ky, vy = np.zeros(kb.shape, np.uint16), np.zeros(vb.shape, np.uint16)
    assert oracle_mod.fp8_to_fp16_kv(k8, ky, v8, vy, B, 0, S) == oracle_mod.OK
    return k8, v8, ky.view(np.float16).astype(np.float64), vy.view(np.float16).astype(np.float64)


def _emulate_fp32(q, K, V, group, scale, states=None, split_sums=False):
    """A binary32 computation with the kernels' structure: softmax states over spans of
    16-position steps (`states`: (first, end) position spans, 256-position items by
    default), binary32 scores, lazy rescaling (threshold 2^8), 2^x in binary32, weights
    split into a binary16 high part and residual for the value sum (`split_sums`: the two
    parts summed apart and added when the state ends, as for groups of up to four query
    heads), binary32 sums; the states merged in binary32; the result rounded to binary16."""
    f32 = np.float32
    NH, D = q.shape
    n = K.shape[0]
    out = np.zeros((NH, D), np.float64)
    c = f32(f32(scale) * f32(attn_bound.LOG2E))
    if states is None:
        states = [(c0, min(n, c0 + attn_bound.CHUNK)) for c0 in range(0, n, attn_bound.CHUNK)]
    for h in range(NH):
        kvh = h // group
        qh = q[h].astype(f32)
        parts = []
        for c0, c1 in states:
            m, l, acc, acc_lo = f32(-np.inf), f32(0), np.zeros(D, f32), np.zeros(D, f32)
            for t0 in range(c0, c1, 16):
                kk = K[t0:min(t0 + 16, c1), kvh].astype(f32)
                vv = V[t0:min(t0 + 16, c1), kvh].astype(f32)
                s = np.array([np.sum(kk[i] * qh, dtype=f32) for i in range(kk.shape[0])], f32)
                x = (s * c).astype(f32)
                mx = x.max()
                if mx > m + f32(8):
                    alpha = f32(0) if m == -np.inf else f32(np.exp2(f32(m - mx)))
                    l = f32(l * alpha)
                    acc = (acc * alpha).astype(f32)
                    acc_lo = (acc_lo * alpha).astype(f32)
                    m = mx
                p = np.exp2((x - m).astype(f32)).astype(f32)
                hi = p.astype(np.float16).astype(f32)
                lo = (p - hi).astype(np.float16).astype(f32)
                l = f32(l + np.sum(p, dtype=f32))
                if split_sums:
                    acc = (acc + (hi[:, None] * vv).sum(axis=0, dtype=f32)).astype(f32)
                    acc_lo = (acc_lo + (lo[:, None] * vv).sum(axis=0, dtype=f32)).astype(f32)
                else:
                    acc = (acc + ((hi + lo)[:, None] * vv).sum(axis=0, dtype=f32)).astype(f32)
            parts.append((m, l, (acc + acc_lo).astype(f32)))
        mstar = max(pm for pm, _, _ in parts)
        L, O = f32(0), np.zeros(D, f32)
        for pm, pl, pa in parts:
            f = f32(np.exp2(f32(pm - mstar)))
            L = f32(L + f * pl)
            O = (O + f * pa).astype(f32)
        out[h] = (O / L).astype(np.float16).astype(np.float64)
    return out


@pytest.mark.parametrize("outliers", [False, True])
def test_bound_exact_output_is_the_oracles(oracle_mod, outliers):
    q, k, v = _fp8_case(1, outliers=outliers)
    k8, v8, K, V = _encode_fp8(oracle_mod, k, v)
    B, NH, D = q.shape
    lens = np.array([300, 171], np.int32)
    st, _, ex = oracle_mod.decode_attention_fp8(q.view(torch.int16).numpy().view(np.uint16), k8, v8, B, NH, 0, lens,
                                                None, 1.0 / math.sqrt(D))
    assert st == oracle_mod.OK
    for i in range(B):
        o, tol = attn_bound.attention_bound(q[i].float().numpy(), K[i, :lens[i]], V[i, :lens[i]], NH, 1.0 / math.sqrt(D))
        assert np.allclose(o, ex[i], rtol=1e-12, atol=1e-12 * np.abs(V).max())
        assert (tol > 0).all()


@pytest.mark.parametrize("outliers", [False, True])
@pytest.mark.parametrize("seed", range(3))
def test_binary32_restatement_within_bound(oracle_mod, outliers, seed):
    q, k, v = _fp8_case(seed, S=700, D=256, NH=8, outliers=outliers)
    _, _, K, V = _encode_fp8(oracle_mod, k, v)
    scale = 1.0 / 16
    for i in range(q.shape[0]):
        qi = q[i].float().numpy().astype(np.float64)
        o, tol = attn_bound.attention_bound(qi, K[i], V[i], 8, scale)
        y = _emulate_fp32(qi, K[i], V[i], 8, scale)
        err = np.abs(y - o)
        assert np.all(err <= tol), f"worst error {err.max():.4g}, bound there {tol[np.argmax(err / tol)]:.4g}"


@pytest.mark.parametrize("outliers", [False, True])
@pytest.mark.parametrize("seed", range(2))
def test_binary32_restatement_split_sums_within_bound(oracle_mod, outliers, seed):
    """The arithmetic of groups of up to four query heads: the weights' high parts and
    residuals summed apart; softmax states of one chunk or of an aligned pair of
    128-position chunks (as warps' contiguous ranges of chunks give them), merged over up
    to ceil(n / 128) workspace entries."""
    q, k, v = _fp8_case(10 + seed, S=700, D=128, NH=4, outliers=outliers)
    _, _, K, V = _encode_fp8(oracle_mod, k, v)
    scale = 1.0 / math.sqrt(128)
    # one warp's range ends after chunk 0, the next starts at chunk 1 (alone: its pair
    # partner belongs to the other warp), then aligned pairs (2, 3) and (4, 5)
    states = [(0, 128), (128, 256), (256, 512), (512, 700)]
    for i in range(q.shape[0]):
        qi = q[i].float().numpy().astype(np.float64)
        o, tol = attn_bound.attention_bound(qi, K[i], V[i], 4, scale)
        y = _emulate_fp32(qi, K[i], V[i], 4, scale, states=states, split_sums=True)
        err = np.abs(y - o)
        assert np.all(err <= tol), f"worst error {err.max():.4g}, bound there {tol[np.argmax(err / tol)]:.4g}"


def test_bound_is_small_on_typical_inputs():
    """On N(0,1) keys and values (2000 positions, a flat softmax) the derived bound is a
    few binary16 ulps of the largest |v| and no looser than the tolerance used before it
    was derived, so the GPU tests lose no sensitivity there."""
    g = torch.Generator().manual_seed(workloads.SEED_BASE + 740)
    K = torch.randn(2000, 1, 128, generator=g).half().double().numpy()
    V = torch.randn(2000, 1, 128, generator=g).half().double().numpy()
    q = torch.randn(4, 128, generator=g).half().double().numpy()
    o, tol = attn_bound.attention_bound(q, K, V, 4, 128 ** -0.5)
    old = attn_bound.old_tolerance(o, np.abs(V).max())
    assert np.median(tol) <= np.median(old), (np.median(tol), np.median(old))
    assert tol.max() < 1e-3


@pytest.mark.parametrize("mistake", ["drop_last", "other_head", "scale"])
def test_planted_mistakes_exceed_the_bound(oracle_mod, mistake):
    """Outputs an attention kernel with a typical mistake would produce (computed in fp64
    by the oracle with the mistake put into its inputs) fall outside the bound for most
    outputs."""
    g = torch.Generator().manual_seed(workloads.SEED_BASE + 750)
    B, S, H, D, NH = 1, 600, 2, 128, 4
    k, v = workloads.normal_kv((B, S, H, D), workloads.SEED_BASE + 751)
    k8, v8, K, V = _encode_fp8(oracle_mod, k, v)
    q = torch.randn(B, NH, D, generator=g).half()
    qb = q.view(torch.int16).numpy().view(np.uint16)
    scale = 1.0 / math.sqrt(D)
    lens = np.array([S], np.int32)
    if mistake == "drop_last":
        st, _, bad = oracle_mod.decode_attention_fp8(qb, k8, v8, B, NH, 0, lens - 1, None, scale)
    elif mistake == "other_head":
        v8w = np.ascontiguousarray(v8[:, :, ::-1])  # values of the other kv head
        st, _, bad = oracle_mod.decode_attention_fp8(qb, k8, v8w, B, NH, 0, lens, None, scale)
    else:
        st, _, bad = oracle_mod.decode_attention_fp8(qb, k8, v8, B, NH, 0, lens, None, scale * (1 + 2.0 ** -6))
    assert st == oracle_mod.OK
    o, tol = attn_bound.attention_bound(q[0].float().numpy(), K[0], V[0], NH // H, scale)
    outside = np.abs(bad[0] - o) > tol
    assert outside.mean() > 0.5, f"only {outside.mean():.2f} of the outputs outside the bound"
