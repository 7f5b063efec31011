"""count_match (page "Implementation: Turboderp org Exllamav2 Ext Cache",
Description and I/O Contract): the length of the matching prefix of two 1-D
64-bit tensors, checked no further than max_a.  A host function: the oracle is
pinned against a brute-force Python comparison, and the library's C function
(and its Python binding) against the oracle."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch


def brute(a, b, max_a):
    n = 0
    for x, y in zip(a, b):
        if n >= max_a or x != y:
            break
        n += 1
    return n


def cases():
    rng = np.random.default_rng(5)
    out = [(np.array([], np.int64), np.array([], np.int64), 10),
           (np.arange(10), np.arange(10), 10), (np.arange(10), np.arange(10), 4), (np.arange(10), np.arange(10), 0),
           (np.arange(10), np.arange(10), -3), (np.arange(10), np.arange(20), 100), (np.arange(20), np.arange(5), 100),
           (np.array([1, 2, 3]), np.array([9, 2, 3]), 3),
           (np.array([-1, 2**62, -2**63]), np.array([-1, 2**62, -2**63]), 5),
           (np.array([0x0123456789ABCDEF]), np.array([0x0123456789ABCDEE]), 1)]
    for _ in range(200):
        n = int(rng.integers(0, 300))
        a = rng.integers(-2**63, 2**63 - 1, n, dtype=np.int64)
        b = a.copy()
        if n and rng.random() < 0.8:
            k = int(rng.integers(0, n))
            b[k] ^= np.int64(1) << np.int64(int(rng.integers(0, 63)))
        b = b[: int(rng.integers(0, n + 1))] if rng.random() < 0.3 else b
        out.append((a, b, int(rng.integers(-1, n + 5))))
    return out


def test_oracle_count_match_bruteforce(oracle_mod):
    for a, b, m in cases():
        assert oracle_mod.count_match(a, b, m) == brute(a.tolist(), b.tolist(), m)


def test_library_count_match_matches_oracle(oracle_mod, kvq_built):
    kvq = kvq_built

    for a, b, m in cases():
        ref = oracle_mod.count_match(a, b, m)
        assert kvq.count_match(torch.from_numpy(a.astype(np.int64)), torch.from_numpy(b.astype(np.int64)), m) == ref
    L = kvq.library()
    assert L.kvq_count_match(None, 0, None, 0, 5) == 0
    assert L.kvq_count_match(None, 3, None, 3, 5) == -1
    with pytest.raises(ValueError):
        kvq.count_match(torch.zeros(3, dtype=torch.int32), torch.zeros(3, dtype=torch.int64), 3)
