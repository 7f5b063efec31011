"""Per-output error bound of the decode-attention kernels, computed from the inputs.

Test infrastructure.  It restates no kernel and no oracle function: it takes the
exact (binary64) keys and values of the attended positions, computes the exact
softmax weights w_p = 2^(tau_p - tau*) with tau_p = scale * log2(e) * (q . k_p), and
bounds |RN16(y_kernel) - o| for o = sum_p w_p v_p / sum_p w_p from the arithmetic
the kernels perform (csrc/attention.cuh):

* scores: binary16 products summed on the tensor core into a binary32 accumulator,
  D / 16 steps of 16 products.  One step is modelled as exact products aligned to
  the largest exponent and truncated, then a truncated normalization: an error below
  MMA_STEP_ULPS * 2^-23 times the largest term (measured on the device by
  kvq_selfcheck_attention_numerics), hence |s_hat - s| <= gamma_S * A_p with
  A_p = sum_d |q_d k_pd| and gamma_S = MMA_STEP_ULPS * 2^-23 * D / 16;
* the binary32 scale constant scale * log2(e) (three roundings, common to every
  position: a relative error of the exponent differences), the rounding of the
  scaled score and of its difference from the running reference maximum;
* every 2^x (the weights, the lazy-rescale factors, the chunk merge factors):
  relative error at most EPS_EXP2 each, and the binary32 subtractions of reference
  maxima that feed them (at most five levels, each below u times the score range);
* the weights enter P . V as a binary16 high part plus a binary16 residual (relative
  2^-22, and an absolute 2^-25 of the item's largest weight once the residual is
  subnormal: at most 2^-17 of the weight sum over one softmax state, which spans at
  most 256 positions), summed by the tensor core in 2 steps per 16 positions (32 steps
  per state), and the weight sums and the merges of up to ceil(n / 128) workspace
  entries (one per 128-position chunk) in binary32;
* the final binary32 division and the rounding to binary16 (half an ulp).

Each weight the kernels use is w_p * (1 + r_p) up to a common factor, with
2^-(E_p + xi) (1 - eps) <= 1 + r_p <= 2^(E_p + xi) (1 + eps): E_p the exponent error of
position p, xi that of the merges, eps that of the 2^x evaluations.  With up_p the
largest |r_p|, nu the numerator-only and lam the denominator-only relative errors of
the sums, and beta the absolute error of the binary16 weight split:

  |y - o| <= [sum w up |v - o| + (nu sum w (1 + up) |v| + beta max|v| + lam |o|) sum w (1 + up)]
             / [(1 - lam) sum w 2^-(E + xi) (1 - eps)]

and, since the weighted mean lies between the smallest and largest value, also
|y - o| <= max |v - o| plus the sum errors.  The binary16 output is within the
smaller of the two plus half an ulp of |o| + bound.
"""
from __future__ import annotations

import math

import numpy as np

U = 2.0 ** -24                # binary32 unit roundoff
EPS_EXP2 = 2.0 ** -21         # bound on the relative error of ex2.approx.ftz and of exp2f (self-check)
MMA_STEP_ULPS = 18.0          # one mma.sync step: error below this many 2^-23 of its largest term (self-check)
CHUNK = 256                   # positions one softmax state spans at most
ENTRY = 128                   # positions per workspace entry (the entries merged per output)
STEPS_PER_ITEM = CHUNK // 16  # softmax steps (and lazy-rescale opportunities) per state
LOG2E = 1.4426950408889634


def ulp16(x):
    """The binary16 spacing at magnitude x (the subnormal spacing 2^-24 below 2^-14)."""
    x = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -14)
    return np.exp2(np.floor(np.log2(x)) - 10.0)


def attention_bound(q, K, V, group, scale):
    """q: [NH, D] query values; K, V: [n, H, D] exact key and value values of the
    attended positions (n may be 0).  Returns (o, tol), both [NH, D]: the exact output
    and the bound on |kernel output - o|."""
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    NH, D = q.shape
    n = K.shape[0]
    o = np.zeros((NH, D))
    tol = np.zeros((NH, D))
    if n == 0:
        return o, tol
    nch = math.ceil(n / ENTRY)
    n_b = math.ceil(math.ceil(nch / 4) / (1024 // D))  # batch rescales per warp in the chunk merge
    gamma_s = MMA_STEP_ULPS * 2.0 ** -23 * (D / 16)
    gamma_n = MMA_STEP_ULPS * 2.0 ** -23 * (2 * STEPS_PER_ITEM) * (1 + 2.0 ** -10)
    n_exp = 1 + STEPS_PER_ITEM + 1 + 1 + n_b + 1  # 2^x evaluations on one position's path
    nu = (2.0 ** -22 + gamma_n + (29 + n_b + nch) * U) * (1 + 2.0 ** -10)
    lam = (96 + n_b + nch) * U * (1 + 2.0 ** -10)
    beta = 2.0 ** -17
    c = scale * LOG2E
    for kvh in range(K.shape[1]):
        hs = slice(kvh * group, (kvh + 1) * group)
        Kh, Vh = K[:, kvh, :], V[:, kvh, :]
        s = Kh @ q[hs].T                        # [n, G]
        A = np.abs(Kh) @ np.abs(q[hs]).T        # [n, G]
        tau = c * s
        tmax = tau.max(axis=0)
        tmin = tau.min(axis=0)
        w = np.exp2(tau - tmax)                 # exact weights, largest 1
        W = w.sum(axis=0)
        oh = (w.T @ Vh) / W[:, None]            # [G, D]
        a = c * (1 + 4 * U) * gamma_s * A
        amax = a.max(axis=0)
        E = a + 3 * U * (tmax - tau) + U * (np.abs(tau) + a + 1) + U * (tmax - tau + 2 * amax + 9)
        xi = 5 * U * (tmax - tmin + 2 * amax + 9)
        eps = math.expm1(n_exp * EPS_EXP2)
        up = np.exp2(E + xi) * (1 + eps) - 1.0       # largest relative perturbation of a weight
        dn = np.exp2(-(E + xi)) * (1 - eps)          # smallest factor on a weight
        vmax = np.abs(Vh).max(axis=0)                # [D]
        for g in range(oh.shape[0]):
            wu = w[:, g] * up[:, g]
            w1 = w[:, g] * (1 + up[:, g])
            mass = w1.sum()
            low = (1 - lam) * (w[:, g] * dn[:, g]).sum()
            dev = np.abs(Vh - oh[g])
            sums = (nu * (w1 @ np.abs(Vh)) + beta * vmax * mass) / low
            b_weights = (wu @ dev + lam * np.abs(oh[g]) * mass) / low + sums
            b_hull = dev.max(axis=0) + vmax * lam / (1 - lam) + sums
            b = np.minimum(b_weights, b_hull)
            o[hs.start + g] = oh[g]
            tol[hs.start + g] = b + 0.5 * ulp16(np.abs(oh[g]) + b)
    return o, tol


def attended_rows(vals, seq, n, page_size=0, block_table=None):
    """Rows [n, H, D] of positions 0..n-1 of sequence `seq` from a decoded cache `vals`
    ([dim0, dim1, H, D]; paged: [pages, page_size, H, D] read through the block table)."""
    if n == 0:
        return vals[:0, 0]
    if page_size == 0:
        return vals[seq, :n]
    p = np.arange(n)
    pages = np.asarray(block_table)[seq, p // page_size]
    return vals[pages, p % page_size]


def old_tolerance(ex, vmax):
    """The tolerance used before the bound was derived: one binary16 ulp of the exact
    value plus 2^-14 of the largest |v| (kept to report how often it is exceeded)."""
    return ulp16(ex) + 2.0 ** -14 * vmax
