"""Independent fp64 models used to pin the oracle (test helpers).

* `online_row` follows the online-softmax recurrence as the pages state it:
  running max m and running sum l start at -inf and 0; for each new block of
  scores the block max updates m, the old sum is rescaled by e^(m_old - m_new),
  the block's exponentials are added, and the partial output is rescaled the
  same way before the block's weighted values are added (FlashAttention
  optimisation article, section 3.2.1; Gemini 3 Flash kernel-fusion post,
  section 3).  Section 3.2.2 of the article claims the result equals the
  ordinary softmax for any block order; the pins check the oracle against
  this model for random block widths and random key orders.
* `split_combine_row` evaluates disjoint key splits separately and merges them
  by their log-sum-exp, which is the same claim applied to whole splits.
* `brute_row` is the textbook definition with no max subtraction, in extended
  precision (numpy longdouble), for tiny inputs only.
"""
from __future__ import annotations

import math

import numpy as np


def widen(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def online_row(q, K, V, scale, blocks, rescale_threshold=0.0):
    """q [d], K/V [n, d] float64; blocks = list of index arrays (any order).

    rescale_threshold > 0 keeps a stale max until the new one exceeds it by
    more than the threshold (natural-log units); the result is the same.
    """
    d = V.shape[1]
    m = -math.inf
    l = 0.0
    o = np.zeros(d)
    for idx in blocks:
        if len(idx) == 0:
            continue
        x = scale * (K[idx] @ q)
        m_local = float(np.max(x))
        m_new = max(m, m_local)
        if m != -math.inf and m_new - m <= rescale_threshold:
            m_new = m          # conditional rescale: keep the old max
        alpha = 0.0 if m == -math.inf else math.exp(m - m_new)
        p = np.exp(x - m_new)
        l = alpha * l + float(p.sum())
        o = alpha * o + p @ V[idx]
        m = m_new
    if l == 0.0:
        return np.zeros(d), -math.inf
    return o / l, m + math.log(l)


def split_combine_row(q, K, V, scale, splits):
    """Evaluate each split with its own softmax, then merge by log-sum-exp."""
    parts = []
    for idx in splits:
        if len(idx) == 0:
            continue
        o_s, lse_s = online_row(q, K, V, scale, [idx])
        parts.append((o_s, lse_s))
    if not parts:
        return np.zeros(V.shape[1]), -math.inf
    mx = max(p[1] for p in parts)
    tot = sum(math.exp(p[1] - mx) for p in parts)
    lse = mx + math.log(tot)
    o = sum(math.exp(p[1] - lse) * p[0] for p in parts)
    return o, lse


def brute_row(q, K, V, scale, visible):
    """Extended precision, no max subtraction: e^{s_j} / sum e^{s}."""
    q = np.asarray(q, dtype=np.longdouble)
    K = np.asarray(K, dtype=np.longdouble)
    V = np.asarray(V, dtype=np.longdouble)
    n, d = K.shape
    w = np.zeros(n, dtype=np.longdouble)
    for j in range(n):
        if j < visible:
            s = np.longdouble(0)
            for t in range(d):
                s += q[t] * K[j, t]
            w[j] = np.exp(np.longdouble(scale) * s)
    tot = w.sum()
    if tot == 0:
        return np.zeros(d), -math.inf
    o = np.zeros(d, dtype=np.longdouble)
    for j in range(n):
        for t in range(d):
            o[t] += w[j] / tot * V[j, t]
    return o.astype(np.float64), float(np.log(tot))
