"""Algorithmic work and byte counts used for roofline reporting.

None of this runs on the hot path; it turns shapes into the FLOP and byte
figures that throughput numbers are divided by.

* Prefill FLOPs count both contractions (Q.K^T and P.V), 2 flops per
  multiply-add, over the (query, key) pairs the mask leaves visible.  Fully
  masked work is skipped by the method, so it is not counted.
* Decode bytes are what one pass must move at minimum: every visible K and V
  row once, the query and output vectors, the used block-table entries and the
  sequence lengths.  Split-KV partials are implementation overhead and are not
  counted.
* `score_matrix_elements` / `score_matrix_bytes` restate the size of the N x N
  score matrix that an unfused implementation materialises (Gemini 3 Flash
  kernel-fusion post, "traditional attention" memory example).
* `kv_cache_bytes` restates the KV-cache size formula
  2 * layers * heads * head_dim * seq_len * batch * dtype_size (GPU-optimisation
  tag page, KV-cache memory section).
"""
from __future__ import annotations

import numpy as np


def visible_pairs(Nq: int, Nkv: int, causal: bool) -> int:
    """Number of (query, key) pairs left visible by the mask.

    Causal masking is aligned to the bottom-right corner: query i sees keys
    j <= i + (Nkv - Nq).  Without a mask every pair is visible.
    """
    if not causal:
        return Nq * Nkv
    off = Nkv - Nq
    i = np.arange(Nq, dtype=np.int64)
    return int(np.clip(i + off + 1, 0, Nkv).sum())


def prefill_flops(B: int, Hq: int, Nq: int, Nkv: int, d: int, causal: bool) -> float:
    return 4.0 * B * Hq * d * visible_pairs(Nq, Nkv, causal)


def varlen_prefill_flops(q_lens, kv_lens, Hq: int, d: int, causal: bool) -> float:
    """Both contractions over the visible pairs of every sequence (sequence s
    has q_lens[s] queries against kv_lens[s] keys, bottom-right aligned)."""
    return 4.0 * Hq * d * sum(visible_pairs(int(a), int(b), causal) for a, b in zip(q_lens, kv_lens))


def decode_kv_bytes(seq_lens, Hkv: int, d: int) -> int:
    return int(np.asarray(seq_lens, dtype=np.int64).clip(min=0).sum()) * Hkv * d * 2 * 2


def decode_bytes(seq_lens, Hq: int, Hkv: int, d: int, page_size: int, lse: bool = True) -> int:
    lens = np.asarray(seq_lens, dtype=np.int64).clip(min=0)
    S = len(lens)
    pages = int(((lens + page_size - 1) // page_size).sum())
    b = decode_kv_bytes(lens, Hkv, d) + 2 * S * Hq * d * 2 + pages * 4 + S * 4
    if lse:
        b += 4 * S * Hq
    return b


def decode_flops(seq_lens, Hq: int, d: int) -> float:
    return 4.0 * float(np.asarray(seq_lens, dtype=np.int64).clip(min=0).sum()) * Hq * d


def score_matrix_elements(N: int) -> int:
    return N * N


def score_matrix_bytes(N: int, heads: int = 1, dtype_size: int = 2) -> int:
    return N * N * heads * dtype_size


def kv_cache_bytes(num_layers: int, num_heads: int, head_dim: int, seq_len: int,
                   batch_size: int = 1, dtype_size: int = 2) -> int:
    return 2 * num_layers * num_heads * head_dim * seq_len * batch_size * dtype_size
