"""The oracle against its pins (CPU only)."""
import json
import os

import numpy as np
import pytest

import oracle
import oracle_pins
from tiled_attention_17_b200 import accounting

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_sizes.json")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle)


def test_fully_masked_row_reading():
    # Nq > Nkv with bottom-right causal alignment leaves the first rows with no key.
    from tiled_attention_17_b200.inputs import random_prefill
    q, k, v = random_prefill(1, 1, 1, 6, 3, 4, seed=5)
    o, lse = oracle.attn(q, k, v, True)
    assert np.all(o[0, 0, :3] == 0.0) and np.all(np.isneginf(lse[0, 0, :3]))
    assert np.all(np.isfinite(lse[0, 0, 3:]))


def test_page_size_examples():
    g = json.load(open(GOLDEN))
    e = g["score_matrix_n16384"]
    assert accounting.score_matrix_elements(e["N"]) == e["elements"]
    assert accounting.score_matrix_bytes(e["N"], 1, 2) == e["bytes_fp16_one_head"] == 512 * 2**20
    assert accounting.score_matrix_bytes(e["N"], 8, 2) == e["bytes_fp16_eight_heads"] == 4 * 2**30
    e = g["score_matrix_n8192_fp32"]
    assert accounting.score_matrix_bytes(e["N"], 1, 4) == e["bytes_fp32"] == 256 * 2**20
    e = g["score_matrix_n131072_fp32"]
    assert accounting.score_matrix_bytes(e["N"], 1, 4) == e["bytes_fp32"] == 64 * 2**30
    e = g["io_example_n4096_d128"]
    assert 3 * e["N"] * e["d"] * 2 == e["qkv_bytes_fp16"]
    assert accounting.score_matrix_bytes(e["N"], 1, 2) == e["score_bytes_fp16"] == 32 * 2**20
    e = g["flops_n8192_d128"]
    assert accounting.prefill_flops(1, 1, e["N"], e["N"], e["d"], False) == e["total_flops"] == 32 * 2**30
    assert accounting.prefill_flops(1, 1, e["N"], e["N"], e["d"], False) / 2 == e["qk_flops"]
    e = g["kv_cache_example"]
    assert accounting.kv_cache_bytes(e["num_layers"], e["num_heads"], e["head_dim"], e["seq_len"],
                                     e["batch_size"], e["dtype_size"]) == e["bytes"]
    for L, gib in g["kv_cache_context_table"]["seq_len_to_gib"].items():
        assert accounting.kv_cache_bytes(32, 32, 128, int(L)) == gib * 2**30


def test_varlen_flops_sum_of_sequences():
    assert accounting.varlen_prefill_flops([3, 0, 4], [5, 2, 4], 2, 8, True) == \
        4.0 * 2 * 8 * (accounting.visible_pairs(3, 5, True) + 0 + 4 * 5 // 2)
    assert accounting.varlen_prefill_flops([3, 4], [5, 4], 1, 1, False) == 4.0 * (15 + 16)


def test_visible_pairs_closed_form():
    for N in (1, 7, 256, 4096):
        assert accounting.visible_pairs(N, N, True) == N * (N + 1) // 2
        assert accounting.visible_pairs(N, N, False) == N * N
    # bottom-right alignment: Nq=2, Nkv=5 -> rows see 4 and 5 keys
    assert accounting.visible_pairs(2, 5, True) == 9
    # Nq > Nkv: first rows see nothing
    assert accounting.visible_pairs(5, 2, True) == 0 + 0 + 0 + 1 + 2
