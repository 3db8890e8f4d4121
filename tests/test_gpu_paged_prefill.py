"""Parity of varlen prefill over the paged KV cache (attn_paged_prefill through
the C ABI) with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from gpu_util import bf16_to_f64, parity, to_dev
from tiled_attention_17_b200.inputs import paged_prefill_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_attention_17_b200 import binding
    binding.load()
    return torch


def run(torch, inp, causal, scale=None):
    from tiled_attention_17_b200 import binding
    dev_i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    o, lse = binding.paged_prefill(to_dev(inp.q), to_dev(inp.k_cache), to_dev(inp.v_cache),
                                   dev_i32(inp.block_table), dev_i32(inp.cu_seqlens), dev_i32(inp.seq_lens),
                                   inp.max_q_len, causal, scale)
    torch.cuda.synchronize()
    return o, lse


def check(torch, inp, causal, what, seqs=None):
    o, lse = run(torch, inp, causal)
    o_ref, lse_ref = oracle.paged_prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.cu_seqlens,
                                          inp.seq_lens, causal, seqs=seqs)
    rows = np.arange(inp.q.shape[0])
    if seqs is not None:
        rows = np.concatenate([np.arange(inp.cu_seqlens[s], inp.cu_seqlens[s + 1]) for s in seqs])
    return parity(bf16_to_f64(o)[rows], o_ref[rows], lse.cpu().numpy()[rows], lse_ref[rows], what)


CASES = [
    # q_lens, kv_lens, Hq, Hkv, d, page_size
    ([1, 100, 300, 257, 5], [1, 612, 300, 900, 5], 4, 2, 128, 16),     # chunked prefill: prefix + new tokens
    ([128, 129, 256, 0, 3], [128, 300, 1000, 70, 3], 2, 2, 128, 8),    # tile edges, an empty sequence
    ([200, 77], [333, 77], 8, 2, 128, 32),                             # GQA group 4
    ([64, 512], [64, 700], 2, 1, 64, 64),                              # d = 64, 64-token pages
    ([300], [200], 2, 2, 128, 16),                                     # more queries than keys: masked rows
    ([300, 5, 700], [300, 900, 1200], 6, 2, 128, 16),                  # GQA group 3: consecutive-tile pairs
    ([150, 400], [500, 900], 4, 1, 128, 64),                           # d = 128, 64-token pages
]


@pytest.mark.parametrize("q_lens,kv_lens,Hq,Hkv,d,ps", CASES)
@pytest.mark.parametrize("causal", [True, False])
def test_paged_prefill_parity(torch_cuda, q_lens, kv_lens, Hq, Hkv, d, ps, causal):
    inp = paged_prefill_inputs(q_lens, kv_lens, Hq, Hkv, d, ps, seed=sum(q_lens) + ps)
    check(torch_cuda, inp, causal, f"{q_lens} {kv_lens} {Hq}/{Hkv} d{d} p{ps} c={causal}")


@pytest.mark.parametrize("ps", [8, 16, 32, 64])
def test_paged_prefill_equals_dense_bitwise(torch_cuda, ps):
    # one sequence whose pages are in order is the dense prefill of its rows:
    # the same arithmetic on the same values, so the same bits (at every page
    # size: each lands its K and V pages in its own shared-memory layout)
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    Hq, Hkv, d, n = 4, 2, 128, 700
    inp = paged_prefill_inputs([n], [n], Hq, Hkv, d, ps, seed=5, extra_pages=0)
    npages = (n + ps - 1) // ps
    inp.block_table[0, :npages] = np.arange(npages, dtype=np.int32)   # pages in order
    o, lse = run(torch, inp, True)
    k = inp.k_cache.transpose(1, 0, 2, 3).reshape(Hkv, npages * ps, d)[:, :n][None]
    v = inp.v_cache.transpose(1, 0, 2, 3).reshape(Hkv, npages * ps, d)[:, :n][None]
    q = np.ascontiguousarray(inp.q.transpose(1, 0, 2))[None]
    od, ld = binding.attention(to_dev(q), to_dev(np.ascontiguousarray(k)), to_dev(np.ascontiguousarray(v)), True)
    torch.cuda.synchronize()
    assert torch.equal(o, od[0].transpose(0, 1).contiguous())
    assert torch.equal(lse, ld[0].transpose(0, 1).contiguous())


def test_paged_prefill_bad_table_entry_is_flagged(torch_cuda):
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    binding.ta_device_status(True)
    inp = paged_prefill_inputs([50, 40], [300, 40], 2, 2, 128, 16, seed=6)
    inp.block_table[0, 3] = 10 ** 6          # outside the pool: clamped, never read
    o, _ = run(torch, inp, True)
    code, flags = binding.ta_device_status(True)
    assert flags & binding.TA_DEV_BAD_BLOCK_TABLE
    assert np.all(np.isfinite(bf16_to_f64(o)))
    # the untouched sequence is still exact
    check(torch, inp, True, "after bad entry", seqs=[1])
    binding.ta_device_status(True)


def test_paged_prefill_serving_mix_sampled(torch_cuda):
    # a serving-like batch: 32 sequences, 1-2048 new tokens after a 0-8192 prefix
    rng = np.random.Generator(np.random.PCG64(1234))
    q_lens = rng.integers(1, 2048, size=32, endpoint=True)
    kv_lens = q_lens + rng.integers(0, 8192, size=32, endpoint=True)
    inp = paged_prefill_inputs(q_lens, kv_lens, 32, 8, 128, 16, seed=77)
    check(torch_cuda, inp, True, "serving mix", seqs=[0, int(np.argmax(q_lens)), 31])


def test_paged_prefill_page_tails_hold_huge_finite_values(torch_cuda):
    # Keys are read a page at a time: the rows of a sequence's last page past
    # its length are loaded and given exactly zero weight (their scores are
    # masked to -inf before the row max).  Any finite values there, even the
    # largest bf16 ones, leave the result unchanged.
    import dataclasses
    ps = 16
    inp = paged_prefill_inputs([50, 77, 3], [300, 77, 40], 4, 2, 128, ps, seed=8)
    k, v = inp.k_cache.copy(), inp.v_cache.copy()
    big = np.array([0x7F7F, 0xFF7F], dtype=np.uint16)   # +-3.39e38, the largest finite bf16
    for sq, n in enumerate(inp.seq_lens):
        if n % ps:
            page = inp.block_table[sq, n // ps]
            tail = np.resize(big, k[page, :, n % ps:, :].shape)
            k[page, :, n % ps:, :] = tail
            v[page, :, n % ps:, :] = tail[..., ::-1]
    huge = dataclasses.replace(inp, k_cache=k, v_cache=v)
    for causal in (True, False):
        check(torch_cuda, huge, causal, f"huge finite page tails causal={causal}")

