"""Parity of the split-KV paged decode (attn_paged_decode through the C ABI) with the
fp64 oracle, bit-exact gather, device-side clamping, and the bounded-wait self-test."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from gpu_util import bf16_to_f64, parity, to_dev
from tiled_attention_17_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_attention_17_b200 import binding
    binding.load()
    return torch


def small_paged(num_seqs, Hq, Hkv, d, page_size, lens, seed, extra_pages=5):
    cfg = inputs.DecodeConfig("small", num_seqs, Hq, Hkv, d, page_size, 1, max(max(lens), 1))
    return inputs.paged_inputs(cfg, seed=seed, seq_lens=np.array(lens, dtype=np.int32), extra_pages=extra_pages)


def to_dev_paged(torch, inp):
    return (to_dev(inp.q), to_dev(inp.k_cache), to_dev(inp.v_cache),
            torch.from_numpy(inp.block_table).cuda(), torch.from_numpy(inp.seq_lens).cuda())


def run_decode(torch, inp, scale=None):
    from tiled_attention_17_b200 import binding
    q, kc, vc, bt, sl = to_dev_paged(torch, inp)
    o, lse, ws = binding.paged_decode(q, kc, vc, bt, sl, scale)
    torch.cuda.synchronize()
    return o, lse, ws


def check_decode(torch, inp, what, scale=None):
    o, lse, ws = run_decode(torch, inp, scale)
    o_ref, lse_ref = oracle.paged_decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.seq_lens, scale)
    res = parity(bf16_to_f64(o), o_ref, lse.cpu().numpy(), lse_ref, what)
    from tiled_attention_17_b200 import binding
    code, flags = binding.attn_paged_decode_check(ws)
    assert code == 0 and flags == 0, (code, flags)
    return res


DECODE_CASES = [
    # num_seqs, Hq, Hkv, d, page_size, lens
    (5, 8, 2, 128, 16, [1, 15, 16, 17, 300]),
    (4, 32, 8, 128, 16, [64, 65, 1000, 2049]),
    (3, 4, 4, 128, 16, [33, 700, 5]),           # G = 1
    (3, 4, 2, 64, 16, [33, 700, 5]),            # G = 2, d = 64
    (2, 16, 2, 128, 16, [257, 1500]),            # G = 8
    (3, 8, 2, 128, 8, [9, 500, 1030]),           # page 8
    (3, 8, 2, 128, 32, [31, 97, 1100]),          # page 32
    (3, 8, 2, 128, 64, [1, 64, 1500]),           # page 64
    (2, 8, 2, 64, 64, [3, 130]),
]


@pytest.mark.parametrize("S,Hq,Hkv,d,ps,lens", DECODE_CASES)
def test_decode_parity_small(torch_cuda, S, Hq, Hkv, d, ps, lens):
    inp = small_paged(S, Hq, Hkv, d, ps, lens, seed=sum(lens) + ps + d)
    check_decode(torch_cuda, inp, f"{S, Hq, Hkv, d, ps, lens}")


def test_decode_zero_length(torch_cuda):
    inp = small_paged(3, 8, 2, 128, 16, [0, 40, 0], seed=1)
    o, lse, _ = run_decode(torch_cuda, inp)
    o_ref, lse_ref = oracle.paged_decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.seq_lens)
    parity(bf16_to_f64(o), o_ref, lse.cpu().numpy(), lse_ref, "zero length")
    assert np.all(bf16_to_f64(o)[0] == 0) and np.all(np.isneginf(lse.cpu().numpy()[0]))


def test_decode_long_split_merge(torch_cuda):
    # lengths spanning many splits, including split-boundary (2048-token splits)
    # and chunk-boundary lengths
    lens = [1024, 2048, 2049, 4095, 8193]
    inp = small_paged(len(lens), 8, 2, 128, 16, lens, seed=2)
    check_decode(torch_cuda, inp, "long split merge")


GATHER_CASES = [
    # page_size, d, lens: partial last pages, lengths that span several splits
    # (a split is 2048 tokens, 256 pages at page 8) and the split boundaries
    (8, 128, [1, 37, 513, 2050]),
    (16, 128, [1, 37, 2048, 2049, 5000]),
    (32, 128, [31, 33, 4200]),
    (64, 128, [70, 1, 4097]),
    (8, 64, [5, 200, 600]),
    (64, 64, [130]),
]


@pytest.mark.parametrize("ps,d,lens", GATHER_CASES)
def test_gather_bit_exact(torch_cuda, ps, d, lens):
    """The gathered logical K/V rows equal the oracle's explicitly gathered rows
    bit for bit.  attn_paged_gather_debug runs the decode kernels' own
    split-table load and chunk copies (both decode split kernels use them)."""
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    Hkv = 2
    inp = small_paged(len(lens), 4 * Hkv, Hkv, d, ps, lens, seed=ps + d + len(lens))
    q, kc, vc, bt, sl = to_dev_paged(torch, inp)
    max_pages = inp.block_table.shape[1]
    binding.ta_device_status(reset=True)
    for s in range(len(lens)):
        for h in range(Hkv):
            ko = torch.zeros((max_pages * ps, d), dtype=torch.bfloat16, device="cuda")
            vo = torch.zeros_like(ko)
            binding.attn_paged_gather_debug(kc, vc, bt, sl, s, h, ps, Hkv, d, max_pages,
                                            inp.k_cache.shape[0], ko, vo)
            torch.cuda.synchronize()
            kr, vr = oracle.paged_gather(inp.k_cache, inp.v_cache, inp.block_table, inp.seq_lens, s, h)
            L = lens[s]
            kg = ko[:L].cpu().view(torch.int16).numpy().view(np.uint16)
            vg = vo[:L].cpu().view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(kg, kr) and np.array_equal(vg, vr), (ps, d, s, h)
            # rows past the sequence are never written
            assert torch.all(ko[L:] == 0) and torch.all(vo[L:] == 0)
    code, flags = binding.ta_device_status(reset=True)
    assert code == 0 and flags == 0


@pytest.mark.parametrize("ps", [8, 16, 32, 64])
def test_gather_bad_entry_clamped_bit_exact(torch_cuda, ps):
    """A table entry outside the pool is never dereferenced: its page reads as
    physical page 0 (bit-exact against the oracle's gather through the same
    table with that entry replaced by 0) and the status word is flagged."""
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    d, Hkv, L = 128, 2, 5 * ps + 3
    inp = small_paged(1, 8, Hkv, d, ps, [L], seed=40 + ps)
    bad = inp.block_table.copy()
    bad[0, 2] = inp.num_pages_total + 11
    fixed = bad.copy()
    fixed[0, 2] = 0
    kc, vc = to_dev(inp.k_cache), to_dev(inp.v_cache)
    bt, sl = torch.from_numpy(bad).cuda(), torch.from_numpy(inp.seq_lens).cuda()
    max_pages = bad.shape[1]
    binding.ta_device_status(reset=True)
    for h in range(Hkv):
        ko = torch.zeros((max_pages * ps, d), dtype=torch.bfloat16, device="cuda")
        vo = torch.zeros_like(ko)
        binding.attn_paged_gather_debug(kc, vc, bt, sl, 0, h, ps, Hkv, d, max_pages, inp.num_pages_total, ko, vo)
        torch.cuda.synchronize()
        kr, vr = oracle.paged_gather(inp.k_cache, inp.v_cache, fixed, inp.seq_lens, 0, h)
        assert np.array_equal(ko[:L].cpu().view(torch.int16).numpy().view(np.uint16), kr)
        assert np.array_equal(vo[:L].cpu().view(torch.int16).numpy().view(np.uint16), vr)
    code, flags = binding.ta_device_status(reset=True)
    assert binding.STATUS_NAMES[code] == "TA_ERR_BAD_BLOCK_TABLE" and flags & binding.TA_DEV_BAD_BLOCK_TABLE


def test_decode_cross_entry_identity_table(torch_cuda):
    """Decode over an identity block table equals attn_fwd with Nq = 1 on the same K/V."""
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    ps, d, Hq, Hkv, L = 16, 128, 8, 2, 1000
    rng = np.random.Generator(np.random.PCG64(6))
    kf = inputs.f32_to_bf16_bits(rng.standard_normal((1, Hkv, L, d)).astype(np.float32))
    vf = inputs.f32_to_bf16_bits(rng.standard_normal((1, Hkv, L, d)).astype(np.float32))
    qf = inputs.f32_to_bf16_bits(rng.standard_normal((1, Hq, 1, d)).astype(np.float32))
    npg = (L + ps - 1) // ps
    pool_k = np.zeros((npg, Hkv, ps, d), dtype=np.uint16)
    pool_v = np.zeros_like(pool_k)
    for p in range(npg):
        rows = slice(p * ps, min(L, (p + 1) * ps))
        n = rows.stop - rows.start
        pool_k[p, :, :n] = kf[0, :, rows]
        pool_v[p, :, :n] = vf[0, :, rows]
    table = np.arange(npg, dtype=np.int32)[None, :]
    q_dec = qf[:, :, 0, :]
    o1, l1, _ = binding.paged_decode(to_dev(q_dec), to_dev(pool_k), to_dev(pool_v),
                                     torch.from_numpy(table).cuda(),
                                     torch.tensor([L], dtype=torch.int32, device="cuda"))
    o2, l2 = binding.attention(to_dev(qf), to_dev(kf), to_dev(vf), False)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn(qf, kf, vf, False)
    parity(bf16_to_f64(o1), o_ref[:, :, 0], l1.cpu().numpy(), lse_ref[:, :, 0], "decode identity table")
    parity(bf16_to_f64(o2), o_ref, l2.cpu().numpy(), lse_ref, "attn_fwd Nq=1")
    assert np.max(np.abs(bf16_to_f64(o1) - bf16_to_f64(o2)[:, :, 0])) <= 2e-2


def test_decode_bad_table_is_clamped_and_flagged(torch_cuda):
    """Out-of-range table entries and lengths: the kernel clamps them (never
    dereferences them) and reports through the checked mode."""
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    inp = small_paged(3, 8, 2, 128, 16, [40, 100, 20], seed=3)
    inp.block_table[1, 2] = inp.num_pages_total + 7
    inp.block_table[2, 0] = -3
    q, kc, vc, bt, sl = to_dev_paged(torch, inp)
    o, lse, ws = binding.paged_decode(q, kc, vc, bt, sl)
    code, flags = binding.attn_paged_decode_check(ws)
    assert binding.STATUS_NAMES[code] == "TA_ERR_BAD_BLOCK_TABLE"
    assert flags & binding.TA_DEV_BAD_BLOCK_TABLE
    # sequence 0 is untouched by the bad entries
    o_ref, lse_ref = oracle.paged_decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.seq_lens, seqs=[0])
    parity(bf16_to_f64(o[:1]), o_ref, lse[:1].cpu().numpy(), lse_ref, "good sequence next to bad ones")
    # a length beyond max_pages * page_size is clamped and flagged
    sl2 = torch.tensor([40, 100, inp.block_table.shape[1] * 16 + 5], dtype=torch.int32, device="cuda")
    inp.block_table[1, 2] = 0
    inp.block_table[2, 0] = 0
    bt2 = torch.from_numpy(inp.block_table).cuda()
    _, _, ws2 = binding.paged_decode(q, kc, vc, bt2, sl2)
    code, flags = binding.attn_paged_decode_check(ws2)
    assert flags & binding.TA_DEV_BAD_SEQ_LEN
    # a clean call afterwards reports nothing
    inp2 = small_paged(2, 8, 2, 128, 16, [40, 100], seed=4)
    _, _, ws3 = run_decode(torch, inp2)
    assert binding.attn_paged_decode_check(ws3) == (0, 0)


def test_decode_deterministic(torch_cuda):
    inp = small_paged(4, 32, 8, 128, 16, [3000, 17, 900, 5000], seed=5)
    o1, l1, _ = run_decode(torch_cuda, inp)
    o2, l2, _ = run_decode(torch_cuda, inp)
    assert torch_cuda.equal(o1, o2) and torch_cuda.equal(l1, l2)


def test_bounded_wait_selftest(torch_cuda):
    """A wait nothing completes gives up after its limit, sets the timeout bit,
    and leaves the context usable."""
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    binding.ta_device_status(reset=True)
    assert binding.ta_selftest_bounded_wait(2000) == 0
    code, flags = binding.ta_device_status(reset=True)
    assert binding.STATUS_NAMES[code] == "TA_ERR_DEVICE_TIMEOUT" and flags & binding.TA_DEV_TIMEOUT
    inp = small_paged(2, 8, 2, 128, 16, [40, 100], seed=6)
    check_decode(torch, inp, "after timeout self-test")
    assert binding.ta_device_status(reset=True) == (0, 0)


@pytest.mark.parametrize("seed_offset", [0, 1, 2])
def test_decode_full_size_sampled(torch_cuda, seed_offset):
    """The full decode workload (64 sequences, lengths 512..32768) in the
    benchmark's launch configuration, three seeds (the config's own and two
    more); sampled sequences vs the oracle."""
    torch = torch_cuda
    inp = inputs.paged_inputs(inputs.DECODE_CONFIG, seed=inputs.CONFIG_SEEDS["decode"] + 1000 * seed_offset)
    o, lse, ws = run_decode(torch, inp)
    lens = inp.seq_lens
    pick = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 0, 31, 63, 17})
    o_ref, lse_ref = oracle.paged_decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.seq_lens, seqs=pick)
    parity(bf16_to_f64(o[pick]), o_ref, lse[pick].cpu().numpy(), lse_ref, "full decode sampled")
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    from tiled_attention_17_b200 import binding
    assert binding.attn_paged_decode_check(ws) == (0, 0)
