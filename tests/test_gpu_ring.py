"""The log-sum-exp merge kernels and the ring schedule on one GPU (the ranks
emulated in one process), against the fp64 oracle."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from gpu_util import bf16_to_f64, parity, to_dev
from tiled_attention_17_b200.inputs import f32_to_bf16_bits, random_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_attention_17_b200 import binding
    binding.load()
    return torch


@pytest.mark.parametrize("B,Hq,Hkv,N,d,shards", [(1, 4, 2, 1024, 128, 4), (2, 2, 2, 900, 128, 3),
                                                 (1, 8, 2, 512, 64, 2)])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
def test_ring_emulated_matches_whole_sequence(torch_cuda, B, Hq, Hkv, N, d, shards, causal, layout):
    from tiled_attention_17_b200 import ring
    q, k, v = random_prefill(B, Hq, Hkv, N, N, d, seed=N + shards)
    o, lse = ring.ring_attention_emulated(to_dev(q), to_dev(k), to_dev(v), shards, causal, layout=layout)
    torch_cuda.cuda.synchronize()
    o_ref, lse_ref = oracle.attn(q, k, v, causal)
    parity(bf16_to_f64(o), o_ref, lse.cpu().numpy(), lse_ref, f"ring {layout} {B, Hq, Hkv, N, d, shards, causal}")


def test_merge_of_key_halves(torch_cuda):
    # attention over keys [0, 300) and [300, 700) separately (oracle, rounded
    # to bf16 / fp32 as attn_fwd would return them), merged on the GPU, equals
    # attention over all 700 keys; rows that see no key of the second half
    # (causal) carry lse = -inf there
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    q, k, v = random_prefill(1, 2, 2, 700, 700, 128, seed=11)
    o1, l1 = oracle.attn(q, k[:, :, :300], v[:, :, :300], False)
    o2, l2 = oracle.attn(q, k[:, :, 300:], v[:, :, 300:], True)   # bottom-right: row i sees keys 300..i
    rows, d = 2 * 700, 128
    acc_o = torch.empty((rows, d), dtype=torch.float32, device="cuda")
    acc_l = torch.empty(rows, dtype=torch.float32, device="cuda")
    for first, (o_p, l_p) in ((1, (o1, l1)), (0, (o2, l2))):
        op = to_dev(f32_to_bf16_bits(o_p.reshape(rows, d).astype(np.float32)))
        lp = torch.from_numpy(l_p.reshape(rows).astype(np.float32)).cuda()
        binding.attn_lse_merge(acc_o, acc_l, op, lp, rows, d, first)
    out = torch.empty((rows, d), dtype=torch.bfloat16, device="cuda")
    binding.attn_lse_merge_finish(acc_o, out, rows, d)
    torch.cuda.synchronize()
    # reference: the first 300 keys fully visible, then keys 300.. causally (row i sees up to i)
    o_ref = np.zeros((1, 2, 700, d))
    l_ref = np.zeros((1, 2, 700))
    from online_model import brute_row, widen
    for h in range(2):
        for i in range(0, 700, 37):
            vis = np.arange(700) < 300
            vis |= (np.arange(700) >= 300) & (np.arange(700) - 300 <= i - (700 - 400))
            o_r, l_r = brute_row(widen(q[0, h, i]), widen(k[0, h][vis]), widen(v[0, h][vis]), 128 ** -0.5, int(vis.sum()))
            o_ref[0, h, i], l_ref[0, h, i] = o_r, l_r
    sel = np.arange(0, 700, 37)
    og = bf16_to_f64(out).reshape(1, 2, 700, d)[:, :, sel]
    lg = acc_l.cpu().numpy().reshape(1, 2, 700)[:, :, sel]
    parity(og, o_ref[:, :, sel], lg, l_ref[:, :, sel], "merge of halves")


def test_merge_both_empty(torch_cuda):
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    rows, d = 64, 64
    acc_o = torch.full((rows, d), 7.0, dtype=torch.float32, device="cuda")
    acc_l = torch.full((rows,), float("-inf"), dtype=torch.float32, device="cuda")
    part = torch.ones((rows, d), dtype=torch.bfloat16, device="cuda")
    lp = torch.full((rows,), float("-inf"), dtype=torch.float32, device="cuda")
    binding.attn_lse_merge(acc_o, acc_l, part, lp, rows, d, 0)
    torch.cuda.synchronize()
    assert torch.all(acc_o == 0) and torch.all(torch.isneginf(acc_l))
