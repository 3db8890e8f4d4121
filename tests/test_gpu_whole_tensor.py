"""Whole-tensor parity at the full workload sizes: every output row of each
prefill configuration (tiny, causal, long, gqa) through attn_fwd, and every
sequence of the paged decode workload through attn_paged_decode, against the
fp64 oracle, in the launch configuration bench.py times (the same calls,
shapes, seeds and workspace sizing).  The metrics are taken over the whole
tensor: max-abs and relative L2 of O, max absolute error of lse.

The oracle evaluates all rows on the host cores (about a minute in total on
16 cores); the outputs of the GPU are copied back once per configuration.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from gpu_util import bf16_to_f64, parity, to_dev
from tiled_attention_17_b200 import inputs

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_attention_17_b200 import binding
    binding.load()
    return torch


@pytest.mark.parametrize("name", ["tiny", "causal", "long", "gqa"])
def test_prefill_whole_tensor(torch_cuda, name):
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    c = inputs.PREFILL_CONFIGS[name]
    q_h, k_h, v_h = inputs.prefill_inputs(c, seed=inputs.CONFIG_SEEDS[name])
    q, k, v = to_dev(q_h), to_dev(k_h), to_dev(v_h)
    o = torch.empty_like(q)
    lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    binding.attn_fwd(q, k, v, o, lse, c.B, c.Hq, c.Hkv, c.Nq, c.Nkv, c.d, c.scale, int(c.causal), stream)
    torch.cuda.synchronize()
    og, lg = bf16_to_f64(o), lse.cpu().numpy()
    del q, k, v, o, lse
    o_ref, lse_ref = oracle.attn(q_h, k_h, v_h, c.causal, scale=c.scale)
    res = parity(og, o_ref, lg, lse_ref, f"{name} whole tensor")
    print(f"{name}: max-abs {res[0]:.3e} rel-L2 {res[1]:.3e} lse {res[2]:.3e} over {og.shape[:-1]} rows")


def test_decode_whole_tensor(torch_cuda):
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    D = inputs.DECODE_CONFIG
    inp = inputs.paged_inputs(D, seed=inputs.CONFIG_SEEDS["decode"])
    q, kc, vc = to_dev(inp.q), to_dev(inp.k_cache), to_dev(inp.v_cache)
    bt = torch.from_numpy(inp.block_table).cuda()
    sl = torch.from_numpy(inp.seq_lens).cuda()
    ws_bytes = binding.attn_paged_decode_workspace_size(D.num_seqs, D.Hq, D.Hkv, D.d, D.max_pages, D.page_size)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((D.num_seqs, D.Hq), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    binding.attn_paged_decode(q, kc, vc, bt, sl, D.page_size, D.num_seqs, D.Hq, D.Hkv, D.d, D.max_pages,
                              inp.num_pages_total, D.scale, o, lse, ws, ws_bytes, stream)
    torch.cuda.synchronize()
    assert binding.attn_paged_decode_check(ws) == (0, 0)
    og, lg = bf16_to_f64(o), lse.cpu().numpy()
    del kc, vc
    o_ref, lse_ref = oracle.paged_decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.seq_lens, D.scale)
    res = parity(og, o_ref, lg, lse_ref, "decode whole tensor")
    print(f"decode: max-abs {res[0]:.3e} rel-L2 {res[1]:.3e} lse {res[2]:.3e} over {D.num_seqs} sequences "
          f"({int(inp.seq_lens.sum())} tokens)")
