"""attn_paged_decode_noalloc: paged decode for callers that cannot allocate
device memory (for example a plugin inside a framework that owns all device
memory and passes in only inputs and outputs, or a latency-critical path that
cannot afford cudaMalloc's implicit synchronisation).  The entry point uses the
library's fixed scratch array instead of a caller workspace.

Checked here through the C ABI on two calls in a row (the second call reuses
the scratch the first one left behind):
  * against the workspace entry point (attn_paged_decode) on the same inputs:
    both run the same plan, kernels and deterministic split reduction, so the
    outputs must be bitwise equal;
  * against the fp64 oracle at the parity tolerances of the other tests.
The file is named to be collected last.
"""
import numpy as np
import pytest

import oracle
from gpu_util import bf16_to_f64, parity, to_dev
from tiled_attention_17_b200 import inputs

pytestmark = pytest.mark.gpu


def _paged(seed, lens):
    cfg = inputs.DecodeConfig("noalloc", len(lens), 32, 8, 128, 16, 1, max(lens))
    return inputs.paged_inputs(cfg, seed=seed, seq_lens=np.array(lens, dtype=np.int32), extra_pages=4)


def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_attention_17_b200 import binding
    binding.load()
    cases = []
    for seed, lens in [(31, [3000, 17, 0, 5000, 1024]), (32, [40, 7000, 513])]:
        inp = _paged(seed, lens)
        dev = dict(q=to_dev(inp.q), kc=to_dev(inp.k_cache), vc=to_dev(inp.v_cache),
                   bt=torch.from_numpy(inp.block_table).cuda(), sl=torch.from_numpy(inp.seq_lens).cuda())
        S, Hq, d = inp.q.shape
        shape = dict(S=S, Hq=Hq, d=d, Hkv=inp.k_cache.shape[1], ps=inp.k_cache.shape[2],
                     mp=inp.block_table.shape[1], P=inp.k_cache.shape[0], scale=d ** -0.5)
        ref_o, ref_l, _ = binding.paged_decode(dev["q"], dev["kc"], dev["vc"], dev["bt"], dev["sl"], shape["scale"])
        cases.append((inp, dev, shape, ref_o, ref_l))
    torch.cuda.synchronize()
    outs = []
    for _, dev, sh, _, _ in cases:          # two no-alloc calls in a row, sharing the scratch
        o = torch.empty_like(dev["q"])
        lse = torch.empty((sh["S"], sh["Hq"]), dtype=torch.float32, device="cuda")
        binding.attn_paged_decode_noalloc(dev["q"], dev["kc"], dev["vc"], dev["bt"], dev["sl"], sh["ps"], sh["S"],
                                          sh["Hq"], sh["Hkv"], sh["d"], sh["mp"], sh["P"], sh["scale"], o, lse)
        outs.append((o, lse))
    torch.cuda.synchronize()
    for (o, lse), (inp, _, sh, ref_o, ref_l) in zip(outs, cases):
        # the same kernels on the same inputs: bitwise equal (-inf lse included)
        assert torch.equal(o.view(torch.int16), ref_o.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), ref_l.view(torch.int32))
        o_ref, lse_ref = oracle.paged_decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.seq_lens,
                                             sh["scale"])
        parity(bf16_to_f64(o), o_ref, lse.cpu().numpy(), lse_ref, "no-alloc decode vs oracle")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_attention_17_b200 import binding
    binding.load()
    # 4096 sequences x 32 heads x 32 splits of partials need far more than 64 MiB
    need = binding.attn_paged_decode_workspace_size(4096, 32, 8, 128, 2048, 16)
    assert need > 64 << 20
    code = binding.attn_paged_decode_noalloc(256, 256, 256, 256, 256, 16, 4096, 32, 8, 128, 2048, 100,
                                             0.1, 256, None, check=False)
    assert binding.STATUS_NAMES[code] == "TA_ERR_UNSUPPORTED"
    assert "scratch" in binding.ta_last_error()
