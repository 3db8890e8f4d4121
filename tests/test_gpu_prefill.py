"""Parity of the fused prefill kernel (attn_fwd through the C ABI) with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from gpu_util import bf16_to_f64, parity, sample_rows, to_dev
from tiled_attention_17_b200 import inputs
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


def run_fwd(torch, q, k, v, causal, scale=None):
    from tiled_attention_17_b200 import binding
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o, lse = binding.attention(qd, kd, vd, causal, scale)
    torch.cuda.synchronize()
    return o, lse


def check_full(torch, q, k, v, causal, scale=None, what=""):
    o, lse = run_fwd(torch, q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attn(q, k, v, causal, scale=scale)
    return parity(bf16_to_f64(o), o_ref, lse.cpu().numpy(), lse_ref, what)


CASES = [
    # B, Hq, Hkv, Nq, Nkv, d, causal
    (1, 1, 1, 256, 256, 64, False),       # tiny config
    (1, 1, 1, 256, 256, 64, True),
    (1, 2, 2, 640, 640, 128, False),      # ragged last query pair (tile 1 empty)
    (1, 2, 2, 640, 640, 128, True),
    (1, 2, 2, 200, 333, 128, True),       # Nq < Nkv, ragged K/V tile, bottom-right mask
    (1, 2, 2, 200, 333, 128, False),
    (2, 8, 2, 384, 384, 128, True),       # GQA group 4
    (1, 4, 1, 130, 130, 64, True),        # GQA group 4, d = 64, ragged
    (1, 4, 2, 700, 900, 128, True),       # GQA group 2: head-paired tiles, Nq < Nkv
    (1, 6, 2, 333, 333, 128, True),       # GQA group 3: consecutive-tile pairs
    (1, 1, 1, 1, 700, 128, False),        # one query row
    (1, 1, 1, 1, 700, 128, True),
    (1, 1, 1, 513, 129, 128, False),
    # more CTAs than SMs, several waves
    (2, 40, 8, 512, 512, 128, True),
    (1, 64, 16, 600, 200, 128, True),     # items with no visible key mixed in
    (2, 40, 40, 384, 384, 64, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nkv,d,causal", CASES)
def test_prefill_parity_small(torch_cuda, B, Hq, Hkv, Nq, Nkv, d, causal):
    q, k, v = random_prefill(B, Hq, Hkv, Nq, Nkv, d, seed=Nq * 7 + Nkv + d + causal)
    check_full(torch_cuda, q, k, v, causal, what=f"{B, Hq, Hkv, Nq, Nkv, d, causal}")


def test_prefill_fully_masked_rows(torch_cuda):
    # Nq > Nkv with bottom-right causal alignment: the first Nq - Nkv rows see no key
    q, k, v = random_prefill(1, 2, 1, 300, 100, 128, seed=3)
    o, lse = run_fwd(torch_cuda, q, k, v, True)
    o_ref, lse_ref = oracle.attn(q, k, v, True)
    parity(bf16_to_f64(o), o_ref, lse.cpu().numpy(), lse_ref, "fully masked rows")
    assert np.all(bf16_to_f64(o)[:, :, :200] == 0.0)
    assert np.all(np.isneginf(lse.cpu().numpy()[:, :, :200]))


def test_prefill_sharp_peaks(torch_cuda):
    # every 64th key row x4: large score gaps exercise the rescale path
    cfg = inputs.PrefillConfig("peaks", 1, 2, 2, 1024, 1024, 128, False, 64, 4.0)
    q, k, v = inputs.prefill_inputs(cfg, seed=99)
    check_full(torch_cuda, q, k, v, False, what="sharp peaks")


def test_prefill_large_scores_rescale(torch_cuda):
    # keys grow along the sequence so the running max rises on almost every tile
    rng = np.random.Generator(np.random.PCG64(5))
    N, d = 1024, 128
    q = f32_to_bf16_bits(np.abs(rng.standard_normal((1, 1, N, d))).astype(np.float32))
    ramp = np.linspace(0.2, 3.0, N, dtype=np.float32)[None, None, :, None]
    k = f32_to_bf16_bits((np.abs(rng.standard_normal((1, 1, N, d))) * ramp).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((1, 1, N, d)).astype(np.float32))
    check_full(torch_cuda, q, k, v, False, what="rising max")
    check_full(torch_cuda, q, k, v, True, what="rising max causal")


def test_prefill_special_cases(torch_cuda):
    # single key: O = v_0 (exactly representable), lse = scale q.k_0
    q, k, v = random_prefill(1, 2, 2, 129, 1, 128, seed=8)
    o, lse = run_fwd(torch_cuda, q, k, v, False)
    o_ref, lse_ref = oracle.attn(q, k, v, False)
    parity(bf16_to_f64(o), o_ref, lse.cpu().numpy(), lse_ref, "single key")
    assert np.array_equal(bf16_to_f64(o), np.broadcast_to(o_ref, o.shape))
    # scale 0: uniform weights over visible keys
    q, k, v = random_prefill(1, 1, 1, 300, 300, 128, seed=9)
    check_full(torch_cuda, q, k, v, True, scale=0.0, what="scale 0 causal")
    check_full(torch_cuda, q, k, v, False, scale=0.0, what="scale 0")
    # causal row 0 returns v_0 exactly
    o, _ = run_fwd(torch_cuda, q, k, v, True)
    assert np.array_equal(bf16_to_f64(o)[0, 0, 0], inputs.bf16_bits_to_f32(v[0, 0, 0]).astype(np.float64))


def test_prefill_empty_shapes(torch_cuda):
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    q = torch.zeros((1, 2, 0, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 2, 5, 128), dtype=torch.bfloat16, device="cuda")
    o, lse = binding.attention(q, k, k, True)         # Nq = 0: nothing to do
    assert o.numel() == 0
    q = torch.ones((1, 2, 7, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 2, 0, 128), dtype=torch.bfloat16, device="cuda")
    o = torch.full_like(q, 3.0)
    lse = torch.zeros((1, 2, 7), dtype=torch.float32, device="cuda")
    binding.attention(q, k, k, False, out=o, lse=lse)  # Nkv = 0: O = 0, lse = -inf
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_prefill_deterministic(torch_cuda):
    q, k, v = random_prefill(1, 4, 2, 1000, 1000, 128, seed=4)
    o1, l1 = run_fwd(torch_cuda, q, k, v, True)
    o2, l2 = run_fwd(torch_cuda, q, k, v, True)
    assert torch_cuda.equal(o1, o2) and torch_cuda.equal(l1, l2)


def test_prefill_bad_args_do_not_launch(torch_cuda):
    from tiled_attention_17_b200 import binding
    torch = torch_cuda
    q = torch.zeros((1, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    code = binding.attn_fwd(q, q, q, q, None, 1, 3, 2, 16, 16, 128, 0.1, 0, check=False)
    assert binding.STATUS_NAMES[code] == "TA_ERR_INVALID_ARG"
    code = binding.attn_fwd(q, q, q, q, None, 1, 1, 1, 16, 16, 96, 0.1, 0, check=False)
    assert binding.STATUS_NAMES[code] == "TA_ERR_UNSUPPORTED"


@pytest.mark.parametrize("seed_offset", [0, 1, 2])
@pytest.mark.parametrize("name", ["causal", "long", "gqa"])
def test_prefill_full_size_sampled(torch_cuda, name, seed_offset):
    """Full-size workloads in the benchmark's launch configuration, three seeds
    each (the config's own and two more); sampled rows vs the oracle."""
    cfg = inputs.PREFILL_CONFIGS[name]
    q, k, v = inputs.prefill_inputs(cfg, seed=inputs.CONFIG_SEEDS[name] + 1000 * seed_offset)
    o, lse = run_fwd(torch_cuda, q, k, v, cfg.causal, cfg.scale)
    rng = np.random.Generator(np.random.PCG64(77))
    rows = sample_rows(cfg.B, cfg.Hq, cfg.Nq, 384, rng)
    o_ref, lse_ref = oracle.attn(q, k, v, cfg.causal, scale=cfg.scale, rows=rows)
    og = o.view(-1, cfg.d)[torch_cuda.from_numpy(rows).cuda()]
    lg = lse.view(-1)[torch_cuda.from_numpy(rows).cuda()]
    parity(bf16_to_f64(og), o_ref, lg.cpu().numpy(), lse_ref, f"{name} sampled")
    # properties that hold at any size: finite outputs, lse at least the largest visible score bound
    assert torch_cuda.isfinite(o.float()).all()
    assert torch_cuda.isfinite(lse).all()
