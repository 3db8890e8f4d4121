"""Parity of the FP8 (E4M3) prefill (attn_fwd_fp8 through the C ABI) with the
fp64 oracle's exact attention of the dequantised inputs.

Two bars, both derived from the arithmetic:

* integer scores (every Q and K row holds a few +-1 entries) with scale = ln 2:
  every softmax weight relative to any score of its row is a power of two,
  which E4M3 holds exactly, so rounding P to FP8 costs nothing and the bf16
  attention bar applies unchanged (max-abs 2e-2, rel-L2 5e-3, lse 1e-3);
* N(0, 1) inputs quantised per tensor: the kernel rounds each weight to E4M3
  (3 mantissa bits, round to nearest: relative error <= 2^-4, RMS about 0.026
  over a binade).  Each output element is a weighted mean of V, so its error
  is at most 2^-4 max|V| (plus the bf16 output rounding, 2^-9 |O|), and for
  independent rounding errors the expected relative L2 error is about 0.026.
  The bar: rel-L2 <= 4e-2 over all checked rows, max-abs <= 2^-4 max|V| +
  2^-8 max|O|.  lse depends only on the scores and the unrounded sum, so it
  keeps the 1e-3 bar.
"""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
from gpu_util import LSE_ABS, bf16_to_f64, parity, sample_rows
from tiled_attention_17_b200 import inputs

pytestmark = pytest.mark.gpu

FP8_REL_L2 = 4e-2


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_attention_17_b200 import binding
    binding.load()
    return torch


def dev8(torch, codes):
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).cuda()


def run_fp8(torch, q8, k8, v8, descale, causal, scale=None):
    from tiled_attention_17_b200 import binding
    o, lse = binding.attention_fp8(dev8(torch, q8), dev8(torch, k8), dev8(torch, v8), descale, causal, scale)
    torch.cuda.synchronize()
    return bf16_to_f64(o), lse.cpu().numpy().astype(np.float64)


def fp8_bar(o, o_ref, lse, lse_ref, vmax, what):
    err = np.abs(o - o_ref)
    max_abs = float(err.max())
    rel = float(np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref))
    both = np.isneginf(lse) & np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse_ref)), f"{what}: -inf lse pattern differs"
    with np.errstate(invalid="ignore"):
        lerr = float(np.abs(np.where(both, 0.0, lse - lse_ref)).max())
    bound = vmax / 16 + np.abs(o_ref).max() / 256
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    assert max_abs <= bound, f"{what}: max-abs {max_abs:.3e} > {bound:.3e}"
    assert rel <= FP8_REL_L2, f"{what}: rel-L2 {rel:.3e} > {FP8_REL_L2}"
    assert lerr <= LSE_ABS, f"{what}: lse err {lerr:.3e} > {LSE_ABS}"
    return max_abs, rel, lerr


EXACT_CASES = [
    # B, Hq, Hkv, Nq, Nkv, causal
    (1, 2, 1, 300, 300, True),      # GQA, ragged last tile, pair with one tile
    (1, 2, 1, 300, 300, False),
    (2, 4, 2, 513, 700, True),      # Nq < Nkv (bottom-right mask), ragged K/V tile
    (1, 1, 1, 1024, 1024, True),    # several full tiles per row, both pair tiles busy
    (1, 1, 1, 1, 333, False),       # one query row
]


@pytest.mark.parametrize("case", EXACT_CASES, ids=lambda c: "x".join(map(str, c[:5])) + ("c" if c[5] else ""))
def test_fp8_integer_scores_exact(torch_cuda, case):
    B, Hq, Hkv, Nq, Nkv, causal = case
    q8, k8, v8, dv = inputs.fp8_integer_score_inputs(B, Hq, Hkv, Nq, Nkv, 128, seed=31 + Nq)
    desc = (2.0, 0.5, dv)           # q and k descales multiply to 1: the scores stay integers
    scale = math.log(2.0)
    o, lse = run_fp8(torch_cuda, q8, k8, v8, desc, causal, scale)
    o_ref, lse_ref = oracle.attn_fp8(q8, k8, v8, desc, causal, scale=scale)
    parity(o, o_ref, lse, lse_ref, f"fp8 exact {case}")


RANDOM_CASES = [
    (1, 2, 2, 640, 640, True),
    (1, 2, 2, 640, 640, False),
    (2, 8, 2, 384, 384, True),      # GQA group 4
    (1, 2, 2, 200, 333, True),
    (1, 1, 1, 2048, 2048, True),
]


@pytest.mark.parametrize("case", RANDOM_CASES, ids=lambda c: "x".join(map(str, c[:5])) + ("c" if c[5] else ""))
def test_fp8_random_parity(torch_cuda, case):
    B, Hq, Hkv, Nq, Nkv, causal = case
    q8, k8, v8, desc = inputs.random_prefill_fp8(B, Hq, Hkv, Nq, Nkv, 128, seed=41 + Nkv)
    o, lse = run_fp8(torch_cuda, q8, k8, v8, desc, causal)
    o_ref, lse_ref = oracle.attn_fp8(q8, k8, v8, desc, causal)
    vmax = float(np.abs(oracle.e4m3_decode(v8)).max()) * desc[2]
    fp8_bar(o, o_ref, lse, lse_ref, vmax, f"fp8 random {case}")


def test_fp8_full_size_sampled(torch_cuda):
    """The benchmark's FP8 workload (B=4, H=16, N=4096, d=128, causal) in the
    launch configuration bench.py times, on sampled rows."""
    B, H, N = 4, 16, 4096
    q8, k8, v8, desc = inputs.random_prefill_fp8(B, H, H, N, N, 128, seed=inputs.CONFIG_SEEDS["causal"])
    o, lse = run_fp8(torch_cuda, q8, k8, v8, desc, True)
    rng = np.random.Generator(np.random.PCG64(5))
    rows = sample_rows(B, H, N, 160, rng)
    o_ref, lse_ref = oracle.attn_fp8(q8, k8, v8, desc, True, rows=rows)
    vmax = float(np.abs(oracle.e4m3_decode(v8)).max()) * desc[2]
    fp8_bar(o.reshape(-1, 128)[rows], o_ref, lse.reshape(-1)[rows], lse_ref, vmax, "fp8 full size")


def test_fp8_no_keys(torch_cuda):
    q8, k8, v8, desc = inputs.random_prefill_fp8(1, 2, 2, 130, 1, 128, seed=3)
    from tiled_attention_17_b200 import binding
    torch = torch_cuda
    o = torch.full((1, 2, 130, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 2, 130), dtype=torch.float32, device="cuda")
    empty = torch.empty((1, 2, 0, 128), dtype=torch.uint8, device="cuda")
    binding.attn_fwd_fp8(dev8(torch, q8), empty, empty, *desc, o, lse, 1, 2, 2, 130, 0, 128, 0.1, 0)
    torch.cuda.synchronize()
    assert torch.all(o == 0).item() and torch.all(torch.isneginf(lse)).item()


def test_fp8_deterministic(torch_cuda):
    q8, k8, v8, desc = inputs.random_prefill_fp8(1, 4, 2, 700, 700, 128, seed=9)
    a = run_fp8(torch_cuda, q8, k8, v8, desc, True)
    b = run_fp8(torch_cuda, q8, k8, v8, desc, True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_fp8_all_codes(torch_cuda):
    """Q, K and V codes drawn uniformly from every finite E4M3 code (subnormals
    and +-448 included), descaled to |x| <= 1: the tensor cores must read the
    whole format as the oracle's decoder does."""
    rng = np.random.Generator(np.random.PCG64(77))
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    B, Hq, Hkv, Nq, Nkv = 1, 2, 1, 300, 300
    q8 = rng.choice(finite, size=(B, Hq, Nq, 128))
    k8 = rng.choice(finite, size=(B, Hkv, Nkv, 128))
    v8 = rng.choice(finite, size=(B, Hkv, Nkv, 128))
    desc = (1 / 448, 1 / 448, 1 / 448)
    for causal in (True, False):
        o, lse = run_fp8(torch_cuda, q8, k8, v8, desc, causal)
        o_ref, lse_ref = oracle.attn_fp8(q8, k8, v8, desc, causal)
        fp8_bar(o, o_ref, lse, lse_ref, 1.0, f"fp8 all codes causal={causal}")


def test_fp8_rising_scores_exact(torch_cuda):
    """Integer scores that rise along the keys (0, 1, ..., 15 in steps every 32
    keys), so the running max grows tile by tile: weights reach 2^8 against a
    stale max before the O rescale.  With scale ln 2 every weight is a power of
    two and exact in E4M3, so the bf16 bar applies."""
    B, H, N = 1, 1, 512
    one = inputs.f32_to_e4m3_bits(np.array([1.0], dtype=np.float32))[0]
    q8 = np.zeros((B, H, N, 128), dtype=np.uint8)
    q8[..., 0] = one
    k8 = np.zeros((B, H, N, 128), dtype=np.uint8)
    k8[0, 0, :, 0] = inputs.f32_to_e4m3_bits((np.arange(N) // 32).astype(np.float32))
    rng = np.random.Generator(np.random.PCG64(78))
    v8, dv = inputs.quantize_e4m3(rng.standard_normal(N * 128).astype(np.float32))
    v8 = v8.reshape(B, H, N, 128)
    desc = (1.0, 1.0, dv)
    for causal in (False, True):
        o, lse = run_fp8(torch_cuda, q8, k8, v8, desc, causal, math.log(2.0))
        o_ref, lse_ref = oracle.attn_fp8(q8, k8, v8, desc, causal, scale=math.log(2.0))
        parity(o, o_ref, lse, lse_ref, f"fp8 rising scores causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_huge_score_gaps(torch_cuda, causal):
    """Scores far apart: queries hold 448 in one dimension; keys 16t+2 hold 2
    there, keys 16t and 16t+1 hold -16, the rest 0.  The opposed keys sit about
    1,000 exp2 units below the row max on the columns whose weights the
    FMA-pipe exponential computes (below its range of exact results); they must
    weigh 0, not NaN.  Every weight is 0 or 1 within E4M3 rounding, so the bf16
    bar applies; |lse| stays below 700, where fp32 holds it to 1e-4."""
    B, Hq, Hkv, N = 1, 2, 1, 300
    big, up, down = inputs.f32_to_e4m3_bits(np.array([448.0, 2.0, -16.0], dtype=np.float32))
    q8 = np.zeros((B, Hq, N, 128), dtype=np.uint8)
    q8[..., 0] = big
    k8 = np.zeros((B, Hkv, N, 128), dtype=np.uint8)
    pos = np.arange(N) % 16
    k8[0, 0, pos == 2, 0] = up
    k8[0, 0, (pos == 0) | (pos == 1), 0] = down
    rng = np.random.Generator(np.random.PCG64(79))
    v8, dv = inputs.quantize_e4m3(rng.standard_normal(N * 128).astype(np.float32))
    v8 = v8.reshape(B, Hkv, N, 128)
    desc = (1.0, 1.0, dv)
    o, lse = run_fp8(torch_cuda, q8, k8, v8, desc, causal)
    o_ref, lse_ref = oracle.attn_fp8(q8, k8, v8, desc, causal)
    assert np.all(np.isfinite(o)), "non-finite output"
    parity(o, o_ref, lse, lse_ref, f"fp8 huge score gaps causal={causal}")

