"""The FMA-pipe exponential that the FP8 prefill uses for part of its softmax
weights (ta_exp2_poly_debug, through the C ABI) against 2^x in fp64: its stated
error bound over the whole input range, and its floor below -125."""
from __future__ import annotations

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

BOUND = 7.5e-5   # max relative error stated with the polynomial
FLOOR = 2.0 ** -125


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_attention_17_b200 import binding
    binding.load()
    return torch


def run(torch, xs):
    from tiled_attention_17_b200 import binding
    x = torch.from_numpy(np.ascontiguousarray(xs, dtype=np.float32)).cuda()
    y = torch.full_like(x, -1.0)
    binding.ta_exp2_poly_debug(x, y, x.numel())
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def test_exp2_poly_error_bound(torch_cuda):
    rng = np.random.Generator(np.random.PCG64(11))
    xs = np.concatenate([np.linspace(-125.0, 20.0, 1_450_001), rng.uniform(-125.0, 0.0, 500_000),
                         np.array([0.0, -0.5, 0.5, -1.0, 1.0, -124.999, -125.0, -8.0, 8.0])]).astype(np.float32)
    y = run(torch_cuda, xs)
    ref = np.exp2(xs.astype(np.float64))
    rel = np.abs(y - ref) / ref
    worst = int(np.argmax(rel))
    assert rel[worst] <= BOUND, f"max relative error {rel[worst]:.3e} at x = {xs[worst]!r}"


def test_exp2_poly_below_range(torch_cuda):
    # far below the row max (and -inf, NaN): a tiny positive floor, never NaN
    xs = np.array([-125.0001, -125.5, -126.0, -126.6, -127.0, -128.0, -1000.0, -1e30, -np.inf, np.nan],
                  dtype=np.float32)
    y = run(torch_cuda, xs)
    assert np.all(np.isfinite(y)), y
    assert np.all((y > 0) & (y <= FLOOR * (1 + BOUND))), y


def test_exp2_poly_odd_count(torch_cuda):
    # pairs are evaluated together; the last element of an odd count stands alone
    xs = np.array([-3.0, 2.0, -0.25], dtype=np.float32)
    y = run(torch_cuda, xs)
    assert np.all(np.abs(y / np.exp2(xs.astype(np.float64)) - 1) <= BOUND)
