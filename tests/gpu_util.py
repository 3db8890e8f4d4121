"""Helpers shared by the GPU tests: device copies of bf16 bit arrays and the
parity metrics (tolerances fixed by the attention parity bar: max-abs 2e-2,
relative L2 5e-3, lse 1e-3 absolute, for bf16 inputs with fp32 accumulation),
and the gradient bar of the backward pass."""
from __future__ import annotations

import numpy as np

MAX_ABS = 2e-2
REL_L2 = 5e-3
LSE_ABS = 1e-3

# Gradient bar of the backward pass: relative L2 <= 5e-3 (the attention parity
# bar) and max error <= 1.2e-2 of the largest gradient, each about 2x the error
# a model of the kernels' bf16 rounding points predicts (2.5e-3 and 6e-3;
# tests/test_bwd_error_model.py).
GRAD_REL_L2 = 5e-3
GRAD_MAX_REL = 1.2e-2


def to_dev(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def bf16_to_f64(t) -> np.ndarray:
    import torch
    return t.detach().float().cpu().numpy().astype(np.float64)


def parity(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    """Assert the parity bar; returns (max_abs, rel_l2, lse_err)."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    err = np.abs(o_gpu - o_ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(o_gpu - o_ref) / denom) if denom > 0 else float(np.linalg.norm(o_gpu))
    lse_err = 0.0
    if lse_gpu is not None:
        lg = np.asarray(lse_gpu, dtype=np.float64)
        lr = np.asarray(lse_ref, dtype=np.float64)
        both = np.isneginf(lg) & np.isneginf(lr)
        assert np.array_equal(np.isneginf(lg), np.isneginf(lr)), f"{what}: -inf lse pattern differs"
        with np.errstate(invalid="ignore"):     # -inf - -inf on rows with no key; masked by `both`
            d = np.abs(np.where(both, 0.0, lg - lr))
        lse_err = float(d.max()) if d.size else 0.0
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {MAX_ABS}"
    assert rel <= REL_L2 or denom == 0, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    assert lse_err <= LSE_ABS, f"{what}: lse err {lse_err:.3e} > {LSE_ABS}"
    return max_abs, rel, lse_err


def sample_rows(B, Hq, Nq, n, rng, extra=()):
    """Flat row ids (b*Hq + h)*Nq + i: tile boundaries, first/last rows, and random ones."""
    ids = set()
    special_i = [0, 1, 127, 128, 255, 256, Nq // 2, Nq - 129, Nq - 128, Nq - 2, Nq - 1]
    for b in {0, B - 1}:
        for h in {0, Hq - 1, Hq // 2}:
            for i in special_i:
                if 0 <= i < Nq:
                    ids.add((b * Hq + h) * Nq + i)
    ids.update(int(x) for x in extra)
    while len(ids) < n:
        ids.add(int(rng.integers(0, B * Hq * Nq)))
    return np.array(sorted(ids), dtype=np.int64)
