"""The FP8 parity bar, checked against a model of the kernel's arithmetic (CPU).

The FP8 prefill rounds every softmax weight to E4M3 before the P.V product;
its GPU tests therefore compare with the exact oracle under a bar derived from
that rounding (rel-L2 4e-2, max-abs 2^-4 max|V| + 2^-8 max|O|).  This file
models the kernel's arithmetic in numpy, to the level the bar is about:

* scores from the dequantised inputs, processed in 128-key tiles in order;
* running max kept stale until it grows by more than 8 in exp2 units, O and l
  rescaled when it moves;
* weights 2^(s*c - m*c) rounded to E4M3 (torch's float8_e4m3fn conversion)
  for O, and summed unrounded for l.

It checks that the modelled error sits inside the bar with margin and at the
predicted level (about 0.026 RMS relative), and that integer scores with scale
ln 2 make the model exact.  The model is test infrastructure: it shares
nothing with the CUDA code and is not the oracle.
"""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
from tiled_attention_17_b200 import inputs

FP8_REL_L2 = 4e-2      # the bar used by tests/test_gpu_fp8.py
TILE = 128
STALE_LOG2 = 8.0


def _e4m3_round(x):
    import torch
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def model_row(qv, K, V, scale, visible):
    """One query row through the kernel's tiled, stale-max, FP8-P arithmetic."""
    c = scale / math.log(2.0)          # exp2 units
    s = K[:visible] @ qv
    m, l, o = -math.inf, 0.0, np.zeros(V.shape[1])
    for j0 in range(0, visible, TILE):
        t = s[j0:j0 + TILE]
        m_new = max(m, float(t.max()))
        if m == -math.inf or (m_new - m) * c > STALE_LOG2:
            alpha = 0.0 if m == -math.inf else 2.0 ** ((m - m_new) * c)
            o *= alpha
            l *= alpha
            m = m_new
        p = np.exp2((t - m) * c)
        o += _e4m3_round(p) @ V[j0:j0 + len(t)]
        l += p.sum()
    return o / l


def _model(q8, k8, v8, desc, causal, scale, rows):
    Q = oracle.e4m3_decode(q8) * desc[0]
    K = oracle.e4m3_decode(k8) * desc[1]
    V = oracle.e4m3_decode(v8) * desc[2]
    _, _, Nq, _ = Q.shape
    Nkv = K.shape[2]
    out = []
    for i in rows:
        vis = min(Nkv, i + Nkv - Nq + 1) if causal else Nkv
        out.append(model_row(Q[0, 0, i], K[0, 0], V[0, 0], scale, vis))
    return np.array(out)


def test_fp8_bar_covers_modelled_error():
    N = 1024
    q8, k8, v8, desc = inputs.random_prefill_fp8(1, 1, 1, N, N, 128, seed=101)
    rows = np.arange(0, N, 7)
    for causal in (True, False):
        o_model = _model(q8, k8, v8, desc, causal, 128 ** -0.5, rows)
        o_ref, _ = oracle.attn_fp8(q8, k8, v8, desc, causal, rows=rows)
        rel = np.linalg.norm(o_model - o_ref) / np.linalg.norm(o_ref)
        vmax = np.abs(oracle.e4m3_decode(v8)).max() * desc[2]
        # at the predicted level (E4M3 rounding, ~0.026 RMS relative) ...
        assert 0.01 < rel < 0.035, rel
        # ... and inside both bars with margin
        assert rel < FP8_REL_L2 / 1.15, rel
        assert np.abs(o_model - o_ref).max() < vmax / 16 / 2


def test_fp8_integer_scores_make_weights_exact():
    q8, k8, v8, dv = inputs.fp8_integer_score_inputs(1, 1, 1, 400, 400, 128, seed=5)
    desc = (2.0, 0.5, dv)
    rows = np.arange(0, 400, 3)
    for causal in (True, False):
        o_model = _model(q8, k8, v8, desc, causal, math.log(2.0), rows)
        o_ref, _ = oracle.attn_fp8(q8, k8, v8, desc, causal, scale=math.log(2.0), rows=rows)
        assert np.abs(o_model - o_ref).max() <= 1e-12 * max(1.0, np.abs(o_ref).max())


@pytest.mark.parametrize("bits", [2, 3])
def test_rounding_error_shrinks_with_mantissa(bits):
    """A sanity check of the model itself: rounding the weights to a format
    with more mantissa bits than E4M3 lowers the error roughly by 2x per bit,
    so the error the bar covers is the weight rounding and nothing else."""
    N = 512
    q8, k8, v8, desc = inputs.random_prefill_fp8(1, 1, 1, N, N, 128, seed=103)
    Q = oracle.e4m3_decode(q8)[0, 0] * desc[0]
    K = oracle.e4m3_decode(k8)[0, 0] * desc[1]
    V = oracle.e4m3_decode(v8)[0, 0] * desc[2]
    rows = np.arange(0, N, 5)
    o_ref, _ = oracle.attn_fp8(q8, k8, v8, desc, False, rows=rows)

    def round_mant(p, b):
        e = np.floor(np.log2(p))
        step = 2.0 ** (e - b)
        return np.round(p / step) * step

    errs = []
    for b in (bits, bits + 2):
        out = []
        for i in rows:
            s = K @ Q[i] * 128 ** -0.5
            p = np.exp(s - s.max())
            out.append(round_mant(p, b) @ V / p.sum())
        errs.append(np.linalg.norm(np.array(out) - o_ref) / np.linalg.norm(o_ref))
    assert errs[1] < errs[0] / 2.5, errs
