"""Parity of the backward pass (attn_bwd through the C ABI) with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from gpu_util import GRAD_MAX_REL, GRAD_REL_L2, bf16_to_f64, to_dev
from tiled_attention_17_b200 import inputs
from tiled_attention_17_b200.inputs import grad_output, random_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tiled_attention_17_b200 import binding
    binding.load()
    return torch


def run_bwd(torch, q, k, v, do, causal, scale=None):
    from tiled_attention_17_b200 import binding
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    o, lse = binding.attention(qd, kd, vd, causal, scale)
    dq, dk, dv = binding.attention_backward(qd, kd, vd, o, lse, dod, causal, scale)
    torch.cuda.synchronize()
    return dq, dk, dv


def grad_errors(g, ref):
    g = np.asarray(g, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape
    assert np.all(np.isfinite(g))
    err = np.abs(g - ref)
    scale = max(float(np.abs(ref).max()), 1e-30)
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(g - ref) / denom) if denom > 0 else float(np.linalg.norm(g))
    return float(err.max()) / scale, rel


# The gradient bar (GRAD_REL_L2, GRAD_MAX_REL) is derived from a model of the
# kernels' bf16 rounding points; see gpu_util and tests/test_bwd_error_model.py.


def check_grads(torch, q, k, v, do, causal, scale=None, what="", groups=None):
    dq, dk, dv = run_bwd(torch, q, k, v, do, causal, scale)
    rq, rk, rv = oracle.attn_bwd(q, k, v, do, causal, scale=scale, groups=groups)
    out = {}
    B, Hkv = k.shape[0], k.shape[1]
    G = q.shape[1] // Hkv
    sel_kv = np.zeros((B, Hkv), dtype=bool)
    for gid in (range(B * Hkv) if groups is None else groups):
        sel_kv[gid // Hkv, gid % Hkv] = True
    sel_q = np.repeat(sel_kv, G, axis=1)
    for name, g, r, sel in (("dq", dq, rq, sel_q), ("dk", dk, rk, sel_kv), ("dv", dv, rv, sel_kv)):
        out[name] = grad_errors(bf16_to_f64(g)[sel], r[sel])
    print(what, {k2: (f"{a:.2e}", f"{b:.2e}") for k2, (a, b) in out.items()})
    for name, (mx, rel) in out.items():
        assert rel <= GRAD_REL_L2, f"{what} {name}: rel-L2 {rel:.3e}"
        assert mx <= GRAD_MAX_REL, f"{what} {name}: max err / max|ref| {mx:.3e}"
    return out


CASES = [
    # B, Hq, Hkv, Nq, Nkv, d, causal
    (1, 1, 1, 256, 256, 64, False),
    (1, 1, 1, 256, 256, 64, True),
    (1, 2, 2, 640, 640, 128, False),
    (1, 2, 2, 640, 640, 128, True),
    (1, 2, 2, 200, 333, 128, True),       # Nq < Nkv, ragged tiles, bottom-right mask
    (1, 2, 2, 333, 200, 128, False),
    (2, 8, 2, 384, 384, 128, True),       # GQA group 4
    (1, 4, 1, 130, 130, 64, True),        # GQA group 4, d = 64, ragged
    (1, 1, 1, 1, 700, 128, False),        # one query row
    (1, 2, 1, 300, 100, 128, True),       # rows with no visible key
    (2, 40, 8, 512, 512, 128, True),      # more CTAs than SMs
    # Persistent CTAs (more items than SMs): a CTA takes over further items.
    (1, 32, 8, 1024, 256, 128, True),     # 256 dQ items, 6 of each head's 8 see no key
    (2, 16, 8, 256, 2048, 128, True),     # 256 dK/dV key-tile items, Nq < Nkv
    (1, 8, 8, 130, 2500, 64, False),      # 160 dK/dV items at d = 64, ragged last key tile
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nkv,d,causal", CASES)
def test_backward_parity_small(torch_cuda, B, Hq, Hkv, Nq, Nkv, d, causal):
    q, k, v = random_prefill(B, Hq, Hkv, Nq, Nkv, d, seed=Nq * 5 + Nkv + d + causal)
    do = grad_output(q.shape, seed=Nq + 17 * Nkv)
    check_grads(torch_cuda, q, k, v, do, causal, what=f"{B, Hq, Hkv, Nq, Nkv, d, causal}")


def test_backward_sharp_peaks(torch_cuda):
    cfg = inputs.PrefillConfig("peaks", 1, 2, 2, 1024, 1024, 128, False, 64, 4.0)
    q, k, v = inputs.prefill_inputs(cfg, seed=98)
    check_grads(torch_cuda, q, k, v, grad_output(q.shape, seed=3), False, what="sharp peaks")


def test_backward_special_cases(torch_cuda):
    torch = torch_cuda
    # single key: dq = dk = 0 up to rounding (P = 1 is rebuilt from the stored
    # lse, and dO.O and dO.v_0 are summed in different orders), dv = sum of dO
    q, k, v = random_prefill(1, 2, 2, 129, 1, 128, seed=8)
    do = grad_output(q.shape, seed=9)
    dq, dk, dv = run_bwd(torch, q, k, v, do, False)
    assert float(dq.abs().max()) <= 1e-4 and float(dk.abs().max()) <= 1e-4
    _, _, rv = oracle.attn_bwd(q, k, v, do, False)
    mx, rel = grad_errors(bf16_to_f64(dv), rv)
    assert rel <= GRAD_REL_L2
    # scale 0: no gradient reaches q or k
    q, k, v = random_prefill(1, 1, 1, 300, 300, 128, seed=10)
    do = grad_output(q.shape, seed=11)
    dq, dk, dv = run_bwd(torch, q, k, v, do, True, scale=0.0)
    assert torch.all(dq == 0) and torch.all(dk == 0)
    check_grads(torch, q, k, v, do, True, scale=0.0, what="scale 0")


def test_backward_empty_shapes(torch_cuda):
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    # no queries: dk = dv = 0
    q = torch.zeros((1, 2, 0, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.ones((1, 2, 5, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 2, 0), dtype=torch.float32, device="cuda")
    dq, dk, dv = binding.attention_backward(q, k, k, q, lse, q, True)
    torch.cuda.synchronize()
    assert torch.all(dk == 0) and torch.all(dv == 0)
    # no keys: dq = 0
    q = torch.ones((1, 2, 7, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 2, 0, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((1, 2, 7), float("-inf"), dtype=torch.float32, device="cuda")
    dq, dk, dv = binding.attention_backward(q, k, k, q, lse, q, False)
    torch.cuda.synchronize()
    assert torch.all(dq == 0)


def test_backward_deterministic(torch_cuda):
    q, k, v = random_prefill(1, 4, 2, 1000, 1000, 128, seed=4)
    do = grad_output(q.shape, seed=5)
    a = run_bwd(torch_cuda, q, k, v, do, True)
    b = run_bwd(torch_cuda, q, k, v, do, True)
    for x, y in zip(a, b):
        assert torch_cuda.equal(x, y)


def test_backward_bad_args(torch_cuda):
    torch = torch_cuda
    from tiled_attention_17_b200 import binding
    q = torch.zeros((1, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 16), dtype=torch.float32, device="cuda")
    ws = torch.empty(binding.attn_bwd_workspace_size(1, 1, 16), dtype=torch.uint8, device="cuda")
    code = binding.attn_bwd(q, q, q, q, q, lse, q, q, q, ws, ws.numel(), 1, 3, 2, 16, 16, 128, 0.1, 0, check=False)
    assert binding.STATUS_NAMES[code] == "TA_ERR_INVALID_ARG"
    code = binding.attn_bwd(q, q, q, q, q, lse, q, q, q, ws, 16, 1, 1, 1, 16, 16, 128, 0.1, 0, check=False)
    assert binding.STATUS_NAMES[code] == "TA_ERR_INVALID_ARG"          # workspace too small
    code = binding.attn_bwd(q, q, q, q, q, lse, q, q, q, ws, ws.numel(), 1, 1, 1, 16, 16, 96, 0.1, 0, check=False)
    assert binding.STATUS_NAMES[code] == "TA_ERR_UNSUPPORTED"


@pytest.mark.parametrize("name", ["causal", "gqa", "long"])
def test_backward_full_size_one_group(torch_cuda, name):
    # the benchmark shapes; the oracle evaluates one whole KV-head group
    c = inputs.PREFILL_CONFIGS[name]
    q, k, v = inputs.prefill_inputs(c)
    do = grad_output(q.shape, seed=inputs.CONFIG_SEEDS[name] + 100)
    g = c.B * c.Hkv - 1
    check_grads(torch_cuda, q, k, v, do, c.causal, scale=c.scale, what=f"full {name}", groups=[g])
