"""Plant plausible mistakes in a copy of oracle.c and check that the pins
catch every one of them (CPU only; the planted copies never leave a temp dir)."""
import os
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "dropped_scale": ("s[j] = scale * acc;", "s[j] = acc;"),
    "causal_off_by_one": ("(long)(Nkv - Nq) + 1;", "(long)(Nkv - Nq);"),
    "alignment_sign": ("(long)(Nkv - Nq) + 1;", "(long)(Nq - Nkv) + 1;"),
    "no_normalisation": ("double p = exp(s[j] - m) / l;", "double p = exp(s[j] - m);"),
    "wrong_exp_sign": ("double p = exp(s[j] - m) / l;", "double p = exp(m - s[j]) / l;"),
    "lse_without_log": ("*lse = m + log(l);", "*lse = m;"),
    "lse_log2": ("*lse = m + log(l);", "*lse = m + log2(l);"),
    "gqa_mapping": ("int hkv = hq / G;", "int hkv = hq % Hkv;"),
    "reversed_feature": ("bf16_to_f64(kj[t]);", "bf16_to_f64(kj[d - 1 - t]);"),
    "v_row_index": ("const uint16_t *vj = v + (size_t)j * d;", "const uint16_t *vj = v + (size_t)(n - 1 - j) * d;"),
    "page_row_index": ("(size_t)(t % page_size)) * d;", "(size_t)(t / page_size)) * d;"),
    "sum_without_max": ("l += exp(s[j] - m);", "l += exp(s[j]);"),
    "decode_head_mapping": ("int hq = hkv * G + g;", "int hq = g * Hkv + hkv;"),
    # varlen prefill over the paged cache
    "pp_alignment_swapped": ("visible_keys(i, q_len, len, causal)", "visible_keys(i, len, q_len, causal)"),
    "pp_row_offset_ignored": ("size_t row = (size_t)(q0 + i) * Hq + hq;", "size_t row = (size_t)i * Hq + hq;"),
    # backward pass
    "bwd_dq_without_scale": ("dqi[t] += scale * ds *", "dqi[t] += ds *"),
    "bwd_no_jacobian_row_term": ("double ds = p[j] * (dp[j] - rowterm);", "double ds = p[j] * dp[j];"),
    "bwd_key_sweep_no_row_term": ("double ds = p * (dot_bf16(doi, vj, d) - rr[x]);", "double ds = p * dot_bf16(doi, vj, d);"),
    "bwd_dv_from_q": ("dvj[t] += p * bf16_to_f64(doi[t]);", "dvj[t] += p * bf16_to_f64(qi[t]);"),
    "bwd_dk_from_do": ("dkj[t] += scale * ds * bf16_to_f64(qi[t]);", "dkj[t] += scale * ds * bf16_to_f64(doi[t]);"),
    "bwd_one_head_per_group": ("for (int hq = hkv * G; hq < (hkv + 1) * G; ++hq)",
                               "for (int hq = hkv * G; hq < hkv * G + 1; ++hq)"),
    "bwd_dp_from_k": ("dp[j] = dot_bf16(doi, vb + (size_t)j * d, d);", "dp[j] = dot_bf16(doi, kb + (size_t)j * d, d);"),
    "bwd_key_sweep_dp_from_k": ("double ds = p * (dot_bf16(doi, vj, d) - rr[x]);", "double ds = p * (dot_bf16(doi, kj, d) - rr[x]);"),
    "bwd_key_sweep_unnormalised": ("- rm[x]) / rl[x];", "- rm[x]);"),
    # FP8 inputs
    "e4m3_exponent_bias": ("v = ldexp(8.0 + m, e - 10);", "v = ldexp(8.0 + m, e - 11);"),
    "e4m3_subnormal_scale": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "e4m3_sign_ignored": ("return (b & 0x80) ? -v : v;", "return v;"),
    "e4m3_no_nan": ("if (e == 15 && m == 7)\n        return NAN;", "if (0)\n        return NAN;"),
    "fp8_v_descale_dropped": ("o[t] += p * (dv * e4m3_to_f64(vj[t]));", "o[t] += p * e4m3_to_f64(vj[t]);"),
    "fp8_k_descale_dropped": ("(dk * e4m3_to_f64(kj[t]))", "e4m3_to_f64(kj[t])"),
    "fp8_q_descale_squared": ("(dq * e4m3_to_f64(q[t]))", "(dq * dq * e4m3_to_f64(q[t]))"),
    "bwd_key_sweep_mask_ignored": ("if (j >= visible_keys(i, Nq, Nkv, causal))\n                    continue;", "if (0)\n                    continue;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    c = tmp_path / "mutant.c"
    c.write_text(mutated)
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"],
                   check=True)
    variant = oracle.Variant(str(so))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(variant)
        except (AssertionError, RuntimeError, FloatingPointError, ValueError) as e:
            failed.append(pin.__name__)
    assert failed, f"no pin caught mutant {name}"
