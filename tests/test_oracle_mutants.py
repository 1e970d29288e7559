"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that a pin catches each one.

The copy is compiled from a text-edited ``oracle.c`` in a temporary directory;
the committed oracle is never modified.  Every mutant must make at least one
of the named pins in test_oracle_pins.py fail, which shows that the pins
constrain that part of the oracle.
"""
import os
import subprocess

import pytest

import oracle as ora
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(ora.__file__), "oracle.c")

MUTANTS = [
    ("rope sign", "v[i] = a * c - b * s;", "v[i] = a * c + b * s;", ["test_rope_matches_complex_form"]),
    ("rope frequency", "pow(theta, -2.0 * i / d)", "pow(theta, -1.0 * i / d)", ["test_rope_matches_complex_form"]),
    ("rmsnorm mean", "ss / n + eps", "ss + eps", ["test_rmsnorm_unit_rms_before_gain"]),
    ("rmsnorm gain", "x[i] * inv * ora_bf16_to_double(gain[i])", "x[i] * inv", ["test_rmsnorm_matches_torch"]),
    ("attention scale", "s[t] = dot * scale;", "s[t] = dot;", ["test_attention_probs_and_sdpa"]),
    ("softmax denominator", "double p = s[t] / den;", "double p = s[t];", ["test_attention_probs_and_sdpa"]),
    ("top-k tie rule", "logits[e] > logits[best]", "logits[e] >= logits[best]", ["test_topk_ties_go_to_lower_index"]),
    ("top-k weights", "w[j] = exp(logits[sel[j]] - mx) / den;", "w[j] = 1.0 / k;",
     ["test_topk_matches_torch_and_softmax_renorm"]),
    ("gqa head map", "int kvh = h / group;", "int kvh = h % nkv;", ["test_whole_step_matches_torch_reference"]),
    ("swiglu operands", "g[i] = ora_silu(g[i]) * u[i];", "g[i] = ora_silu(u[i]) * g[i];", ["test_swiglu_matches_torch"]),
    ("kv append index", "size_t base = (((size_t)b * nkv + h) * T + S) * hd;",
     "size_t base = (((size_t)b * nkv + h) * T + S - 1) * hd;", ["test_kv_append_writes_only_the_new_row"]),
    ("attention length", "S + 1, hd, att", "S, hd, att", ["test_whole_step_matches_torch_reference"]),
    ("attention residual", "for (int i = 0; i < H; ++i) xb[i] += o[i];\n    if (h_attn)",
     "for (int i = 0; i < H; ++i) xb[i] = o[i];\n    if (h_attn)", ["test_whole_step_matches_torch_reference"]),
    ("bf16 rounding", "rint(ldexp(x, -ulp_exp))", "floor(ldexp(x, -ulp_exp))", ["test_bf16_ties_to_even_and_nearest"]),
    ("gemv transpose", "ora_bf16_to_double(row[c])", "ora_bf16_to_double(w[(size_t)c * rows + r])",
     ["test_gemv_bruteforce"]),
    ("qk-norm gain", "ora_rmsnorm(k + (size_t)h * hd, hd, W->k_norm", "ora_rmsnorm(k + (size_t)h * hd, hd, W->q_norm",
     ["test_whole_step_matches_torch_reference"]),
    ("moe weighting", "acc[i] += wsel[j] * o[i];", "acc[i] += o[i];", ["test_moe_step_matches_torch_reference"]),
    ("silu sign", "return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));", ["test_silu_values"]),
    ("mlp norm gain", "ora_rmsnorm(xb, H, W->mlp_norm,", "ora_rmsnorm(xb, H, W->attn_norm,",
     ["test_whole_step_matches_torch_reference"]),
    ("mlp residual", "      }\n      for (int i = 0; i < H; ++i) xb[i] += o[i];",
     "      }\n      for (int i = 0; i < H; ++i) xb[i] = o[i];", ["test_whole_step_matches_torch_reference"]),
    ("final norm skipped", "ora_gemv(m->lm_head, m->d.vocab, H, xn, logits);",
     "ora_gemv(m->lm_head, m->d.vocab, H, x, logits);", ["test_whole_step_matches_torch_reference"]),
    ("key rope position", "ora_rope(k + (size_t)h * hd, hd, pos, d->rope_theta);",
     "ora_rope(k + (size_t)h * hd, hd, pos + 1, d->rope_theta);", ["test_whole_step_matches_torch_reference"]),
    ("router input", "ora_gemv(W->router, E, H, xn, r);", "ora_gemv(W->router, E, H, xb, r);",
     ["test_moe_step_matches_torch_reference"]),
    ("e4m3 exponent bias", "ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)",
     ["test_e4m3_every_code_matches_torch"]),
    ("e4m3 subnormals", "ldexp((double)m / 8.0, 1 - 7)", "ldexp(1.0 + (double)m / 8.0, 0 - 7)",
     ["test_e4m3_closed_forms"]),
    ("fp8 block index", "scale[(size_t)r * nb + c / block]", "scale[(size_t)r * nb + c % nb]",
     ["test_gemv_fp8_matches_dequantized_torch"]),
    ("nvfp4 nibble order", "c % 2 ? byte >> 4 : byte & 15", "c % 2 ? byte & 15 : byte >> 4",
     ["test_gemv_nvfp4_nibble_order_and_scales"]),
    ("nvfp4 tensor scale", "* (double)tensor_scale * x[c]", "* x[c]", ["test_gemv_nvfp4_matches_dequantized"]),
    ("fp8 step ignores fp8 o_proj", "gemv_w(d, W->wo, &W->wo8, H, nq * hd, att, o);",
     "ora_gemv(W->wo, H, nq * hd, att, o);", ["test_fp8_step_uses_the_fp8_weights"]),
    ("fp8 swiglu operands", "gu[i] = ora_silu(gu[i]) * gu[d->ffn_dim + i];",
     "gu[i] = ora_silu(gu[d->ffn_dim + i]) * gu[i];", ["test_fp8_step_equals_bf16_step_when_the_weights_agree"]),
]


@pytest.mark.parametrize("name,old,new,pin_names", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, pin_names, tmp_path, monkeypatch):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name!r} must occur exactly once"
    mut = tmp_path / "oracle.c"
    mut.write_text(src.replace(old, new))
    (tmp_path / "oracle.h").write_text(open(SRC[:-1] + "h").read())
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-o", str(so), str(mut),
                           "-lm"])
    import ctypes
    lib = ora._setup(ctypes.CDLL(str(so)))
    monkeypatch.setattr(ora, "_lib", lib)
    caught = False
    for pn in pin_names:
        fn = getattr(pins, pn)
        params = getattr(fn, "pytestmark", [])
        cases = [()]
        for mk in params:
            if mk.name == "parametrize":
                cases = mk.args[1]
        for case in cases:
            try:
                fn(*case) if isinstance(case, tuple) else fn(case)
            except (AssertionError, ValueError):
                caught = True
                break
        if caught:
            break
    assert caught, f"no pin caught the planted mistake {name!r}"
