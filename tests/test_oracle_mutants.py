"""The oracle's pins are not vacuous: each plausible mistake, planted in a
temporary copy of the oracle's C source (never in the CUDA path, and only on the
CPU), must make at least one pin in ``test_oracle_pins.py`` fail."""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "qk_oracle.c")

# (name, text in qk_oracle.c, replacement): each is a slip someone could make.
MUTANTS = [
    ("round_half_away", "float n = nearbyintf(t);", "float n = roundf(t);"),
    ("scale_over_128", "float s = amax / 127.0f;", "float s = amax / 128.0f;"),
    ("no_zero_row_guard", "*scale = 1.0f;\n        return;", "*scale = 0.0f;\n        return;"),
    ("clamp_at_126", "if (n > 127.0f)\n            n = 127.0f;", "if (n > 126.0f)\n            n = 126.0f;"),
    ("w4_nibbles_swapped", "(codes[2 * j] | (codes[2 * j + 1] << 4))",
     "(codes[2 * j + 1] | (codes[2 * j] << 4))"),
    ("w4_offset_is_max", "uint16_t ob = oracle_f32_to_f16(lo);", "uint16_t ob = oracle_f32_to_f16(hi);"),
    ("w4_scale_over_16", "(hi - lo) / 15.0f", "(hi - lo) / 16.0f"),
    ("w4_unpack_swapped", "return (k & 1) ? (b >> 4) : (b & 0x0F);", "return (k & 1) ? (b & 0x0F) : (b >> 4);"),
    ("acc_transposed_index", "(int64_t)Wq[n * K + k]", "(int64_t)Wq[k * N + n]"),
    ("bias_dropped", "t = t + (double)bias[n];", "t = t;"),
    ("w4_offset_term_dropped", "f = f + (t + u);", "f = f + t;"),
    ("w4_sx_dropped", "double r = (double)sx[m] * f;", "double r = f;"),
    ("bf16_truncates", "r = (fmod(units, 2.0) == 0.0) ? lo : hi;", "r = lo;"),
    ("bf16_nearest_up", "if (dlo < dhi)\n        r = lo;", "if (dlo < dhi * 0.5)\n        r = lo;"),
    ("gated_residual_dropped", "t = t + (double)oracle_bf16_to_f32(r[m * N + n]);", "t = t;"),
    ("gated_gate_skips_bias", "double t = (double)gate[n] * v;",
     "double t = (double)gate[n] * (v - (bias ? (double)bias[n] : 0.0)) + (bias ? (double)bias[n] : 0.0);"),
    ("act_divide_by_scale", "float t = v[k] * r;", "float t = v[k] / s;"),
    ("w4_divide_by_scale", "float t = (w[i] - o) * r;", "float t = (w[i] - o) / s;"),
    ("w4_codes_from_unrounded_scale", "float s = oracle_f16_to_f32(sb);",
     "float s = (hi - lo) / 15.0f;"),
    ("w4_codes_from_unrounded_offset", "float o = oracle_f16_to_f32(ob);", "float o = lo;"),
    ("group_sum_window", "for (int64_t k = 64 * g; k < 64 * g + 64; ++k)\n                s += xq[m * K + k];",
     "for (int64_t k = 64 * g; k < 64 * g + 63; ++k)\n                s += xq[m * K + k];"),
    ("sage_scale_dropped", "s[j] = (double)dot * (double)sq[i] * (double)sk[j] * scale;",
     "s[j] = (double)dot * (double)sq[i] * (double)sk[j];"),
    ("sage_key_scale_of_query", "s[j] = (double)dot * (double)sq[i] * (double)sk[j] * scale;",
     "s[j] = (double)dot * (double)sq[i] * (double)sk[i] * scale;"),
    ("sage_key_index_is_query", "dot += (int64_t)qc[i * D + d] * (int64_t)kc[j * D + d];",
     "dot += (int64_t)qc[i * D + d] * (int64_t)kc[i * D + d];"),
    ("sage_value_transposed", "o[d] += p * (double)oracle_bf16_to_f32(v[j * D + d]);",
     "o[d] += p * (double)oracle_bf16_to_f32(v[d * L + j]);"),
    ("sage_normalizer_dropped", "double res = o[d] / l;", "double res = o[d];"),
]


def _pin_calls():
    calls = []
    for name in dir(pins):
        fn = getattr(pins, name)
        if name.startswith("test_") and callable(fn):
            if name == "test_quant_error_bound_and_range":
                for K in (32, 96, 256):
                    calls.append((f"{name}[{K}]", lambda f=fn, K=K: f(oracle, K)))
            else:
                calls.append((name, lambda f=fn: f(oracle)))
    return calls


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, mutant, orc):
    name, old, new = mutant
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    path_c = tmp_path / f"{name}.c"
    path_c.write_text(src.replace(old, new))
    lib = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", *oracle.CFLAGS, str(path_c), "-o", str(lib), "-lm"], check=True)
    failed = []
    with oracle.using_library(str(lib)):
        for pin_name, call in _pin_calls():
            try:
                call()
            except AssertionError:
                failed.append(pin_name)
                break
    assert failed, f"no pin caught the planted mistake {name}"
