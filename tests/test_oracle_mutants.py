"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch each one.  The oracle source is untouched: every mutant is a textual
edit of a temporary copy of oracle/nvfp4_oracle.c, compiled on the CPU and
swapped in for the duration of the check.
"""
import ctypes
import os
import subprocess
import tempfile

import pytest

import oracle
import oracle.build as ob
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(ob.__file__), "nvfp4_oracle.c")

# (name, original text, mutated text, pins expected to fail)
MUTANTS = [
    ("multiply_by_scale_instead_of_divide",
     "float y = x16[i] / den;", "float y = x16[i] * den;",
     [pins.test_block_invariants]),
    ("nibble_order_swapped",
     "packed8[j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4))",
     "packed8[j] = (uint8_t)(codes[2 * j + 1] | (codes[2 * j] << 4))",
     [pins.check_all_quantize_golden]),
    ("e2m1_ties_to_odd",
     "(d == best_d && (c & 1) == 0)", "(d == best_d && (c & 1) == 1)",
     [pins.test_e2m1_ties_to_even_and_saturation]),
    ("e4m3_ties_to_odd",
     "pick = (lo & 1) == 0 ? lo : hi;", "pick = (lo & 1) == 1 ? lo : hi;",
     [pins.test_e4m3_encode_matches_torch_below_saturation]),
    ("e4m3_no_saturation",
     "if (a >= oracle_e4m3_value(0x7E)) return (uint8_t)(sign | 0x7E);",
     "if (a >= oracle_e4m3_value(0x7E)) return (uint8_t)(sign | 0x7F);",
     [pins.test_e4m3_satfinite]),
    ("tensor_scale_without_six",
     "const float six_times_448 = 6.0f * 448.0f;", "const float six_times_448 = 448.0f;",
     [pins.test_tensor_scale]),
    ("block_ratio_without_six",
     "float d6 = 6.0f * s_tensor;", "float d6 = s_tensor;",
     [pins.test_block_invariants]),
    ("dequant_sign_dropped",
     "if (code & 0x8) e |= 0x80;", "(void)code;",
     [pins.test_dequant_fp8_sign_and_value]),
    ("softmax_scale_dropped",
     "s[t] = acc * scale;", "s[t] = acc;",
     [pins.test_attention_matches_torch_sdpa_gqa]),
    ("gqa_heads_interleaved",
     "int h = hk * g + j;\n                attend_one(q + ((int64_t)b * H_q + h) * D, K, V, L, D, scale,\n"
     "                           out + ((int64_t)b * H_q + h) * D);\n            }\n            free(K);\n"
     "            free(V);\n        }\n    }\n}\n\nvoid oracle_decode_attention_nvfp4",
     "int h = j * H_kv + hk;\n                attend_one(q + ((int64_t)b * H_q + h) * D, K, V, L, D, scale,\n"
     "                           out + ((int64_t)b * H_q + h) * D);\n            }\n            free(K);\n"
     "            free(V);\n        }\n    }\n}\n\nvoid oracle_decode_attention_nvfp4",
     [pins.test_attention_matches_torch_sdpa_gqa]),
    ("e2m1_subnormal_step_wrong",
     "mag = 0.5 * m;", "mag = 1.0 * m;",
     [pins.test_e2m1_grid_and_range]),
    ("e4m3_bias_off_by_one",
     "mag = (1.0 + m / 8.0) * ldexp(1.0, e - 7);", "mag = (1.0 + m / 8.0) * ldexp(1.0, e - 8);",
     [pins.test_e4m3_decode_matches_torch]),
    ("kv_memory_without_scale_bits",
     "return 4.0 + 8.0 / 16.0;", "return 4.0;",
     [pins.test_memory_ratios_match_pages]),
    ("mxfp4_exponent_off_by_one",
     "e = (ex - 1) - 2;", "e = (ex - 1) - 1;",
     [pins.check_all_mxfp4_golden, pins.test_mxfp4_block_invariants]),
    ("mxfp4_no_low_clamp",
     "if (e < -127) e = -127;", "if (e < -140) e = -140;",
     [pins.check_all_mxfp4_golden]),
    ("mxfp4_multiply_by_scale",
     "codes[i] = oracle_e2m1_encode((float)((double)x32[i] / X));",
     "codes[i] = oracle_e2m1_encode((float)((double)x32[i] * X));",
     [pins.check_all_mxfp4_golden, pins.test_mxfp4_grid_round_trip]),
    ("mxfp4_nibble_order_swapped",
     "packed16[j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));",
     "packed16[j] = (uint8_t)(codes[2 * j + 1] | (codes[2 * j] << 4));",
     [pins.check_all_mxfp4_golden]),
    ("mxfp4_nonfinite_ignored",
     "if (!isfinite(x32[i])) {", "if (0) {",
     [pins.test_mxfp4_nonfinite_blocks]),
    ("mxfp4_scale_bias_wrong",
     "return ldexp(1.0, (int)byte - 127);", "return ldexp(1.0, (int)byte - 128);",
     [pins.test_e8m0_values]),
    ("prefill_one_token_short",
     "attend_one(q + row, K, V, start[b] + i + 1, D, scale, out + row);",
     "attend_one(q + row, K, V, start[b] + i, D, scale, out + row);",
     [pins.test_prefill_single_query_is_decode_attention,
      pins.test_prefill_matches_torch_sdpa_with_causal_mask]),
    ("prefill_query_positions_reversed",
     "int64_t row = (((int64_t)b * C + i) * H_q + h) * D;",
     "int64_t row = (((int64_t)b * C + (C - 1 - i)) * H_q + h) * D;",
     [pins.test_prefill_matches_torch_sdpa_with_causal_mask, pins.test_prefill_is_causal]),
    ("nvfp4_reconstruction_without_tensor_scale",
     "oracle_e2m1_value(code) * oracle_e4m3_value(sb) * (double)s_tensor;",
     "oracle_e2m1_value(code) * oracle_e4m3_value(sb);",
     [pins.test_nvfp4_reconstruction_matches_block_decode]),
]


def _build_mutant(tmp, original, mutated):
    with open(SRC) as f:
        text = f.read()
    assert text.count(original) == 1, "mutation anchor not found exactly once"
    path = os.path.join(tmp, "mutant.c")
    with open(path, "w") as f:
        f.write(text.replace(original, mutated))
    hdr_dir = os.path.dirname(SRC)
    so = os.path.join(tmp, "libmutant.so")
    subprocess.run(["gcc", *ob.CFLAGS, "-I", hdr_dir, "-o", so, path, "-lm"], check=True)
    return so


@pytest.mark.parametrize("name,original,mutated,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, original, mutated, catchers):
    real = oracle.lib()
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(tmp, original, mutated)
        oracle._lib = None
        saved_build = oracle._build
        oracle._build = lambda: so
        try:
            oracle.lib()
            for pin in catchers:
                with pytest.raises(AssertionError):
                    pin()
        finally:
            oracle._build = saved_build
            oracle._lib = real
    # the real oracle still passes the same pins
    for pin in catchers:
        pin()
