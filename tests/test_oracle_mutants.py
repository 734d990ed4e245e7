"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the pins
of tests/pins.py catch every one of them.  The committed oracle is never modified."""
import os
import subprocess
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from pins import ALL_PINS  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "la_oracle.c")

# (name, original text, planted text)
MUTANTS = [
    ("delta_sign", "u[j] = b * (v[j] - c * pj);", "u[j] = b * (v[j] + c * pj);"),
    ("undecayed_prediction", "default: /* gated_delta */ *a = g;   *b = beta; *c = g;",
     "default: /* gated_delta */ *a = g;   *b = beta; *c = 1.0;"),
    ("gated_write_scaled", "case LAO_RULE_GATED:       *a = g;   *b = 1.0;",
     "case LAO_RULE_GATED:       *a = g;   *b = g;"),
    ("readout_by_key", "oj += S[(size_t)i * dv + j] * q[i];", "oj += S[(size_t)i * dv + j] * k[i];"),
    ("transposed_prediction", "alpha[i] * S[(size_t)i * dv + j] : S[(size_t)i * dv + j]) * k[i];",
     "alpha[i] * S[(size_t)j * dv + i] : S[(size_t)j * dv + i]) * k[i];"),
    ("transposed_outer", "ai * S[(size_t)i * dv + j] + k[i] * u[j];", "ai * S[(size_t)i * dv + j] + k[j] * u[i];"),
    ("kda_undecayed_prediction", "(rule == LAO_RULE_KDA ? alpha[i] * S[(size_t)i * dv + j] :",
     "(rule == LAO_RULE_KDA ? S[(size_t)i * dv + j] :"),
    ("kda_channels_reversed", "const double ai = rule == LAO_RULE_KDA ? alpha[i] : a;",
     "const double ai = rule == LAO_RULE_KDA ? alpha[dk - 1 - i] : a;"),
    ("kda_readout_undecayed", "const double sij = kda ? al[i] * S[(size_t)i * dv + j] : S[(size_t)i * dv + j];",
     "const double sij = S[(size_t)i * dv + j];"),
    ("gqa_interleaved", "return h / (n_v_heads / n_qk_heads);", "return h % n_qk_heads;"),
    ("query_group_reads_wrong_queries", "return t * hd.nqh + (n_q_heads > 0 ? (size_t)h * hd.grp :",
     "return t * hd.nqh + (n_q_heads > 0 ? (size_t)h :"),
    ("query_group_output_misplaced", "double *ot = o + ((size_t)t * hd.no + (size_t)h * hd.grp) * dv;",
     "double *ot = o + ((size_t)t * hd.no + (size_t)h) * dv;"),
    ("scan_drops_last_token", "for (int t = cu_seqlens[s]; t < cu_seqlens[s + 1]; ++t) {",
     "for (int t = cu_seqlens[s]; t < cu_seqlens[s + 1] - 1; ++t) {"),
    ("scan_ignores_initial_state", "memcpy(S, src_pool + (size_t)read_slot[s] * slot + (size_t)h * tile, sizeof(double) * tile);",
     "memset(S, 0, sizeof(double) * tile);"),
    ("bf16_ties_away", "double y = ldexp(rint(ldexp(x, -qe)), qe);", "double y = ldexp(round(ldexp(x, -qe)), qe);"),
    ("bf16_truncates", "double y = ldexp(rint(ldexp(x, -qe)), qe);", "double y = ldexp(trunc(ldexp(x, -qe)), qe);"),
    ("decode_store_unrounded", "            round_tile(S, dk, dv, dst_dtype, q8_masks ? q8_masks + (size_t)h * (dk / 32) : NULL);\n            free(u);\n        }\n    }\n\n    for (int b = 0;",
     "            free(u);\n        }\n    }\n\n    for (int b = 0;"),
    ("checkpoint_overwritten", "memcpy(dst_pool + (size_t)ws * slot, next + (size_t)b * slot, sizeof(double) * slot);",
     "memcpy(dst_pool + (size_t)(read_slot ? read_slot[b] : b) * slot, next + (size_t)b * slot, sizeof(double) * slot);"),
    ("checkpoint_off_by_one", "const int pos = t - cu_seqlens[s] + 1;", "const int pos = t - cu_seqlens[s];"),
    ("q8_truncates", "rintf(row[gi * 32 + j] * inv)", "truncf(row[gi * 32 + j] * inv)"),
    ("q8_scale_by_128", "const float k127 = 1.0f / 127.0f;", "const float k127 = 1.0f / 128.0f;"),
    ("q8_mask_ignored", "return (int)((mask[i / 32] >> (i % 32)) & 1u);", "return 0 * (int)mask[i / 32];"),
    ("q8_first_head_mask", "round_tile(S, dk, dv, dst_dtype, q8_masks ? q8_masks + (size_t)h * (dk / 32) : NULL);\n            free(u);\n        }\n    }\n\n    for (int b",
     "round_tile(S, dk, dv, dst_dtype, q8_masks);\n            free(u);\n        }\n    }\n\n    for (int b"),
    ("conv_window_shifted", "for (int j = 0; j < W - 1; ++j) y += w[j] * h[j];",
     "for (int j = 0; j < W - 1; ++j) y += w[j + 1] * h[j];"),
    ("conv_history_not_shifted", "for (int j = 0; j < W - 2; ++j) ho[j] = h[j + 1];",
     "for (int j = 0; j < W - 2; ++j) ho[j] = h[j];"),
    ("conv_silu_sign", "if (act) y = y / (1.0 + exp(-y));", "if (act) y = y / (1.0 + exp(y));"),
    ("conv_norm_shared", "const double rq = 1.0 / sqrt(sq + 1e-6), rk = 1.0 / sqrt(sk + 1e-6);",
     "const double rq = 1.0 / sqrt(sq + 1e-6), rk = rq;"),
    ("gather_wrong_slot", "memcpy(dense + (size_t)i * slot_bytes, pool + (size_t)slots[i] * slot_bytes, slot_bytes);",
     "memcpy(dense + (size_t)i * slot_bytes, pool + (size_t)i * slot_bytes, slot_bytes);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(orc, tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-fopenmp", "-fPIC", "-shared", "-I", os.path.join(ROOT, "oracle"),
                    "-o", str(lib), str(mutant), "-lm"], check=True)
    prev = orc.oracle.use_library(str(lib))
    try:
        caught = None
        for pin in ALL_PINS:
            try:
                pin(orc)
            except AssertionError as e:  # the planted mistake is visible
                caught = (pin.__name__, str(e)[:200])
                break
        assert caught is not None, f"no pin caught the planted mistake {name}"
    finally:
        orc.oracle.restore_library(prev)
