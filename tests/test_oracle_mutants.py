"""Plant plausible mistakes in copies of the oracle and check the pins catch each.

Every mutant is a one-line edit of oracle/jl_oracle.c (a wrong comparison, a
dropped term, a flipped sign, a wrong index), compiled on the CPU into a
temporary library.  The real oracle is never modified.
"""
import os
import subprocess

import pytest

import oracle_pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "jl_oracle.c")

MUTANTS = {
    "local_boundary_inclusive": ("return (q - k) < w_local;", "return (q - k) <= w_local;"),
    "remap_ceil": ("long long jlo_remap(long long x, long long G) { return x / G; }",
                   "long long jlo_remap(long long x, long long G) { return (x + G - 1) / G; }"),
    "group_size_floor": ("long long g = (L + w_pretrained - 1) / w_pretrained;",
                         "long long g = L / w_pretrained;"),
    "rope_sin_sign": ("y[i] = x1 * c - x2 * s;", "y[i] = x1 * c + x2 * s;"),
    "rope_second_half": ("y[i + h] = x1 * s + x2 * c;", "y[i + h] = x2 * s + x1 * c;"),
    "theta_exponent": ("pow(base, -2.0 * (double)i / (double)D)",
                       "pow(base, -1.0 * (double)i / (double)D)"),
    "lse_drops_max": ("return M + log(Z);", "return log(Z);"),
    "remote_uses_standard_query": ("s[kk] = scale * jlo_dot(qr, krem + kk * D, D);",
                                   "s[kk] = scale * jlo_dot(qs, krem + kk * D, D);"),
    "remote_uses_standard_key": ("jlo_rope(raw, krem + kk * D, D, (double)jlo_remap(kk, G), rope_base);",
                                 "jlo_rope(raw, krem + kk * D, D, (double)kk, rope_base);"),
    "drops_diagonal_key": ("for (long long kk = 0; kk <= qp; ++kk) {",
                           "for (long long kk = 0; kk < qp; ++kk) {"),
    "gqa_head_map": ("if (row_b[r] != b || row_h[r] / group != hk) continue;",
                     "if (row_b[r] != b || row_h[r] % Hkv != hk) continue;"),
    "decode_dq_sign": ("const double dq = (double)(jlo_remap(pos, G) - pos);",
                       "const double dq = (double)(pos - jlo_remap(pos, G));"),
    "decode_corrects_local_keys": ("if (jlo_is_local(pos, kk, w_local)) {\n          for (int d = 0; d < D; ++d) kc[kk * D + d] = raw[d];",
                                   "if (0) {\n          for (int d = 0; d < D; ++d) kc[kk * D + d] = raw[d];"),
    "decode_dk_from_position": ("const double dk = (double)(jlo_remap(kk, G) - kk);",
                                "const double dk = (double)(jlo_remap(kk, G));"),
    "decode_group_from_pos": ("jlo_group_size((long long)pos + 1, w_pretrained);",
                              "jlo_group_size((long long)pos > 0 ? pos : 1, w_pretrained);"),
    "prefill_keys_ignore_batch": ("const int64_t base = (((int64_t)b * L + kk) * Hkv + hk) * D;",
                                  "const int64_t base = ((int64_t)kk * Hkv + hk) * D;"),
    "decode_cache_stride_from_pos": (
        "const int64_t base = (((int64_t)b * cache_capacity + kk) * Hkv + hk) * D;",
        "const int64_t base = (((int64_t)b * (pos + 1) + kk) * Hkv + hk) * D;"),
    "remote_query_at_original_position": (
        "jlo_rope(raw, qr, D, (double)jlo_remap(qp, G), rope_base);",
        "jlo_rope(raw, qr, D, (double)qp, rope_base);"),
    "values_read_from_keys": ("vd[kk * D + d] = jlo_load(v, base + d, dtype);",
                              "vd[kk * D + d] = jlo_load(k, base + d, dtype);"),
    "default_scale_over_D": ("if (scale <= 0.0) scale = 1.0 / sqrt((double)D);\n  const long long G = jlo_group_size(L,",
                             "if (scale <= 0.0) scale = 1.0 / (double)D;\n  const long long G = jlo_group_size(L,"),
    "decode_query_not_rotated_to_pos": ("jlo_rope(raw, qs, D, (double)pos, rope_base);",
                                        "jlo_rope(raw, qs, D, 0.0, rope_base);"),
    "bf16_widening": ("uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;",
                      "uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 15;"),
    "fp32_read_as_bf16": ("if (dtype == JLO_F32) return (double)((const float *)base)[idx];",
                          "if (dtype == JLO_F32) return (double)((const uint16_t *)base)[idx];"),
    "explicit_scale_ignored": ("if (scale <= 0.0) scale = 1.0 / sqrt((double)D);\n  const long long G = jlo_group_size(L,",
                               "scale = 1.0 / sqrt((double)D);\n  const long long G = jlo_group_size(L,"),
    "softmax_normaliser": ("for (int d = 0; d < D; ++d) out[d] /= Z;",
                           "for (int d = 0; d < D; ++d) out[d] /= (Z + 1.0);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path, oracle_mod):
    before, after = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation site for {name} not found exactly once"
    mpath = tmp_path / f"{name}.c"
    mpath.write_text(src.replace(before, after))
    lib = tmp_path / f"lib_{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                    str(mpath), "-o", str(lib), "-lm"], check=True)
    orc = oracle_mod.Oracle(str(lib))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
