"""The oracle's pins catch plausible mistakes.

Each case copies ``oracle/pkv_oracle.c``, plants one mistake in the copy (a
dropped term, a wrong index, a transposed layout, a wrong sign ...), compiles
it, and runs the pin suite against it in a child process: the suite must fail.
Everything runs on the CPU; the oracle itself is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "pkv_oracle.c")

MUTANTS = {
    "offset_off_by_one": ("int32_t offset = j % pb->block_size;",
                          "int32_t offset = (j + 1) % pb->block_size;"),
    "nhd_instead_of_hnd": ("((physical_block * pb->num_kv_heads + kv_head) * pb->block_size + offset) * D",
                           "((physical_block * pb->block_size + offset) * pb->num_kv_heads + kv_head) * D"),
    "interleaved_gqa": ("const int32_t kv_head = q_head / group;",
                        "const int32_t kv_head = q_head % pb->num_kv_heads;"),
    "scale_dropped": ("z[j - t0] = scale * dot;", "z[j - t0] = dot;"),
    "no_max_shift": ("double w = exp(z[j - t0] - m);", "double w = exp(z[j - t0]);"),
    "not_normalised": ("        o[d] /= l;\n", "        o[d] /= 1.0;\n"),
    "context_off_by_one": ("attend_range(qrow, K, V, D, pb->scale, 0, L, &m, &l, out);",
                           "attend_range(qrow, K, V, D, pb->scale, 0, L > 1 ? L - 1 : L, &m, &l, out);"),
    "merge_weight_without_l": ("double w = l[p] * exp(m[p] - M);", "double w = exp(m[p] - M);"),
    "merge_sign": ("double w = l[p] * exp(m[p] - M);", "double w = l[p] * exp(M - m[p]);"),
    "slot_uses_logical_block": ("slots[t] = physical_block * block_size + offset;",
                                "slots[t] = logical_block * block_size + offset;"),
    "reshape_transposed": ("size_t dst = (((size_t)block * num_kv_heads + h) * block_size + offset) * row;",
                           "size_t dst = (((size_t)block * block_size + offset) * num_kv_heads + h) * row;"),
    "copy_without_snapshot": ("memcpy(snap_k + (size_t)i * block_bytes,\n               (const char *)k_cache + (size_t)src * block_bytes, (size_t)block_bytes);",
                              "memcpy((char *)k_cache + (size_t)pairs[2 * i + 1] * block_bytes,\n               (const char *)k_cache + (size_t)src * block_bytes, (size_t)block_bytes);\n        memcpy(snap_k + (size_t)i * block_bytes,\n               (const char *)k_cache + (size_t)src * block_bytes, (size_t)block_bytes);"),
    "bf16_widen_shift": ("uint32_t bits = (uint32_t)((const uint16_t *)base)[index] << 16;",
                         "uint32_t bits = (uint32_t)((const uint16_t *)base)[index] << 15;"),
    "multi_not_causal": ("const int32_t visible = L - n + i + 1;      /* keys 0 .. L-n+i */",
                         "const int32_t visible = L;"),
    "multi_causal_off_by_one": ("const int32_t visible = L - n + i + 1;      /* keys 0 .. L-n+i */",
                                "const int32_t visible = L - n + i;"),
    "q_row_of_wrong_head": ("qrow[d] = widen(pb->q, ((int64_t)seq * pb->num_q_heads + q_head) * D + d, q_dtype(pb));",
                            "qrow[d] = widen(pb->q, ((int64_t)seq * pb->num_q_heads + kv_head) * D + d, q_dtype(pb));"),
    "e4m3_ties_away": ("double steps = rint(ldexp(a, 3 - unbiased));",
                       "double steps = floor(ldexp(a, 3 - unbiased) + 0.5);"),
    "e4m3_bias_off_by_one": ("return sign | (uint8_t)(((unbiased + 7) << 3) | ((int)steps - 8));",
                             "return sign | (uint8_t)(((unbiased + 8) << 3) | ((int)steps - 8));"),
    "e4m3_no_saturation": ("        return sign | 0x7e;                       /* saturate */",
                           "        return sign | 0x7f;                       /* saturate */"),
    "e5m2_bias_off_by_one": ("return sign | (uint8_t)(((unbiased + 15) << 2) | ((int)steps - 4));",
                             "return sign | (uint8_t)(((unbiased + 16) << 2) | ((int)steps - 4));"),
    "e5m2_value_three_mantissa_bits": ("v = ldexp(1.0 + man / 4.0, exp - 15);",
                                       "v = ldexp(1.0 + man / 8.0, exp - 15);"),
    "e5m2_subnormal_step": ("v = ldexp((double)man, -16);", "v = ldexp((double)man, -15);"),
    "merge_f32_m_and_l_swapped": ("        md[p] = (double)m[p];\n", "        md[p] = (double)l[p];\n"),
    "merge_f32_o_transposed": ("od[(int64_t)p * head_dim + d] = (double)o[(int64_t)p * head_dim + d];",
                               "od[(int64_t)p * head_dim + d] = (double)o[(int64_t)d * nparts + p];"),
    "fp8_scale_dropped": ("V[(int64_t)j * D + d] = widen(pb->v_cache, row + d, pb->dtype) * pb->v_scale;",
                          "V[(int64_t)j * D + d] = widen(pb->v_cache, row + d, pb->dtype);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutant_c = tmp_path / "mutant.c"
    mutant_c.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", str(lib),
                    str(mutant_c), "-lm"], check=True)
    env = dict(os.environ, PKV_ORACLE_LIB_OVERRIDE=str(lib))
    proc = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert proc.returncode != 0, f"mutant {name} passed every pin:\n{proc.stdout[-2000:]}"
