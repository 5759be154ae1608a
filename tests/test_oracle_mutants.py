"""Plant plausible mistakes in copies of the oracle; each copy must fail at least one pin.

Every mutant below edits one expression of ``oracle/pa_oracle.c`` (a dropped term, a wrong sign,
a wrong index, a swapped operand), compiles the copy into a temporary directory and runs the
pins of ``tests/oracle_pins.py`` against it in a child process.  The real oracle passes every
pin (test_oracle_pins.py); a mutant that passes them all means the pins have a blind spot.
Mutants are chosen so that none reads outside its buffers.
"""
import json
import os
import subprocess
import sys

import pytest

import oracle as oracle_pkg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "gqa_mapping": ("const int g = h / group;", "const int g = h % num_kv_heads;"),
    "block_offset": ("const int64_t offset = t % block_size;",
                     "const int64_t offset = (t + 1) % block_size;"),
    "logical_block": ("const int64_t logical_block = t / block_size;",
                      "const int64_t logical_block = t / block_size / 2;"),
    "drop_last_token": ("attend_rows(o, &m, &l, q, kc, vc, t0, t1, head_dim, scale, z);",
                        "attend_rows(o, &m, &l, q, kc, vc, t0, t1 - 1, head_dim, scale, z);"),
    "drop_scale": ("z[t - t0] = scale * dot;", "z[t - t0] = dot;"),
    "max_sign": ("const double w = exp(z[t - t0] - m);", "const double w = exp(m - z[t - t0]);"),
    "no_normalise": ("for (int d = 0; d < head_dim; ++d) o[d] /= l;", ""),
    "k_for_v": ("o[d] += w * vc[", "o[d] += w * kc["),
    "query_row": ("const size_t qrow = ((size_t)s * (size_t)num_heads + (size_t)h)",
                  "const size_t qrow = ((size_t)s * (size_t)num_heads + (size_t)g)"),
    "write_block_offset_swap": (
        "const int64_t block = slot / block_size;\n    const int64_t offset = slot % block_size;",
        "const int64_t block = slot % block_size;\n    const int64_t offset = slot / block_size % block_size;"),
    "write_value_into_key": ("memcpy((char *)key_cache + dst, (const char *)key + src, row);",
                             "memcpy((char *)key_cache + dst, (const char *)value + src, row);"),
    "copy_direction": (
        "memcpy((char *)key_cache + (size_t)dst * block_bytes,\n"
        "           (const char *)key_cache + (size_t)src * block_bytes, block_bytes);",
        "memcpy((char *)key_cache + (size_t)src * block_bytes,\n"
        "           (const char *)key_cache + (size_t)dst * block_bytes, block_bytes);"),
    "swap_value_from_key": (
        "memcpy((char *)dst_value + (size_t)dst * block_bytes,\n"
        "           (const char *)src_value + (size_t)src * block_bytes, block_bytes);",
        "memcpy((char *)dst_value + (size_t)dst * block_bytes,\n"
        "           (const char *)src_key + (size_t)src * block_bytes, block_bytes);"),
    "swap_dst_index": ("memcpy((char *)dst_key + (size_t)dst * block_bytes,",
                       "memcpy((char *)dst_key + (size_t)src * block_bytes,"),
    "fp8_exponent_bias": ("v = ldexp((double)(8 + m), e - 10);", "v = ldexp((double)(8 + m), e - 11);"),
    "fp8_subnormal_scale": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "fp8_subnormal_floor": ("code = (int)rint(a * 512.0);", "code = (int)floor(a * 512.0);"),
    "fp8_normal_floor": ("int m = (int)rint((ldexp(a, -e) - 1.0) * 8.0);",
                         "int m = (int)floor((ldexp(a, -e) - 1.0) * 8.0);"),
    "fp8_late_saturation": ("if (a >= 448.0) return sign | 0x7e;", "if (a >= 480.0) return sign | 0x7e;"),
    "fp8_quantise_multiplies": ("const float q = x / scale;", "const float q = x * scale;"),
    "fp8_padding_counted": ("if (slot < 0) continue; /* a padding token stores nothing */",
                            "if (slot < 0) { ++skipped; continue; }"),
    "fp8_v_scaled_by_k": ("const double vs = v_scale ? (double)v_scale[g] : 1.0;",
                          "const double vs = k_scale ? (double)k_scale[g] : 1.0;"),
    "prefill_gqa_mapping": ("const int kvh = h / group; /* the kv head query head h reads */",
                            "const int kvh = h % num_kv_heads;"),
    "prefill_causal_limit": ("attend_rows(o, &m, &l, q, kc, vc, 0, p + 1, head_dim, scale, z);",
                             "attend_rows(o, &m, &l, q, kc, vc, 0, p, head_dim, scale, z);"),
    "prefill_query_row": (
        "const size_t qrow = ((size_t)(q0 + j) * (size_t)num_heads + (size_t)h) * (size_t)head_dim;",
        "const size_t qrow = ((size_t)(q0 + q_len - 1 - j) * (size_t)num_heads + (size_t)h) * (size_t)head_dim;"),
    "prefill_positions": ("const int64_t p = len - q_len + j; /* this token's position: it sees 0 .. p */",
                          "const int64_t p = j; /* this token's position: it sees 0 .. p */"),
    "bf16_shift": ("uint32_t u = (uint32_t)h << 16;", "uint32_t u = (uint32_t)h << 15;"),
    "f16_bias": ("v = ldexp((double)(m | 0x400), e - 25);", "v = ldexp((double)(m | 0x400), e - 24);"),
    "merge_sign": ("const double w = l[p] * exp(m[p] - big_m);",
                   "const double w = l[p] * exp(big_m - m[p]);"),
    "merge_drop_l": ("const double w = l[p] * exp(m[p] - big_m);",
                     "const double w = exp(m[p] - big_m);"),
    "empty_context_reads": ("const int64_t len = context_lens[s] > 0 ? context_lens[s] : 0;",
                            "const int64_t len = context_lens[s] > 0 ? context_lens[s] : 1;"),
    "padding_counted_as_refused": ("if (slot < 0) continue; /* padding token */",
                                   "if (slot < 0) { ++skipped; continue; } /* padding token */"),
}

_CHILD = r"""
import json, sys
sys.path.insert(0, {root!r})
import oracle
from tests.oracle_pins import ALL_PINS
orc = oracle.Oracle({lib!r})
failed = []
for pin in ALL_PINS:
    try:
        pin(orc)
    except Exception as exc:
        failed.append(pin.__name__)
        break
print(json.dumps(failed))
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    before, after = MUTANTS[name]
    with open(oracle_pkg.SOURCE) as f:
        src = f.read()
    assert src.count(before) == 1, f"mutation site for {name} not unique/not found"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(before, after))
    lib = oracle_pkg.build(str(path), str(tmp_path / "libmutant.so"))
    res = subprocess.run([sys.executable, "-c", _CHILD.format(root=ROOT, lib=lib)],
                         capture_output=True, text=True, timeout=300)
    if res.returncode != 0:
        return  # the mutant broke the oracle outright; that is caught too
    failed = json.loads(res.stdout.strip().splitlines()[-1])
    assert failed, f"mutant {name!r} passed every pin"
