"""Planted mistakes: each entry copies the oracle source, plants one plausible
error (a dropped term, a wrong sign or index, a transposed operand), builds it
on the CPU, and runs the pin suite against it.  At least one pin must fail for
every mutant — otherwise the pins would not notice that mistake in the oracle.
"""

import os
import subprocess
import sys

import pytest

import oracle
from oracle_pins import PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "pa_oracle.cpp")

MUTANTS = {
    "gqa_interleaved_heads": ("const int h = kvh * group + j;  // query head h reads kv head h / group",
                              "const int h = j * sh.num_kv_heads + kvh;"),
    "prefill_gqa_interleaved": ("const int h = kvh * group + j;\n                    const int64_t t = first + i;",
                                "const int h = j * num_kv_heads + kvh;\n                    const int64_t t = first + i;"),
    "layout_token_outer": ("return (vector * block_size + token) * vec + dim % vec;",
                           "return ((tile * block_size + token) * (head_dim / vec) + dim / vec) * vec + dim % vec;"),
    "offset_off_by_one": ("const int offset = t % sh.block_size;",
                          "const int offset = (t + 1) % sh.block_size;"),
    "logical_block_off_by_one": ("table_row[t / sh.block_size]", "table_row[(t + 1) / sh.block_size]"),
    "softmax_sign": ("w[t] = std::exp(z[t] - zmax);", "w[t] = std::exp(zmax - z[t]);"),
    "dropped_scale": ("z[t] = scale * dot;", "z[t] = dot;"),
    "missing_normalisation": ("const double p = w[t] / denom;", "const double p = w[t];"),
    "merge_weight_dropped": ("const double w = std::exp(m[p] - big) / denom;",
                             "const double w = 1.0 / denom;"),
    "partition_end_short": ("const int t1 = std::min(context_len, t0 + part);",
                            "const int t1 = std::min(context_len, t0 + part - 1);"),
    "reshape_block_shift": ("const int64_t dst = pool_index(block, h, offset, d, num_kv_heads, block_size, head_dim, vec);",
                            "const int64_t dst = pool_index((slot + 1) / block_size, h, offset, d, num_kv_heads, block_size, head_dim, vec);"),
    "reshape_kv_swapped": ("static_cast<const uint8_t*>(value) + src * es, es);",
                           "static_cast<const uint8_t*>(key) + src * es, es);"),
    "reshape_skips_slot_zero": ("if (head_dim % vec != 0) return kBadArg;\n    for (int64_t i = 0; i < num_tokens; ++i) {\n        const int64_t slot = slot_mapping[i];\n        if (slot < 0) continue;",
                                "if (head_dim % vec != 0) return kBadArg;\n    for (int64_t i = 0; i < num_tokens; ++i) {\n        const int64_t slot = slot_mapping[i];\n        if (slot <= 0) continue;"),
    "f16_exponent_bias": ("exponent - 25);", "exponent - 24);"),
    "bf16_wrong_half": ("static_cast<uint32_t>(bits) << 16);", "static_cast<uint32_t>(bits) << 15);"),
    "context_len_short": ("attend_plain(qrow.data(), keys, values, len, D, scale_d, dst);",
                          "attend_plain(qrow.data(), keys, values, len > 1 ? len - 1 : len, D, scale_d, dst);"),
    "copy_v_from_k_pool": ("static_cast<const uint8_t*>(src_v) + from * es, es);",
                           "static_cast<const uint8_t*>(src_k) + from * es, es);"),
    "copy_last_token_skipped": ("for (int t = 0; t < block_size; ++t) {\n                for (int d = 0; d < head_dim; ++d) {\n                    const int64_t from",
                                "for (int t = 0; t < block_size - 1; ++t) {\n                for (int d = 0; d < head_dim; ++d) {\n                    const int64_t from"),
    "copy_direction_reversed": ("const int64_t src = block_mapping[2 * i];\n        const int64_t dst = block_mapping[2 * i + 1];",
                                "const int64_t dst = block_mapping[2 * i];\n        const int64_t src = block_mapping[2 * i + 1];"),
    "copy_head_dropped": ("for (int h = 0; h < num_kv_heads; ++h) {\n            for (int t = 0; t < block_size; ++t) {",
                          "for (int h = 1; h < num_kv_heads; ++h) {\n            for (int t = 0; t < block_size; ++t) {"),
    "e4m3_exponent_bias": ("v = std::ldexp(static_cast<double>(mantissa + 8), exponent - 10);",
                           "v = std::ldexp(static_cast<double>(mantissa + 8), exponent - 9);"),
    "e4m3_subnormal_step": ("v = std::ldexp(static_cast<double>(mantissa), -9);",
                            "v = std::ldexp(static_cast<double>(mantissa), -8);"),
    "e4m3_ties_away": ("double r = std::nearbyint(a / quantum) * quantum;",
                       "double r = std::round(a / quantum) * quantum;"),
    "e4m3_no_saturation": ("if (r > 448.0) r = 448.0;", "if (r > 480.0) r = 448.0;"),
    "e4m3_scale_multiplied": ("to_e4m3_bits(kx / k_scale[h]);", "to_e4m3_bits(kx * k_scale[h]);"),
    "e4m3_v_scale_for_keys": ("from_e4m3_bits(static_cast<const uint8_t*>(k_cache)[ka]) * static_cast<double>(sh.k_scale[kv_head]);",
                              "from_e4m3_bits(static_cast<const uint8_t*>(k_cache)[ka]) * static_cast<double>(sh.v_scale[kv_head]);"),
    "e4m3_byte_order_natural": ("int64_t e4m3_slot16(int64_t j) { return 4 * ((j % 8) / 2) + 2 * (j / 8) + j % 2; }",
                                "int64_t e4m3_slot16(int64_t j) { return j; }"),
    "e4m3_v_not_transposed": ("const int64_t va = e4m3_v_index(physical, kv_head, offset, d, sh.num_kv_heads, sh.block_size, D);",
                              "const int64_t va = e4m3_k_index(physical, kv_head, offset, d, sh.num_kv_heads, sh.block_size, D);"),
    "prefill_causal_off_by_one": ("const int visible = len - count + i + 1;", "const int visible = len - count + i + 2;"),
    "prefill_not_causal": ("const int visible = len - count + i + 1;", "const int visible = len;"),
    "prefill_rows_reversed": ("const int64_t t = first + i;", "const int64_t t = first + count - 1 - i;"),
    "q_from_wrong_head": ("(static_cast<int64_t>(s) * sh.num_q_heads + h) * D + d",
                          "(static_cast<int64_t>(s) * sh.num_q_heads + kvh) * D + d"),
}


# Runs the pins against one oracle build in a child process: a planted
# indexing mistake may read or write outside an array, and a crash of the
# child counts as a pin failing.
_CHILD = """
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle
from oracle_pins import PINS
orc = oracle.Oracle({lib!r})
failed = []
for pin in PINS:
    try:
        pin(orc)
    except Exception as e:
        failed.append(pin.__name__)
print("FAILED:" + ",".join(failed))
"""


def _pins_failed(lib):
    here = os.path.dirname(os.path.abspath(__file__))
    code = _CHILD.format(root=os.path.dirname(here), tests=here, lib=lib)
    proc = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    if proc.returncode != 0:
        return [f"child exited with {proc.returncode}"]
    line = [l for l in proc.stdout.splitlines() if l.startswith("FAILED:")][-1]
    return [x for x in line[len("FAILED:"):].split(",") if x]


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """Every mutant built and run against the pins once, several at a time
    (each is a g++ build and a child process): name -> pins that failed, or
    None when the mutation's anchor is not in the source exactly once."""
    from concurrent.futures import ThreadPoolExecutor
    base = tmp_path_factory.mktemp("mutants")
    src = open(SRC).read()

    def one(name):
        old, new = MUTANTS[name]
        if src.count(old) != 1:
            return name, None
        d = base / name
        d.mkdir()
        mutant_src = d / "pa_oracle_mutant.cpp"
        mutant_src.write_text(src.replace(old, new))
        lib = oracle.build(str(mutant_src), str(d / "liboracle_mutant.so"), force=True)
        return name, _pins_failed(lib)

    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        return dict(ex.map(one, sorted(MUTANTS)))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, mutant_results):
    failed = mutant_results[name]
    assert failed is not None, f"mutation anchor not found exactly once: {MUTANTS[name][0]!r}"
    assert failed, f"no pin caught the planted mistake {name}"
