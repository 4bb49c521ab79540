"""Plant plausible mistakes in a copy of the C oracle and check that the pins catch each one.

Every mutant is one textual edit of ``oracle/pa_oracle.c`` (a wrong index, a
dropped term, a flipped sign, swapped operands), compiled into a temporary
library on the CPU.  A mutant that no pin rejects would mean the pins leave
that part of the oracle unchecked.
"""
import json
import os
import subprocess
import sys

import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "pa_oracle.c")

MUTANTS = {
    "row_uses_division": ("int64_t row = j % block_size;", "int64_t row = j / block_size;"),
    "table_uses_modulo": ("table_row[j / block_size];\n        int64_t row", "table_row[j % block_size];\n        int64_t row"),
    "gqa_modulo_grouping": ("int64_t h = hq / group;", "int64_t h = hq % num_kv_heads;"),
    "dropped_scale": ("z[j] = scale * acc;", "z[j] = acc;"),
    "softmax_sign": ("z[j] = exp(z[j] - m);", "z[j] = exp(m - z[j]);"),
    "no_max_shift": ("z[j] = exp(z[j] - m);", "z[j] = exp(z[j]);"),
    "dropped_normaliser": ("double w = z[j] / Z;", "double w = z[j];"),
    "k_v_swapped": ("K[j * head_dim + i] = widen(kr[i], dtype);", "K[j * head_dim + i] = widen(vr[i], dtype);"),
    "query_of_kv_head": ("attend(q + (s * num_q_heads + hq) * head_dim,", "attend(q + (s * num_q_heads + h) * head_dim,"),
    "last_token_dropped": ("for (int64_t j = 0; j < L; ++j) {\n        int64_t p",
                           "for (int64_t j = 0; j < L - 1; ++j) {\n        int64_t p"),
    "fp16_no_implicit_bit": ("ldexp((double)(f + 1024), e - 25)", "ldexp((double)f, e - 25)"),
    "fp16_bias_off_by_one": ("ldexp((double)(f + 1024), e - 25)", "ldexp((double)(f + 1024), e - 24)"),
    "fp16_subnormal_scale": ("ldexp((double)f, -24);", "ldexp((double)f, -25);"),
    "bf16_shift": ("((uint32_t)b) << 16;", "((uint32_t)b) << 15;"),
    "dtype_swapped": ("return dtype == 2 ? oracle_bf16_to_double(bits)", "return dtype == 1 ? oracle_bf16_to_double(bits)"),
    "write_row_division": ("int64_t row = slot % block_size;", "int64_t row = slot / block_size % block_size;"),
    "write_k_from_v": ("k_cache[dst] = k[src];", "k_cache[dst] = v[src];"),
    "write_head_stride": ("int64_t dst = ((block * num_kv_heads + h) * block_size + row) * head_dim + i;",
                          "int64_t dst = ((block * num_kv_heads) * block_size + row) * head_dim + i;"),
    "write_negative_slots": ("if (slot < 0) continue;", "if (slot < 0) slot = 0;"),
    "copy_swaps_direction": ("dst_k[dst * per_block + e] = src_k[src * per_block + e];",
                             "dst_k[src * per_block + e] = src_k[dst * per_block + e];"),
    "copy_skips_v": ("            dst_v[dst * per_block + e] = src_v[src * per_block + e];\n", ""),
    "copy_half_block": ("const int64_t per_block = num_kv_heads * block_size * head_dim;",
                        "const int64_t per_block = block_size * head_dim;"),
    "causal_off_by_one": ("K, V, pos + 1, head_dim", "K, V, pos, head_dim"),
    "causal_sees_future": ("K, V, pos + 1, head_dim", "K, V, L, head_dim"),
    "position_top_left": ("int64_t pos = L - n + t;", "int64_t pos = t;"),
    "prefill_token_row": ("int64_t tok = query_start[s] + t;", "int64_t tok = t;"),
    "prefill_interleaved_groups": ("for (int64_t hq = h * group; hq < (h + 1) * group; ++hq)",
                                   "for (int64_t hq = h; hq < num_q_heads; hq += num_kv_heads)"),
    "zero_length_garbage": ("for (int64_t i = 0; i < head_dim; ++i) o[i] = 0.0;\n            if (L == 0) continue;",
                            "if (L == 0) { o[0] = 1.0; continue; }\n            for (int64_t i = 0; i < head_dim; ++i) o[i] = 0.0;"),
}


_RUNNER = """
import json, sys
sys.path[:0] = sys.argv[2:]
from oracle_pins import ALL_PINS
failed = []
for pin in ALL_PINS:
    try:
        pin(sys.argv[1])
    except (AssertionError, ValueError):
        failed.append(pin.__name__)
print(json.dumps(failed))
"""


def _failing_pins(lib_path):
    """Run every pin against ``lib_path`` in a child process (a mutant may read out of bounds)."""
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    res = subprocess.run([sys.executable, "-c", _RUNNER, lib_path, here, root], capture_output=True, text=True,
                         timeout=600)
    if res.returncode < 0:
        return [f"crashed (signal {-res.returncode})"]
    assert res.returncode == 0, f"pin runner failed: {res.stderr[-2000:]}"
    return json.loads(res.stdout.strip().splitlines()[-1])


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """Build every mutant (and the unmodified source as a control) and run the pins on each, eight child
    processes at a time; returns {name: failing pins}."""
    from concurrent.futures import ThreadPoolExecutor
    d = tmp_path_factory.mktemp("mutants")
    with open(SRC) as f:
        src = f.read()
    libs = {"__control__": str(d / "lib_control.so")}
    oracle.build(SRC, libs["__control__"])
    for name, (old, new) in MUTANTS.items():
        assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
        path = d / f"{name}.c"
        path.write_text(src.replace(old, new))
        libs[name] = str(d / f"lib_{name}.so")
        oracle.build(str(path), libs[name])
    with ThreadPoolExecutor(max_workers=8) as ex:
        futures = {name: ex.submit(_failing_pins, lib) for name, lib in libs.items()}
        return {name: f.result() for name, f in futures.items()}


def test_runner_accepts_the_real_oracle(mutant_results):
    """Control: the unmodified source, built the same way, passes every pin in the runner."""
    assert mutant_results["__control__"] == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, mutant_results):
    failed = mutant_results[name]
    assert failed, f"mutant {name} passes every pin"
    print(f"{name}: caught by {failed}")
