"""The oracle's pins must catch plausible mistakes (CPU only).

Each case plants one mistake in a copy of the oracle source (a dropped term,
a wrong sign or index, a reversed order, a wrong rounding or partition
direction), builds it, and runs the oracle pin tests against that build in a
subprocess.  The pins pass on the real oracle (the other test files), so a
mutant passing them would mean the pins cannot see that mistake.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

SLOT_LOOP = """    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j) {
            int32_t e = topk[t * k + j];
            slot[t * k + j] = cursor[e];"""

MUTANTS = {
    "combine_drops_first_term": (
        "            for (int32_t j = 0; j < k; ++j) {\n                int64_t row = slot[t * k + j];\n                float v = oracle_bf16_to_f32(eo[row * H + h]);\n                acc = fmaf(w[t * k + j], v, acc);\n            }\n            y[t * H + h]",
        "            for (int32_t j = 1; j < k; ++j) {\n                int64_t row = slot[t * k + j];\n                float v = oracle_bf16_to_f32(eo[row * H + h]);\n                acc = fmaf(w[t * k + j], v, acc);\n            }\n            y[t * H + h]"),
    "combine_wrong_weight_index": (
        "                acc = fmaf(w[t * k + j], v, acc);\n            }\n            y[t * H + h]",
        "                acc = fmaf(w[t * k], v, acc);\n            }\n            y[t * H + h]"),
    "combine_sign_flip": (
        "                acc = fmaf(w[t * k + j], v, acc);\n            }\n            y[t * H + h]",
        "                acc = fmaf(w[t * k + j], -v, acc);\n            }\n            y[t * H + h]"),
    "bf16_ties_away_from_zero": (
        "    else if (dropped == 0x8000u && (kept & 1u))",
        "    else if (dropped == 0x8000u)"),
    "partition_extra_to_last_ranks": (
        "        if (extra_left > 0) {",
        "        if (r >= R - (E - base * R)) {"),
    "slots_reverse_token_order": (
        SLOT_LOOP,
        SLOT_LOOP.replace("int64_t t = 0; t < T; ++t", "int64_t t = T - 1; t >= 0; --t")),
    "node_of_rank_modulo": (
        "node_of_expert[e] = r / ranks_per_node;",
        "node_of_expert[e] = r % ranks_per_node;"),
    "staging_skips_first_row": (
        "            if (ns >= 0) {\n                int64_t row",
        "            if (ns > 0) {\n                int64_t row"),
    "dispatch_skips_first_destination": (
        "    for (int64_t t = 0; t < T; ++t)\n        for (int32_t j = 0; j < k; ++j) {\n            int64_t dst",
        "    for (int64_t t = 0; t < T; ++t)\n        for (int32_t j = 1; j < k; ++j) {\n            int64_t dst"),
    "validation_misses_adjacent_repeat": (
        "for (int32_t i = 0; i < j; ++i)",
        "for (int32_t i = 0; i + 1 < j; ++i)"),
    "rank_partial_range_off_by_one": (
        "if (row >= rank_offsets[r] && row < rank_offsets[r + 1])",
        "if (row >= rank_offsets[r] && row <= rank_offsets[r + 1])"),
    "e4m3_ties_to_odd_code": (
        "pick = (lo & 1) ? hi : lo;   /* tie: even code */",
        "pick = (lo & 1) ? lo : hi;   /* tie: even code */"),
    "fp8_scale_inverted": (
        "scale[r] = amax > 0.0f ? amax / 448.0f : 1.0f;",
        "scale[r] = amax > 0.0f ? 448.0f / amax : 1.0f;"),
    "fp8_combine_drops_scale": (
        "float coef = w[t * k + j] * eo_scale[row];",
        "float coef = w[t * k + j];"),
    "node_src_ignores_node_offset": (
        "node_src[(int64_t)node_offsets[n] + ns] = (int32_t)t;",
        "node_src[ns] = (int32_t)t;"),
    "ep_counts_later_sources": (
        "for (int32_t h = 0; h < g; ++h)",
        "for (int32_t h = g + 1; h < G; ++h)"),
    "ep_cursor_ignores_source_offset": (
        "cursor[e] = (int32_t)(expert_offsets[e] + before);",
        "cursor[e] = (int32_t)(expert_offsets[e]);"),
    "widening_drops_low_bit": (
        "    uint32_t u = ((uint32_t)h) << 16;",
        "    uint32_t u = ((uint32_t)(h & 0xFFFEu)) << 16;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} must occur once"
    mutant_c = tmp_path / "mutant.c"
    mutant_c.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-shared", "-fPIC",
                    "-o", str(lib), str(mutant_c), "-lm"], check=True)
    env = dict(os.environ, MOE_ORACLE_LIB=str(lib))
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           "-k", "not full_workloads",
           os.path.join(ROOT, "tests", "test_oracle_partition.py"),
           os.path.join(ROOT, "tests", "test_oracle_layout.py"),
           os.path.join(ROOT, "tests", "test_oracle_dispatch_combine.py"),
           os.path.join(ROOT, "tests", "test_oracle_fp8.py"),
           os.path.join(ROOT, "tests", "test_oracle_ep.py"),
           os.path.join(ROOT, "tests", "test_oracle_properties.py")]
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 1, (
        f"mutant {name} passed every pin:\n{res.stdout[-2000:]}\n{res.stderr[-2000:]}")
