"""The oracle's pins must catch plausible mistakes (CPU only).

Each case plants one mistake in a copy of the oracle source (a dropped term,
a wrong sign or index, a reversed order, a wrong rounding or partition
direction), builds it, and runs the oracle pin tests against that build in a
subprocess.  The pins pass on the real oracle (the other test files), so a
mutant passing them would mean the pins cannot see that mistake.
"""
import concurrent.futures
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
    "fp8_amax_of_signed_values": (
        "float v = fabsf(oracle_bf16_to_f32(src[r * H + h]));",
        "float v = oracle_bf16_to_f32(src[r * H + h]);"),
    "e4m3_saturates_to_nan_code": (
        "        return (uint8_t)(sign | 0x7E);",
        "        return (uint8_t)(sign | 0x7F);"),
    "e4m3_subnormal_scale_off": (
        "v = ldexpf((float)man, -9);",
        "v = ldexpf((float)man, -10);"),
    "expert_offsets_inclusive": (
        "        expert_offsets[e] = (int32_t)run;\n        run += expert_counts[e];",
        "        run += expert_counts[e];\n        expert_offsets[e] = (int32_t)run;"),
    "rank_offsets_from_expert_index": (
        "    if (first == NULL)\n        return ORC_INVALID_ARG;\n    oracle_partition(E, R, first);\n"
        "    for (int32_t r = 0; r <= R; ++r)\n        rank_offsets[r] = expert_offsets[first[r]];",
        "    if (first == NULL)\n        return ORC_INVALID_ARG;\n    oracle_partition(E, R, first);\n"
        "    for (int32_t r = 0; r <= R; ++r)\n        rank_offsets[r] = first[r];"),
    "validation_accepts_expert_E": (
        "            if (e < 0 || e >= E)\n                return ORC_EXPERT_OOB;",
        "            if (e < 0 || e > E)\n                return ORC_EXPERT_OOB;"),
    "node_cursor_counts_every_token": (
        "                if (touched) {\n                    node_slot[t * N + n] = ncursor[n];\n                    ncursor[n] += 1;\n                } else {\n                    node_slot[t * N + n] = -1;\n                }",
        "                node_slot[t * N + n] = touched ? ncursor[n] : -1;\n                ncursor[n] += 1;"),
    "rank_partials_rounded_before_sum": (
        "                total = total + part;",
        "                total = total + oracle_bf16_to_f32(oracle_f32_to_bf16(part));"),
    "rank_partials_reverse_rank_order": (
        "            for (int32_t r = 0; r < R; ++r) {\n                float part = 0.0f;",
        "            for (int32_t r = R - 1; r >= 0; --r) {\n                float part = 0.0f;"),
    "fp8_dispatch_inverse_scale": (
        "            recv_scale[dst] = st;",
        "            recv_scale[dst] = 1.0f / st;"),
}


PIN_FILES = ["test_oracle_partition.py", "test_oracle_layout.py", "test_oracle_dispatch_combine.py",
             "test_oracle_fp8.py", "test_oracle_ep.py", "test_oracle_properties.py"]


def _run_mutant(name, workdir):
    """Build the oracle with one planted mistake and run the pins on it;
    returns (returncode of the pin run, the end of its output)."""
    old, new = MUTANTS[name]
    src = open(SRC).read()
    if src.count(old) != 1:
        return None, f"mutation anchor for {name} must occur once"
    mutant_c = os.path.join(workdir, "mutant.c")
    with open(mutant_c, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(workdir, "libmutant.so")
    subprocess.run(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-shared", "-fPIC",
                    "-o", lib, mutant_c, "-lm"], check=True)
    env = dict(os.environ, MOE_ORACLE_LIB=lib)
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           "-k", "not full_workloads", *[os.path.join(ROOT, "tests", p) for p in PIN_FILES]]
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return res.returncode, res.stdout[-2000:] + res.stderr[-2000:]


@pytest.fixture(scope="module")
def mutant_runs(tmp_path_factory):
    """Every mutant's pin run, run concurrently (each is its own build and
    process, so they share nothing)."""
    names = sorted(MUTANTS)
    dirs = {n: str(tmp_path_factory.mktemp(n)) for n in names}
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as ex:
        futures = {n: ex.submit(_run_mutant, n, dirs[n]) for n in names}
        return {n: f.result() for n, f in futures.items()}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, mutant_runs):
    rc, out = mutant_runs[name]
    assert rc is not None, out
    assert rc == 1, f"mutant {name} passed every pin:\n{out}"
