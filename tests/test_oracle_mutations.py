"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/ep_oracle.c (on the CPU),
builds it, and runs tests/test_oracle_pins.py against that build: the pins
must fail.  This checks the claim that a dropped term, a wrong sign or index,
or a swapped operand anywhere in the oracle fails at least one pin."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ep_oracle.c")

# (name, text to find in ep_oracle.c, replacement)
MUTANTS = [
    ("rank_of_expert_modulo",
     "in_rank[((size_t)s * T + t) * R + e / El] = 1;",
     "in_rank[((size_t)s * T + t) * R + e % R] = 1;"),
    ("experts_counted_once_per_token",
     "ntpe[(size_t)s * E + e] += 1;",
     "ntpe[(size_t)s * E + e] = 1;"),
    ("prefix_matrix_exclusive",
     "                run += in_rank[((size_t)s * T + t) * R + d];\n            P[(size_t)s * R + d] = run;",
     "                ;\n            P[(size_t)s * R + d] = run;\n            for (int t = 0; t < T; ++t) run += in_rank[((size_t)s * T + t) * R + d];"),
    ("rows_ordered_token_major",
     "        for (int s = 0; s < R; ++s) {\n            for (int t = 0; t < T; ++t) {\n                size_t i = ((size_t)s * T + t) * R + d;",
     "        for (int t0 = 0; t0 < T; ++t0) {\n            for (int s0 = 0; s0 < R; ++s0) {\n                int s = s0, t = t0;\n                size_t i = ((size_t)s * T + t) * R + d;"),
    ("global_instead_of_local_expert_id",
     "recv_topk_idx[o] = local ? (e - (int64_t)d * El) : -1;",
     "recv_topk_idx[o] = local ? e : -1;"),
    ("nonlocal_weight_kept",
     "recv_topk_weights[o] = local ? topk_weights[st * K + k] : 0.0f;",
     "recv_topk_weights[o] = topk_weights[st * K + k];"),
    ("combine_drops_last_copy",
     "            for (int d = 0; d < R; ++d) {\n                int32_t row = send_pos[(size_t)st * R + d];\n                if (row < 0 || row >= cap)\n                    continue;\n                acc = acc + orc_bf16_to_f32",
     "            for (int d = 0; d < R - 1; ++d) {\n                int32_t row = send_pos[(size_t)st * R + d];\n                if (row < 0 || row >= cap)\n                    continue;\n                acc = acc + orc_bf16_to_f32"),
    ("combine_skips_bias1",
     "                acc = acc + orc_bf16_to_f32(bias1[(size_t)st * H + h]);",
     "                ;"),
    ("bf16_round_half_up",
     "    u += 0x7FFFu + lsb;",
     "    u += 0x8000u + 0 * lsb;"),
    ("e4m3_ties_away_from_zero",
     "    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;",
     "    return fl + 1.0;"),
    ("e4m3_wrong_bias",
     "    int E = e + 7;",
     "    int E = e + 8;"),
    ("e4m3_overflow_not_saturated",
     "    if (a >= 448.0)\n        return (uint8_t)(sign | 0x7E);",
     "    if (a >= 464.0)\n        return (uint8_t)(sign | 0x7F);"),
    ("scale_inverted",
     "        inv = 448.0f / amax;\n            scale = amax / 448.0f;",
     "        inv = 448.0f / amax;\n            scale = 448.0f / amax;"),
    ("amax_floor_dropped",
     "        if (amax < 1e-4f)\n            amax = 1e-4f;\n        float scale, inv;",
     "        float scale, inv;"),
    ("round_scale_rounds_down",
     "            int e = (fr == 0.5) ? ex - 1 : ex;     /* 2^e >= sf, 2^(e-1) < sf */",
     "            int e = ex - 1;"),
    ("ll_repeated_expert_gets_new_row",
     "                if (first >= 0) {\n                    ll_pos[st * K + k] = ll_pos[st * K + first];\n                    continue;\n                }",
     "                (void)first;"),
    ("ll_combine_first_weight_only",
     "                acc = fmaf(v, topk_weights[(size_t)st * K + k], acc);",
     "                acc = fmaf(v, topk_weights[(size_t)st * K + 0], acc);"),
    ("ll_mask_ignores_destination",
     "                if (mask && (mask[s] || mask[e / El])) {\n                    ll_pos[st * K + k] = -1;",
     "                if (mask && mask[s]) {\n                    ll_pos[st * K + k] = -1;"),
    ("expert_counts_aligned_down",
     "                n = (n + align - 1) / align * align;",
     "                n = n / align * align;"),
    ("handle_stores_source_rank",
     "                    recv_src_idx[(size_t)d * cap + row] = t;",
     "                    recv_src_idx[(size_t)d * cap + row] = s;"),
    ("dispatch_copies_neighbour_row",
     "                   x + (size_t)st * H, sizeof(uint16_t) * (size_t)H);",
     "                   x + (size_t)(st + (st + 1 < (long)R * T)) * H, sizeof(uint16_t) * (size_t)H);"),
    ("combined_weights_last_copy_only",
     "                    acc = acc + recv_w[((size_t)d * cap + row) * K + k];",
     "                    acc = recv_w[((size_t)d * cap + row) * K + k];"),
    ("ll_range_begin_after_source",
     "        for (int e = 0; e < E; ++e)\n            layout_range[((size_t)e * R + s) * 2 + 0] = count[e];\n        for (int t = 0; t < T; ++t) {",
     "        for (int t = 0; t < T; ++t) {"),
    ("dequant_by_inverse_scale",
     "            float v = orc_e4m3_to_f32(q[(size_t)r * H + h]) *\n                      scales[(size_t)r * (H / 128) + h / 128];",
     "            float v = orc_e4m3_to_f32(q[(size_t)r * H + h]) /\n                      scales[(size_t)r * (H / 128) + h / 128];"),
]


@pytest.mark.slow
@pytest.mark.parametrize("name,find,repl", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_fail_on_mutant(name, find, repl, tmp_path):
    src = open(SRC).read()
    assert src.count(find) >= 1, f"mutation anchor not found: {name}"
    mutated = src.replace(find, repl, 1)
    csrc = tmp_path / "ep_oracle.c"
    csrc.write_text(mutated)
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
                           "-o", str(lib), str(csrc), "-lm"])
    env = dict(os.environ, EP_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests",
                        "test_oracle_pins.py"), "-x", "-q", "-p", "no:cacheprovider",
                        f"--basetemp={tmp_path / 'inner'}"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-1500:]}"
