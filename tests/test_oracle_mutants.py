"""Plant plausible mistakes in copies of the CPU oracle and require every one
to fail at least one pin (no GPU).  This shows the pins constrain each part of
the oracle: a dropped term, a wrong sign or index, a transposed operand, a
reversed order or a wrong constant is caught."""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "oracle.c")

# (name, exact snippet in oracle.c, replacement)
MUTANTS = [
    ("max_vio_minus_one_dropped", "(double)P - 1.0 : 0.0", "(double)P - 0.0 : 0.0"),
    ("max_vio_mean_off_by_one", "((double)mx * (double)E) / (double)P", "((double)mx * (double)E) / (double)(P + 1)"),
    ("stats_counts_bad_ids", "    if (e < 0 || e >= E) {\n      ++bad;\n      continue;\n    }\n    loads[e] += 1;",
     "    if (e < 0 || e >= E) {\n      ++bad;\n      e = 0;\n    }\n    loads[e] += 1;"),
    ("chunks_ascending_id", "for (int e = (r + 1) * ER - 1; e >= r * ER && rem > 0; --e)",
     "for (int e = r * ER; e < (r + 1) * ER && rem > 0; ++e)"),
    ("chunk_min_dropped", "int64_t take = loads[e] < rem ? loads[e] : rem;", "int64_t take = rem;"),
    ("deficits_descending_rank", "  for (int r = 0; r < R; ++r) {\n    if (SK - L[r] > 0) {",
     "  for (int r = R - 1; r >= 0; --r) {\n    if (SK - L[r] > 0) {"),
    ("match_tie_advances_one", "    if (left_d == 0) {\n      ++j;", "    else if (left_d == 0) {\n      ++j;"),
    ("home_count_not_reduced", "home_count[rep_expert[m]] -= rep_count[m];", "home_count[rep_expert[m]] -= 0;"),
    ("home_takes_last_pairs", "int32_t p = list[start[e] + i];", "int32_t p = list[start[e] + (home_count[e] - 1 - i)];"),
    ("replica_range_from_zero", "    rep_first[m] = next[rep_expert[m]];", "    rep_first[m] = 0;"),
    ("replica_rows_reversed", "int32_t p = list[start[e] + rep_first[m] + i];",
     "int32_t p = list[start[e] + rep_first[m] + (rep_count[m] - 1 - i)];"),
    ("cu_seqlens_end_off_by_one", "cu_seqlens[nslot] = (int32_t)P;", "cu_seqlens[nslot] = (int32_t)(P - 1);"),
    ("align_pad_off_by_one", "int64_t padded = (cnt[e] + block_m - 1) / block_m * block_m;",
     "int64_t padded = (cnt[e] + block_m) / block_m * block_m;"),
    ("align_sentinel_wrong", "for (int64_t i = 0; i < sorted_cap; ++i) sorted_ids[i] = (int32_t)P;",
     "for (int64_t i = 0; i < sorted_cap; ++i) sorted_ids[i] = (int32_t)(P - 1);"),
    ("align_block_expert_shift", "b < off[e + 1] / block_m; ++b) expert_ids[b] = e;",
     "b < off[e + 1] / block_m; ++b) expert_ids[b] = e + (b > 0);"),
    ("dispatch_token_rounding", "x + (p / K) * H", "x + ((p + K - 1) / K) * H"),
    ("combine_weight_transposed", "float prod = w[t * K + k] * bf16_to_f32(y[(int64_t)row * H + h]);",
     "float prod = w[k * T + t] * bf16_to_f32(y[(int64_t)row * H + h]);"),
    ("combine_wrong_sign", "        float prod = w[t * K + k] * bf16_to_f32(y[(int64_t)row * H + h]);\n        acc = acc + prod;",
     "        float prod = w[t * K + k] * bf16_to_f32(y[(int64_t)row * H + h]);\n        acc = acc - prod;"),
    ("combine_first_term_dropped",
     "      for (int k = 0; k < K; ++k) {\n        int32_t row = pos[t * K + k];\n        if (row < 0) continue;\n        float prod",
     "      for (int k = 1; k < K; ++k) {\n        int32_t row = pos[t * K + k];\n        if (row < 0) continue;\n        float prod"),
    ("bf16_round_half_up", "  uint32_t lsb = (u >> 16) & 1u;\n  u += 0x7FFFu + lsb;", "  uint32_t lsb = 1u;\n  u += 0x7FFFu + lsb;"),
    ("grad_home_dropped", "for (int64_t j = 0; j < n; ++j) dst[j] = dst[j] + g[j];", "for (int64_t j = 0; j < n; ++j) dst[j] = g[j];"),
    ("grad_bf16_wrong_widen", "dst[j] = dst[j] + bf16_to_f32(g[j]);", "dst[j] = dst[j] + (float)g[j];"),
    ("grad_no_clear", "if (clear) memset(g, 0, (size_t)n * 4);", "if (0) memset(g, 0, (size_t)n * 4);"),
    ("dispatch_bwd_first_term_dropped", "        acc = acc + bf16_to_f32(dbuf[(int64_t)row * H + h]);",
     "        if (k > 0) acc = acc + bf16_to_f32(dbuf[(int64_t)row * H + h]);"),
    ("combine_bwd_weight_index", "dy[(int64_t)row * H + h] = f32_to_bf16(w[t * K + k] * g);",
     "dy[(int64_t)row * H + h] = f32_to_bf16(w[t * K] * g);"),
    ("quota_ties_to_higher_id", "if (!used[e] && (best < 0 || loads[e] > loads[best])) best = e;",
     "if (!used[e] && (best < 0 || loads[e] >= loads[best])) best = e;"),
    ("quota_descending_id_chunks", "if (!used[e] && (best < 0 || loads[e] > loads[best])) best = e;",
     "if (!used[e] && (best < 0 || e > best)) best = e;"),
    ("quota_no_slot_budget", "if (left_r == 0 || pieces == B) {", "if (left_r == 0) {"),
    ("quota_rooms_descending", "  for (int r = 0; r < R; ++r) {\n    if (tau - H[r] > 0) {",
     "  for (int r = R - 1; r >= 0; --r) {\n    if (tau - H[r] > 0) {"),
    ("quota_pieces_not_reset", "      ++j;\n      pieces = 0;", "      ++j;\n      pieces = pieces;"),
    ("quota_chunk_whole_expert", "int64_t take = loads[best] < rem ? loads[best] : rem;", "int64_t take = loads[best];"),
    ("quota_zero_rooms", "if (tau - H[r] > 0) {\n      rm_r[nrm] = r;", "if (tau - H[r] >= 0) {\n      rm_r[nrm] = r;"),
    ("quota_scan_from_above", "int64_t tau = (P + R - 1) / R;", "int64_t tau = (P + R - 1) / R + 1;"),
    ("quota_no_locality", "if (i >= 0 && ls < il[i]) {", "if (i >= 0 && ls < 0) {"),
    ("quota_local_not_capped", "il[i] = iq[i] < Lm[ir[i] * E + ie[i]] ? iq[i] : Lm[ir[i] * E + ie[i]];",
     "il[i] = Lm[ir[i] * E + ie[i]];"),
    ("quota_lookup_off_by_one", "if (jj >= ic[c] && jj < ic[c] + (iq[c] - il[c])) {",
     "if (jj > ic[c] && jj <= ic[c] + (iq[c] - il[c])) {"),
    ("capped_home_by_mod", "load_capped[rep_expert[m] / ER]", "load_capped[rep_expert[m] % R]"),
    ("prefetch_slot_off_by_one", "    if (j < B) {\n      slot[m] = E + j;", "    if (j <= B) {\n      slot[m] = E + j;"),
    ("combine_bwd_dw_wrong_row", "s += (double)g * (double)bf16_to_f32(y[(int64_t)row * H + h]);",
     "s += (double)g * (double)bf16_to_f32(y[(int64_t)(t * K + k) * H + h]);"),
]

RUNNER = r"""
import sys
sys.path[:0] = [%r, %r]
import oracle as O, oracle_pins as PINS
L = O.lib(sys.argv[1])
for pin in PINS.ALL_PINS:
    try:
        pin(L)
    except Exception as exc:
        print("caught by", pin.__name__, type(exc).__name__)
        sys.exit(1)
print("SURVIVED")
sys.exit(0)
""" % (ROOT, HERE)


def _run(mut, tmp):
    name, old, new = mut
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation {name}: snippet not found exactly once"
    path = os.path.join(tmp, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(tmp, f"lib{name}.so")
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-w", "-o", so, path])
    r = subprocess.run([sys.executable, "-c", RUNNER, so], capture_output=True, text=True, timeout=600)
    return name, r.returncode, (r.stdout + r.stderr)[-400:]


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda m: _run(m, tmp), MUTANTS))
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
