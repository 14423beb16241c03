"""Plant plausible mistakes in a copy of the oracle (CPU only) and check that
the pins catch every one.  Each mutant is built from the oracle's source by
an exact text substitution and run in a child process, so a mutant that
crashes counts as caught without taking pytest down."""
import json
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "head_map_modulo": ("int g = h / (p->Hq / p->Hkv);", "int g = h % p->Hkv;"),
    "no_block_table": (
        "int32_t phys = p->block_tables[(int64_t)b * p->max_blocks_per_seq + logical_block];",
        "int32_t phys = logical_block;"),
    "head_before_token_layout": (
        "return (((int64_t)phys * p->block_size + offset) * p->Hkv + g) * p->D + d;",
        "return (((int64_t)phys * p->Hkv + g) * p->block_size + offset) * p->D + d;"),
    "scale_dropped": ("return p->scale * dot;", "return dot;"),
    "no_normalisation": ("        out[d] /= den;\n}", "        out[d] /= 1.0;\n}"),
    "k_read_as_v": ("out[d] += w * value_at(p->v_cache,", "out[d] += w * value_at(p->k_cache,"),
    "last_token_dropped": ("    for (int t = 0; t < L; ++t) {\n        double w", "    for (int t = 0; t < L - 1; ++t) {\n        double w"),
    "softmax_sign_flipped": ("double w = exp(s[t] - m);\n        den", "double w = exp(m - s[t]);\n        den"),
    "q_index_transposed": ("value_at(p->q, ((int64_t)b * p->Hq + h) * p->D + d", "value_at(p->q, ((int64_t)h * p->B + b) * p->D + d"),
    "merge_without_rescale": ("double c = exp(pm[part] - M);", "double c = 1.0;"),
    "append_offset_dropped": ("int64_t offset = s % block_size;", "int64_t offset = 0;"),
    "append_v_from_k": ("memcpy((char *)v_cache + dst, (const char *)v_new",
                        "memcpy((char *)v_cache + dst, (const char *)k_new"),
    "prefill_sees_one_future_token": ("attend_prefill(p, row, b, h, pos + 1, s, out + i * p->D);",
                                      "attend_prefill(p, row, b, h, pos + 2 <= p->context_lens[b] ? pos + 2 : pos + 1, s, out + i * p->D);"),
    "prefill_misses_itself": ("attend_prefill(p, row, b, h, pos + 1, s, out + i * p->D);",
                              "attend_prefill(p, row, b, h, pos > 0 ? pos : 1, s, out + i * p->D);"),
    "prefill_positions_from_zero": ("int pos = p->context_lens[b] - n + (int)(row - query_start[b]);",
                                    "int pos = (int)(row - query_start[b]);"),
    "prefill_not_causal": ("attend_prefill(p, row, b, h, pos + 1, s, out + i * p->D);",
                           "attend_prefill(p, row, b, h, p->context_lens[b], s, out + i * p->D);"),
    "prefill_q_row_of_request": ("double qd = value_at(p->q, (row * p->Hq + h) * p->D + d, p->dtype);",
                                 "double qd = value_at(p->q, ((int64_t)b * p->Hq + h) * p->D + d, p->dtype);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "paged_attn_oracle.c")).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = str(tmp_path / "libmutant.so")
    oracle.build(force=True, src=str(mutated), out=lib)
    proc = subprocess.run([sys.executable, "-m", "tests.oracle_pins", lib], cwd=ROOT, capture_output=True,
                          text=True, timeout=600)
    if proc.returncode != 0:
        return  # the mutant crashed the pins: caught
    failed = json.loads(proc.stdout.strip().splitlines()[-1])
    assert failed, f"no pin caught mutant {name}"
