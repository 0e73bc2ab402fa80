"""Planted mistakes: each mutant of the oracle source must fail at least one pin.

The mutants are made on the CPU from a copy of dsa_oracle.c (the oracle itself is never
edited); each is compiled to a temporary shared library and run against the pins."""
import os

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "dsa_oracle.c")

MUTANTS = {
    "relu_dropped": ("double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;"),
    "weight_index": ("total += (double)wt[h] * relu;", "total += (double)wt[0] * relu;"),
    "key_index_reversed": ("bf16_to_double(ks[d])", "bf16_to_double(ks[head_dim - 1 - d])"),
    "dot_sign": ("dot += bf16_to_double(qt[(long)h * head_dim + d])",
                 "dot -= bf16_to_double(qt[(long)h * head_dim + d])"),
    "causal_off_by_one": ("long v = q_pos0 + t + 1;", "long v = q_pos0 + t;"),
    "tie_to_higher_index": ("return a->index < b->index;", "return a->index > b->index;"),
    "rank_ascending": ("return a->score > b->score;", "return a->score < b->score;"),
    "nan_ranks_first": ("if (an != bn) return bn;", "if (an != bn) return an;"),
    "output_not_sorted": ("qsort(out, (size_t)take, sizeof(int32_t), cmp_int32);", ""),
    "pad_with_zero": ("for (long j = take; j < k; ++j) out[j] = -1;",
                      "for (long j = take; j < k; ++j) out[j] = 0;"),
    "scale_dropped": ("z[j] = scale * dot;", "z[j] = dot;"),
    "value_offset": ("for (int d = 0; d < dv; ++d) o[d] += p * bf16_to_double(c[d]);",
                     "for (int d = 0; d < dv; ++d) o[d] += p * bf16_to_double(c[d + 64]);"),
    "not_normalised": ("double p = exp(z[j] - zmax) / denom;", "double p = exp(z[j] - zmax);"),
    "reuse_ignored": ("if (compute_indices) {", "if (1) {"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) >= 1, f"mutation site for {name} not found"
    mutated = text.replace(old, new, 1)
    src = tmp_path / f"mutant_{name}.c"
    src.write_text(mutated)
    so = oracle.compile_c(str(src), str(tmp_path / f"mutant_{name}.so"))
    m = oracle.Oracle(so)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(m)
        except (AssertionError, RuntimeError, IndexError, ValueError):
            caught.append(pin.__name__)
            break
    assert caught, f"no pin catches the planted mistake {name}"
