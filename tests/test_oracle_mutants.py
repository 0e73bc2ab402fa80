"""Planted mistakes: each mutant of the oracle source must fail at least one pin.

The mutants are made on the CPU from a copy of dsa_oracle.c (the oracle itself is never
edited); each is compiled to a temporary shared library and run against the pins."""
import os

import pytest

import oracle
import pins

HERE = os.path.dirname(oracle.__file__)
SRC = os.path.join(HERE, "dsa_oracle.c")
VERIFY_SRC = os.path.join(HERE, "verify_oracle.c")
FP8_SRC = os.path.join(HERE, "fp8_oracle.c")
SHARD_SRC = os.path.join(HERE, "shard_oracle.c")
SOURCES = [SRC, VERIFY_SRC, FP8_SRC, SHARD_SRC]

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
    # MTP verify step (verify_oracle.c)
    "verify_max_not_min": ("a += (double)(p[v] < q[v] ? p[v] : q[v]);", "a += (double)(p[v] > q[v] ? p[v] : q[v]);",
                           VERIFY_SRC),
    "verify_accept_reversed": ("accept[r] = uq < pr[x] ? 1 : 0;", "accept[r] = uq > pr[x] ? 1 : 0;", VERIFY_SRC),
    "verify_residual_sign": ("float r = p[v] - q[v];\n        if (r > 0.0f) run",
                             "float r = q[v] - p[v];\n        if (r > 0.0f) run", VERIFY_SRC),
    "verify_resample_from_p": (": resample(pr, qr, V, u2[r], x)", ": resample(pr, pr, V, u2[r], x)",
                               VERIFY_SRC),
    "verify_len_counts_all": ("while (n < S && accept[(long)b * S + n]) ++n;",
                              "for (int j = 0; j < S; ++j) n += accept[(long)b * S + j];", VERIFY_SRC),
    # FP8 index keys (fp8_oracle.c)
    "e4m3_bias": ("ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)", FP8_SRC),
    "e4m3_subnormal_scale": ("ldexp((double)m / 8.0, -6)", "ldexp((double)m / 8.0, -7)", FP8_SRC),
    "e4m3_relu_dropped": ("total += (double)wt[h] * (dot > 0.0 ? dot : 0.0);", "total += (double)wt[h] * dot;", FP8_SRC),
    "e4m3_key_index": ("oracle_e4m3_to_double(ks[d])", "oracle_e4m3_to_double(ks[0])", FP8_SRC),
    # context-sharded decode (shard_oracle.c)
    "shard_lse_base2": ("lse[(b * T + t) * (long)H + h] = zmax + log(denom);",
                        "lse[(b * T + t) * (long)H + h] = zmax + log2(denom);", SHARD_SRC),
    "shard_lse_drops_max": ("lse[(b * T + t) * (long)H + h] = zmax + log(denom);",
                            "lse[(b * T + t) * (long)H + h] = log(denom);", SHARD_SRC),
    "shard_range_exclusive_low": ("if (g < offset || g >= offset + Ns) continue;\n                    const uint16_t *c",
                                  "if (g <= offset || g >= offset + Ns) continue;\n                    const uint16_t *c",
                                  SHARD_SRC),
    "merge_weight_sign": ("const double c = exp(lses[(long)w * R + r] - m) / s;",
                          "const double c = exp(m - lses[(long)w * R + r]) / s;", SHARD_SRC),
    "merge_unnormalised": ("const double c = exp(lses[(long)w * R + r] - m) / s;",
                           "const double c = exp(lses[(long)w * R + r] - m);", SHARD_SRC),
    "cand_tie_to_higher": ("return a->pos < b->pos;", "return a->pos > b->pos;", SHARD_SRC),
    "cand_not_sorted": ("qsort(o, (size_t)take, sizeof(int32_t), sh_cmp_i32);", "", SHARD_SRC),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new, target = (MUTANTS[name] + (SRC,))[:3]
    text = open(target).read()
    assert text.count(old) >= 1, f"mutation site for {name} not found"
    mutated = text.replace(old, new, 1)
    src = tmp_path / f"mutant_{name}.c"
    src.write_text(mutated)
    others = [x for x in SOURCES if x != target]
    so = oracle.compile_c([str(src)] + others, str(tmp_path / f"mutant_{name}.so"))
    m = oracle.Oracle(so)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(m)
        except (AssertionError, RuntimeError, IndexError, ValueError):
            caught.append(pin.__name__)
            break
    assert caught, f"no pin catches the planted mistake {name}"
