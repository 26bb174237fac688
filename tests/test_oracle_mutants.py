"""Plants plausible mistakes in the oracle's C source and checks that every one
of them trips at least one pin. This shows the pins constrain each part of the
oracle (scale, head-to-group map, position range, normalisation, operand roles,
min-over-heads, the tie rule, the cosine's norms). CPU only; each mutant is
compiled into a temporary library."""
import os

import pytest

import oracle
from tests import pins

MUTANTS = [
    ("scale_1_over_d", "double scale = 1.0 / sqrt((double)d);", "double scale = 1.0 / (double)d;"),
    ("interleaved_head_map", "    int h = g * M + m;\n    double *o", "    int h = m * J->Hkv + g;\n    double *o"),
    ("drops_position_0",
     "for (int j = 0; j < L; ++j) {\n        double acc = 0.0;",
     "for (int j = 1; j < L; ++j) {\n        double acc = 0.0;"),
    ("drops_last_position",
     "for (int j = 0; j < L; ++j) {\n        double acc = 0.0;",
     "for (int j = 0; j < L - 1; ++j) {\n        double acc = 0.0;"),
    ("unnormalised_weights", "double p = logit[j] / z;", "double p = logit[j];"),
    ("keys_read_from_values", "const uint16_t *kj = K + (size_t)j * d;", "const uint16_t *kj = V + (size_t)j * d;"),
    ("max_over_heads", "if (c < s)\n                    s = c;", "if (c > s || m == 0)\n                    s = c;"),
    ("strict_threshold", "int sink = (s >= tau);", "int sink = (s > tau);"),
    ("cosine_without_key_norm", "return dot / (sqrt(qq) * sqrt(kk));", "return dot / sqrt(qq);"),
    ("sink_returns_cache_row_1",
     "const uint16_t *v0g = J->v0 + ((size_t)b * J->Hkv + g) * d;",
     "const uint16_t *v0g = V + (size_t)d;"),
    ("p0_reports_last_weight", "J->p0[(size_t)b * J->Hq + h] = logit[0] / z;",
     "J->p0[(size_t)b * J->Hq + h] = logit[L - 1] / z;"),
    ("rope_sign", "out[i] = narrow_to_bf16(a * (double)c[i] - b * (double)s[i]);",
     "out[i] = narrow_to_bf16(a * (double)c[i] + b * (double)s[i]);"),
    ("rope_adjacent_pairs", "double a = widen_bf16(x[i]), b = widen_bf16(x[i + h]);",
     "double a = widen_bf16(x[i]), b = widen_bf16(x[(i + 1) % d]);"),
    ("no_position0_capture", "memcpy(k0 + unit * d, kslot, sizeof(uint16_t) * (size_t)d);", ""),
    ("length_not_advanced", "seq_lens[b] = p + 1;", "seq_lens[b] = p;"),
    ("ties_away_from_zero", "double y = ldexp(rint(ldexp(x, -spacing)), spacing);",
     "double y = ldexp(round(ldexp(x, -spacing)), spacing);"),
    ("rope_row_of_next_position", "const float *c = rope_cos + (size_t)p * (d / 2);",
     "const float *c = rope_cos + (size_t)(p + 1) * (d / 2);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique in the oracle source"
    mutated = tmp_path / f"{name}.c"
    mutated.write_text(src.replace(old, new))
    lib = oracle.build(str(mutated), str(tmp_path / f"lib_{name}.so"))
    o = oracle.Oracle(lib)
    failures = []
    for pin in pins.PINS:
        try:
            pin(o)
        except (AssertionError, ValueError) as e:  # a pin fired
            failures.append((pin.__name__, str(e)[:80]))
    assert failures, f"mutant {name} passed every pin"
    os.remove(lib)
