"""Plant a plausible mistake in a copy of the oracle and check a pin catches it.

Each mutation is a one-line edit of oracle/oracle.c compiled into a temporary
library (CPU only); the pins of tests/oracle_pins.py run against it and at
least one must fail.  This shows the pins constrain every step of the oracle:
the store's slot decoding, the gather, the head map, the scale, the causal
position, the softmax normalisation, the value gather, the rotary embedding's
direction, pairing, frequencies, positions and row addressing, and the bf16
rounding.
"""

import os
import subprocess

import pytest

from oracle import oracle as O
from oracle_pins import ALL_CHECKS

SRC = os.path.join(os.path.dirname(O.__file__), "oracle.c")

MUTATIONS = {
    "scale_1_over_D": ("job.scale = scale > 0.0 ? scale : 1.0 / sqrt((double)head_dim);",
                       "job.scale = scale > 0.0 ? scale : 1.0 / (double)head_dim;"),
    "head_map_modulo": ("const int32_t hk = hq / group;", "const int32_t hk = hq % job->num_kv_heads;"),
    "mask_off_by_one": ("const int32_t visible = pos + 1;", "const int32_t visible = pos;"),
    "causal_top_left": ("const int32_t pos = L_b - n_b + i;", "const int32_t pos = (i < L_b ? i : L_b - 1);"),
    "gather_offset": ("const uint16_t *krow = job->k_pool + (((int64_t)blk * BS + j % BS)",
                      "const uint16_t *krow = job->k_pool + (((int64_t)blk * BS + (j + 1) % BS)"),
    "gather_block_index": ("const int32_t blk = job->block_tables[(int64_t)b * job->max_blocks_per_seq + j / BS];\n"
                           "        if (blk < 0",
                           "const int32_t blk = job->block_tables[(int64_t)b * job->max_blocks_per_seq + j % "
                           "job->max_blocks_per_seq / BS];\n        if (blk < 0"),
    "value_from_key_pool": ("const uint16_t *vrow = job->v_pool", "const uint16_t *vrow = job->k_pool"),
    "no_normalisation": ("orow[d] /= denom;", "orow[d] /= (double)visible;"),
    "store_offset": ("const int64_t offset = s % block_size;", "const int64_t offset = s % block_size / 2;"),
    "store_skips_last_token": ("for (int32_t t = 0; t < num_tokens; ++t) {",
                               "for (int32_t t = 0; t + 1 < num_tokens; ++t) {"),
    "rope_sin_sign": ("o[i] = x1 * c - x2 * s;", "o[i] = x1 * c + x2 * s;"),
    "rope_adjacent_pairs": ("const double x2 = bf16_to_double(row[i + half]);",
                            "const double x2 = bf16_to_double(row[half - 1 - i]);"),
    "rope_frequency_exponent": ("pow(base, -2.0 * (double)i / (double)head_dim)",
                                "pow(base, -(double)i / (double)head_dim)"),
    "rope_position_shift": ("const double p = (double)positions[t];", "const double p = (double)positions[t] + 1.0;"),
    "rope_head_stride": ("const uint16_t *row = x + t * token_stride + (int64_t)h * head_dim;",
                         "const uint16_t *row = x + t * token_stride + (int64_t)h * half;"),
    "bf16_round_down": ("ldexp(nearbyint(ldexp(a, -q)), q)", "ldexp(floor(ldexp(a, -q)), q)"),
    "bf16_ties_away": ("ldexp(nearbyint(ldexp(a, -q)), q)", "ldexp(round(ldexp(a, -q)), q)"),
    "query_row_index": ("const uint16_t *qrow = job->q + (r * job->num_q_heads + hq) * (int64_t)D;",
                        "const uint16_t *qrow = job->q + (r * job->num_q_heads + hq % 2) * (int64_t)D;"),
}


def _build_mutant(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation {name}: pattern not unique in oracle.c"
    path = tmp_path / f"oracle_{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"liboracle_{name}.so"
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread", str(path), "-o", str(so), "-lm"])
    return O.load(str(so))


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_a_pin_catches_mutation(name, tmp_path):
    lib = _build_mutant(tmp_path, name)
    caught = []
    for check in ALL_CHECKS:
        try:
            check(lib)
        except (AssertionError, O.OracleError, ValueError, IndexError):
            caught.append(check.__name__)
    assert caught, f"no pin catches mutation {name}"
