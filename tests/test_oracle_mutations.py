"""Plant plausible mistakes in a copy of the oracle and check that the pins in
test_oracle_pins.py catch every one.  Each mutant is compiled from a modified
copy of oracle.c into a temporary directory; the committed oracle is never
touched.  CPU only."""
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import build as obuild
import test_oracle_pins as pins

# (name, text in oracle.c, replacement).  A change that cannot alter any
# result is left out.  Dropping pass 2's skip of rows whose LSE is -inf is
# one: pass 2 only reaches a row through an allowed (row, key) pair, and such
# a row always has a finite LSE.
MUTANTS = [
    ("causal_off_by_one", "case OR_MASK_CAUSAL: return j <= i + (s->Nk - s->Nq);",
     "case OR_MASK_CAUSAL: return j < i + (s->Nk - s->Nq);"),
    ("causal_offset_dropped", "case OR_MASK_CAUSAL: return j <= i + (s->Nk - s->Nq);",
     "case OR_MASK_CAUSAL: return j <= i;"),
    ("causal_offset_sign", "case OR_MASK_CAUSAL: return j <= i + (s->Nk - s->Nq);",
     "case OR_MASK_CAUSAL: return j <= i + (s->Nq - s->Nk);"),
    ("block_mask_transposed", "s->bm[(size_t)(i / s->block) * s->nbk + (j / s->block)]",
     "s->bm[(size_t)(j / s->block) * s->nbk + (i / s->block)]"),
    ("lse_drops_max", "return m + log(l);", "return log(l);"),
    ("no_normalisation", "for (int j = 0; j < s->Nk; ++j) S[j] /= l;", ""),
    ("scale_dropped_in_scores", "S[j] = s->scale * dot(q, Kh + (size_t)j * s->d, s->d);",
     "S[j] = dot(q, Kh + (size_t)j * s->d, s->d);"),
    ("dS_sign", "double ds = P[j] * (dP[j] - Di);", "double ds = P[j] * (dP[j] + Di);"),
    ("dQ_scale_dropped", "for (int k = 0; k < d; ++k) dq[k] *= scale;\n                if (O)",
     "\n                if (O)"),
    ("dK_transposed_operand", "dk[k] += ds * qi[k];", "dk[k] += ds * kj[k];"),
    ("dV_uses_dS", "dv[k] += p * doi[k];", "dv[k] += ds * doi[k];"),
    ("D_dropped_in_pass2", "double ds = p * (dp - Dv[(size_t)h * Nq + i]);", "double ds = p * dp;"),
    ("pv_wrong_row", "const double *v = V + hk + (size_t)j * d;\n                    for (int k = 0; k < d; ++k) o[k] += P[j] * v[k];\n                }\n            }\n        free(P);\n    }\n    return err;\n}\n\nint oracle_fwd(",
     "const double *v = V + hk + (size_t)(Nk - 1 - j) * d;\n                    for (int k = 0; k < d; ++k) o[k] += P[j] * v[k];\n                }\n            }\n        free(P);\n    }\n    return err;\n}\n\nint oracle_fwd("),
    # a row that sees no key: the running maximum must start at -inf
    ("empty_row_max_init", "double m = -INFINITY;", "double m = 0.0;"),
    ("pass2_scale_dropped", "double p = exp(s.scale * dot(qi, kj, d) - L);", "double p = exp(dot(qi, kj, d) - L);"),
    ("dK_scale_dropped", "for (int k = 0; k < d; ++k) dk[k] *= scale;", ""),
    ("dV_wrong_operand", "dv[k] += p * doi[k];", "dv[k] += p * qi[k];"),
    ("dQ_uses_V", "double ds = P[j] * (dP[j] - Di);\n                    const double *kj = K + hk",
     "double ds = P[j] * (dP[j] - Di);\n                    const double *kj = V + hk"),
    # the block grid's row length is the number of key blocks
    ("block_row_length_from_queries", "s.nbk = (Nk + s.block - 1) / s.block;", "s.nbk = (Nq + s.block - 1) / s.block;"),
    # the single-row path used for sampled parity at full size
    ("rows_dS_sign", "double ds = P[j] * (dot(doi, V + hk + (size_t)j * d, d) - Di);",
     "double ds = P[j] * (dot(doi, V + hk + (size_t)j * d, d) + Di);"),
    # the key-column path used for sampled dK, dV parity at full size
    ("cols_dS_sign", "const double dsij = pij * (dpij - Dv[(size_t)h * Nq + i]);",
     "const double dsij = pij * (dpij + Dv[(size_t)h * Nq + i]);"),
    ("cols_dV_uses_dS", "gv[k] += pij * doi[k];", "gv[k] += dsij * doi[k];"),
    ("cols_D_without_P", "if (P[j] != 0.0) Di += P[j] * dot(doi, V + hk + (size_t)j * d, d);\n                lse",
     "if (P[j] != 0.0) Di += dot(doi, V + hk + (size_t)j * d, d);\n                lse"),
    ("cols_scale_dropped", "for (int k = 0; k < d; ++k) gk[k] *= scale;", ""),
]

# The pins each mutant is run against (all cheap).
PIN_CALLS = [
    ("worked_none", lambda gd: pins.test_worked_example_closed_form(gd, "none")),
    ("worked_causal", lambda gd: pins.test_worked_example_closed_form(gd, "causal")),
    ("tiling_block", lambda gd: pins.test_online_blocked_equals_two_pass("block", (64, 64))),
    ("tiling_causal", lambda gd: pins.test_online_blocked_equals_two_pass("causal", (7, 7))),
    ("probs_block", lambda gd: pins.test_probability_rows("block")),
    ("const_scores_block", lambda gd: pins.test_constant_scores_give_mean_of_visible_values("block")),
    ("single_key", lambda gd: pins.test_single_key()),
    ("fd_block", lambda gd: pins.test_gradients_by_finite_differences("block")),
    ("identities_causal", lambda gd: pins.test_gradient_identities("causal")),
    ("sdpa_causal", lambda gd: pins.test_against_torch_sdpa_fp64("causal", (1, 3, 128, 64))),
    ("sdpa_block", lambda gd: pins.test_against_torch_sdpa_fp64("block", (2, 2, 200, 32))),
    ("cross_suffix", lambda gd: pins.test_cross_causal_suffix_equals_square_problem()),
    ("cross_more_queries", lambda gd: pins.test_cross_causal_more_queries_than_keys()),
    ("cross_block", lambda gd: pins.test_cross_block_mask_is_query_blocks_by_key_blocks()),
    ("rows_block", lambda gd: pins.test_row_path_matches_full_path("block")),
    ("cols_block", lambda gd: pins.test_col_path_matches_full_path("block")),
]


def _compile(src_text, out_dir, name):
    c = os.path.join(out_dir, f"{name}.c")
    so = os.path.join(out_dir, f"lib{name}.so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-w",
                    "-o", so, c, "-lm"], check=True)
    return so


def test_unmutated_copy_passes_all_pins(tmp_path, golden_dir):
    src = open(obuild.SRC).read()
    so = _compile(src, str(tmp_path), "clean")
    with oracle.using(so):
        for _, call in PIN_CALLS:
            call(golden_dir)


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(mutant, tmp_path, golden_dir):
    name, old, new = mutant
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    so = _compile(src.replace(old, new), str(tmp_path), name)
    caught = []
    with oracle.using(so):
        for pin, call in PIN_CALLS:
            try:
                with np.errstate(all="ignore"):
                    call(golden_dir)
            except (AssertionError, RuntimeError, ValueError, FloatingPointError):
                caught.append(pin)
    assert caught, f"no pin caught the planted mistake {name}"
