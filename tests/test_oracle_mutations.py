"""Planted mistakes in the oracle must fail its pins.

Each case compiles a copy of ``oracle/hstu_oracle.c`` with one plausible slip (a dropped
term, a flipped sign, an off-by-one in the mask or page index, the wrong LayerNorm axis or
variance) into a temporary directory, swaps it in for the real library, and runs the pin
tests from ``test_oracle_pins.py``.  At least one pin must fail for every mutant.  Only the
oracle is mutated, and only on the CPU.
"""
import ctypes
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
from tests import test_oracle_bwd_pins as bwd_pins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "hstu_oracle.c")

MUTANTS = {
    "no_target_mask": ("int allowed = (j <= i && j < hist) || (i >= hist && j == i);",
                       "int allowed = (j <= i);"),
    "drop_self": ("int allowed = (j <= i && j < hist) || (i >= hist && j == i);",
                  "int allowed = (j < i && j < hist);"),
    "drop_rab": ("s += (double)a->rab[(int64_t)h * a->NB + oracle_bucket(i - j, a->n_max, a->NB)];",
                 ""),
    "rab_reversed_distance": ("oracle_bucket(i - j, a->n_max, a->NB)", "oracle_bucket(j - i, a->n_max, a->NB)"),
    "rab_wrong_head": ("a->rab[(int64_t)h * a->NB +", "a->rab["),
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-s));", "return 1.0 / (1.0 + exp(s));"),
    "drop_scale": ("double w = s * sigmoid(s) * inv_n;", "double w = s * sigmoid(s);"),
    "unbiased_variance": ("    var /= (double)HD;", "    var /= (double)(HD - 1);"),
    "eps_outside_sqrt": ("double rstd = 1.0 / sqrt(var + a->eps);", "double rstd = 1.0 / (sqrt(var) + a->eps);"),
    "gate_wrong_index": ("out_row[e] = (o[e] - mean) * rstd * u[e];", "out_row[e] = (o[e] - mean) * rstd * u[0];"),
    "key_head_offset": ("const double* kj = K + j * HD + (int64_t)h * D;", "const double* kj = K + j * HD;"),
    "value_head_offset": ("const double* vj = V + j * HD + (int64_t)h * D;", "const double* vj = V + j * HD;"),
    "bucket_off_by_one": ("int64_t b = 1 + (int64_t)floor(x);", "int64_t b = (int64_t)floor(x);"),
    "page_slot": ("int64_t idx = (((int64_t)page * H + h) * P + j % P) * D + c;",
                  "int64_t idx = (((int64_t)page * H + h) * P + (j + 1) % P) * D + c;"),
    "page_layout_transposed": ("int64_t idx = (((int64_t)page * H + h) * P + j % P) * D + c;",
                               "int64_t idx = (((int64_t)page * P + j % P) * H + h) * D + c;"),
    "paged_query_position": ("int64_t i = C + (t - J->new_offsets[b]);", "int64_t i = t - J->new_offsets[b];"),
    "append_slot": ("int64_t slot = pos % page_size;", "int64_t slot = t % page_size;"),
    # backward pass
    "bwd_silu_derivative": ("const double ds = dw * sig * (1.0 + s * (1.0 - sig)) * inv_n;",
                            "const double ds = dw * sig * inv_n;"),
    "bwd_ln_mean_term": ("dO[idx] = rstd * (dy - mdy - xhat * mdyx);", "dO[idx] = rstd * (dy - xhat * mdyx);"),
    "bwd_dv_weight": ("dv[kj + e] += w * dO[qi + e];", "dv[kj + e] += ds * dO[qi + e];"),
    "bwd_dk_operand": ("dk[kj + e] += ds * ld(q, qi + e, elem_type);", "dk[kj + e] += ds * ld(k, qi + e, elem_type);"),
    "bwd_drab_term": ("drab[(int64_t)h * num_buckets + bk] += ds;", "drab[(int64_t)h * num_buckets + bk] += dw;"),
    "bwd_du_gate": ("du[idx] = xhat * g;", "du[idx] = g;"),
}

PIN_TESTS = [
    pins.test_bucket_hand_values,
    pins.test_single_key_sigmoid_direction,
    pins.test_q_zero_one_hot_v_reads_weight_matrix,
    pins.test_layernorm_closed_form_one_hot,
    pins.test_layernorm_unit_gate_moments,
    lambda: pins.test_against_torch_library_routines(0),
    lambda: pins.test_paged_equals_full_recompute("fp32"),
    pins.test_candidates_do_not_see_each_other,
    pins.test_append_scatter_and_roundtrip,
    pins.test_append_from_empty_then_paged_equals_jagged,
    lambda: bwd_pins.test_gradients_match_finite_differences(3),
    bwd_pins.test_zero_gate_blocks_attention_gradients,
]


@pytest.fixture(scope="module")
def tmpdir_mod():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def _build_mutant(name, old, new, where):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    path_c = os.path.join(where, f"{name}.c")
    path_so = os.path.join(where, f"lib{name}.so")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-shared", "-fPIC", "-o", path_so, path_c,
                           "-lm", "-lpthread"])
    return oracle.bind(ctypes.CDLL(path_so))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmpdir_mod, monkeypatch):
    old, new = MUTANTS[name]
    mutant = _build_mutant(name, old, new, tmpdir_mod)
    oracle._load()
    monkeypatch.setattr(oracle, "_lib", mutant)
    failures = 0
    for t in PIN_TESTS:
        try:
            t()
        except (AssertionError, ValueError):
            failures += 1
    assert failures >= 1, f"mutant {name} passed every pin"


def test_unmutated_passes_all(monkeypatch):
    for t in PIN_TESTS:
        t()
