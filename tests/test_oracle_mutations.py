"""The pins catch plausible mistakes: each case plants one error in a copy of
the oracle's C source (on the CPU, in a temporary directory), loads the broken
build in place of the real one, and checks that the pin checks below fail.
The real oracle is restored afterwards."""
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
import test_oracle_gla_pins as gpins  # noqa: E402
import test_oracle_pins as pins  # noqa: E402
import test_oracle_softmax_pins as spins  # noqa: E402

SRC = os.path.join(os.path.dirname(HERE), "oracle", "lasp_oracle.c")

# (what the mistake is, exact text in the source, its replacement, occurrence index)
MUTATIONS = [
    ("forward state loses its decay",
     "S[i * d + j] = l * S[i * d + j] + (double)ks[i] * vs[j];\n      for",
     "S[i * d + j] = S[i * d + j] + (double)ks[i] * vs[j];\n      for", 0),
    ("forward output reads the state transposed",
     "acc += (double)qs[i] * S[i * d + j];", "acc += (double)qs[i] * S[j * d + i];", 0),
    ("forward uses v for k",
     "S[i * d + j] = l * S[i * d + j] + (double)ks[i] * vs[j];\n      for",
     "S[i * d + j] = l * S[i * d + j] + (double)vs[i] * vs[j];\n      for", 0),
    ("dq contracts with dout against the wrong index",
     "acc += S[i * d + j] * ds[j];", "acc += S[j * d + i] * ds[j];", 0),
    ("dk uses k instead of v", "acc += G[i * d + j] * vs[j];", "acc += G[i * d + j] * ks[j];", 0),
    ("dv gradient state misses the current token",
     "for (int j = r0; j < r1; ++j) G[i * d + j] += (double)qs[i] * ds[j];",
     "for (int j = r0; j < r1; ++j) G[i * d + j] += 0.0 * qs[i] * ds[j];", 0),
    ("dv sums over the wrong operand", "acc += (double)ks[i] * G[i * d + j];",
     "acc += (double)qs[i] * G[i * d + j];", 0),
    ("chunk-state weight off by one", "pow(l, (double)(C - 1 - t))", "pow(l, (double)(C - t))", 0),
    ("gradient-state weight off by one", "pow(l, (double)(t + 1))", "pow(l, (double)(t))", 0),
    ("scan without the chunk decay", "acc[e] = g * acc[e] + Mc[e];", "acc[e] = acc[e] + Mc[e];", 0),
    ("gradient snapshots decay before adding the token",
     "S[i * d + j] = l * (S[i * d + j] + (double)as[i] * bs[j]);",
     "S[i * d + j] = l * S[i * d + j] + (double)as[i] * bs[j];", 0),
    ("bidirectional state transposed", "M[i * d + j] += (double)ks[i] * vs[j];",
     "M[i * d + j] += (double)vs[i] * ks[j];", 0),
    ("bidirectional dk uses dM transposed", "ak += G[i * d + j] * vs[j];", "ak += G[j * d + i] * vs[j];", 0),
    ("bidirectional dv uses dM transposed", "av += (double)ks[j] * G[j * d + i];",
     "av += (double)ks[j] * G[i * d + j];", 0),
    ("gated forward gates the value feature instead of the key feature",
     "for (int j = j0; j < j1; ++j) S[i * d + j] = g * S[i * d + j] + (double)ks[i] * vs[j];",
     "for (int j = j0; j < j1; ++j) S[i * d + j] = exp((double)gs[j]) * S[i * d + j] + (double)ks[i] * vs[j];", 0),
    ("gated forward gates the token's own outer product too",
     "for (int j = j0; j < j1; ++j) S[i * d + j] = g * S[i * d + j] + (double)ks[i] * vs[j];",
     "for (int j = j0; j < j1; ++j) S[i * d + j] = g * (S[i * d + j] + (double)ks[i] * vs[j]);", 0),
    ("gated dq rows are stepped without the gate",
     "for (int j = 0; j < d; ++j) row[j] = g * row[j] + (double)ks[i] * vs[j];",
     "for (int j = 0; j < d; ++j) row[j] = row[j] + (double)ks[i] * vs[j];", 0),
    ("gated dk gradient state loses its gate", "for (int j = 0; j < d; ++j) Gi[j] *= g;",
     "for (int j = 0; j < d; ++j) Gi[j] *= 1.0;", 0),
    ("gated dv gradient state loses its gate", "for (int j = r0; j < r1; ++j) G[i * d + j] *= g;",
     "for (int j = r0; j < r1; ++j) G[i * d + j] *= 1.0;", 0),
    ("gate gradient pairs G_s with S_s instead of S_{s-1}",
     "const double *prev = s > t0 ? buf + (size_t)(s - 1 - t0) * rows : kept + (size_t)m * rows;",
     "const double *prev = buf + (size_t)(s - t0) * rows;", 0),
    ("gate gradient misses the gate factor", "das[i] = g * acca;", "das[i] = acca;", 0),
    ("gated chunk state decays the token by its own gate",
     "long r0 = kind == 0 ? t + 1 : 0, r1 = kind == 0 ? C - 1 : t;",
     "long r0 = kind == 0 ? t : 0, r1 = kind == 0 ? C - 1 : t;", 0),
    ("gated gradient chunk state leaves out the token's own gate",
     "long r0 = kind == 0 ? t + 1 : 0, r1 = kind == 0 ? C - 1 : t;",
     "long r0 = kind == 0 ? t + 1 : 0, r1 = kind == 0 ? C - 1 : t - 1;", 0),
    ("gated scan uses one feature's gate for every row", "double g = exp(gc[i]);", "double g = exp(gc[0]);", 0),
    ("softmax scores miss the scale", "s[j] = scale * acc;", "s[j] = acc;", 0),
    ("softmax dq leaves out the row's softmax correction", "double ds = a * (da - rs[task]);",
     "double ds = a * da;", 0),
    ("softmax dk leaves out the row's softmax correction", "double ds = a * (da - rs[row]);",
     "double ds = a * da;", 0),
    ("softmax dk misses the scale", "dkj[f] += scale * ds * qi[f];", "dkj[f] += ds * qi[f];", 0),
    ("softmax dv weighs do by ds instead of the attention weight", "dvj[f] += a * di[f];",
     "dvj[f] += ds * di[f];", 0),
    ("softmax key pass skips the query on the diagonal", "long i0 = j > q_offset ? j - q_offset : 0;",
     "long i0 = j > q_offset ? j - q_offset + 1 : 0;", 0),
    ("softmax correction term forgets the normaliser", "r += exp(s[j] - m) / l * da;",
     "r += exp(s[j] - m) * da;", 0),
    ("softmax output without the normaliser", "double a = s[j] / l;", "double a = s[j];", 0),
    ("gated gradient snapshots gate before adding the token",
     "for (int j = 0; j < d; ++j) S[i * d + j] = g * (S[i * d + j] + (double)xs[i] * ys[j]);",
     "for (int j = 0; j < d; ++j) S[i * d + j] = g * S[i * d + j] + (double)xs[i] * ys[j];", 0),
]


def _build_mutant(tmp_path, old, new, nth):
    src = open(SRC).read()
    idx = -1
    for _ in range(nth + 1):
        idx = src.find(old, idx + 1)
        assert idx >= 0, f"mutation anchor not found: {old!r}"
    src = src[:idx] + new + src[idx + len(old):]
    path = tmp_path / "mutant.c"
    path.write_text(src)
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", str(path), "-o", str(so), "-lm"],
                   check=True)
    return str(so)


def _pins_pass():
    """A reduced set of the pins; True when all of them hold."""
    checks = [
        pins.test_two_token_worked_example,
        pins.test_unit_vector_closed_form,
        lambda: pins.test_recurrence_equals_quadratic_form(True, 1),
        pins.test_entering_states_equal_quadratic_form,
        lambda: pins.test_recurrence_equals_chunk_form(8),
        pins.test_chunk_states_equal_recurrence_run_over_the_chunk,
        pins.test_state_scan_closed_forms,
        pins.test_scan_of_chunk_states_equals_recurrence_snapshots,
        pins.test_bidirectional_equals_left_product,
        gpins.test_constant_gate_is_the_decayed_recurrence,
        lambda: gpins.test_recurrence_equals_quadratic_form(1),
        gpins.test_gate_gradient_identity,
        lambda: gpins.test_chunk_states_and_scans_equal_snapshots(4),
        lambda: gpins.test_recurrence_equals_chunk_form(8),
        spins.test_two_token_worked_example,
        lambda: spins.test_equals_torch_scaled_dot_product_attention(1, 2, 20, 50, 30, 8, 0.7),
        spins.test_shards_equal_the_whole_sequence,
    ]
    for check in checks:
        try:
            check()
        except AssertionError:
            return False
    return True


@pytest.mark.parametrize("name,old,new,nth", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_the_mistake(tmp_path, name, old, new, nth):
    import ctypes
    so = _build_mutant(tmp_path, old, new, nth)
    real = oracle._load()
    lib = ctypes.CDLL(so)
    for f in ("oracle_fwd", "oracle_bwd", "oracle_chunk_states", "oracle_state_scan", "oracle_state_snapshots",
              "oracle_bidir_fwd", "oracle_bidir_bwd", "oracle_gla_fwd", "oracle_gla_bwd", "oracle_gla_chunk_states",
              "oracle_gla_state_scan", "oracle_gla_state_snapshots", "oracle_softmax_fwd", "oracle_softmax_bwd"):
        getattr(lib, f).argtypes = getattr(real, f).argtypes
        getattr(lib, f).restype = None
    lib.oracle_num_threads.restype = ctypes.c_int
    oracle._lib = lib
    try:
        assert not _pins_pass(), f"the pins did not catch: {name}"
    finally:
        oracle._lib = real


def test_unmutated_source_passes_the_same_checks():
    assert _pins_pass()
    assert np.isfinite(oracle.fwd(np.ones((1, 4, 1, 2), np.float32), np.ones((1, 4, 1, 2), np.float32),
                                  np.ones((1, 4, 1, 2), np.float32))).all()
