"""The pins catch plausible mistakes in the oracle.

Each case plants one mistake in a temporary copy of the oracle's C source (a
dropped gate, a wrong order of steps, a wrong constant), builds it on the CPU,
swaps it in for the real library, and checks that at least one pin of
tests/test_oracle_pins.py fails.  The real oracle is never modified.
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn2_oracle.c")

MUTANTS = {
    # erase along the raw key instead of the erase-gated key
    "erase_without_gate": ("const double kh = b[i] * k[i];", "const double kh = k[i];"),
    # write the raw value instead of the write-gated value
    "write_without_gate": ("vh[j] = w[j0 + j] * v[j0 + j];", "vh[j] = v[j0 + j];"),
    # gates swapped in role: erase scaled by the write gate's first entries
    "erase_with_write_gate": ("const double kh = b[i] * k[i];",
                              "const double kh = w[i % dv] * k[i];"),
    # readout gain missing its factor 2
    "gain_without_two": ("(2.0 / (1.0 + exp(-z[i])))", "(1.0 / (1.0 + exp(-z[i])))"),
    # gain applied without the static profile
    "gain_without_static": ("qt[i] = q[i] * gs[i] *", "qt[i] = q[i] *"),
    # RMSNorm over the sum instead of the mean
    "rmsnorm_sum": ("sqrt(ss / dv + eps)", "sqrt(ss + eps)"),
    # decay applied twice
    "double_decay": ("Sblk[i * COLS_PER_TASK + j] *= alpha[i];",
                     "Sblk[i * COLS_PER_TASK + j] *= alpha[i] * alpha[i];"),
    # write uses the erase sign
    "write_sign": ("+= -kh * r[j] + k[i] * vh[j];", "+= -kh * r[j] - k[i] * vh[j];"),
    # transposed role of q and k in the readout
    "read_with_key": ("o[j] += qt[i] * Sblk", "o[j] += k[i] * Sblk"),
}

# read before the update: move the readout above the erase/write step
READ_BEFORE_WRITE = ("""        /* S = S_hat - (b*k)^T r + k^T (w*v) */
        for (int i = 0; i < dk; ++i) {
            const double kh = b[i] * k[i];
            for (int j = 0; j < nb; ++j)
                Sblk[i * COLS_PER_TASK + j] += -kh * r[j] + k[i] * vh[j];
        }
        /* o = q_til S */
        for (int j = 0; j < nb; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < nb; ++j) o[j] += qt[i] * Sblk[i * COLS_PER_TASK + j];
""", """        for (int j = 0; j < nb; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < nb; ++j) o[j] += qt[i] * Sblk[i * COLS_PER_TASK + j];
        for (int i = 0; i < dk; ++i) {
            const double kh = b[i] * k[i];
            for (int j = 0; j < nb; ++j)
                Sblk[i * COLS_PER_TASK + j] += -kh * r[j] + k[i] * vh[j];
        }
""")

# erase with the undecayed state: compute r before the decay
ERASE_BEFORE_DECAY = ("""        /* S_hat = Diag(alpha) S */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < nb; ++j) Sblk[i * COLS_PER_TASK + j] *= alpha[i];
        /* r = k S_hat */
        for (int j = 0; j < nb; ++j) r[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < nb; ++j) r[j] += k[i] * Sblk[i * COLS_PER_TASK + j];
""", """        for (int j = 0; j < nb; ++j) r[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < nb; ++j) r[j] += k[i] * Sblk[i * COLS_PER_TASK + j];
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < nb; ++j) Sblk[i * COLS_PER_TASK + j] *= alpha[i];
""")

ALL = dict(MUTANTS)
ALL["read_before_write"] = READ_BEFORE_WRITE
ALL["erase_before_decay"] = ERASE_BEFORE_DECAY

PIN_CALLS = [
    lambda: pins.test_equal_gates_reduce_to_kda(0),
    pins.test_scalar_decay_reduces_to_gated_deltanet,
    pins.test_unit_decay_reduces_to_deltanet,
    pins.test_exact_retrieval_with_orthonormal_keys,
    pins.test_zero_erase_is_causal_linear_attention,
    pins.test_zero_erase_closed_form_with_decay,
    pins.test_erase_gate_invariants,
    pins.test_rmsnorm_mean_of_squares,
    pins.test_golden_readback_squared_norm,
    lambda: pins.test_chunked_form_matches_recurrence(50, 16),
]


def _build_mutant(name, old, new, tmp):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    path_c = os.path.join(tmp, f"{name}.c")
    path_so = os.path.join(tmp, f"lib{name}.so")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           "-o", path_so, path_c, "-lm"])
    return path_so


def _with_lib(path):
    real = oracle._load()
    lib = ctypes.CDLL(path)
    lib.oracle_gdn2_forward.restype = real.oracle_gdn2_forward.restype
    lib.oracle_gdn2_forward.argtypes = real.oracle_gdn2_forward.argtypes
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("name", sorted(ALL))
def test_pins_catch_mutant(name):
    old, new = ALL[name]
    real = oracle._load()
    with tempfile.TemporaryDirectory() as tmp:
        mutant = _with_lib(_build_mutant(name, old, new, tmp))
        caught = []
        try:
            oracle._lib = mutant
            for call in PIN_CALLS:
                try:
                    call()
                except AssertionError:
                    caught.append(call)
        finally:
            oracle._lib = real
    assert caught, f"no pin caught mutant {name}"


def test_unmodified_source_passes_every_pin():
    real = oracle._load()
    for call in PIN_CALLS:
        call()
    assert oracle._lib is real


# Mistakes in the q/k preprocessing (a Python step of the oracle), planted by
# swapping the function for a wrong one; the preprocessing pins must notice.
def _prep_no_silu(x):
    x = oracle._f64(x)
    return x / np.maximum(np.linalg.norm(x, axis=-1, keepdims=True), 1e-12)


def _prep_sigmoid(x):
    x = oracle._f64(x)
    s = 1.0 / (1.0 + np.exp(-x))
    return s / np.maximum(np.linalg.norm(s, axis=-1, keepdims=True), 1e-12)


def _prep_wrong_axis(x):
    x = oracle._f64(x)
    s = x / (1.0 + np.exp(-x))
    return s / np.maximum(np.linalg.norm(s, axis=0, keepdims=True), 1e-12)


def _prep_no_floor(x):
    x = oracle._f64(x)
    s = x / (1.0 + np.exp(-x))
    with np.errstate(invalid="ignore", divide="ignore"):
        return s / np.linalg.norm(s, axis=-1, keepdims=True)


PREP_MUTANTS = {"no_silu": _prep_no_silu, "sigmoid_not_silu": _prep_sigmoid,
                "normalised_over_the_wrong_axis": _prep_wrong_axis, "no_norm_floor": _prep_no_floor}


@pytest.mark.parametrize("name", sorted(PREP_MUTANTS))
def test_preprocessing_pins_catch_mutant(name, monkeypatch):
    monkeypatch.setattr(oracle, "preprocess_qk", PREP_MUTANTS[name])
    failed = 0
    for pin in (pins.test_preprocess_qk_is_unit_norm_along_the_head_channels,
                pins.test_preprocess_qk_direction_is_silu, pins.test_preprocess_qk_special_rows):
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1, name
