"""The pins must catch plausible oracle mistakes.

Each mutant build of the oracle (compiled with ORACLE_MUTANT=k into a
temporary directory) plants one mistake: a dropped term, a wrong sign, a
wrong or shifted index, swapped operands, a missing step. For every mutant at
least one pin of ``test_oracle_pins`` must fail; the real oracle passes them
all (checked there).
"""
import numpy as np
import pytest

import oracle.oracle as ow
from test_oracle_pins import PINS, pin_tol

MUTANTS = {
    1: "D skip dropped",
    2: "wrong sign in exp(Delta*A)",
    3: "Delta dropped from the input term",
    4: "readout taken before the state update",
    5: "B and C swapped",
    6: "softplus never applied",
    7: "delta bias dropped",
    8: "sigmoid gate instead of silu",
    9: "B read one token late",
    10: "state index reversed in A",
    11: "decode ignores the stored state",
    12: "final state never written",
    13: "conv filter taps reversed",
    14: "conv activation dropped",
    15: "conv history before token 0 ignored",
    16: "gradient of silu missing its z*s*(1-s) term",
    17: "adjoint state decayed by its own token's A_bar",
    18: "gradient of Delta through A_bar dropped",
    19: "SSD heads assigned to groups round-robin",
    20: "SSD input term decayed by its own token",
    21: "SSD Delta dropped from the input term",
}


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("oracle_mutants"))


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_some_pin_catches_mutant(mutant, mutant_dir):
    lib = ow.mutant_library(mutant, mutant_dir)
    caught = []
    for name, pin in PINS.items():
        with np.errstate(all="ignore"):
            try:
                err = pin(lib)
            except Exception:  # a crash or an assertion inside a pin also counts
                err = float("inf")
        if not (err <= pin_tol(name)):
            caught.append(name)
    assert caught, f"no pin caught mutant {mutant} ({MUTANTS[mutant]})"


# The per-chunk C B^T of the SSD matrix view is a numpy definition in
# oracle.oracle; its mutants replace that function for one pin run.
def _cb_transposed(B, C, chunk=32):
    return np.swapaxes(_CB_REAL(B, C, chunk), -1, -2)


def _cb_chunk_shifted(B, C, chunk=32):
    # chunk k built from the tokens one position later
    return _CB_REAL(np.roll(B, -1, axis=1), np.roll(C, -1, axis=1), chunk)


def _cb_tail_not_zero(B, C, chunk=32):
    # tokens past L taken from the start of the sequence instead of zero
    batch, L = B.shape[:2]
    pad = (-L) % chunk
    Bp = np.concatenate([B, B[:, :pad]], axis=1)
    Cp = np.concatenate([C, C[:, :pad]], axis=1)
    return _CB_REAL(Bp, Cp, chunk)


_CB_REAL = ow.ssd_chunk_cb
CB_MUTANTS = {"transposed": _cb_transposed, "chunk shifted by a token": _cb_chunk_shifted,
              "tail past L not zero": _cb_tail_not_zero}


@pytest.mark.parametrize("name", sorted(CB_MUTANTS))
def test_chunk_cb_pin_catches_mutant(name, oracle_lib, monkeypatch):
    monkeypatch.setattr(ow, "ssd_chunk_cb", CB_MUTANTS[name])
    import oracle
    monkeypatch.setattr(oracle, "ssd_chunk_cb", CB_MUTANTS[name])
    pin = "ssd_chunk_cb_is_intra_chunk_product"
    assert PINS[pin](oracle_lib) > pin_tol(pin), f"pin {pin} misses the mutant '{name}'"
