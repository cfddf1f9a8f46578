"""Mutation check of the oracle's pins.

Each mutant is the oracle compiled with one deliberate, plausible mistake
(``-DDRO_MUTANT=n``): no square root on the erase strength, write-side
scaling put on the erase key, a square root on the decoupled write strength,
the output read before the update, decay after the write, a transposed read,
a flipped error sign, the channel gate on the value dimension, a transposed
output read.  Every mutant must fail at least one pin that the real oracle
passes, which shows that the pins would notice such a mistake.
"""
import ctypes
import os

import numpy as np
import pytest

import oracle
from oracle import build as obuild

from .test_oracle_pins import MODES, _case, _dense_product_form

MUTANTS = list(range(1, 10))


def _load_mutant(n, tmp_path):
    out = str(tmp_path / f"libdr_oracle_m{n}.so")
    obuild.build(force=True, out=out, extra_flags=(f"-DDRO_MUTANT={n}",))
    return out


def _pins_pass(monkeypatch, libpath):
    lib = ctypes.CDLL(libpath)
    base = oracle._load()
    for name in ("dro_sequential", "dro_chunkwise", "dro_max_threads"):
        fn = getattr(lib, name)
        fn.argtypes, fn.restype = getattr(base, name).argtypes, getattr(base, name).restype
    monkeypatch.setattr(oracle, "_lib", lib)
    try:
        from . import test_oracle_pins as P
        P.test_hand_worked_examples()
        P.test_pin_a_read_after_write_returns_value(True)
        for modes in MODES:
            P.test_brute_force_product_form(modes)
        P.test_exact_rationals_on_tiny_input()
    except AssertionError:
        return False
    finally:
        monkeypatch.setattr(oracle, "_lib", base)
    return True


def test_unmutated_build_passes(monkeypatch, tmp_path):
    assert _pins_pass(monkeypatch, _load_mutant(0, tmp_path))


@pytest.mark.parametrize("n", MUTANTS)
def test_every_mutant_fails_a_pin(monkeypatch, tmp_path, n):
    assert not _pins_pass(monkeypatch, _load_mutant(n, tmp_path)), f"mutant {n} passed every pin"
