"""Mutation check of the oracle's pins.

Each mutant is a copy of the oracle's source with one deliberate, plausible
mistake patched in (the oracle itself is the plain recurrence; the patches live
here): no square root on the erase strength, write-side scaling put on the
erase key, a square root on the decoupled write strength, the output read
before the update, decay after the write, a transposed read, a flipped error
sign, the channel gate on the value dimension, a transposed output read.
Every mutant must fail at least one pin that the real oracle passes, which
shows that the pins would notice such a mistake.
"""
import ctypes
import os

import numpy as np
import pytest

import oracle
from oracle import build as obuild

from .test_oracle_pins import MODES, _case, _dense_product_form

_OUT = """    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * a->q[th * dk + i];
      a->o[th * dv + j] = acc;
    }
"""
_DECAY = """    for (int i = 0; i < dk; ++i) {
      const double al = gate(a->alpha, a->alpha_mode, th, dk, i);
      for (int j = 0; j < dv; ++j) S[i * dv + j] *= al;
    }
"""
_WRITE = """      for (int j = 0; j < dv; ++j) S[i * dv + j] += av[i] * u[j];
"""
# (what the mistake is, [(text of the oracle, replacement), ...])
PATCHES = {
    1: ("no square root on the erase strength",
        [("const double bk = sqrt(gate(a->beta_k, a->beta_k_mode, th, dk, i)) * a->k[th * dk + i];",
          "const double bk = gate(a->beta_k, a->beta_k_mode, th, dk, i) * a->k[th * dk + i];")]),
    2: ("write-side scale on the erase key, plain key on the write",
        [("av[i] = a->s_scale ? a->s_scale[th * dk + i] * bk : bk;",
          "av[i] = a->s_scale ? a->s_scale[th * dk + i] * bk : bk;\n    if (a->s_scale) { bv[i] = av[i]; av[i] = bk; }")]),
    3: ("square root on the decoupled write strength",
        [("wv[j] = gate(a->beta_v, a->beta_v_mode, th, dv, j) * vj;",
          "wv[j] = sqrt(gate(a->beta_v, a->beta_v_mode, th, dv, j)) * vj;")]),
    4: ("output read before the update",
        [("    token_vectors(a, th, bv, av, wv);\n", "    token_vectors(a, th, bv, av, wv);\n" + _OUT),
         ("    /* output from the updated state: o_t = S_t^T q_t */\n" + _OUT, "")]),
    5: ("decay applied after the erase and write",
        [("    /* decay first: S <- Diag(alpha_t) S */\n" + _DECAY, ""),
         (_WRITE, _WRITE + _DECAY)]),
    6: ("transposed read",
        [("for (int i = 0; i < dk; ++i) r += S[i * dv + j] * bv[i];",
          "for (int i = 0; i < dk; ++i) r += (dk == dv ? S[j * dv + i] : S[i * dv + j]) * bv[i];")]),
    7: ("flipped error sign", [("u[j] = wv[j] - r;", "u[j] = wv[j] + r;")]),
    8: ("channel decay on the value dimension",
        [(_WRITE, _WRITE + """    if (dk == dv)
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
          S[i * dv + j] *= gate(a->alpha, a->alpha_mode, th, dk, j) / gate(a->alpha, a->alpha_mode, th, dk, i);
""")]),
    9: ("transposed output read",
        [("for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * a->q[th * dk + i];",
          "for (int i = 0; i < dk; ++i) acc += (dk == dv ? S[j * dv + i] : S[i * dv + j]) * a->q[th * dk + i];")]),
}
MUTANTS = sorted(PATCHES)


def _mutant_source(n):
    src = open(obuild.SRC).read()
    for old, new in ([] if n == 0 else PATCHES[n][1]):
        assert src.count(old) == 1, f"mutant {n}: the oracle text to patch is not unique: {old[:60]!r}"
        src = src.replace(old, new)
    return src


def _load_mutant(n, tmp_path):
    src = tmp_path / f"dr_oracle_m{n}.c"
    src.write_text(_mutant_source(n))
    out = str(tmp_path / f"libdr_oracle_m{n}.so")
    obuild.build(force=True, out=out, src=str(src))
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
def test_every_patch_changes_the_source(n):
    assert _mutant_source(n) != _mutant_source(0), PATCHES[n][0]


@pytest.mark.parametrize("n", MUTANTS)
def test_every_mutant_fails_a_pin(monkeypatch, tmp_path, n):
    assert not _pins_pass(monkeypatch, _load_mutant(n, tmp_path)), f"mutant {n} ({PATCHES[n][0]}) passed every pin"
