"""Planted mistakes in the FP8 oracle: every plausible slip must fail at least one pin.

Each mutant is a copy of ``oracle/fp8.py`` with one edit, loaded as a separate module from a
temporary file.  The pins of ``test_oracle_fp8`` are run with it swapped in, and the test passes
only if some pin fails.  The committed oracle is never modified.
"""
import importlib.util
import os

import pytest

import test_oracle_fp8 as pins
from oracle import fp8 as real

MUTANTS = [
    ("ties_away_from_zero", "(d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))",
     "(d_hi <= d_lo)"),
    ("ties_toward_zero", "(d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))", "(d_hi < d_lo)"),
    ("truncation", "(d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))", "(d_hi == 0)"),
    ("overflow_to_nan", "code = np.where(a >= E4M3_MAX, 126, code)",
     "code = np.where(a > 464, 127, code)"),
    ("exponent_bias_8", "2.0 ** (e - 7)", "2.0 ** (e - 8)"),
    ("subnormal_exponent", "(m / 8.0) * 2.0 ** -6", "(m / 8.0) * 2.0 ** -7"),
    ("sign_dropped", "return (code | sign).astype(np.uint8)", "return code.astype(np.uint8)"),
    ("scale_inverted", "safe / np.float32(E4M3_MAX)", "np.float32(E4M3_MAX) / safe"),
    ("amax_without_abs", "amax = np.max(np.abs(x), axis=-1)", "amax = np.max(x, axis=-1)"),
    ("mantissa_of_four_bits", "(1.0 + m / 8.0)", "(1.0 + m / 16.0)"),
    ("decode_sign_dropped", "return np.where(c & 0x80, -out, out).astype(np.float32)",
     "return out.astype(np.float32)"),
    ("overflowing_inverse_kept", "live = nz & np.isfinite(inv)", "live = nz"),
]

PINS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


def _mutant(tmp_path, name, old, new):
    text = open(real.__file__).read()
    assert text.count(old) >= 1, f"{name}: pattern not in the oracle"
    path = os.path.join(tmp_path, f"fp8_{name}.py")
    with open(path, "w") as f:
        f.write(text.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"fp8_mutant_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_each_planted_mistake_fails_a_pin(name, old, new, tmp_path, monkeypatch):
    monkeypatch.setattr(pins, "fp8", _mutant(str(tmp_path), name, old, new))
    failed = []
    for pin in PINS:
        try:
            pin()
        except Exception:            # an assertion, or an error the slip causes
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"


def test_the_committed_oracle_passes_every_pin():
    for pin in PINS:
        pin()
