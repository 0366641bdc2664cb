"""Planted mistakes in the FP8 attention-tier oracle: every plausible slip must fail at least one
pin.

Each mutant is a copy of ``oracle/e4m3.py`` with one edit, loaded as a separate module from a
temporary file; the pins of ``test_oracle_e4m3`` run with it swapped in, and the test passes only
if some pin fails.  The committed oracle is never modified.
"""
import importlib.util
import os

import pytest

import test_oracle_e4m3 as pins
from oracle import e4m3 as real

MUTANTS = [
    ("scale_240", "inv = (np.float32(QMAX) / safe)", "inv = (np.float32(240) / safe)"),
    ("scale_inverted", "safe / np.float32(QMAX)", "safe * np.float32(QMAX)"),
    ("no_inverse_applied", "_fp8.e4m3_encode((xb * inv[None, :, None])",
     "_fp8.e4m3_encode((xb * np.float32(1))"),
    ("q_block_64", "sq = q_scale[h, rows // Q_ROWS]", "sq = q_scale[h, rows // 64]"),
    ("k_scale_dropped", "sk = k_scale[h, np.arange(n) // K_KEYS].astype(np.float64)[None, :]",
     "sk = np.ones((1, n))"),
    ("mask_one_key_late", "kv_end[off[c] - t_ctx:off[c + 1] - t_ctx] = off[c + 1]",
     "kv_end[off[c] - t_ctx:off[c + 1] - t_ctx] = off[c + 1] + 1"),
    ("softmax_scale_dropped", "return softmax_scale * sq * sk * dots", "return sq * sk * dots"),
    ("head_of_q_wrong", "qv = _fp8.e4m3_decode(q_codes[rows, h, :])",
     "qv = _fp8.e4m3_decode(q_codes[rows, 0, :])"),
    ("block_max_first_row", "a = np.max(np.abs(xb), axis=(0, 2))",
     "a = np.max(np.abs(xb[:1]), axis=(0, 2))"),
]

PINS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


def _mutant(tmp_path, name, old, new):
    text = open(real.__file__).read()
    assert text.count(old) >= 1, f"{name}: pattern not in the oracle"
    path = os.path.join(tmp_path, f"e4m3_{name}.py")
    with open(path, "w") as f:
        f.write(text.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"e4m3_mutant_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_each_planted_mistake_fails_a_pin(name, old, new, tmp_path, monkeypatch):
    monkeypatch.setattr(pins, "e4m3", _mutant(str(tmp_path), name, old, new))
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
