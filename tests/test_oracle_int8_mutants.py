"""Planted mistakes in the INT8 oracle: every plausible slip must fail at least one pin.

Each mutant is a copy of ``oracle/int8.py`` with one edit, loaded as a separate module from a
temporary file; the pins of ``test_oracle_int8`` run with it swapped in, and the test passes only
if some pin fails.  The committed oracle is never modified.
"""
import importlib.util
import os

import pytest

import test_oracle_int8 as pins
from oracle import int8 as real

MUTANTS = [
    ("no_smoothing", "quantize_blocks(smooth(k, mu), K_KEYS)", "quantize_blocks(_f32(k), K_KEYS)"),
    ("smoothing_sign", "(_f32(k) - np.asarray(mu, np.float32)[None])",
     "(_f32(k) + np.asarray(mu, np.float32)[None])"),
    ("mean_over_t_minus_1", "dtype=np.float64) / T", "dtype=np.float64) / (T - 1)"),
    ("scale_128", "inv = (np.float32(QMAX) / safe)", "inv = (np.float32(128) / safe)"),
    ("truncation", "np.clip(np.rint(y), -QMAX, QMAX)", "np.clip(np.trunc(y), -QMAX, QMAX)"),
    ("q_block_64", "sq = q_scale[h, rows // Q_ROWS]", "sq = q_scale[h, rows // 64]"),
    ("k_scale_dropped", "sk = k_scale[h, np.arange(n) // K_KEYS].astype(np.float64)[None, :]",
     "sk = np.ones((1, n))"),
    ("mask_one_key_late", "kv_end[off[c] - t_ctx:off[c + 1] - t_ctx] = off[c + 1]",
     "kv_end[off[c] - t_ctx:off[c + 1] - t_ctx] = off[c + 1] + 1"),
    ("softmax_scale_dropped", "return softmax_scale * sq * sk * dots.astype(np.float64)",
     "return sq * sk * dots.astype(np.float64)"),
    ("head_of_q_wrong", "dots = q_codes[rows, h, :]", "dots = q_codes[rows, 0, :]"),
]

PINS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


def _mutant(tmp_path, name, old, new):
    text = open(real.__file__).read()
    assert text.count(old) >= 1, f"{name}: pattern not in the oracle"
    path = os.path.join(tmp_path, f"int8_{name}.py")
    with open(path, "w") as f:
        f.write(text.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"int8_mutant_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_each_planted_mistake_fails_a_pin(name, old, new, tmp_path, monkeypatch):
    monkeypatch.setattr(pins, "int8", _mutant(str(tmp_path), name, old, new))
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
