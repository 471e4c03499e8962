"""Planted mistakes in the oracle must fail its pins (CPU only).

Each mutant below replaces one step of the oracle with a plausible slip -- a wrong sign, a
transposed index, a dropped term, an off-by-one -- and the whole pin battery of
``tests/test_oracle.py`` is run against it; at least one pin has to fail.  The battery is also
run unmodified, where every pin has to pass, so that a failure can only come from the planted
mistake.  The mistakes are planted in the oracle's Python steps (``oracle.rope3d``, the ring's
window and key gathering, the softmax scale handed to the row attention); the C arithmetic is
reached through them.
"""
import inspect

import numpy as np
import pytest

import oracle
from tests import test_oracle as pins

BF16_ONE = 0x3F80


def _pin_calls():
    """(name, function, kwargs) for every pin, parametrized pins expanded."""
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_") or fn.__module__ != pins.__name__:
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        params = list(inspect.signature(fn).parameters)
        if not marks:
            if not params:
                calls.append((name, fn, {}))
            continue
        argnames, argvalues = marks[0].args[0], marks[0].args[1]
        argnames = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) else argnames
        if set(argnames) != set(params):
            continue
        for k, vals in enumerate(argvalues):
            vals = vals if len(argnames) > 1 else (vals,)
            calls.append((f"{name}[{k}]", fn, dict(zip(argnames, vals))))
    return calls


def _failing_pins():
    failed = []
    for name, fn, kw in _pin_calls():
        try:
            fn(**kw)
        except Exception:   # an assertion, or an error the slip provokes
            failed.append(name)
    return failed


# ---- the mutants --------------------------------------------------------------------------

_rope3d = oracle.rope3d
_window_kv = oracle.OracleLayer.window_kv
_window_frames = oracle.OracleLayer.window_frames
_attention_rows = oracle.attention_rows


def rope_flipped_sign(x_bits, frame_idx, frames, Hg, Wg, spec):
    """Rotation by -angle: R(-a) x = 2 cos(a) x - R(a) x, cos(a) read from rotated unit pairs."""
    y = _rope3d(x_bits, frame_idx, frames, Hg, Wg, spec)
    unit = np.zeros_like(np.asarray(x_bits, dtype=np.uint16))
    unit[..., 0::2] = BF16_ONE
    c = np.repeat(_rope3d(unit, frame_idx, frames, Hg, Wg, spec)[..., 0::2], 2, axis=-1)
    return 2.0 * c * oracle.bf16_to_f64(x_bits) - y


def _half_split_perm(spec):
    perm = []
    o = 0
    for d in (spec.d_t, spec.d_h, spec.d_w):
        for j in range(d // 2):
            perm += [o + j, o + j + d // 2]
        o += d
    return np.asarray(perm)


def rope_half_split_pairs(x_bits, frame_idx, frames, Hg, Wg, spec):
    """Pairs (j, j + d_a/2) of each axis block rotated instead of adjacent channels."""
    perm = _half_split_perm(spec)
    y = _rope3d(np.ascontiguousarray(np.asarray(x_bits)[..., perm]), frame_idx, frames, Hg, Wg, spec)
    out = np.empty_like(y)
    out[..., perm] = y
    return out


def rope_transposed_grid(x_bits, frame_idx, frames, Hg, Wg, spec):
    """Token index decoded with the grid's height and width swapped."""
    return _rope3d(x_bits, frame_idx, frames, Wg, Hg, spec)


def rope_frame_off_by_one(x_bits, frame_idx, frames, Hg, Wg, spec):
    return _rope3d(x_bits, frame_idx + 1, frames, Hg, Wg, spec)


def window_kv_dropped_key(self, window):
    K, V = _window_kv(self, window)
    return K[:, :, :-1], V[:, :, :-1]


def window_kv_values_of_other_head(self, window):
    K, V = _window_kv(self, window)
    return K, V[:, ::-1]


def window_frames_missing_oldest(self, window):
    frames = _window_frames(self, window)
    return frames[1:] if len(frames) > 1 else frames


def attention_scale_one_over_d(q, K, V, rows, scale):
    return _attention_rows(q, K, V, rows, scale * scale)


MUTANTS = {
    "rotation sign flipped": (oracle, "rope3d", rope_flipped_sign),
    "half-split channel pairs": (oracle, "rope3d", rope_half_split_pairs),
    "token grid transposed": (oracle, "rope3d", rope_transposed_grid),
    "temporal position off by one": (oracle, "rope3d", rope_frame_off_by_one),
    "last key of the window dropped": (oracle.OracleLayer, "window_kv", window_kv_dropped_key),
    "values of another head": (oracle.OracleLayer, "window_kv", window_kv_values_of_other_head),
    "window misses its oldest frame": (oracle.OracleLayer, "window_frames",
                                       window_frames_missing_oldest),
    "softmax scale 1/D instead of 1/sqrt(D)": (oracle, "attention_rows",
                                               attention_scale_one_over_d),
}


def test_battery_passes_unmodified():
    calls = _pin_calls()
    assert len(calls) >= 30
    assert _failing_pins() == []


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(mutant):
    owner, attr, fn = MUTANTS[mutant]
    with pytest.MonkeyPatch.context() as mp:
        mp.setattr(owner, attr, fn)
        failed = _failing_pins()
    assert failed, f"no pin catches: {mutant}"
