"""Planted mistakes in the oracle must fail its pins (CPU only).

Each mutant below replaces one step of the oracle with a plausible slip -- a wrong sign, a
transposed index, a dropped term, an off-by-one -- and the pin battery of the module that pins
that step is run against it; at least one pin has to fail.  Each battery is also run unmodified,
where every pin has to pass, so that a failure can only come from the planted mistake.  The
mistakes are planted in the oracle's Python steps (``oracle.rope3d``, the ring's window and key
gathering, the softmax scale handed to the row attention, the convolution, the truncated SVD,
the renoise); the C arithmetic is reached through them.
"""
import inspect

import numpy as np
import pytest

import oracle
from tests import test_lowrank, test_schedule, test_vae_conv
from tests import test_oracle as pins

BF16_ONE = 0x3F80


def _pin_calls(module=pins):
    """(name, function, kwargs) for every pin of ``module``, parametrized pins expanded."""
    calls = []
    for name, fn in inspect.getmembers(module, inspect.isfunction):
        if not name.startswith("test_") or fn.__module__ != module.__name__:
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


def _failing_pins(module=pins):
    failed = []
    for name, fn, kw in _pin_calls(module):
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


_conv3d = oracle.conv3d_causal
_svd_truncate = oracle.svd_truncate


def conv_taps_flipped_in_h(x_bits, w_bits, bias=None):
    """The kernel's h taps applied in reverse (a convolution instead of a correlation in h)."""
    return _conv3d(x_bits, np.ascontiguousarray(np.asarray(w_bits)[:, :, ::-1]), bias)


def conv_reads_one_frame_later(x_bits, w_bits, bias=None):
    """Output frame t reads input frames t+1 .. t+3 (the causal window off by one)."""
    x = np.asarray(x_bits)
    shifted = np.concatenate([x[:, 1:], np.zeros_like(x[:, :1])], axis=1)
    return _conv3d(shifted, w_bits, bias)


def conv_padding_on_one_side(x_bits, w_bits, bias=None):
    """Zero padding of two positions on the left of w and none on the right."""
    x = np.asarray(x_bits)
    shifted = np.concatenate([np.zeros_like(x[:, :, :, :1]), x[:, :, :, :-1]], axis=3)
    return _conv3d(shifted, w_bits, bias)


def conv_bias_dropped(x_bits, w_bits, bias=None):
    return _conv3d(x_bits, w_bits, None)


def svd_smallest_singular_vectors(W, rank):
    U, S, Vh = np.linalg.svd(np.asarray(W, dtype=np.float64), full_matrices=False)
    return (S[-rank:, None] * Vh[-rank:]), U[:, -rank:], S


def svd_singular_values_dropped(W, rank):
    w1, w2, S = _svd_truncate(W, rank)
    return w1 / S[:rank, None], w2, S


def renoise_sigma_swapped(x0_bits, eps_bits, sigma):
    return sigma * oracle.bf16_to_f64(x0_bits) + (1.0 - sigma) * oracle.bf16_to_f64(eps_bits)


# mutant -> (what is replaced, the replacement, the module whose pins must catch it)
MUTANTS = {
    "rotation sign flipped": (oracle, "rope3d", rope_flipped_sign, pins),
    "half-split channel pairs": (oracle, "rope3d", rope_half_split_pairs, pins),
    "token grid transposed": (oracle, "rope3d", rope_transposed_grid, pins),
    "temporal position off by one": (oracle, "rope3d", rope_frame_off_by_one, pins),
    "last key of the window dropped": (oracle.OracleLayer, "window_kv", window_kv_dropped_key,
                                       pins),
    "values of another head": (oracle.OracleLayer, "window_kv", window_kv_values_of_other_head,
                               pins),
    "window misses its oldest frame": (oracle.OracleLayer, "window_frames",
                                       window_frames_missing_oldest, pins),
    "softmax scale 1/D instead of 1/sqrt(D)": (oracle, "attention_rows",
                                               attention_scale_one_over_d, pins),
    "conv taps flipped in h": (oracle, "conv3d_causal", conv_taps_flipped_in_h, test_vae_conv),
    "conv window one frame late": (oracle, "conv3d_causal", conv_reads_one_frame_later,
                                   test_vae_conv),
    "conv padding on one side": (oracle, "conv3d_causal", conv_padding_on_one_side,
                                 test_vae_conv),
    "conv bias dropped": (oracle, "conv3d_causal", conv_bias_dropped, test_vae_conv),
    "svd keeps the smallest singular vectors": (oracle, "svd_truncate",
                                                svd_smallest_singular_vectors, test_lowrank),
    "svd factors without the singular values": (oracle, "svd_truncate",
                                                svd_singular_values_dropped, test_lowrank),
    "renoise weights swapped": (oracle, "renoise", renoise_sigma_swapped, test_schedule),
}


@pytest.mark.parametrize("module", [pins, test_vae_conv, test_lowrank, test_schedule],
                         ids=lambda m: m.__name__.rsplit(".", 1)[-1])
def test_battery_passes_unmodified(module):
    assert len(_pin_calls(module)) >= 3
    assert _failing_pins(module) == []


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(mutant):
    owner, attr, fn, module = MUTANTS[mutant]
    with pytest.MonkeyPatch.context() as mp:
        mp.setattr(owner, attr, fn)
        failed = _failing_pins(module)
    assert failed, f"no pin catches: {mutant}"
