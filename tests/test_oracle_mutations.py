"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in the CPU oracle (a wrong GQA index, a flipped
RoPE sign, a dropped residual, a transposed operand, ...) by swapping one of
its functions for a mutated copy, then runs the pins of
``test_oracle_pins.py``; at least one pin must fail for every mutant.
"""
import numpy as np
import pytest

from oracle import model as om
from tests import test_oracle_pins as pins


def _attention_gqa_modulo(q, k, v, allowed):
    n_q, _, hd = q.shape
    n_kv = k.shape[0]
    out = np.empty_like(q)
    for h in range(n_q):
        g = h % n_kv                     # mistake: interleaved instead of contiguous groups
        s = (q[h] @ k[g].T) / np.sqrt(hd)
        s = np.where(allowed, s, -np.inf)
        p = np.exp(s - s.max(-1, keepdims=True))
        out[h] = (p / p.sum(-1, keepdims=True)) @ v[g]
    return out


def _attention_scale_hd(q, k, v, allowed):
    n_q, _, hd = q.shape
    group = n_q // k.shape[0]
    out = np.empty_like(q)
    for h in range(n_q):
        g = h // group
        s = (q[h] @ k[g].T) / hd          # mistake: 1/hd instead of 1/sqrt(hd)
        s = np.where(allowed, s, -np.inf)
        p = np.exp(s - s.max(-1, keepdims=True))
        out[h] = (p / p.sum(-1, keepdims=True)) @ v[g]
    return out


def _attention_no_mask(q, k, v, allowed):
    return om.__dict__["_orig_attention"](q, k, v, np.ones_like(allowed, dtype=bool))


def _rope_sign(x, pos, base):
    hd = x.shape[-1]
    half = hd // 2
    inv_freq = base ** (-(2.0 * np.arange(half)) / hd)
    ang = np.asarray(pos, float)[:, None] * inv_freq[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)   # mistake: rotation backwards


def _rope_interleaved(x, pos, base):
    hd = x.shape[-1]
    half = hd // 2
    inv_freq = base ** (-(2.0 * np.arange(half)) / hd)
    ang = np.asarray(pos, float)[:, None] * inv_freq[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., 0::2], x[..., 1::2]    # mistake: adjacent pairs instead of rotate-half
    out = np.empty_like(x)
    out[..., 0::2] = x1 * c - x2 * s
    out[..., 1::2] = x2 * c + x1 * s
    return out


def _rms_norm_no_eps_sqrt(x, g, eps):
    return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * g   # mistake: eps outside the root


def _rms_norm_no_gain(x, g, eps):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)        # mistake: gain dropped


def _swiglu_no_gate(y, wg, wu, wd, rb):
    return rb(y @ wu.T) @ wd.T                                              # mistake: gate branch dropped


def _swiglu_swapped(y, wg, wu, wd, rb):
    return rb(om.silu(y @ wu.T) * (y @ wg.T)) @ wd.T                        # mistake: silu on the up branch


def _time_embedding_swapped(t, dim, pmin, pmax):
    e = om.__dict__["_orig_time_embedding"](t, dim, pmin, pmax)
    half = dim // 2
    return np.concatenate([e[half:], e[:half]])                             # mistake: [cos || sin]


def _positions_ignore_pad(valid):
    return np.arange(len(valid))                                            # mistake: pads advance the position


def _cross_kv_prev_layer(W, s, l, K, V, rb=lambda x: x):
    return om.__dict__["_orig_cross_kv"](W, s, l, np.roll(K, 1, axis=0), np.roll(V, 1, axis=0), rb)  # wrong layer


def _split_transposed_heads(x, n):
    T = x.shape[0]
    return x.reshape(T, -1, n).transpose(2, 0, 1)                            # mistake: heads interleaved


MUTANTS = {
    "gqa_modulo": ("attention", _attention_gqa_modulo),
    "attention_scale": ("attention", _attention_scale_hd),
    "attention_no_mask": ("attention", _attention_no_mask),
    "rope_sign": ("rope", _rope_sign),
    "rope_interleaved": ("rope", _rope_interleaved),
    "rmsnorm_eps": ("rms_norm", _rms_norm_no_eps_sqrt),
    "rmsnorm_gain": ("rms_norm", _rms_norm_no_gain),
    "swiglu_no_gate": ("_swiglu", _swiglu_no_gate),
    "swiglu_swapped": ("_swiglu", _swiglu_swapped),
    "time_embedding_swapped": ("time_embedding", _time_embedding_swapped),
    "positions_ignore_pad": ("prefix_positions", _positions_ignore_pad),
    "cross_attention_wrong_layer": ("cross_kv", _cross_kv_prev_layer),
    "heads_interleaved": ("_split", _split_transposed_heads),
}

PIN_TESTS = [
    lambda: pins.test_brute_force_tiny(True),
    pins.test_joint_pass_matches_prefill_then_denoise,
    pins.test_gqa_equals_mha_with_repeated_heads,
    pins.test_zero_branches_reduce_to_heads,
    pins.test_padding_invariance,
    pins.test_rope_closed_form_hd4,
    pins.test_rope_identity_at_zero_norm_and_relative_position,
    pins.test_rms_norm_constant_vector,
    pins.test_time_embedding_closed_form,
    pins.test_prefix_positions,
    pins.test_attention_single_valid_key_returns_v,
    pins.test_attention_matches_loops,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    fname, fn = MUTANTS[name]
    monkeypatch.setitem(om.__dict__, "_orig_" + fname, getattr(om, fname))
    monkeypatch.setattr(om, fname, fn)
    caught = []
    for pin in PIN_TESTS:
        try:
            pin()
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(getattr(pin, "__name__", "brute_force"))
    assert caught, f"no pin caught the planted mistake {name!r}"


def test_unmutated_oracle_passes_every_pin():
    for pin in PIN_TESTS:
        pin()
