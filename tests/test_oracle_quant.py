"""Pins of the weight-only int8 oracle (the vlm-8bit preset of the mlx-smolvla
PyPI page §Run a checkpoint; readings 22-24 in ``oracle/quant.py``) against
things other than the oracle itself: weights built on a known grid, exhaustive
search over the 256 codes, the rounding error bound, the exact group minimum,
the degenerate constant group, the preset's scope, and planted mistakes that
one of these must catch."""
import numpy as np
import pytest

import synth
from oracle import quant as oq


def _bf16(x):
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.asarray(x, np.float32))).astype(np.float32)


def _grid_matrix(rng, N, K, exps=(-13, -11, -9)):
    """Rows of 64-groups w = alpha (j - c0), alpha = 2^e, codes j with 0 and 255 present:
    bf16 values whose exact quantisation is (j, alpha, -alpha c0)."""
    G = K // oq.GROUP
    j = rng.integers(0, 256, size=(N, G, oq.GROUP))
    j[..., 0] = 0
    j[..., 1] = 255
    for n in range(N):
        for g in range(G):
            rng.shuffle(j[n, g])
    alpha = np.float32(2.0) ** rng.choice(exps, size=(N, G)).astype(np.float32)
    c0 = rng.integers(0, 256, size=(N, G))
    w = (alpha[..., None] * (j - c0[..., None]).astype(np.float32)).astype(np.float32)
    assert np.array_equal(_bf16(w), w)  # |j - c0| <= 255: 8 significant bits
    return w.reshape(N, K), j.reshape(N, K), alpha, (-alpha * c0).astype(np.float32)


def _random_matrix(rng, N, K, outliers=True):
    w = 0.02 * rng.standard_normal((N, K)).astype(np.float32)
    if outliers:
        w[rng.integers(0, N, 8), rng.integers(0, K, 8)] = 0.5  # a few wide groups
        w[0, :64] = 0.01 + 1e-4 * rng.standard_normal(64)      # a narrow, offset group
    return _bf16(w)


# ----------------------------------------------------------------------------
# pins (each takes the functions under test, so planted mistakes can be swapped in)
# ----------------------------------------------------------------------------
def pin_grid_round_trip(quantize, dequantize):
    rng = np.random.default_rng(11)
    w, j, alpha, beta = _grid_matrix(rng, 8, 256)
    q, a, b = quantize(w)
    assert np.array_equal(q.astype(np.int64), j)
    assert np.array_equal(a, alpha) and np.array_equal(b, beta)
    assert np.array_equal(dequantize(q, a, b), w.astype(np.float64))


def pin_nearest_code(quantize, dequantize):
    """Every code is the nearest of the 256 grid points alpha c + beta (exact float64 search)."""
    rng = np.random.default_rng(12)
    w = _random_matrix(rng, 6, 128)
    q, a, b = quantize(w)
    G = w.shape[1] // oq.GROUP
    codes = np.arange(256, dtype=np.float64)
    for n in range(w.shape[0]):
        for g in range(G):
            al, be = float(a[n, g]), float(b[n, g])
            for i in range(oq.GROUP):
                k = g * oq.GROUP + i
                err = np.abs(be + al * codes - float(w[n, k]))
                assert err[int(q[n, k])] <= err.min() + 1e-6 * max(al, 1e-30)


def pin_error_bound(quantize, dequantize):
    """|w^ - w| <= alpha/2 + (hi - lo - 255 alpha)^+ + the final bf16 rounding (2^-8 relative)."""
    rng = np.random.default_rng(13)
    w = _random_matrix(rng, 64, 512)
    q, a, b = quantize(w)
    wh = dequantize(q, a, b)
    N, K = w.shape
    g = w.reshape(N, K // oq.GROUP, oq.GROUP).astype(np.float64)
    span = g.max(-1) - g.min(-1)
    a64 = a.astype(np.float64)
    bound = a64 * (0.5 + 1e-6) + np.maximum(span - 255.0 * a64, 0.0)
    err = np.abs(wh.reshape(g.shape) - g)
    assert np.all(err <= bound[..., None] + np.abs(wh.reshape(g.shape)) * 2.0 ** -8 + 1e-30)
    # the scale is the span over 255 codes, to bf16 rounding
    nz = span > 0
    assert np.all(np.abs(a64[nz] * 255.0 - span[nz]) <= span[nz] * 2.0 ** -8)


def pin_group_min_exact(quantize, dequantize):
    """The minimum of every group (64 consecutive inputs of one row) is code 0 and is
    reproduced exactly; the maximum takes one of the two top codes."""
    rng = np.random.default_rng(14)
    w = _random_matrix(rng, 64, 192)
    q, a, b = quantize(w)
    wh = dequantize(q, a, b)
    for n in range(w.shape[0]):
        for g in range(w.shape[1] // oq.GROUP):
            sl = slice(g * oq.GROUP, (g + 1) * oq.GROUP)
            i_lo = np.argmin(w[n, sl])
            i_hi = np.argmax(w[n, sl])
            assert q[n, sl][i_lo] == 0
            assert wh[n, sl][i_lo] == float(w[n, sl][i_lo])
            assert q[n, sl][i_hi] in (254, 255)


def pin_constant_group(quantize, dequantize):
    w = np.full((2, 128), 0.01171875, np.float32)
    w[1, 64:] = -3.0
    q, a, b = quantize(w)
    assert np.all(a == 0) and np.all(q == 0)
    assert np.array_equal(dequantize(q, a, b), w.astype(np.float64))


PINS = [pin_grid_round_trip, pin_nearest_code, pin_error_bound, pin_group_min_exact, pin_constant_group]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_quant_pin(pin):
    pin(oq.quantize_affine8, oq.dequantize_affine8)


def test_scale_and_offset_are_bf16_values():
    rng = np.random.default_rng(15)
    _, a, b = oq.quantize_affine8(_random_matrix(rng, 4, 256))
    assert np.array_equal(_bf16(a), a) and np.array_equal(_bf16(b), b)


def test_rejects_ragged_input_width():
    with pytest.raises(ValueError):
        oq.quantize_affine8(np.zeros((2, 96), np.float32))


def test_preset_scope_and_identity_on_grid_weights():
    """vlm-8bit touches exactly the prefix LM's seven matrices per layer; weights that
    already lie on their groups' grids pass through unchanged, so the quantised
    model's prefill equals the dense one."""
    import oracle

    s = synth.SHAPES["tiny"]
    W = oracle.load_weights(synth.gen_weights(s, 3, random_affine=True))
    names = set(oq.prefix_matrix_names(s.p_layers))
    assert len(names) == 7 * s.p_layers
    Wq = oq.quantize_prefix(W, s.p_layers)
    for k in W:
        if k in names:
            assert not np.array_equal(Wq[k], W[k])
        else:
            assert Wq[k] is W[k]
    rng = np.random.default_rng(16)
    Wg = dict(W)
    for k in names:
        N, K = W[k].shape
        Wg[k] = _grid_matrix(rng, N, K)[0].astype(np.float64)
    Wgq = oq.quantize_prefix(Wg, s.p_layers)
    for k in names:
        assert np.array_equal(Wgq[k], Wg[k])
    emb = 0.5 * rng.standard_normal((7, s.p_width))
    valid = np.array([1, 1, 0, 1, 1, 1, 0], bool)
    K0, V0 = oracle.prefill(Wg, s, emb, valid)
    K1, V1 = oracle.prefill(Wgq, s, emb, valid)
    assert np.array_equal(K0, K1) and np.array_equal(V0, V1)


# ----------------------------------------------------------------------------
# planted mistakes: each must fail at least one pin
# ----------------------------------------------------------------------------
def _q_floor(w):
    w = np.asarray(w, np.float32)
    N, K = w.shape
    g = w.reshape(N, K // 64, 64)
    lo, hi = g.min(-1), g.max(-1)
    a = oq._bf16_rne((hi - lo) / np.float32(255))
    safe = np.where(a > 0, a, np.float32(1)).astype(np.float32)
    q = np.clip(np.floor((g - lo[..., None]) / safe[..., None]), 0, 255)   # mistake: floor
    return np.where(a[..., None] > 0, q, 0).astype(np.uint8).reshape(N, K), a, lo


def _q_256(w):
    w = np.asarray(w, np.float32)
    N, K = w.shape
    g = w.reshape(N, K // 64, 64)
    lo, hi = g.min(-1), g.max(-1)
    a = oq._bf16_rne((hi - lo) / np.float32(256))                         # mistake: 256 levels
    safe = np.where(a > 0, a, np.float32(1)).astype(np.float32)
    q = np.clip(np.rint((g - lo[..., None]) / safe[..., None]), 0, 255)
    return np.where(a[..., None] > 0, q, 0).astype(np.uint8).reshape(N, K), a, lo


def _q_columns(w):
    """mistake: each group is 64 consecutive outputs of one input column; the codes
    are returned against each row group's scale and offset"""
    w = np.asarray(w, np.float32)
    N, K = w.shape
    assert N % 64 == 0
    wh = oq.dequantize_affine8(*oq.quantize_affine8(np.ascontiguousarray(w.T))).T
    _, a, b = oq.quantize_affine8(w)
    g = wh.astype(np.float32).reshape(N, K // 64, 64)
    q = np.rint((g - b[..., None]) / np.where(a > 0, a, 1)[..., None])
    return np.clip(q, 0, 255).astype(np.uint8).reshape(N, K), a, b


def _q_hi_offset(w):
    q, a, b = oq.quantize_affine8(w)
    N, K = q.shape
    hi = np.asarray(w, np.float32).reshape(N, K // 64, 64).max(-1)
    return q, a, hi                                                        # mistake: beta = max


def _dq_no_offset(q, a, b):
    return oq.dequantize_affine8(q, a, np.zeros_like(b))                   # mistake: drops beta


def _dq_f32_scale_code(q, a, b):
    N, K = q.shape
    v = np.asarray(a, np.float32)[..., None] * (np.asarray(q, np.float32).reshape(N, K // 64, 64) + 0.5) \
        + np.asarray(b, np.float32)[..., None]                              # mistake: code midpoint
    return oq._bf16_rne(v.astype(np.float32)).astype(np.float64).reshape(N, K)


MUTANTS = {
    "floor_rounding": (_q_floor, oq.dequantize_affine8),
    "256_levels": (_q_256, oq.dequantize_affine8),
    "groups_along_outputs": (_q_columns, oq.dequantize_affine8),
    "offset_is_max": (_q_hi_offset, oq.dequantize_affine8),
    "dequant_drops_offset": (oq.quantize_affine8, _dq_no_offset),
    "dequant_code_midpoint": (oq.quantize_affine8, _dq_f32_scale_code),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_quant_mistake(name):
    qf, dqf = MUTANTS[name]
    failed = 0
    for pin in PINS:
        try:
            pin(qf, dqf)
        except AssertionError:
            failed += 1
    assert failed >= 1, f"no pin caught the planted mistake {name}"
