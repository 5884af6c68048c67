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


def _ragged_grid_matrix(rng, N, n_full, tail):
    """Rows of n_full 64-groups and one `tail`-wide group, each on its own grid
    w = alpha (j - c0) with codes 0 and the top code present. The tail's offset
    c0 is -1, so its values alpha (j + 1) are all positive (and j + 1 <= 256 keeps
    them bf16 values): a tail that is padded with zeros, or merged with the group
    before it, gets another minimum."""
    K = 64 * n_full + tail
    w = np.zeros((N, K), np.float32)
    codes = np.zeros((N, K), np.int64)
    alpha = np.zeros((N, n_full + 1), np.float32)
    beta = np.zeros((N, n_full + 1), np.float32)
    for n in range(N):
        for g in range(n_full + 1):
            width = 64 if g < n_full else tail
            j = rng.integers(0, 256, size=width)
            j[0], j[1] = 0, 255
            rng.shuffle(j)
            e = float(rng.choice((-13, -11, -9)))
            al = np.float32(2.0 ** e)
            c0 = int(rng.integers(0, 256)) if g < n_full else -1
            k0 = 64 * g
            w[n, k0:k0 + width] = al * (j - c0).astype(np.float32)
            codes[n, k0:k0 + width] = j
            alpha[n, g] = al
            beta[n, g] = -al * c0
    assert np.array_equal(_bf16(w), w)  # |j - c0| <= 256: 8 significant bits
    return w, codes, alpha, beta


def pin_ragged_grid_round_trip(quantize, dequantize):
    """K = 64 G + 16 (the expert's 720 = 11 * 64 + 16): every group, the 16-wide
    last one included, recovers its grid exactly (reading 29)."""
    rng = np.random.default_rng(21)
    for n_full, tail in ((3, 16), (11, 16), (0, 48)):
        w, j, alpha, beta = _ragged_grid_matrix(rng, 5, n_full, tail)
        q, a, b = quantize(w)
        assert q.shape == w.shape and a.shape == (5, n_full + 1)
        assert np.array_equal(q.astype(np.int64), j)
        assert np.array_equal(a, alpha) and np.array_equal(b, beta)
        assert np.array_equal(dequantize(q, a, b), w.astype(np.float64))


def pin_ragged_nearest_code(quantize, dequantize):
    """With a ragged last group every code is still the nearest of its own group's
    256 grid points (exact float64 search, the group found by column index)."""
    rng = np.random.default_rng(22)
    w = _random_matrix(rng, 4, 80)
    w[1, 64:] = 0.3 + 1e-3 * rng.standard_normal(16).astype(np.float32)  # a tail far from the row
    w = _bf16(w)
    q, a, b = quantize(w)
    codes = np.arange(256, dtype=np.float64)
    for n in range(4):
        for k in range(80):
            g = k // 64
            al, be = float(a[n, g]), float(b[n, g])
            err = np.abs(be + al * codes - float(w[n, k]))
            assert err[int(q[n, k])] <= err.min() + 1e-6 * max(al, 1e-30)
        tail = w[n, 64:].astype(np.float64)
        assert float(b[n, 1]) == tail.min()


def pin_ragged_groups_are_independent(quantize, dequantize):
    """Changing the inputs of one group changes nothing of the others (the 16-wide
    last group is not padded, merged or shared)."""
    rng = np.random.default_rng(23)
    w = _random_matrix(rng, 3, 208)
    q0, a0, b0 = quantize(w)
    w2 = w.copy()
    w2[:, 128:192] *= np.float32(4.0)
    q1, a1, b1 = quantize(w2)
    assert np.array_equal(q0[:, 192:], q1[:, 192:]) and np.array_equal(a0[:, 3], a1[:, 3])
    assert np.array_equal(b0[:, 3], b1[:, 3])
    w3 = w.copy()
    w3[:, 192:] = np.float32(-1.5)
    q2, a2, b2 = quantize(w3)
    assert np.array_equal(q0[:, :192], q2[:, :192]) and np.array_equal(a0[:, :3], a2[:, :3])
    assert np.all(a2[:, 3] == 0) and np.all(b2[:, 3] == np.float32(-1.5))
    assert np.array_equal(dequantize(q2, a2, b2)[:, 192:], np.full((3, 16), -1.5))


PINS = [pin_grid_round_trip, pin_nearest_code, pin_error_bound, pin_group_min_exact, pin_constant_group,
        pin_ragged_grid_round_trip, pin_ragged_nearest_code, pin_ragged_groups_are_independent]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_quant_pin(pin):
    pin(oq.quantize_affine8, oq.dequantize_affine8)


def test_scale_and_offset_are_bf16_values():
    rng = np.random.default_rng(15)
    _, a, b = oq.quantize_affine8(_random_matrix(rng, 4, 256))
    assert np.array_equal(_bf16(a), a) and np.array_equal(_bf16(b), b)


def test_rejects_empty_input_width():
    with pytest.raises(ValueError):
        oq.quantize_affine8(np.zeros((2, 0), np.float32))


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


def test_expert_preset_scope_and_identity_on_grid_weights():
    """The expert preset (reading 29) touches exactly the expert layers' seven
    matrices; on weights already on their groups' grids (the tiny expert's
    96-wide inputs have a 32-wide last group) it is the identity, so the
    quantised model's denoise equals the dense one."""
    import oracle

    s = synth.SHAPES["tiny"]
    W = oracle.load_weights(synth.gen_weights(s, 4, random_affine=True))
    names = set(oq.expert_matrix_names(s.e_layers))
    assert len(names) == 7 * s.e_layers
    assert any(W[k].shape[1] % 64 for k in names)  # ragged groups are exercised
    Wq = oq.quantize_expert(W, s.e_layers)
    for k in W:
        if k in names:
            assert not np.array_equal(Wq[k], W[k])
        else:
            assert Wq[k] is W[k]
    rng = np.random.default_rng(24)
    Wg = dict(W)
    for k in names:
        N, K = W[k].shape
        if K % 64:
            Wg[k] = _ragged_grid_matrix(rng, N, K // 64, K % 64)[0].astype(np.float64)
        else:
            Wg[k] = _grid_matrix(rng, N, K)[0].astype(np.float64)
        Wg[k] *= 8.0  # same grids, scales nearer the workloads' weights
    Wgq = oq.quantize_expert(Wg, s.e_layers)
    for k in names:
        assert np.array_equal(Wgq[k], Wg[k])
    L, H = 6, 5
    valid = np.array([1, 1, 0, 1, 1, 1], bool)
    Kc = 0.5 * rng.standard_normal((s.p_layers, L, s.p_kv_width))
    Vc = 0.5 * rng.standard_normal((s.p_layers, L, s.p_kv_width))
    noise = rng.standard_normal((H, s.action_dim))
    x0 = oracle.denoise(Wg, s, Kc, Vc, valid, noise, 3)[2]
    x1 = oracle.denoise(Wgq, s, Kc, Vc, valid, noise, 3)[2]
    assert np.array_equal(x0, x1)


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


def _q_tail_zero_padded(w):
    """mistake: the ragged last group is padded with zeros to 64 inputs"""
    w = np.asarray(w, np.float32)
    N, K = w.shape
    pad = (-K) % 64
    q, a, b = oq.quantize_affine8(np.concatenate([w, np.zeros((N, pad), np.float32)], axis=1))
    return q[:, :K], a, b


def _q_tail_merged(w):
    """mistake: the ragged tail joins the group before it (one (64 + r)-wide group)"""
    w = np.asarray(w, np.float32)
    N, K = w.shape
    q, a, b = oq.quantize_affine8(w)
    r = K % 64
    if r == 0 or K < 64 + r:
        return q, a, b
    k0 = K - 64 - r
    qm, am, bm = oq.quantize_affine8(w[:, k0:])  # 64 + r wide: groups [0, 64) and the tail
    lo, hi = w[:, k0:].min(1), w[:, k0:].max(1)
    al = oq._bf16_rne((hi - lo) / np.float32(255))
    safe = np.where(al > 0, al, np.float32(1)).astype(np.float32)
    qq = np.clip(np.rint((w[:, k0:] - lo[:, None]) / safe[:, None]), 0, 255).astype(np.uint8)
    q[:, k0:] = qq
    a[:, -2:] = al[:, None]
    b[:, -2:] = lo[:, None]
    return q, a, b


def _q_tail_previous_scale(w):
    """mistake: the tail is coded on the previous group's scale and offset"""
    w = np.asarray(w, np.float32)
    N, K = w.shape
    q, a, b = oq.quantize_affine8(w)
    if K % 64 == 0 or K < 64:
        return q, a, b
    k0 = K - K % 64
    al, be = a[:, -2], b[:, -2]
    safe = np.where(al > 0, al, np.float32(1)).astype(np.float32)
    q[:, k0:] = np.clip(np.rint((w[:, k0:] - be[:, None]) / safe[:, None]), 0, 255).astype(np.uint8)
    a[:, -1], b[:, -1] = al, be
    return q, a, b


MUTANTS = {
    "tail_zero_padded": (_q_tail_zero_padded, oq.dequantize_affine8),
    "tail_merged_with_previous": (_q_tail_merged, oq.dequantize_affine8),
    "tail_on_previous_scale": (_q_tail_previous_scale, oq.dequantize_affine8),
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
        except Exception:  # a wrong value, or a mutant that cannot take a ragged row
            failed += 1
    assert failed >= 1, f"no pin caught the planted mistake {name}"
