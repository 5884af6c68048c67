"""Pins of the prefix-assembly oracle (connector pixel shuffle + linear, state
token, prefix order) against things other than the oracle itself: a
hand-worked example, permutation and closed-form properties, parameter counts,
and a planted mistake that one of them must catch."""
import json
import os

import numpy as np
import pytest

import synth
from oracle import assembly as oa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pixel_shuffle_worked_example.json")


def test_pixel_shuffle_worked_examples():
    for case in json.load(open(GOLDEN))["cases"]:
        g, r, C = case["grid"], case["r"], case["C"]
        feats = (C * np.arange(g * g)[:, None] + np.arange(C)[None, :]).astype(float)
        assert np.array_equal(oa.pixel_shuffle(feats, g, r), np.array(case["tokens"], float))


def test_pixel_shuffle_is_a_permutation_with_a_local_inverse():
    rng = np.random.default_rng(5)
    g, r, C = 8, 2, 3
    feats = rng.standard_normal((g * g, C))
    out = oa.pixel_shuffle(feats, g, r)
    assert out.shape == ((g // r) ** 2, r * r * C)
    assert np.array_equal(np.sort(out.ravel()), np.sort(feats.ravel()))
    # every output token holds exactly the r x r block of neighbouring patches
    grid = feats.reshape(g, g, C)
    for t in range(out.shape[0]):
        i, j = divmod(t, g // r)
        block = grid[r * i:r * i + r, r * j:r * j + r, :]
        assert np.array_equal(np.sort(out[t]), np.sort(block.ravel()))


def test_connector_block_selector_closed_form():
    rng = np.random.default_rng(6)
    g, r, C = 8, 2, 4
    feats = rng.standard_normal((g * g, C))
    grid = feats.reshape(g, g, C)
    for a0 in range(r):
        for b0 in range(r):
            Wc = np.zeros((C, r * r * C))
            Wc[np.arange(C), (a0 * r + b0) * C + np.arange(C)] = 1.0
            out = oa.connector(Wc, feats, g, r)
            for t in range(out.shape[0]):
                i, j = divmod(t, g // r)
                assert np.array_equal(out[t], grid[r * i + a0, r * j + b0])


def test_state_token_closed_form():
    D, S = 12, 5
    state = np.arange(1.0, S + 1.0)
    Ws = np.eye(D, S)
    bs = 0.5 * np.arange(D)
    want = np.concatenate([state, np.zeros(D - S)]) + bs
    assert np.array_equal(oa.state_token(Ws, bs, state), want)


def test_assemble_prefix_layout():
    a = synth.ASSEMBLY_SHAPES["tiny"]
    D = synth.SHAPES["tiny"].p_width
    w = {k: synth.bf16_bits_to_f32(v).astype(np.float64)
         for k, v in synth.gen_assembly_weights(a, D, seed=3).items()}
    inp = synth.gen_assembly_inputs(a, D, B=2, seed=3)
    for b in range(2):
        vis = synth.bf16_bits_to_f32(inp["vis"][b]).astype(np.float64)
        text = synth.bf16_bits_to_f32(inp["text"][b]).astype(np.float64)
        emb, valid = oa.assemble_prefix(w["w_conn"], w["w_state"], w["b_state"], vis, text, inp["text_valid"][b],
                                        inp["state"][b], a.grid, a.shuffle)
        tpi = a.tokens_per_image
        L = a.n_img * tpi + a.text_len + 1
        assert emb.shape == (L, D) and valid.shape == (L,)
        assert valid[:a.n_img * tpi].all() and valid[-1] == 1
        assert np.array_equal(valid[a.n_img * tpi:-1], inp["text_valid"][b])
        for im in range(a.n_img):
            assert np.allclose(emb[im * tpi:(im + 1) * tpi], oa.pixel_shuffle(vis[im], a.grid, a.shuffle) @ w["w_conn"].T)
        assert np.array_equal(emb[a.n_img * tpi:-1], text)
        assert np.allclose(emb[-1], w["w_state"] @ inp["state"][b].astype(np.float64) + w["b_state"])


def test_assembly_parameter_counts():
    a = synth.ASSEMBLY_SHAPES["smolvla"]
    D = synth.SHAPES["smolvla"].p_width
    # pixel shuffle x4 of 768-wide patch features: the linear input width, 64 tokens per 32 x 32 grid
    assert a.conn_in == 16 * 768 == 12288 and a.tokens_per_image == 64
    man = dict(synth.assembly_manifest(a, D))
    assert int(np.prod(man["w_conn"])) == 11_796_480
    assert int(np.prod(man["w_state"])) + int(np.prod(man["b_state"])) == 31_680


def _pixel_shuffle_ba(feats, grid, r):
    """Planted mistake: the r x r block concatenated column-major, (b, a)."""
    n, C = feats.shape
    g2 = grid // r
    return np.asarray(feats, float).reshape(g2, r, g2, r, C).transpose(0, 2, 3, 1, 4).reshape(g2 * g2, r * r * C)


def test_pins_catch_a_transposed_pixel_shuffle(monkeypatch):
    monkeypatch.setattr(oa, "pixel_shuffle", _pixel_shuffle_ba)
    with pytest.raises(AssertionError):
        test_pixel_shuffle_worked_examples()
