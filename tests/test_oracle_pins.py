"""Pins for the CPU oracle: each test checks it against something other than
itself — closed forms, invariants the pages state, brute force on tiny
inputs, published known-answer vectors. No GPU needed.
"""
import json
import math
import os

import numpy as np
import pytest

import synth
import oracle
from oracle import model as om
from tests import brute_force as bf

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tiny(random_affine=False, seed=0):
    s = synth.SHAPES["tiny"]
    W = oracle.load_weights(synth.gen_weights(s, seed, random_affine=random_affine))
    wl = synth.WORKLOADS["tiny"]
    inp = synth.gen_inputs(wl)
    emb = synth.bf16_bits_to_f32(inp["embeds"][0]).astype(np.float64)
    return s, W, emb, inp["valid"][0].astype(bool), inp["noise"][0].astype(np.float64), wl


# --------------------------------------------------------------------------
# published generator
# --------------------------------------------------------------------------
def test_philox_known_answers():
    kat = json.load(open(os.path.join(GOLDEN, "philox4x32_10_kat.json")))
    for case in kat["cases"]:
        ctr = [np.array([int(c, 16)], dtype=np.uint64) for c in case["ctr"]]
        key = [int(k, 16) for k in case["key"]]
        got = [int(r[0]) for r in oracle.philox4x32_10(ctr, key)]
        assert got == [int(o, 16) for o in case["out"]]


def test_gaussian_noise_moments_and_layout():
    z = oracle.gaussian_noise(1234, 4, 50, 32)
    assert z.shape == (4, 50, 32)
    flat = z.reshape(-1)
    assert abs(flat.mean()) < 0.05 and abs(flat.std() - 1.0) < 0.05
    # query b is independent of the batch size (counter carries the query index)
    assert np.array_equal(oracle.gaussian_noise(1234, 2, 50, 32), z[:2])
    # different seeds give different noise
    assert not np.allclose(oracle.gaussian_noise(1235, 1, 50, 32), z[:1])
    # |z| is bounded by sqrt(-2 ln 2^-24) since u1 >= 2^-24
    assert np.abs(flat).max() <= math.sqrt(-2 * math.log(2.0 ** -24)) + 1e-12


# --------------------------------------------------------------------------
# building blocks in closed form
# --------------------------------------------------------------------------
def test_rope_closed_form_hd4():
    # x = [1, 2, 3, 4] at position 1, base 1e4: inv_freq = [1, 1e-2]; pairs (0,2), (1,3)
    x = np.array([1.0, 2.0, 3.0, 4.0])[None, None, :]
    got = om.rope(x, np.array([1]), 10000.0)[0, 0]
    c0, s0, c1, s1 = math.cos(1.0), math.sin(1.0), math.cos(0.01), math.sin(0.01)
    want = [1 * c0 - 3 * s0, 2 * c1 - 4 * s1, 3 * c0 + 1 * s0, 4 * c1 + 2 * s1]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)


def test_rope_identity_at_zero_norm_and_relative_position():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((3, 5, 64))
    np.testing.assert_array_equal(om.rope(x, np.zeros(5, int), 1e4), x)
    y = om.rope(x, np.arange(5) * 37, 1e4)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # q(m) . k(n) depends on m - n only
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    def dot(m, n):
        return float(om.rope(q[None, None], np.array([m]), 1e4)[0, 0] @ om.rope(k[None, None], np.array([n]), 1e4)[0, 0])
    assert abs(dot(7, 3) - dot(104, 100)) < 1e-12
    assert abs(dot(7, 3) - dot(3, 7)) > 1e-6


def test_rms_norm_constant_vector():
    c, eps = 0.75, 1e-5
    g = np.linspace(0.5, 1.5, 16)
    y = om.rms_norm(np.full((2, 16), c), g, eps)
    np.testing.assert_allclose(y, np.broadcast_to(c / math.sqrt(c * c + eps) * g, (2, 16)), rtol=1e-15)


def test_time_embedding_closed_form():
    dim, pmin, pmax = 96, 4e-3, 4.0
    e0 = om.time_embedding(0.0, dim, pmin, pmax)
    np.testing.assert_array_equal(e0[:48], 0.0)
    np.testing.assert_array_equal(e0[48:], 1.0)
    # first period is pmin, last is pmax: at t = pmax/4 the last sine is 1
    e = om.time_embedding(pmax / 4, dim, pmin, pmax)
    assert abs(e[47] - 1.0) < 1e-15 and abs(e[95]) < 1e-15
    e = om.time_embedding(pmin / 4, dim, pmin, pmax)
    assert abs(e[0] - 1.0) < 1e-15


def test_prefix_positions():
    np.testing.assert_array_equal(om.prefix_positions([1, 1, 1, 1]), [0, 1, 2, 3])
    np.testing.assert_array_equal(om.prefix_positions([1, 1, 0, 0, 1]), [0, 1, 1, 1, 2])
    np.testing.assert_array_equal(om.prefix_positions([0, 1, 1]), [-1, 0, 1])


def test_attention_single_valid_key_returns_v():
    # mlx-smolvla forum thread: with L = 1 the attention output must be V exactly
    rng = np.random.default_rng(1)
    q = rng.standard_normal((15, 7, 64)) * 3
    k = rng.standard_normal((5, 9, 64)) * 3
    v = rng.standard_normal((5, 9, 64))
    allowed = np.zeros((7, 9), bool)
    allowed[:, 4] = True
    o = om.attention(q, k, v, allowed)
    for h in range(15):
        np.testing.assert_array_equal(o[h], np.broadcast_to(v[h // 3, 4], (7, 64)))
    # first causal row returns its own v
    causal = np.tril(np.ones((9, 9), bool))
    o = om.attention(rng.standard_normal((15, 9, 64)), k, v, causal)
    np.testing.assert_array_equal(o[:, 0], v[np.arange(15) // 3, 0])


def test_attention_matches_loops():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((6, 5, 8)) * 2
    k = rng.standard_normal((2, 7, 8)) * 2
    v = rng.standard_normal((2, 7, 8))
    valid = [1, 0, 1, 1, 0, 1, 1]
    got = om.attention(q, k, v, np.broadcast_to(np.array(valid, bool)[None], (5, 7)))
    want = bf.attend(q.tolist(), k.tolist(), v.tolist(), lambda i, j: bool(valid[j]))
    np.testing.assert_allclose(om._merge(got), np.array(want), rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# whole-path pins
# --------------------------------------------------------------------------
@pytest.mark.parametrize("random_affine", [False, True])
def test_brute_force_tiny(random_affine):
    """Pin (d): loop-only restatement on the tiny shape agrees to rounding."""
    s, W, emb, valid, noise, wl = _tiny(random_affine)
    K, V, vs, xs, x = oracle.sample(W, s, emb, valid, noise, wl.n_steps)
    Kb, Vb, xb = bf.sample(bf.tolist(W), s, emb.tolist(), valid.tolist(), noise.tolist(), wl.n_steps)
    L = emb.shape[0]
    np.testing.assert_allclose(K.reshape(s.p_layers, L, -1), np.array(Kb), rtol=0, atol=1e-11)
    np.testing.assert_allclose(V.reshape(s.p_layers, L, -1), np.array(Vb), rtol=0, atol=1e-11)
    np.testing.assert_allclose(x, np.array(xb), rtol=0, atol=1e-10)


def test_joint_pass_matches_prefill_then_denoise():
    """Pin (a): the block mask makes one joint pass equal prefill + denoise."""
    s, W, emb, valid, noise, wl = _tiny(random_affine=True)
    K, V = oracle.prefill(W, s, emb, valid)
    t = 0.7
    v_split = oracle.velocity(W, s, noise, t, K, V, valid)
    Kj, Vj, vj = oracle.oracle_joint(W, s, emb, valid, noise, t)
    np.testing.assert_allclose(Kj, K, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Vj, V, rtol=0, atol=1e-12)
    np.testing.assert_allclose(vj, v_split, rtol=0, atol=1e-11)
    # the prefix cannot see the actions: other noise leaves the joint K/V bitwise equal
    Kj2, Vj2, vj2 = oracle.oracle_joint(W, s, emb, valid, noise * -3.0 + 1.0, t)
    assert np.array_equal(Kj2, Kj) and np.array_equal(Vj2, Vj)
    assert not np.allclose(vj2, vj)


def test_constant_velocity_linear_trajectory():
    """Pin (b): with W_out = 0 and b_out = c the velocity is c through the whole
    network, so x_k = x_0 + k dt c exactly for dyadic values (N = 4)."""
    s, W, emb, valid, _, wl = _tiny()
    W = dict(W)
    A = s.action_dim
    c = np.array([0.5, -1.25, 2.0, 0.0, -0.375, 1.0, 3.5, -2.0])[:A]
    W["w_out"] = np.zeros_like(W["w_out"])
    W["b_out"] = c
    x0 = (np.arange(wl.H * A).reshape(wl.H, A) % 7 - 3) * 0.25
    K, V = oracle.prefill(W, s, emb, valid)
    vs, xs, x = oracle.denoise(W, s, K, V, valid, x0, 4)
    for k in range(4):
        assert np.array_equal(vs[k], np.broadcast_to(c, x0.shape))
        assert np.array_equal(xs[k], x0 + (k + 1) * (-0.25) * c)
    # after the full unit interval the state moved by exactly -c: with a
    # velocity eps - a (flow-matching target) noise eps lands on a
    assert np.array_equal(x, x0 - c)


def test_gqa_equals_mha_with_repeated_heads():
    """Pin (c): an n_kv = n_q model whose k/v rows repeat each kv head equals GQA."""
    s, W, emb, valid, noise, wl = _tiny(random_affine=True)
    hd, rep = s.head_dim, s.p_heads // s.p_kv_heads
    sm = s.replace(p_kv_heads=s.p_heads, e_kv_heads=s.e_heads)
    Wm = dict(W)

    def rep_rows(w):
        n_in_heads = w.shape[0] // hd
        return np.concatenate([w[(h // rep) * hd:(h // rep + 1) * hd] for h in range(n_in_heads * rep)])

    for l in range(s.p_layers):
        for nm in ("wk", "wv"):
            Wm[f"p{l}.{nm}"] = rep_rows(W[f"p{l}.{nm}"])
    for l in range(s.e_layers):
        for nm in ("wk", "wv"):
            w = W[f"e{l}.{nm}"]
            if l % 2 == 0:
                Wm[f"e{l}.{nm}"] = rep_rows(w)
            else:
                # cross projection: the MHA cache repeats each kv head; read the
                # first copy only, then repeat the output heads
                wi = np.zeros((w.shape[0], sm.p_kv_width))
                for hi in range(sm.p_kv_heads):
                    if hi % rep == 0:
                        g = hi // rep
                        wi[:, hi * hd:(hi + 1) * hd] = w[:, g * hd:(g + 1) * hd]
                Wm[f"e{l}.{nm}"] = rep_rows(wi)
    K, V, vs, xs, x = oracle.sample(W, s, emb, valid, noise, wl.n_steps)
    Km, Vm, vsm, xsm, xm = oracle.sample(Wm, sm, emb, valid, noise, wl.n_steps)
    for h in range(s.p_heads):
        np.testing.assert_allclose(Km[:, :, h], K[:, :, h // rep], rtol=0, atol=1e-12)
        np.testing.assert_allclose(Vm[:, :, h], V[:, :, h // rep], rtol=0, atol=1e-12)
    np.testing.assert_allclose(xm, x, rtol=1e-9, atol=1e-11)


def test_zero_branches_reduce_to_heads():
    """With W_o = W_d = 0 every layer is the identity on the residual, so the
    velocity is action_out(norm(time-MLP(action_in(x), e(t)))) in closed form."""
    s, W, emb, valid, noise, wl = _tiny(random_affine=True)
    W = dict(W)
    for l in range(s.e_layers):
        W[f"e{l}.wo"] = np.zeros_like(W[f"e{l}.wo"])
        W[f"e{l}.wd"] = np.zeros_like(W[f"e{l}.wd"])
    K, V = oracle.prefill(W, s, emb, valid)
    t = 0.3
    v = oracle.velocity(W, s, noise, t, K, V, valid)
    # closed form written with loops over scalars
    De = s.e_width
    want = np.empty_like(noise)
    for i in range(noise.shape[0]):
        a = [math.fsum(W["w_in"][o, j] * noise[i, j] for j in range(s.action_dim)) + W["b_in"][o] for o in range(De)]
        half = De // 2
        e = []
        for fn in (math.sin, math.cos):
            for j in range(half):
                per = s.t_min_period * (s.t_max_period / s.t_min_period) ** (j / (half - 1))
                e.append(fn(2 * math.pi * t / per))
        cat = a + e
        h = []
        for o in range(De):
            z = math.fsum(W["w_t1"][o, j] * cat[j] for j in range(2 * De)) + W["b_t1"][o]
            h.append(z / (1 + math.exp(-z)))
        r = [math.fsum(W["w_t2"][o, j] * h[j] for j in range(De)) + W["b_t2"][o] for o in range(De)]
        inv = 1.0 / math.sqrt(math.fsum(x * x for x in r) / De + s.rms_eps)
        y = [r[j] * inv * W["final_norm"][j] for j in range(De)]
        for o in range(s.action_dim):
            want[i, o] = math.fsum(W["w_out"][o, j] * y[j] for j in range(De)) + W["b_out"][o]
    np.testing.assert_allclose(v, want, rtol=0, atol=1e-12)


def test_padding_invariance():
    """Reading 2: a query's valid outputs do not depend on interior padding."""
    s, W, emb, _, noise, wl = _tiny(random_affine=True)
    L = emb.shape[0]
    valid = np.ones(L, bool)
    valid[[3, 4, 10, 17, 18, 19]] = False          # interior holes
    K, V, _, _, x = oracle.sample(W, s, emb, valid, noise, wl.n_steps)
    keep = np.nonzero(valid)[0]
    Kc, Vc, _, _, xc = oracle.sample(W, s, emb[keep], np.ones(len(keep), bool), noise, wl.n_steps)
    np.testing.assert_allclose(K[:, keep], Kc, rtol=0, atol=1e-12)
    np.testing.assert_allclose(V[:, keep], Vc, rtol=0, atol=1e-12)
    np.testing.assert_allclose(x, xc, rtol=0, atol=1e-11)


def test_self_attention_position_offset():
    """Reading 4: a common position offset of the chunk leaves causal scores
    unchanged (RoPE depends on differences only)."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal((4, 6, 32))
    k = rng.standard_normal((2, 6, 32))
    v = rng.standard_normal((2, 6, 32))
    causal = np.tril(np.ones((6, 6), bool))
    o1 = om.attention(om.rope(q, np.arange(6), 1e4), om.rope(k, np.arange(6), 1e4), v, causal)
    o2 = om.attention(om.rope(q, np.arange(6) + 177, 1e4), om.rope(k, np.arange(6) + 177, 1e4), v, causal)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)


def test_empty_prefix_rejected():
    s, W, emb, _, noise, wl = _tiny()
    with pytest.raises(ValueError):
        oracle.prefill(W, s, emb, np.zeros(emb.shape[0], bool))


def test_smolvla_shapes_and_parameter_count():
    g = json.load(open(os.path.join(GOLDEN, "smolvla_shapes.json")))
    s = synth.SHAPES["smolvla"]
    for k in ("p_layers", "p_width", "p_heads", "p_kv_heads", "head_dim", "e_layers", "e_width", "action_dim"):
        assert getattr(s, k) == g[k], k
    assert synth.WORKLOADS["smolvla_b1"].H == g["chunk"]
    assert synth.WORKLOADS["smolvla_b1"].n_steps == g["euler_steps"]
    n = synth.param_count(s, "expert")
    assert n == 99_849_312
    assert abs(n - g["expert_params_approx"]) <= g["expert_params_rel_tol"] * g["expert_params_approx"]
    assert synth.param_count(s, "prefix") == 157_317_120


def test_bf16_emulation_stays_close():
    """Sanity of the diagnostic switch: rounding at the GPU's storage points
    moves the chunk by far less than the parity gate."""
    s, W, emb, valid, noise, wl = _tiny(random_affine=True)
    _, _, _, _, x = oracle.sample(W, s, emb, valid, noise, wl.n_steps)
    _, _, _, _, xe = oracle.sample(W, s, emb, valid, noise, wl.n_steps, emulate_bf16=True)
    d = np.abs(x - xe).max()
    assert 0 < d < 2e-2


# --------------------------------------------------------------------------
# prefix overwrite at a chunk junction (reading 17)
# --------------------------------------------------------------------------
def test_prefix_overwrite_with_no_prefix_is_plain_denoise():
    s, W, emb, valid, noise, wl = _tiny(random_affine=True)
    K, V = oracle.prefill(W, s, emb, valid)
    a = oracle.denoise(W, s, K, V, valid, noise, wl.n_steps)
    b = oracle.denoise_prefix_overwrite(W, s, K, V, valid, noise, wl.n_steps, np.zeros((0, s.action_dim)))
    for u, w in zip(a, b):
        assert np.array_equal(u, w)


@pytest.mark.parametrize("n_steps", [3, 4, 10])
def test_prefix_overwrite_lands_on_the_previous_actions(n_steps):
    """t reaches exactly 0, so the flow path t eps + (1 - t) a_prev ends on a_prev."""
    s, W, emb, valid, noise, wl = _tiny(random_affine=True)
    K, V = oracle.prefill(W, s, emb, valid)
    rng = np.random.default_rng(3)
    a_prev = rng.standard_normal((3, s.action_dim))
    vs, xs, x = oracle.denoise_prefix_overwrite(W, s, K, V, valid, noise, n_steps, a_prev)
    assert np.array_equal(x[:3], a_prev)
    assert not np.allclose(x[3:], oracle.denoise(W, s, K, V, valid, noise, n_steps)[2][3:])  # conditioning


def test_prefix_overwrite_constant_velocity_closed_form():
    """With v = c everywhere: rows past the prefix move linearly, prefix rows
    follow the flow path of the given actions, step by step, exactly."""
    s, W, emb, valid, _, wl = _tiny()
    W = dict(W)
    A = s.action_dim
    c = np.array([0.5, -1.25, 2.0, 0.0, -0.375, 1.0, 3.5, -2.0])[:A]
    W["w_out"] = np.zeros_like(W["w_out"])
    W["b_out"] = c
    x0 = (np.arange(wl.H * A).reshape(wl.H, A) % 7 - 3) * 0.25
    a_prev = (np.arange(2 * A).reshape(2, A) % 5 - 2) * 0.5
    K, V = oracle.prefill(W, s, emb, valid)
    vs, xs, x = oracle.denoise_prefix_overwrite(W, s, K, V, valid, x0, 4, a_prev)
    for k in range(4):
        t = 1.0 - 0.25 * (k + 1)
        assert np.array_equal(xs[k][2:], x0[2:] + (k + 1) * (-0.25) * c)
        assert np.array_equal(xs[k][:2], t * x0[:2] + (1 - t) * a_prev)
