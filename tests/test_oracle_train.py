"""Pins of the training-step oracle (the flow-matching fine-tune of the expert;
readings 25-27 in ``oracle/train.py``) against things other than the oracle
itself: the numpy velocity of ``model.py``, central differences of the numpy
loss (no autograd), closed forms of the head gradients, the flow path's end
points against the denoise, and planted mistakes that one pin must catch."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from oracle import model as om  # noqa: E402
from oracle import train as ot  # noqa: E402

S = synth.SHAPES["tiny"]
B, L, H = 2, 6, 8


def _case(seed=0, zero_w_out=False):
    rng = np.random.default_rng([seed, 77])
    W = oracle.load_weights(synth.gen_weights(S, 11 + seed, random_affine=True))
    W = {k: np.array(v) for k, v in W.items()}
    if zero_w_out:
        W["w_out"] = np.zeros_like(W["w_out"])
    K = rng.standard_normal((B, S.p_layers, L, S.p_kv_heads, S.head_dim))
    V = rng.standard_normal((B, S.p_layers, L, S.p_kv_heads, S.head_dim))
    valid = np.ones((B, L), np.uint8)
    valid[1, 2] = 0
    a = 0.5 * rng.standard_normal((B, H, S.action_dim))
    eps = rng.standard_normal((B, H, S.action_dim))
    t = np.array([0.3, 0.85])
    return W, K, V, valid, a, eps, t


# ----------------------------------------------------------------------------
# pins (each takes the module under test so planted mistakes can be swapped in)
# ----------------------------------------------------------------------------
def pin_forward_matches_numpy(m):
    W, K, V, valid, a, eps, t = _case()
    P = {n: torch.tensor(W[n]) for n in m.trainable_names(S)}
    for b in range(B):
        for tt in (float(t[b]), 1.0, 0.0):
            x = m.flow_input(a[b], eps[b], tt)
            v_np = om.velocity(W, S, x, tt, K[b], V[b], valid[b])
            v_t = m.velocity_torch(P, S, torch.tensor(x), tt, torch.tensor(K[b]), torch.tensor(V[b]), valid[b])
            assert np.allclose(v_t.detach().numpy(), v_np, rtol=0, atol=1e-12)


def pin_loss_and_central_differences(m):
    """dL/dW of autograd against (L(W + h) - L(W - h)) / 2h of the numpy loss,
    two elements of every trainable tensor."""
    W, K, V, valid, a, eps, t = _case(1)
    loss, G = m.train_step(W, S, K, V, valid, a, eps, t)
    assert abs(loss - ot.loss_np(W, S, K, V, valid, a, eps, t)) <= 1e-12 * max(1.0, loss)
    rng = np.random.default_rng(5)
    h = 1e-5
    for name in m.trainable_names(S):
        w = W[name]
        for _ in range(2):
            idx = tuple(int(rng.integers(0, d)) for d in w.shape)
            old = w[idx]
            w[idx] = old + h
            lp = ot.loss_np(W, S, K, V, valid, a, eps, t)
            w[idx] = old - h
            lm = ot.loss_np(W, S, K, V, valid, a, eps, t)
            w[idx] = old
            fd = (lp - lm) / (2 * h)
            g = float(G[name][idx])
            assert abs(fd - g) <= 1e-6 * abs(g) + 1e-9, (name, idx, fd, g)


def pin_head_closed_forms(m):
    """v is affine in b_out and W_out: dL/db_out = 2/N sum (v - (eps - a)) and
    dL/dW_out = 2/N sum (v - (eps - a)) norm(x)^T; with W_out = 0 no other tensor
    receives a gradient and v = b_out."""
    for zero in (False, True):
        W, K, V, valid, a, eps, t = _case(2, zero_w_out=zero)
        _, G = m.train_step(W, S, K, V, valid, a, eps, t)
        N = a.size
        gb = np.zeros(S.action_dim)
        for b in range(B):
            x = t[b] * eps[b] + (1 - t[b]) * a[b]                  # the page's x_t
            v = om.velocity(W, S, x, float(t[b]), K[b], V[b], valid[b])
            gb += 2.0 / N * np.sum(v - (eps[b] - a[b]), axis=0)    # the page's target eps - a
        assert np.allclose(G["b_out"], gb, rtol=1e-10, atol=1e-13)
        if zero:
            for name in m.trainable_names(S):
                if name not in ("w_out", "b_out"):
                    assert not np.any(G[name]), name


def pin_flow_end_points(m):
    """x_t is the noise at t = 1 and the target chunk at t = 0; the training
    velocity at t = 1 is the denoise's first velocity."""
    W, K, V, valid, a, eps, t = _case(3)
    assert np.array_equal(m.flow_input(a[0], eps[0], 1.0), eps[0])
    assert np.array_equal(m.flow_input(a[0], eps[0], 0.0), a[0])
    vs, _, _ = om.denoise(W, S, K[0], V[0], valid[0], eps[0], 2)
    P = {n: torch.tensor(W[n]) for n in m.trainable_names(S)}
    v1 = m.velocity_torch(P, S, torch.tensor(m.flow_input(a[0], eps[0], 1.0)), 1.0, torch.tensor(K[0]),
                          torch.tensor(V[0]), valid[0])
    assert np.allclose(v1.detach().numpy(), vs[0], rtol=0, atol=1e-12)


PINS = [pin_forward_matches_numpy, pin_loss_and_central_differences, pin_head_closed_forms, pin_flow_end_points]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_train_pin(pin):
    pin(ot)


def test_trainable_set_is_the_expert_and_heads():
    names = ot.trainable_names(S)
    man = [n for n, _ in synth.manifest(S)]
    assert names == [n for n in man if not n.startswith("p")]
    assert sum(int(np.prod(shp)) for n, shp in synth.manifest(S) if n in names) == synth.param_count(S, "expert")


# ----------------------------------------------------------------------------
# planted mistakes
# ----------------------------------------------------------------------------
class _Mutant:
    """The oracle module with one function replaced."""

    def __init__(self, **over):
        self.__dict__.update({k: getattr(ot, k) for k in ("trainable_names", "flow_input", "velocity_torch",
                                                          "train_step")})
        self.__dict__.update(over)


def _flow_swapped(a, eps, t):
    return t * np.asarray(a, np.float64) + (1.0 - t) * np.asarray(eps, np.float64)


def _train_step_sum(W, s, K, V, valid, a, eps, t):
    loss, G = ot.train_step(W, s, K, V, valid, a, eps, t)
    n = a.size
    return loss * n, {k: g * n for k, g in G.items()}               # mistake: sum, not mean


def _train_step_target_sign(W, s, K, V, valid, a, eps, t):
    return ot.train_step(W, s, K, V, valid, eps, a, t)              # mistake: target a - eps, x_t swapped


def _velocity_no_rope(P, s, x, t, K, V, valid):
    orig = ot._rope
    try:
        ot._rope = lambda x_, pos, base: x_                          # mistake: RoPE dropped
        return ot.velocity_torch(P, s, x, t, K, V, valid)
    finally:
        ot._rope = orig


def _train_step_no_rope(W, s, K, V, valid, a, eps, t):
    orig = ot._rope
    try:
        ot._rope = lambda x_, pos, base: x_
        return ot.train_step(W, s, K, V, valid, a, eps, t)
    finally:
        ot._rope = orig


def _train_step_detached_norm(W, s, K, V, valid, a, eps, t):
    orig = ot._rms_norm
    try:
        ot._rms_norm = lambda x, g, e: x / (x.pow(2).mean(-1, keepdim=True) + e).sqrt().detach() * g  # mistake
        return ot.train_step(W, s, K, V, valid, a, eps, t)
    finally:
        ot._rms_norm = orig


MUTANTS = {
    "flow_path_swapped": _Mutant(flow_input=_flow_swapped),
    "loss_sum": _Mutant(train_step=_train_step_sum),
    "target_sign": _Mutant(train_step=_train_step_target_sign),
    "rope_dropped": _Mutant(velocity_torch=_velocity_no_rope, train_step=_train_step_no_rope),
    "norm_scale_not_differentiated": _Mutant(train_step=_train_step_detached_norm),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_train_mistake(name):
    failed = 0
    for pin in PINS:
        try:
            pin(MUTANTS[name])
        except AssertionError:
            failed += 1
    assert failed >= 1, f"no pin caught the planted mistake {name}"


def test_inputs_are_well_conditioned_for_bf16():
    """The GPU parity test of the training step draws W_in 10x wider so that a
    chunk's rows differ: then rounding the attention's q, k, v and output to
    bf16 (the GPU's storage points) moves no gradient by more than 1e-2, while
    with the narrow W_in it moves the self-attention W_q / W_k gradients by
    several percent (cancellation in the softmax gradient)."""
    def rb(x):
        return x + (x.to(torch.bfloat16).to(torch.float64) - x).detach()

    def grads(w_in_scale, emulate):
        W, K, V, valid, a, eps, t = _case(4)
        W["w_in"] = W["w_in"] * w_in_scale
        orig_split, orig_att = ot._split, ot._attention
        if emulate:
            ot._split = lambda x, n: rb(orig_split(x, n))
            ot._attention = lambda q, k, v, al: rb(orig_att(rb(q), rb(k), rb(v), al))
        try:
            return ot.train_step(W, S, K, V, valid, a, eps, t)[1]
        finally:
            ot._split, ot._attention = orig_split, orig_att

    def worst(scale):
        g0, g1 = grads(scale, False), grads(scale, True)
        return max(np.linalg.norm(g1[n] - g0[n]) / np.linalg.norm(g0[n]) for n in g0)

    assert worst(10.0) <= 1e-2
    assert worst(1.0) > 2e-2


# ----------------------------------------------------------------------------
# reading 28: the optional rounding at the GPU's bf16 storage points
# ----------------------------------------------------------------------------
def test_bf16_round_is_nearest_even_with_a_straight_through_gradient():
    """bf16 keeps 8 significant bits: at 1 the spacing is 2^-7, so 1 + 2^-8 is
    a tie that goes to the even neighbour 1, 1 + 3 2^-8 a tie that goes to the
    even neighbour 1 + 2^-6, and anything above a tie goes up."""
    x = torch.tensor([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, -(1 + 2 ** -8), 3.0, 0.0],
                     dtype=torch.float64, requires_grad=True)
    r = ot.bf16_round(x)
    assert r.detach().tolist() == [1.0, 1 + 2 ** -6, 1 + 2 ** -7, -1.0, 3.0, 0.0]
    r.sum().backward()
    assert x.grad.tolist() == [1.0] * 6


def test_storage_rounding_moves_the_forward_by_bf16_amounts():
    """The rounded forward differs from the exact one (rounding happened), by
    the size of a few bf16 roundings carried through the layers, not more."""
    W, K, V, valid, a, eps, t = _case(3)
    P = {n: torch.tensor(W[n]) for n in ot.trainable_names(S)}
    for b in range(B):
        x = torch.tensor(ot.flow_input(a[b], eps[b], float(t[b])))
        args = (P, S, x, float(t[b]), torch.tensor(K[b]), torch.tensor(V[b]), valid[b])
        v0 = ot.velocity_torch(*args).detach().numpy()
        v1 = ot.velocity_torch(*args, bf16_storage=True).detach().numpy()
        rel = np.linalg.norm(v1 - v0) / np.linalg.norm(v0)
        assert 2 ** -16 < rel < 2e-2, rel


def test_storage_rounding_keeps_the_head_closed_forms():
    """Every rounding point lies before the final norm, so the head stays
    affine: dL/db_out = 2/N sum (v - (eps - a)) with v the rounded forward's
    velocity; with W_out = 0 no other tensor receives a gradient."""
    for zero in (False, True):
        W, K, V, valid, a, eps, t = _case(4, zero_w_out=zero)
        _, G = ot.train_step(W, S, K, V, valid, a, eps, t, bf16_storage=True)
        P = {n: torch.tensor(W[n]) for n in ot.trainable_names(S)}
        d = np.zeros(S.action_dim)
        for b in range(B):
            x = torch.tensor(ot.flow_input(a[b], eps[b], float(t[b])))
            v = ot.velocity_torch(P, S, x, float(t[b]), torch.tensor(K[b]), torch.tensor(V[b]), valid[b],
                                  bf16_storage=True).detach().numpy()
            d += (v - (eps[b] - a[b])).sum(axis=0)
        assert np.allclose(G["b_out"], 2.0 / a.size * d, rtol=1e-12, atol=1e-14)
        if zero:
            for n in ot.trainable_names(S):
                if n not in ("w_out", "b_out"):
                    assert not np.any(G[n]), n


def test_storage_rounding_is_what_moves_the_narrow_input_gradients():
    """At the workloads' own N(0, 0.02) W_in the rows of a chunk are nearly
    equal and the softmax gradient cancels: rounding at the storage points
    moves some self-attention W_q / W_k gradient by more than 2e-2. This is
    the case the GPU parity test compares against the rounded oracle."""
    W, K, V, valid, a, eps, t = _case(4)
    g0 = ot.train_step(W, S, K, V, valid, a, eps, t)[1]
    g1 = ot.train_step(W, S, K, V, valid, a, eps, t, bf16_storage=True)[1]
    rel = {n: np.linalg.norm(g1[n] - g0[n]) / np.linalg.norm(g0[n]) for n in g0}
    assert max(rel["e0.wq"], rel["e0.wk"]) > 2e-2, rel


def test_workload_self_attention_gradients_are_rounding_bound():
    """At the SmolVLA shape with the workloads' own weights (two queries,
    prefix 177, chunk 50, as the GPU parity test), realizations of the
    storage-rounded oracle whose values before every bf16 rounding differ by
    one float32 ulp disagree on the self-attention W_q / W_k gradients by more
    than 1e-2, and on every other gradient by less than 5e-3: those two
    tensors per self-attention layer are set by individual rounding decisions
    (the rows of a chunk are nearly equal and the softmax gradient cancels),
    the rest is well conditioned."""
    s = synth.SHAPES["smolvla"]
    B, L, Hc, seed = 2, 177, 50, 7
    W = oracle.load_weights(synth.gen_weights(s, seed))
    rng = np.random.default_rng([seed, 31])
    kv = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
        rng.standard_normal((2, s.p_layers, B, L, s.p_kv_width)).astype(np.float32))).astype(np.float64)
    K = kv[0].transpose(1, 0, 2, 3).reshape(B, s.p_layers, L, s.p_kv_heads, s.head_dim)
    V = kv[1].transpose(1, 0, 2, 3).reshape(B, s.p_layers, L, s.p_kv_heads, s.head_dim)
    valid = np.ones((B, L), np.uint8)
    valid[0, 1] = 0
    valid[1, L - 3:] = 0
    a = (0.5 * rng.standard_normal((B, Hc, s.action_dim))).astype(np.float32).astype(np.float64)
    eps = rng.standard_normal((B, Hc, s.action_dim)).astype(np.float32).astype(np.float64)
    t = rng.uniform(0.05, 0.95, B).astype(np.float32).astype(np.float64)
    orig = ot.bf16_round
    runs = []
    for k in (1, -1):
        ot.bf16_round = (lambda kk: (lambda x: orig(x * (1 + kk * 2.0 ** -23))))(k)
        try:
            runs.append(ot.train_step(W, s, K, V, valid, a, eps, t, bf16_storage=True)[1])
        finally:
            ot.bf16_round = orig
    d = {n: np.linalg.norm(runs[0][n] - runs[1][n]) / np.linalg.norm(runs[1][n]) for n in runs[0]}
    sa = {f"e{l}.{w}" for l in range(0, s.e_layers, 2) for w in ("wq", "wk")}
    assert min(d[n] for n in sa) > 1e-2, sorted((n, d[n]) for n in sa)
    assert max(d[n] for n in d if n not in sa) < 5e-3, max((d[n], n) for n in d if n not in sa)
