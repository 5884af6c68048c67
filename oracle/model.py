"""Plain float64 definition of the SmolVLA prefix prefill and Euler denoise.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library must
never import this module.

Readings taken where the pages leave a step open (each is marked "Reading"
below; the numbers are used wherever a reading is cited):

 1. Prefix mask: bidirectional over valid prefix keys; the row's own validity
    does not matter ("noeira docs, SmolVLA" §Architecture only fixes that the
    prefix cannot see the actions).
 2. Prefix positions with padding: pos = cumsum(valid) - 1.
 3. RoPE: rotate-half pairing (i, i + hd/2), inv_freq_i = base^(-2i/hd).
 4. Expert self-attention: within the chunk only, causal, positions 0..H-1.
 5. Cross-attention: odd expert layer l reads prefix layer l's cache (post-RoPE
    K); the expert k/v projections act on each token's head-concatenated
    K (resp. V) vector; no RoPE on the expert query; key j allowed iff valid.
 6. GQA: query head h reads kv head floor(h / (n_q / n_kv)).
 7. Attention: scale 1/sqrt(hd), masked logits -inf, max-subtracted softmax.
 8. RMSNorm y = x / sqrt(mean(x^2) + eps) * g; pre-norm residual blocks; a
    final RMSNorm on the expert output before action_out.
 9. Biases only on action_in, the time MLP and action_out.
11. Time MLP: s = W2 silu(W1 [a || e(t)] + b1) + b2, action embedding first.
12. Sinusoid: e(t) = [sin(2 pi t / p_i) || cos(2 pi t / p_i)],
    p_i = pmin (pmax / pmin)^(i / (De/2 - 1)).
13. Euler: t_0 = 1, dt = -1/N, v evaluated at (x_k, t_k), t_k = 1 + k dt,
    x_{k+1} = x_k + dt v_k; the output is x_N ("noeira docs, SmolVLA"
    §Architecture: x_t = t eps + (1 - t) a, target eps - a).
17. Prefix overwrite at a chunk junction: after each Euler step the first d
    rows of the state are the flow path of the previous chunk's d actions at
    the time reached (see ``denoise_prefix_overwrite``).

Optional ``emulate_bf16`` rounds to bf16 at the points where the GPU stores
bf16 (normalised activations, q/k/v, attention output, SwiGLU output, time-MLP
hidden, action embedding). It exists only to separate storage-precision error
from kernel bugs in diagnostics; the parity gates use the plain definition.
"""
from __future__ import annotations

from typing import Dict, Tuple

import numpy as np

F64 = np.float64


# ----------------------------------------------------------------------------
# rounding used only by the optional bf16 emulation
# ----------------------------------------------------------------------------
def _round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), returned as float64."""
    f = np.asarray(x, dtype=np.float32)      # float64 -> float32 is itself RNE
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(F64)


def _identity(x):
    return x


# ----------------------------------------------------------------------------
# weights
# ----------------------------------------------------------------------------
def load_weights(bits: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """bf16 bit patterns -> exact float64 values."""
    out = {}
    for k, b in bits.items():
        u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
        out[k] = u.view(np.float32).astype(F64)
    return out


# ----------------------------------------------------------------------------
# building blocks ("noeira docs, SmolVLA" §Architecture, SmolLM2 layer)
# ----------------------------------------------------------------------------
def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """Reading 8: x / sqrt(mean(x^2) + eps) * g over the last axis."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Reading 3: rotate-half RoPE. x is [heads, T, hd]; pos is [T]."""
    hd = x.shape[-1]
    half = hd // 2
    inv_freq = base ** (-(2.0 * np.arange(half, dtype=F64)) / hd)
    ang = np.asarray(pos, dtype=F64)[:, None] * inv_freq[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
              allowed: np.ndarray) -> np.ndarray:
    """Readings 6, 7: GQA softmax attention.

    q [n_q, Tq, hd], k/v [n_kv, Tk, hd], allowed bool [Tq, Tk] (True = key
    visible). Every row must have at least one visible key.
    """
    n_q, _, hd = q.shape
    n_kv = k.shape[0]
    group = n_q // n_kv
    out = np.empty_like(q)
    for h in range(n_q):
        g = h // group
        s = (q[h] @ k[g].T) / np.sqrt(hd)
        s = np.where(allowed, s, -np.inf)
        m = np.max(s, axis=-1, keepdims=True)
        p = np.exp(s - m)
        p = p / np.sum(p, axis=-1, keepdims=True)
        out[h] = p @ v[g]
    return out


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def _split(x: np.ndarray, n: int) -> np.ndarray:
    """[T, n*hd] -> [n, T, hd]"""
    T = x.shape[0]
    return x.reshape(T, n, -1).transpose(1, 0, 2)


def _merge(x: np.ndarray) -> np.ndarray:
    """[n, T, hd] -> [T, n*hd]"""
    n, T, hd = x.shape
    return x.transpose(1, 0, 2).reshape(T, n * hd)


def _swiglu(y, wg, wu, wd, rb):
    h = rb(silu(y @ wg.T) * (y @ wu.T))
    return h @ wd.T


def prefix_positions(valid: np.ndarray) -> np.ndarray:
    """Reading 2: position of token i = (number of valid tokens up to i) - 1."""
    return np.cumsum(np.asarray(valid, dtype=np.int64)) - 1


# ----------------------------------------------------------------------------
# prefix prefill
# ----------------------------------------------------------------------------
def prefill(W: Dict[str, np.ndarray], s, embeds: np.ndarray, valid: np.ndarray,
            emulate_bf16: bool = False) -> Tuple[np.ndarray, np.ndarray]:
    """One query's prefix through the 16 SmolLM2 layers; returns its K/V cache.

    embeds [L, p_width] (float64 values of the bf16 inputs), valid [L] (1 =
    real token). Returns K, V as [p_layers, L, p_kv_heads, head_dim]; K is
    stored after RoPE. All layers run in full (the last layer's attention and
    MLP outputs are computed although nothing reads them).
    """
    rb = _round_bf16 if emulate_bf16 else _identity
    valid = np.asarray(valid).astype(bool)
    if not valid.any():
        raise ValueError("query has no valid prefix token")
    L = embeds.shape[0]
    pos = prefix_positions(valid)
    allowed = np.broadcast_to(valid[None, :], (L, L))          # Reading 1
    x = np.array(embeds, dtype=F64)
    Ks = np.empty((s.p_layers, L, s.p_kv_heads, s.head_dim))
    Vs = np.empty_like(Ks)
    for l in range(s.p_layers):
        p = f"p{l}."
        y = rb(rms_norm(x, W[p + "in_norm"], s.rms_eps))
        q = rope(_split(y @ W[p + "wq"].T, s.p_heads), pos, s.rope_base)
        k = rope(_split(y @ W[p + "wk"].T, s.p_kv_heads), pos, s.rope_base)
        v = _split(y @ W[p + "wv"].T, s.p_kv_heads)
        q, k, v = rb(q), rb(k), rb(v)
        Ks[l] = k.transpose(1, 0, 2)
        Vs[l] = v.transpose(1, 0, 2)
        o = rb(_merge(attention(q, k, v, allowed)))
        x = x + o @ W[p + "wo"].T
        y = rb(rms_norm(x, W[p + "post_norm"], s.rms_eps))
        x = x + _swiglu(y, W[p + "wg"], W[p + "wu"], W[p + "wd"], rb)
    return Ks, Vs


# ----------------------------------------------------------------------------
# action expert
# ----------------------------------------------------------------------------
def time_embedding(t: float, dim: int, pmin: float, pmax: float) -> np.ndarray:
    """Reading 12: [sin || cos] of 2 pi t over geometric periods pmin..pmax."""
    half = dim // 2
    frac = np.arange(half, dtype=F64) / (half - 1)
    period = pmin * (pmax / pmin) ** frac
    ang = 2.0 * np.pi * t / period
    return np.concatenate([np.sin(ang), np.cos(ang)])


def cross_kv(W, s, l: int, K: np.ndarray, V: np.ndarray, rb=_identity):
    """Reading 5: expert layer l's keys/values from prefix layer l's cache.

    K[l], V[l] are [L, p_kv_heads, hd]; each token's head-concatenated vector
    goes through the expert's k/v projection. Returns [e_kv_heads, L, hd].
    """
    L = K.shape[1]
    kc = K[l].reshape(L, s.p_kv_width)
    vc = V[l].reshape(L, s.p_kv_width)
    k = rb(_split(kc @ W[f"e{l}.wk"].T, s.e_kv_heads))
    v = rb(_split(vc @ W[f"e{l}.wv"].T, s.e_kv_heads))
    return k, v


def velocity(W, s, x: np.ndarray, t: float, K: np.ndarray, V: np.ndarray,
             valid: np.ndarray, emulate_bf16: bool = False) -> np.ndarray:
    """v_theta(x_t, t | prefix): the expert's velocity for one query's chunk.

    x [H, A], t scalar, K/V [p_layers, L, p_kv_heads, hd], valid [L].
    """
    rb = _round_bf16 if emulate_bf16 else _identity
    valid = np.asarray(valid).astype(bool)
    H = x.shape[0]
    L = K.shape[1]
    De = s.e_width
    a = x @ W["w_in"].T + W["b_in"]                                   # action_in
    e = np.broadcast_to(time_embedding(t, De, s.t_min_period, s.t_max_period), (H, De))
    h = rb(silu(np.concatenate([rb(a), e], axis=1) @ W["w_t1"].T + W["b_t1"]))  # Reading 11
    r = h @ W["w_t2"].T + W["b_t2"]                                   # expert residual
    pos = np.arange(H)
    causal = np.tril(np.ones((H, H), dtype=bool))                     # Reading 4
    cross_allowed = np.broadcast_to(valid[None, :], (H, L))           # Reading 5
    for l in range(s.e_layers):
        p = f"e{l}."
        y = rb(rms_norm(r, W[p + "in_norm"], s.rms_eps))
        q = _split(y @ W[p + "wq"].T, s.e_heads)
        if l % 2 == 0:
            k = rope(_split(y @ W[p + "wk"].T, s.e_kv_heads), pos, s.rope_base)
            v = _split(y @ W[p + "wv"].T, s.e_kv_heads)
            q = rope(q, pos, s.rope_base)
            o = attention(rb(q), rb(k), rb(v), causal)
        else:
            k, v = cross_kv(W, s, l, K, V, rb)
            o = attention(rb(q), k, v, cross_allowed)
        r = r + rb(_merge(o)) @ W[p + "wo"].T
        y = rb(rms_norm(r, W[p + "post_norm"], s.rms_eps))
        r = r + _swiglu(y, W[p + "wg"], W[p + "wu"], W[p + "wd"], rb)
    yf = rms_norm(r, W["final_norm"], s.rms_eps)                      # Reading 8
    return yf @ W["w_out"].T + W["b_out"]                             # action_out


def denoise(W, s, K, V, valid, noise: np.ndarray, n_steps: int,
            emulate_bf16: bool = False):
    """Reading 13: Euler from x_0 = noise at t = 1 to t = 0 in n_steps.

    Returns (vs [n, H, A], xs [n, H, A], x_final [H, A]) where vs[k] is the
    velocity at (x_k, t_k) and xs[k] = x_{k+1}, the per-step trace of the
    CSDN precision post §2 (step_k velocity / step_k x).
    """
    dt = -1.0 / n_steps
    x = np.array(noise, dtype=F64)
    vs, xs = [], []
    for k in range(n_steps):
        t = 1.0 + k * dt
        v = velocity(W, s, x, t, K, V, valid, emulate_bf16)
        x = x + dt * v
        vs.append(v)
        xs.append(x.copy())
    return np.stack(vs), np.stack(xs), x


def denoise_prefix_overwrite(W, s, K, V, valid, noise: np.ndarray, n_steps: int,
                             a_prev: np.ndarray, emulate_bf16: bool = False):
    """Euler denoise with the gradient-free prefix overwrite at a chunk junction.

    "Paper vs hardware 11: SmolVLA" §What I ran: the first d actions of a new
    chunk run during the inference delay, and overwriting that prefix with the
    previous chunk's actions removes most of the jump at the junction.
    Reading 17: after every Euler step (and so before every later velocity
    evaluation) the first d rows of the state are set to the flow path of the
    known actions, x_t[:d] = t eps[:d] + (1 - t) a_prev (x_t = t eps + (1 - t) a,
    "noeira docs, SmolVLA" §Architecture), with t the time the step reached;
    the final chunk therefore starts with exactly a_prev. At t = 1 the
    overwrite is the noise itself, so step 0 is unchanged. a_prev is [d, A],
    0 <= d <= H. Returns (vs, xs, x) like ``denoise``; xs holds the states
    after the overwrite.
    """
    a_prev = np.asarray(a_prev, dtype=F64)
    d = a_prev.shape[0]
    eps = np.array(noise, dtype=F64)
    dt = -1.0 / n_steps
    x = eps.copy()
    vs, xs = [], []
    for k in range(n_steps):
        t = 1.0 + k * dt
        v = velocity(W, s, x, t, K, V, valid, emulate_bf16)
        x = x + dt * v
        t_next = 1.0 + (k + 1) * dt
        if d:
            x[:d] = t_next * eps[:d] + (1.0 - t_next) * a_prev
        vs.append(v)
        xs.append(x.copy())
    return np.stack(vs), np.stack(xs), x


def sample(W, s, embeds, valid, noise, n_steps, emulate_bf16=False):
    """Prefill once, then denoise: one query's action chunk and K/V."""
    K, V = prefill(W, s, embeds, valid, emulate_bf16)
    vs, xs, x = denoise(W, s, K, V, valid, noise, n_steps, emulate_bf16)
    return K, V, vs, xs, x


# ----------------------------------------------------------------------------
# joint pass (pin for the block mask)
# ----------------------------------------------------------------------------
def oracle_joint(W, s, embeds: np.ndarray, valid: np.ndarray, x: np.ndarray,
                 t: float):
    """One pass over the concatenated [prefix || chunk] sequence.

    "noeira docs, SmolVLA" §Architecture: a block attention mask joins prefix
    and suffix so that a single joint pass and prefill + denoise give the same
    prefix activations. Here each row uses its own group's weights and one
    (L+H) x (L+H) mask is built from explicit block rules:

      prefix row i, column j:   j < L and valid[j]
      chunk row, even layer:    L <= j <= i            (causal within chunk)
      chunk row, odd layer:     j < L and valid[j]     (cross to the prefix)

    On odd layers the chunk rows read the prefix keys/values of the same layer
    through the expert's k/v projection. Returns (K, V, v) with K/V as in
    ``prefill`` and v the velocity at (x, t).
    """
    valid = np.asarray(valid).astype(bool)
    L, H = embeds.shape[0], x.shape[0]
    T = L + H
    pos_p = prefix_positions(valid)
    pos_c = np.arange(H)
    rows = np.arange(T)[:, None]
    cols = np.arange(T)[None, :]
    col_valid = np.concatenate([valid, np.zeros(H, bool)])[None, :]
    prefix_rule = (rows < L) & (cols < L) & col_valid
    chunk_even = (rows >= L) & (cols >= L) & (cols <= rows)
    chunk_odd = (rows >= L) & (cols < L) & col_valid

    xp = np.array(embeds, dtype=F64)
    De = s.e_width
    a = x @ W["w_in"].T + W["b_in"]
    e = np.broadcast_to(time_embedding(t, De, s.t_min_period, s.t_max_period), (H, De))
    r = silu(np.concatenate([a, e], axis=1) @ W["w_t1"].T + W["b_t1"]) @ W["w_t2"].T + W["b_t2"]
    hd = s.head_dim
    Ks = np.empty((s.p_layers, L, s.p_kv_heads, hd))
    Vs = np.empty_like(Ks)
    if s.p_layers != s.e_layers or s.p_kv_heads != s.e_kv_heads:
        raise ValueError("joint pass needs equal layer and kv-head counts")
    for l in range(s.p_layers):
        odd = l % 2 == 1
        allowed = prefix_rule | (chunk_odd if odd else chunk_even)
        P, E = f"p{l}.", f"e{l}."
        # prefix rows
        yp = rms_norm(xp, W[P + "in_norm"], s.rms_eps)
        qp = rope(_split(yp @ W[P + "wq"].T, s.p_heads), pos_p, s.rope_base)
        kp = rope(_split(yp @ W[P + "wk"].T, s.p_kv_heads), pos_p, s.rope_base)
        vp = _split(yp @ W[P + "wv"].T, s.p_kv_heads)
        Ks[l] = kp.transpose(1, 0, 2)
        Vs[l] = vp.transpose(1, 0, 2)
        # chunk rows
        yc = rms_norm(r, W[E + "in_norm"], s.rms_eps)
        qc = _split(yc @ W[E + "wq"].T, s.e_heads)
        if odd:
            kcp = _split(_merge(kp) @ W[E + "wk"].T, s.e_kv_heads)   # projected prefix keys
            vcp = _split(_merge(vp) @ W[E + "wv"].T, s.e_kv_heads)
            kcc = np.zeros((s.e_kv_heads, H, hd))                    # no chunk keys on odd layers
            vcc = np.zeros((s.e_kv_heads, H, hd))
        else:
            qc = rope(qc, pos_c, s.rope_base)
            kcc = rope(_split(yc @ W[E + "wk"].T, s.e_kv_heads), pos_c, s.rope_base)
            vcc = _split(yc @ W[E + "wv"].T, s.e_kv_heads)
            kcp, vcp = kp, vp                                        # raw prefix keys (masked)
        # every row group scores all L + H columns; the mask decides
        op = attention(qp, np.concatenate([kp, kcc], axis=1),
                       np.concatenate([vp, vcc], axis=1), allowed[:L])
        kc_all = np.concatenate([kcp, kcc], axis=1)
        vc_all = np.concatenate([vcp, vcc], axis=1)
        oc = attention(qc, kc_all, vc_all, allowed[L:])
        xp = xp + _merge(op) @ W[P + "wo"].T
        xp = xp + _swiglu(rms_norm(xp, W[P + "post_norm"], s.rms_eps),
                          W[P + "wg"], W[P + "wu"], W[P + "wd"], _identity)
        r = r + _merge(oc) @ W[E + "wo"].T
        r = r + _swiglu(rms_norm(r, W[E + "post_norm"], s.rms_eps),
                        W[E + "wg"], W[E + "wu"], W[E + "wd"], _identity)
    v = rms_norm(r, W["final_norm"], s.rms_eps) @ W["w_out"].T + W["b_out"]
    return Ks, Vs, v
