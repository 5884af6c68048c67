"""Training step of the action expert (the flow-matching fine-tune), plain definition.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library must
never import this module.

"noeira docs, SmolVLA" §Architecture (the flow-matching objective of the
fine-tune): x_t = t eps + (1 - t) a and L = ||v_theta(x_t, t | prefix) - (eps - a)||^2;
the block mask lets the fine-tune reuse the inference forward. §Fine-tuning:
the shipped recipe trains the 16 expert layers and the action and time
projections, while SigLIP, the language model and the connector stay frozen.

Readings (numbered after those of ``quant.py``):

25. The loss of a batch is the mean of (v - (eps - a))^2 over its queries,
    chunk rows and action dimensions (the squared norm of the page averaged
    over its B H A terms); every action row counts.
26. Trainable set: every expert tensor (per layer in_norm, W_q, W_k, W_v, W_o,
    post_norm, W_g, W_u, W_d; on odd layers W_k and W_v act on the frozen
    prefix cache), final_norm, and the heads w_in, b_in, w_t1, b_t1, w_t2,
    b_t2, w_out, b_out. The prefix LM is frozen: its K/V cache is an input.
    Each query has its own flow time t_b, an input (the sampler of t is not
    on the path, like the noise).
27. A step's result is the loss and its gradient with respect to every
    trainable tensor; the optimiser update is not part of it.

28. Storage rounding (optional, ``bf16_storage=True``; off by default). The
    CSDN precision post (§3-§7, §9) shows that where a bf16 pipeline rounds
    decides how far it lands from an fp32 one, and its §11 asks to keep that
    precision-change error apart from the error of the port itself. To tell
    the two apart, the forward can round to bfloat16
    (nearest, ties to even, from the float32 value) at the points where the
    GPU stores bf16: the action embedding and the time features entering the
    time MLP, the time MLP's hidden layer, both RMSNorm outputs of every
    layer, q and k after RoPE and v (the cross layers' projected prefix keys
    and values too), the unnormalised probabilities in P V (the softmax sum
    stays unrounded) and the attention output, and the SwiGLU output. Each
    rounding passes its gradient straight through, so the backward is the
    derivative of the rounded forward taken at the rounded values, except
    that the attention's derivative is that of the unrounded softmax: a
    backward that recomputes P from the stored q and k (as the GPU's does)
    never sees the rounded P. The default path is unchanged.

The forward is the velocity of ``model.py`` restated in float64 torch, so
that autograd returns the exact derivative of the written forward; the tests
pin this forward to ``model.velocity`` and the gradients to central
differences of ``loss_np`` (numpy only).
"""
from __future__ import annotations

import math
from typing import Dict, List, Tuple

import numpy as np

from . import model as om


def trainable_names(s) -> List[str]:
    """Reading 26, in manifest order."""
    names = []
    for l in range(s.e_layers):
        names += [f"e{l}.{m}" for m in ("in_norm", "wq", "wk", "wv", "wo", "post_norm", "wg", "wu", "wd")]
    names += ["final_norm", "w_in", "b_in", "w_t1", "b_t1", "w_t2", "b_t2", "w_out", "b_out"]
    return names


def flow_input(a: np.ndarray, eps: np.ndarray, t: float) -> np.ndarray:
    """x_t = t eps + (1 - t) a."""
    return t * np.asarray(eps, np.float64) + (1.0 - t) * np.asarray(a, np.float64)


def loss_np(W, s, K: np.ndarray, V: np.ndarray, valid: np.ndarray, a: np.ndarray, eps: np.ndarray,
            t: np.ndarray) -> float:
    """Reading 25 with the numpy velocity: K/V [B, p_layers, L, kv, hd],
    valid [B, L], a/eps [B, H, A], t [B]."""
    tot, n = 0.0, 0
    for b in range(a.shape[0]):
        x = flow_input(a[b], eps[b], float(t[b]))
        v = om.velocity(W, s, x, float(t[b]), K[b], V[b], valid[b])
        d = v - (np.asarray(eps[b], np.float64) - np.asarray(a[b], np.float64))
        tot += float(np.sum(d * d))
        n += d.size
    return tot / n


# ----------------------------------------------------------------------------
# the same forward in float64 torch
# ----------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def _rms_norm(x, g, eps):
    return x / (x.pow(2).mean(-1, keepdim=True) + eps).sqrt() * g


def _rope(x, pos, base):
    torch = _torch()
    hd = x.shape[-1]
    half = hd // 2
    inv_freq = base ** (-(2.0 * torch.arange(half, dtype=torch.float64)) / hd)
    ang = torch.as_tensor(pos, dtype=torch.float64)[:, None] * inv_freq[None, :]
    c, sn = torch.cos(ang), torch.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * c - x2 * sn, x2 * c + x1 * sn], dim=-1)


def _attention(q, k, v, allowed):
    torch = _torch()
    n_q, hd = q.shape[0], q.shape[-1]
    group = n_q // k.shape[0]
    outs = []
    for h in range(n_q):
        g = h // group
        sc = (q[h] @ k[g].T) / math.sqrt(hd)
        sc = sc.masked_fill(~allowed, float("-inf"))
        outs.append(torch.softmax(sc, dim=-1) @ v[g])
    return torch.stack(outs)


def _split(x, n):
    T = x.shape[0]
    return x.reshape(T, n, -1).transpose(0, 1)


def _merge(x):
    n, T, hd = x.shape
    return x.transpose(0, 1).reshape(T, n * hd)


def _silu(x):
    return x / (1.0 + (-x).exp())


def bf16_round(x):
    """Reading 28: the value of x rounded to bfloat16 (nearest, ties to even,
    from its float32 value), with the gradient passed straight through."""
    torch = _torch()
    r = x.detach().to(torch.float32).to(torch.bfloat16).to(torch.float64)
    return x + (r - x).detach()


def _identity(x):
    return x


def _attention_rounded(q, k, v, allowed, rnd):
    """Attention whose value has the unnormalised probabilities rounded where
    they enter P V (the softmax sum over the unrounded values), and whose
    derivative is that of the unrounded softmax attention: the backward
    recomputes P from the stored q and k, it never sees the rounded P
    (reading 28)."""
    torch = _torch()
    n_q, hd = q.shape[0], q.shape[-1]
    group = n_q // k.shape[0]
    outs = []
    for h in range(n_q):
        g = h // group
        sc = (q[h] @ k[g].T) / math.sqrt(hd)
        sc = sc.masked_fill(~allowed, float("-inf"))
        exact = torch.softmax(sc, dim=-1) @ v[g]
        pt = (sc - sc.max(dim=-1, keepdim=True).values).exp().detach()
        stored = (rnd(pt) @ v[g].detach()) / pt.sum(dim=-1, keepdim=True)
        outs.append(exact + (stored - exact).detach())
    return torch.stack(outs)


def velocity_torch(P, s, x, t: float, K, V, valid, bf16_storage: bool = False):
    """model.velocity restated on torch tensors (P: name -> float64 tensor);
    ``bf16_storage`` rounds at the GPU's storage points (reading 28)."""
    torch = _torch()
    rnd = bf16_round if bf16_storage else _identity
    H, L = x.shape[0], K.shape[1]
    De = s.e_width
    a = x @ P["w_in"].T + P["b_in"]
    e = torch.as_tensor(om.time_embedding(t, De, s.t_min_period, s.t_max_period)).expand(H, De)
    h = rnd(_silu(torch.cat([rnd(a), rnd(e)], dim=1) @ P["w_t1"].T + P["b_t1"]))
    r = h @ P["w_t2"].T + P["b_t2"]
    pos = np.arange(H)
    causal = torch.tril(torch.ones(H, H, dtype=torch.bool))
    cross = torch.as_tensor(np.asarray(valid, bool))[None, :].expand(H, L)

    def attend(q, k, v, allowed):
        if not bf16_storage:
            return _attention(q, k, v, allowed)
        return rnd(_attention_rounded(q, k, v, allowed, rnd))

    for l in range(s.e_layers):
        p = f"e{l}."
        y = rnd(_rms_norm(r, P[p + "in_norm"], s.rms_eps))
        q = _split(y @ P[p + "wq"].T, s.e_heads)
        if l % 2 == 0:
            k = rnd(_rope(_split(y @ P[p + "wk"].T, s.e_kv_heads), pos, s.rope_base))
            v = rnd(_split(y @ P[p + "wv"].T, s.e_kv_heads))
            o = attend(rnd(_rope(q, pos, s.rope_base)), k, v, causal)
        else:
            kc = K[l].reshape(L, s.p_kv_width)
            vc = V[l].reshape(L, s.p_kv_width)
            k = rnd(_split(kc @ P[p + "wk"].T, s.e_kv_heads))
            v = rnd(_split(vc @ P[p + "wv"].T, s.e_kv_heads))
            o = attend(rnd(q), k, v, cross)
        r = r + _merge(o) @ P[p + "wo"].T
        y = rnd(_rms_norm(r, P[p + "post_norm"], s.rms_eps))
        r = r + rnd(_silu(y @ P[p + "wg"].T) * (y @ P[p + "wu"].T)) @ P[p + "wd"].T
    yf = _rms_norm(r, P["final_norm"], s.rms_eps)
    return yf @ P["w_out"].T + P["b_out"]


def train_step(W: Dict[str, np.ndarray], s, K: np.ndarray, V: np.ndarray, valid: np.ndarray, a: np.ndarray,
               eps: np.ndarray, t: np.ndarray, bf16_storage: bool = False) -> Tuple[float, Dict[str, np.ndarray]]:
    """Readings 25-27: (loss, {trainable name: dL/dW}) for one batch.

    K/V [B, p_layers, L, p_kv_heads, hd] (frozen prefix cache), valid [B, L],
    a (the target chunk) and eps (the noise) [B, H, A], t [B].
    ``bf16_storage``: round the forward at the GPU's storage points (reading 28).
    """
    torch = _torch()
    names = trainable_names(s)
    P = {n: torch.tensor(np.asarray(W[n], np.float64), requires_grad=True) for n in names}
    tot = None
    count = 0
    for b in range(a.shape[0]):
        x = torch.as_tensor(flow_input(a[b], eps[b], float(t[b])))
        v = velocity_torch(P, s, x, float(t[b]), torch.as_tensor(np.asarray(K[b], np.float64)),
                           torch.as_tensor(np.asarray(V[b], np.float64)), valid[b], bf16_storage)
        target = torch.as_tensor(np.asarray(eps[b], np.float64) - np.asarray(a[b], np.float64))
        term = (v - target).pow(2).sum()
        tot = term if tot is None else tot + term
        count += v.numel()
    loss = tot / count
    loss.backward()
    return float(loss.detach()), {n: P[n].grad.numpy().copy() for n in names}
