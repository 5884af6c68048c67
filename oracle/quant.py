"""Weight-only int8 quantisation of the prefix LM ("vlm-8bit") and of the action
expert, plain definition.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library must
never import this module.

mlx-smolvla PyPI page §Run a checkpoint: besides the dense bf16 default the
port offers a ``vlm-8bit`` (and ``vlm-4bit``) quantised preset, an explicit
opt-in that is never selected implicitly. The page names the preset and
nothing of its scheme.

Readings (numbered after those of ``assembly.py``):

22. ``vlm-8bit`` quantises the weight matrices of the prefix LM's linear
    layers — W_q, W_k, W_v, W_o, W_g, W_u, W_d of every prefix layer — and
    nothing else: the norm gains, the action expert and its heads stay bf16,
    and the activations stay bf16 (weight-only).
23. Affine groups: every run of 64 consecutive input weights of one output row
    (row n, columns 64 g .. 64 g + 63) is one group with a scale alpha and an
    offset beta, w ~ alpha q + beta, q in {0 .. 255}. The pages give no group
    size; 64 is the default group of the MLX affine quantiser the port is
    built on. Per group, with every operation an IEEE fp32 operation rounded
    to nearest even (so the codes are reproducible bit for bit):
        lo = min w, hi = max w,
        alpha = bf16(fp32(hi - lo) / 255),   beta = lo   (both bf16 values),
        q = clamp(rint(fp32(w - beta) / alpha), 0, 255),  q = 0 if alpha = 0.
24. The dequantised weight is the bf16 value w^ = bf16(fp32(alpha q + beta))
    (alpha q is exact in fp32: 8-bit significand times an 8-bit integer).
    The quantised model is the dense bf16 model with every quantised matrix
    replaced by w^; where a norm gain is folded into a projection, it is
    applied to w^ as it is to the dense weight.
29. The expert preset (the scope "prefix/expert" of the int8 row): the same
    scheme applied to the weight matrices of every action-expert layer —
    W_q, W_k, W_v (the odd layers' W_k, W_v act on the prefix cache), W_o,
    W_g, W_u, W_d; the expert's heads (action_in, the time MLP, action_out)
    and its norm gains stay bf16. The expert's 720-wide inputs are not a
    multiple of 64: where K mod 64 is not zero, the last group of each row
    holds the K mod 64 remaining inputs (columns 64 (G - 1) .. K - 1,
    G = ceil(K / 64)), with its own scale and offset by the same rules.
"""
from __future__ import annotations

from typing import Dict, List, Tuple

import numpy as np

GROUP = 64
QMAX = 255
PREFIX_LINEARS = ("wq", "wk", "wv", "wo", "wg", "wu", "wd")
EXPERT_LINEARS = PREFIX_LINEARS


def _bf16_rne(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even), as float32."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def group_bounds(K: int) -> List[Tuple[int, int]]:
    """Column ranges of the groups of a K-wide row: runs of 64, the last one
    holding the K mod 64 remaining inputs when that is not zero (reading 29)."""
    return [(k0, min(k0 + GROUP, K)) for k0 in range(0, K, GROUP)]


def quantize_affine8(w: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """[N, K] weights (bf16 values) -> codes uint8 [N, K], alpha and beta
    float32 [N, G] holding bf16 values, G = ceil(K / 64) (readings 23, 29)."""
    w = np.asarray(w, np.float32)
    N, K = w.shape
    if K < 1:
        raise ValueError("empty input width")
    bounds = group_bounds(K)
    q = np.zeros((N, K), np.uint8)
    alpha = np.zeros((N, len(bounds)), np.float32)
    beta = np.zeros((N, len(bounds)), np.float32)
    for g, (k0, k1) in enumerate(bounds):
        grp = w[:, k0:k1]
        lo = grp.min(axis=1)
        hi = grp.max(axis=1)
        a = _bf16_rne((hi - lo) / np.float32(QMAX))
        safe = np.where(a > 0, a, np.float32(1)).astype(np.float32)
        t = np.rint((grp - lo[:, None]) / safe[:, None])
        codes = np.clip(t, 0, QMAX)
        q[:, k0:k1] = np.where(a[:, None] > 0, codes, 0).astype(np.uint8)
        alpha[:, g] = a
        beta[:, g] = lo
    return q, alpha, beta


def dequantize_affine8(q: np.ndarray, alpha: np.ndarray, beta: np.ndarray) -> np.ndarray:
    """w^ = bf16(fp32(alpha q + beta)) as float64 values (reading 24), group by group."""
    N, K = q.shape
    out = np.zeros((N, K), np.float64)
    for g, (k0, k1) in enumerate(group_bounds(K)):
        a = np.asarray(alpha, np.float32)[:, g:g + 1]
        b = np.asarray(beta, np.float32)[:, g:g + 1]
        v = a * np.asarray(q[:, k0:k1], np.float32) + b
        out[:, k0:k1] = _bf16_rne(v.astype(np.float32)).astype(np.float64)
    return out


def prefix_matrix_names(p_layers: int) -> List[str]:
    """The matrices the vlm-8bit preset quantises (reading 22)."""
    return [f"p{l}.{m}" for l in range(p_layers) for m in PREFIX_LINEARS]


def quantize_prefix(W: Dict[str, np.ndarray], p_layers: int) -> Dict[str, np.ndarray]:
    """The weights of the vlm-8bit model: the prefix LM's linear matrices
    replaced by their dequantised values, every other tensor unchanged."""
    out = dict(W)
    for name in prefix_matrix_names(p_layers):
        out[name] = dequantize_affine8(*quantize_affine8(W[name]))
    return out


def expert_matrix_names(e_layers: int) -> List[str]:
    """The matrices the expert preset quantises (reading 29)."""
    return [f"e{l}.{m}" for l in range(e_layers) for m in EXPERT_LINEARS]


def quantize_expert(W: Dict[str, np.ndarray], e_layers: int) -> Dict[str, np.ndarray]:
    """The weights of the int8-expert model: the expert layers' linear matrices
    replaced by their dequantised values, every other tensor unchanged."""
    out = dict(W)
    for name in expert_matrix_names(e_layers):
        out[name] = dequantize_affine8(*quantize_affine8(W[name]))
    return out
