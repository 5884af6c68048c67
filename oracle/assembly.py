"""Plain float64 definition of the prefix assembly upstream of the prefill.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library must
never import this module.

"noeira docs, SmolVLA" §Architecture: the vision tower (SigLIP, width 768,
512x512 input in 16x16 patches, so a 32x32 grid of patch features per image)
feeds a connector — pixel shuffle x4, 64 tokens per image, then a linear
projection to the LM width 960 — and a query's prefix is the two camera images,
the tokenised instruction and one state token. "Paper vs hardware 11: SmolVLA"
§What the paper claims: the state is projected to one token of the VLM prefix.
The CSDN precision post §8 (mixed-precision table): the state projection runs
in fp32, the connector in bf16.

Readings where the pages are silent (numbered after those of ``model.py``):

18. Pixel shuffle x r is a space-to-depth of the g x g patch grid: output token
    (i, j) of the (g/r) x (g/r) grid (row-major token index i (g/r) + j) is the
    concatenation, in row-major (a, b) order, of the r x r block of patches
    (r i + a, r j + b), each C channels: channel (a r + b) C + c of the token
    is channel c of patch (r i + a, r j + b).
19. The connector is a linear map without bias (like the LM's projections).
20. The state token is W_s s + b_s (a linear layer with bias), computed in
    float (fp32 on the GPU), then stored as a bf16 prefix embedding.
21. Prefix order: the images' tokens in camera order, then the text tokens
    (with their validity), then the state token; image and state tokens are
    valid.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

F64 = np.float64


def pixel_shuffle(feats: np.ndarray, grid: int, r: int) -> np.ndarray:
    """[grid*grid, C] patch features (row-major patch index) -> [(grid/r)^2, r*r*C] (reading 18)."""
    n, C = feats.shape
    assert n == grid * grid and grid % r == 0
    g2 = grid // r
    x = np.asarray(feats, F64).reshape(g2, r, g2, r, C)      # (i, a, j, b, c)
    x = x.transpose(0, 2, 1, 3, 4)                           # (i, j, a, b, c)
    return x.reshape(g2 * g2, r * r * C)


def connector(Wc: np.ndarray, feats: np.ndarray, grid: int, r: int) -> np.ndarray:
    """One image: pixel shuffle then the linear projection (reading 19)."""
    return pixel_shuffle(feats, grid, r) @ np.asarray(Wc, F64).T


def state_token(Ws: np.ndarray, bs: np.ndarray, state: np.ndarray) -> np.ndarray:
    """W_s s + b_s (reading 20)."""
    return np.asarray(Ws, F64) @ np.asarray(state, F64) + np.asarray(bs, F64)


def assemble_prefix(Wc, Ws, bs, vis_feats: np.ndarray, text_embeds: np.ndarray, text_valid: np.ndarray,
                    state: np.ndarray, grid: int, r: int) -> Tuple[np.ndarray, np.ndarray]:
    """One query: [n_img, grid*grid, C] features, [T, D] text embeddings with
    [T] validity, [S] state -> ([L, D] prefix embeddings in float64, [L] valid),
    L = n_img (grid/r)^2 + T + 1 (reading 21)."""
    parts = [connector(Wc, f, grid, r) for f in vis_feats]
    parts.append(np.asarray(text_embeds, F64))
    parts.append(state_token(Ws, bs, state)[None, :])
    n_vis = sum(p.shape[0] for p in parts[:-2])
    valid = np.concatenate([np.ones(n_vis, np.uint8), np.asarray(text_valid, np.uint8), np.ones(1, np.uint8)])
    return np.concatenate(parts, axis=0), valid
