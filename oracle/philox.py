"""Philox4x32-10 and Box–Muller Gaussian noise — TEST INFRASTRUCTURE ONLY.

The pages say only that the denoise starts from Gaussian noise at t = 1
("noeira docs, SmolVLA" §Architecture). Reading 15: the noise of
``svla_sample`` is Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
numbers: as easy as 1, 2, 3", SC'11) keyed by the 64-bit seed, with counter
(block, query, 0, 0), followed by Box–Muller. This is an independent
restatement of that published generator; the CUDA library has its own.

Element e of query b's [H, A] noise (row-major) is lane e % 4 of counter block
n = e // 4. The two pairs (r0, r1) and (r2, r3) of a block each give two
normals: u1 = ((r_a >> 8) + 1) / 2^24 in (0, 1], u2 = (r_b >> 8) / 2^24 in
[0, 1), rho = sqrt(-2 ln u1), z_a = rho cos(2 pi u2), z_b = rho sin(2 pi u2).
"""
from __future__ import annotations

import numpy as np

# Philox4x32 round multipliers and Weyl key increments (Salmon et al., SC'11)
_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = 0x9E3779B9
_W1 = 0xBB67AE85
_MASK = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key):
    """Apply 10 Philox4x32 rounds. ctr: 4 arrays of uint32 values, key: 2 ints."""
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _MASK for c in ctr)
    k0, k1 = int(key[0]) & 0xFFFFFFFF, int(key[1]) & 0xFFFFFFFF
    for rnd in range(10):
        p0 = _M0 * c0                      # 32 x 32 -> 64-bit products
        p1 = _M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK
        c0, c1, c2, c3 = (hi1 ^ c1 ^ np.uint64(k0), lo1,
                          hi0 ^ c3 ^ np.uint64(k1), lo0)
        if rnd < 9:
            k0 = (k0 + _W0) & 0xFFFFFFFF
            k1 = (k1 + _W1) & 0xFFFFFFFF
    return tuple(c.astype(np.uint32) for c in (c0, c1, c2, c3))


def _box_muller(ra, rb):
    u1 = ((ra.astype(np.float64) // 256) + 1.0) / 16777216.0
    u2 = (rb.astype(np.float64) // 256) / 16777216.0
    rho = np.sqrt(-2.0 * np.log(u1))
    return rho * np.cos(2.0 * np.pi * u2), rho * np.sin(2.0 * np.pi * u2)


def gaussian_noise(seed: int, B: int, H: int, A: int) -> np.ndarray:
    """Reading 15: the [B, H, A] float64 noise that ``svla_sample`` draws."""
    n_el = H * A
    n_blk = (n_el + 3) // 4
    key = (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    out = np.empty((B, n_blk * 4))
    blk = np.arange(n_blk, dtype=np.uint64)
    zero = np.zeros(n_blk, dtype=np.uint64)
    for b in range(B):
        r0, r1, r2, r3 = philox4x32_10((blk, zero + np.uint64(b), zero, zero), key)
        z0, z1 = _box_muller(r0, r1)
        z2, z3 = _box_muller(r2, r3)
        out[b] = np.stack([z0, z1, z2, z3], axis=1).reshape(-1)
    return out[:, :n_el].reshape(B, H, A)
