"""Shared test helpers: cached workloads, oracle runs and comparison metrics."""
from __future__ import annotations

import functools

import numpy as np

import synth

# Parity gates (the statement of the path: bf16 storage, fp32 accumulation)
KV_REL_L2 = 5e-3       # per layer, valid positions
CHUNK_MAX_ABS = 2e-2   # final chunk
CHUNK_REL_L2 = 1e-2


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))


@functools.lru_cache(maxsize=2)
def weights(wl_name: str, random_affine: bool = False):
    """(shape, bf16 weight bits dict, flat blob) of a workload's model."""
    wl = synth.WORKLOADS[wl_name]
    s = wl.model
    wb = synth.gen_weights(s, wl.seed, random_affine=random_affine)
    return s, wb, synth.pack_blob(s, wb)


@functools.lru_cache(maxsize=2)
def oracle_weights(wl_name: str, random_affine: bool = False):
    import oracle
    _, wb, _ = weights(wl_name, random_affine)
    return oracle.load_weights(wb)


@functools.lru_cache(maxsize=4)
def inputs(wl_name: str):
    return synth.gen_inputs(synth.WORKLOADS[wl_name])


def oracle_query(wl_name: str, b: int, random_affine: bool = False, n_steps=None):
    """Oracle K/V, per-step trace and chunk for query b of a workload."""
    import oracle
    wl = synth.WORKLOADS[wl_name]
    s = wl.model
    W = oracle_weights(wl_name, random_affine)
    inp = inputs(wl_name)
    n = wl.n_steps if n_steps is None else n_steps
    valid = inp["valid"][b]
    if wl.prefix_kind == "kv_given":
        K = synth.bf16_bits_to_f32(inp["k"][:, b]).astype(np.float64)
        V = synth.bf16_bits_to_f32(inp["v"][:, b]).astype(np.float64)
    else:
        emb = synth.bf16_bits_to_f32(inp["embeds"][b]).astype(np.float64)
        K, V = oracle.prefill(W, s, emb, valid)
    vs, xs, x = oracle.denoise(W, s, K, V, valid, inp["noise"][b].astype(np.float64), n)
    return K, V, vs, xs, x
