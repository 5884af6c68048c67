"""Seeded synthetic inputs for SmolVLA action-chunk generation.

This module only *produces data*: model shapes, the flat weight-blob order,
seeded weights rounded to bf16, prefix embeddings, pad masks, noise and (for
the denoise-only workload) ready-made K/V caches. It holds none of the
method's arithmetic, so both the CPU oracle and the CUDA library can be fed
from it without sharing any computation.

Sources for the shapes (page titles and sections):
  * "noeira docs, SmolVLA" §Architecture: SmolLM2 prefix LM of 16 layers,
    width 960, 15 query heads over 5 KV heads of dim 64; action expert of
    16 layers, width 720; 10 Euler steps; chunk 50; 32-wide padded actions.
  * "Paper vs hardware 11: SmolVLA" §claims: 2 cameras x 64 visual tokens,
    one state token, ~100M action expert.
  * The remaining sizes (SwiGLU widths, expert projections, time MLP) are the
    SmolVLA-shaped workload statement that accompanies those pages.

Weights are N(0, 0.02) rounded to bf16 with round-to-nearest-even; RMSNorm
gains are 1 and biases 0 unless ``random_affine`` is set (tests use that to
exercise the gain/bias paths).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Dict, List, Tuple

import numpy as np

__all__ = [
    "ModelShape", "Workload", "SHAPES", "WORKLOADS", "manifest", "param_count",
    "gen_weights", "pack_blob", "gen_inputs", "f32_to_bf16_bits",
    "bf16_bits_to_f32", "pack_kv_cache", "kv_cache_elems", "AssemblyShape", "ASSEMBLY_SHAPES",
    "assembly_manifest", "gen_assembly_weights", "pack_assembly_blob", "gen_assembly_inputs",
]


# --------------------------------------------------------------------------
# bf16 storage format (IEEE binary32 with the low 16 bits dropped)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Expand bf16 bits (uint16) exactly to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# Shapes
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class ModelShape:
    p_layers: int
    p_width: int
    p_heads: int
    p_kv_heads: int
    head_dim: int
    p_ffn: int
    e_layers: int
    e_width: int
    e_heads: int
    e_kv_heads: int
    e_ffn: int
    action_dim: int
    rope_base: float = 10000.0
    rms_eps: float = 1e-5
    t_min_period: float = 4e-3
    t_max_period: float = 4.0

    @property
    def p_kv_width(self) -> int:
        return self.p_kv_heads * self.head_dim

    @property
    def e_q_width(self) -> int:
        return self.e_heads * self.head_dim

    @property
    def e_kv_width(self) -> int:
        return self.e_kv_heads * self.head_dim

    def replace(self, **kw) -> "ModelShape":
        return dataclasses.replace(self, **kw)


SHAPES: Dict[str, ModelShape] = {
    # 2-layer shape check: prefix width 128 (4q/2kv x 32, ffn 256); expert
    # width 96 (4q/2kv x 32, ffn 192), cross K/V projection 64 -> 64.
    "tiny": ModelShape(p_layers=2, p_width=128, p_heads=4, p_kv_heads=2, head_dim=32,
                       p_ffn=256, e_layers=2, e_width=96, e_heads=4, e_kv_heads=2,
                       e_ffn=192, action_dim=8),
    # SmolVLA: SmolLM2 first 16 layers + 16-layer width-720 expert.
    "smolvla": ModelShape(p_layers=16, p_width=960, p_heads=15, p_kv_heads=5, head_dim=64,
                          p_ffn=2560, e_layers=16, e_width=720, e_heads=15, e_kv_heads=5,
                          e_ffn=2048, action_dim=32),
}


def manifest(s: ModelShape) -> List[Tuple[str, Tuple[int, ...]]]:
    """Blob order: per prefix layer, per expert layer, then the heads.

    Every entry is bf16; matrices are [out, in] row-major (nn.Linear storage).
    Odd expert layers cross-attend, so their k/v projections read the cached
    prefix K/V (width p_kv_heads*head_dim) instead of the expert residual.
    """
    m: List[Tuple[str, Tuple[int, ...]]] = []
    D, hd = s.p_width, s.head_dim
    for l in range(s.p_layers):
        m += [(f"p{l}.in_norm", (D,)),
              (f"p{l}.wq", (s.p_heads * hd, D)),
              (f"p{l}.wk", (s.p_kv_heads * hd, D)),
              (f"p{l}.wv", (s.p_kv_heads * hd, D)),
              (f"p{l}.wo", (D, s.p_heads * hd)),
              (f"p{l}.post_norm", (D,)),
              (f"p{l}.wg", (s.p_ffn, D)),
              (f"p{l}.wu", (s.p_ffn, D)),
              (f"p{l}.wd", (D, s.p_ffn))]
    E = s.e_width
    for l in range(s.e_layers):
        kv_in = E if l % 2 == 0 else s.p_kv_width
        m += [(f"e{l}.in_norm", (E,)),
              (f"e{l}.wq", (s.e_q_width, E)),
              (f"e{l}.wk", (s.e_kv_width, kv_in)),
              (f"e{l}.wv", (s.e_kv_width, kv_in)),
              (f"e{l}.wo", (E, s.e_q_width)),
              (f"e{l}.post_norm", (E,)),
              (f"e{l}.wg", (s.e_ffn, E)),
              (f"e{l}.wu", (s.e_ffn, E)),
              (f"e{l}.wd", (E, s.e_ffn))]
    A = s.action_dim
    m += [("final_norm", (E,)),
          ("w_in", (E, A)), ("b_in", (E,)),
          ("w_t1", (E, 2 * E)), ("b_t1", (E,)),
          ("w_t2", (E, E)), ("b_t2", (E,)),
          ("w_out", (A, E)), ("b_out", (A,))]
    return m


def param_count(s: ModelShape, part: str) -> int:
    """Number of parameters of the prefix LM ('prefix') or the expert + heads ('expert')."""
    tot = 0
    for name, shp in manifest(s):
        if (part == "prefix") == name.startswith("p"):
            tot += int(np.prod(shp))
    return tot


def gen_weights(s: ModelShape, seed: int, std: float = 0.02,
                random_affine: bool = False) -> Dict[str, np.ndarray]:
    """Seeded weights as bf16 bits (uint16 arrays), in manifest order.

    Norm gains are 1 and biases 0, unless ``random_affine``: then gains are
    1 + N(0, 0.1) and biases N(0, 0.02) (still bf16-rounded).
    """
    rng = np.random.default_rng([seed, 0xB10B])
    out: Dict[str, np.ndarray] = {}
    for name, shp in manifest(s):
        is_norm = name.endswith("norm")
        is_bias = name.split(".")[-1].startswith("b_")
        if is_norm:
            v = (np.ones(shp, np.float32) if not random_affine
                 else 1.0 + 0.1 * rng.standard_normal(shp, dtype=np.float32))
        elif is_bias:
            v = (np.zeros(shp, np.float32) if not random_affine
                 else std * rng.standard_normal(shp, dtype=np.float32))
        else:
            v = rng.standard_normal(shp, dtype=np.float32)
            v *= np.float32(std)
        out[name] = f32_to_bf16_bits(v)
    return out


def pack_blob(s: ModelShape, w: Dict[str, np.ndarray]) -> np.ndarray:
    """Concatenate the weights (bf16 bits) in manifest order into one flat uint16 array."""
    parts = []
    for name, shp in manifest(s):
        a = np.asarray(w[name], dtype=np.uint16)
        if a.shape != tuple(shp):
            raise ValueError(f"{name}: shape {a.shape} != {shp}")
        parts.append(a.reshape(-1))
    return np.concatenate(parts)


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    name: str
    shape: str
    seed: int
    B: int
    L: int
    H: int
    n_steps: int
    prefix_kind: str          # "tail_pad", "none", "text_pad", "kv_given"
    visual: int = 0           # visual tokens (cameras x 64)
    text_slots: int = 0       # text slots (right-padded)
    tail_pad: int = 0         # fixed tail pad (tiny shape check)

    @property
    def model(self) -> ModelShape:
        return SHAPES[self.shape]


WORKLOADS: Dict[str, Workload] = {
    # 24 prefix embeddings, the last 4 masked; chunk 8, 3 Euler steps.
    "tiny": Workload("tiny", "tiny", 0, B=1, L=24, H=8, n_steps=3,
                     prefix_kind="tail_pad", tail_pad=4),
    # 2 x 64 visual + 48 text + 1 state = 177, no padding; chunk 50, 10 steps.
    "smolvla_b1": Workload("smolvla_b1", "smolvla", 1, B=1, L=177, H=50, n_steps=10,
                           prefix_kind="none", visual=128, text_slots=48),
    # 32 independent queries; text length U{16..48} right-padded to 48, so the
    # pads sit between the text and the state token.
    "smolvla_b32": Workload("smolvla_b32", "smolvla", 2, B=32, L=177, H=50, n_steps=10,
                            prefix_kind="text_pad", visual=128, text_slots=48),
    # 3 x 64 visual + 128 text + 1 state = 321; chunk 100.
    "long_prefix_b8": Workload("long_prefix_b8", "smolvla", 3, B=8, L=321, H=100, n_steps=10,
                               prefix_kind="none", visual=192, text_slots=128),
    # Denoise only: given K/V caches ~N(0,1), 0..31 masked tail positions per query.
    "denoise_b256": Workload("denoise_b256", "smolvla", 4, B=256, L=177, H=50, n_steps=10,
                             prefix_kind="kv_given"),
}


def _valid_mask(wl: Workload, rng: np.random.Generator) -> np.ndarray:
    B, L = wl.B, wl.L
    valid = np.ones((B, L), np.uint8)
    if wl.prefix_kind == "tail_pad":
        valid[:, L - wl.tail_pad:] = 0
    elif wl.prefix_kind == "text_pad":
        lens = rng.integers(16, wl.text_slots + 1, size=B)      # U{16..48}
        for b in range(B):
            valid[b, wl.visual + lens[b]: wl.visual + wl.text_slots] = 0
    elif wl.prefix_kind == "kv_given":
        pads = rng.integers(0, 32, size=B)                       # U{0..31}
        for b in range(B):
            if pads[b]:
                valid[b, L - pads[b]:] = 0
    return valid


def kv_cache_elems(s: ModelShape, B: int, L: int) -> int:
    """bf16 elements of one K/V cache: K block then V block, each [p_layers][B][L][p_kv_width]."""
    return 2 * s.p_layers * B * L * s.p_kv_width


def pack_kv_cache(k_bits: np.ndarray, v_bits: np.ndarray) -> np.ndarray:
    """Lay K and V (bf16 bits, [layers, B, L, kv_heads, head_dim]) out as the cache buffer."""
    return np.concatenate([np.ascontiguousarray(k_bits).reshape(-1),
                           np.ascontiguousarray(v_bits).reshape(-1)])


def gen_inputs(wl: Workload, B: int | None = None) -> Dict[str, np.ndarray]:
    """Seeded inputs of a workload.

    Returns ``valid`` (uint8 [B, L], 1 = real token), ``noise`` (float32
    [B, H, A]) and either ``embeds`` (bf16 bits [B, L, p_width]) or, for the
    denoise-only workload, ``k``/``v`` (bf16 bits [p_layers, B, L, kv_heads,
    head_dim]). ``B`` may select a prefix of the batch (queries are drawn in
    order, so query i is the same whatever B is).
    """
    s = wl.model
    Bf = wl.B if B is None else B
    rng = np.random.default_rng([wl.seed, 0x1A9])
    valid_full = _valid_mask(wl, rng)
    out: Dict[str, np.ndarray] = {"valid": valid_full[:Bf].copy()}
    # one stream per query, so sub-batches reproduce the full batch exactly
    noises, embeds, ks, vs = [], [], [], []
    for b in range(Bf):
        qr = np.random.default_rng([wl.seed, 0x7E5, b])
        noises.append(qr.standard_normal((wl.H, s.action_dim), dtype=np.float32))
        if wl.prefix_kind == "kv_given":
            shp = (s.p_layers, wl.L, s.p_kv_heads, s.head_dim)
            ks.append(f32_to_bf16_bits(qr.standard_normal(shp, dtype=np.float32)))
            vs.append(f32_to_bf16_bits(qr.standard_normal(shp, dtype=np.float32)))
        else:
            embeds.append(f32_to_bf16_bits(
                qr.standard_normal((wl.L, s.p_width), dtype=np.float32)))
    out["noise"] = np.stack(noises)
    if wl.prefix_kind == "kv_given":
        out["k"] = np.ascontiguousarray(np.stack(ks, axis=1))
        out["v"] = np.ascontiguousarray(np.stack(vs, axis=1))
    else:
        out["embeds"] = np.stack(embeds)
    return out


# --------------------------------------------------------------------------
# Prefix assembly upstream of the prefill: the connector (pixel shuffle of the
# vision tower's patch grid, then a linear map to the LM width) and the state
# projection ("noeira docs, SmolVLA" §Architecture: SigLIP width 768 on a
# 512x512 image in 16x16 patches -> 32 x 32 patches, pixel shuffle x4 -> 64
# tokens per image, linear to 960; "Paper vs hardware 11: SmolVLA" §claims:
# the state projected to one prefix token). The state width 32 matches the
# padded action width.
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class AssemblyShape:
    vis_width: int     # C: channels of a patch feature
    grid: int          # patches per image side
    shuffle: int       # r: pixel-shuffle factor
    state_dim: int     # S
    n_img: int         # cameras per query
    text_len: int      # T: text tokens (padded)

    @property
    def tokens_per_image(self) -> int:
        return (self.grid // self.shuffle) ** 2

    @property
    def conn_in(self) -> int:
        return self.shuffle * self.shuffle * self.vis_width


ASSEMBLY_SHAPES: Dict[str, AssemblyShape] = {
    "tiny": AssemblyShape(vis_width=16, grid=8, shuffle=2, state_dim=8, n_img=2, text_len=6),
    "smolvla": AssemblyShape(vis_width=768, grid=32, shuffle=4, state_dim=32, n_img=2, text_len=48),
}


def assembly_manifest(a: AssemblyShape, width: int) -> List[Tuple[str, Tuple[int, ...]]]:
    """Blob order of the assembly weights: W_c [width, r*r*C], W_s [width, S], b_s [width]."""
    return [("w_conn", (width, a.conn_in)), ("w_state", (width, a.state_dim)), ("b_state", (width,))]


def gen_assembly_weights(a: AssemblyShape, width: int, seed: int, std: float = 0.02) -> Dict[str, np.ndarray]:
    """Seeded assembly weights as bf16 bits (the state bias N(0, std) too, so it is exercised)."""
    rng = np.random.default_rng([seed, 0xA55E])
    return {n: f32_to_bf16_bits(np.float32(std) * rng.standard_normal(shp, dtype=np.float32))
            for n, shp in assembly_manifest(a, width)}


def pack_assembly_blob(a: AssemblyShape, width: int, w: Dict[str, np.ndarray]) -> np.ndarray:
    return np.concatenate([np.asarray(w[n], np.uint16).reshape(-1) for n, _ in assembly_manifest(a, width)])


def gen_assembly_inputs(a: AssemblyShape, width: int, B: int, seed: int) -> Dict[str, np.ndarray]:
    """Seeded inputs of one batch: ``vis`` (bf16 bits [B, n_img, grid^2, C]),
    ``text`` (bf16 bits [B, T, width]), ``text_valid`` (uint8 [B, T], a
    per-query count of leading valid tokens in [1, T]) and ``state`` (float32
    [B, S])."""
    out = {"vis": [], "text": [], "text_valid": [], "state": []}
    for b in range(B):
        qr = np.random.default_rng([seed, 0xA55F, b])
        out["vis"].append(f32_to_bf16_bits(qr.standard_normal((a.n_img, a.grid * a.grid, a.vis_width),
                                                              dtype=np.float32)))
        out["text"].append(f32_to_bf16_bits(qr.standard_normal((a.text_len, width), dtype=np.float32)))
        n = int(qr.integers(1, a.text_len + 1))
        tv = np.zeros(a.text_len, np.uint8)
        tv[:n] = 1
        out["text_valid"].append(tv)
        out["state"].append(qr.standard_normal(a.state_dim, dtype=np.float32))
    return {k: np.stack(v) for k, v in out.items()}
