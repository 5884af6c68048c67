"""Python face of libsvla: argument marshalling over the C ABI, nothing else.

Every step of the path runs in the library's CUDA kernels; torch is used only
to own device memory and to name the current CUDA stream.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import _abi

__all__ = ["SmolVLA", "config_from_shape"]


def config_from_shape(shape, max_batch: int, max_prefix: int, max_chunk: int) -> _abi.SvlaConfig:
    """Build an svla_config from any object with the model-shape attributes."""
    c = _abi.SvlaConfig()
    for name, _ in _abi.SvlaConfig._fields_:
        if name in ("max_batch", "max_prefix", "max_chunk"):
            continue
        setattr(c, name, getattr(shape, name))
    c.max_batch, c.max_prefix, c.max_chunk = max_batch, max_prefix, max_chunk
    return c


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors passed to libsvla must be contiguous CUDA tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class SmolVLA:
    """One svla_handle: weights on one GPU plus the workspace for the limits given.

    ``blob`` is the flat bf16 weight blob in manifest order, as a numpy uint16
    array, a torch uint16/bfloat16 tensor (host or CUDA), or raw bytes.
    ``prefix_int8`` builds the weight-only int8 copy of the prefix LM's
    projections (the vlm-8bit preset) and selects it for the prefill;
    ``expert_int8`` builds the int8 copy of the expert's projections and
    selects it for the denoise; ``train`` allocates the workspace of
    ``train_step``.
    """

    def __init__(self, shape, blob, max_batch: int, max_prefix: int, max_chunk: int,
                 device: int = 0, prefix_int8: bool = False, train: bool = False, expert_int8: bool = False):
        self.lib = _abi.load()
        self.cfg = config_from_shape(shape, max_batch, max_prefix, max_chunk)
        self.action_dim = shape.action_dim
        self.device = device
        if isinstance(blob, torch.Tensor):
            t = blob.contiguous()
            ptr, nbytes = t.data_ptr(), t.numel() * t.element_size()
            self._blob_keep = t
        else:
            import numpy as np
            arr = np.ascontiguousarray(blob)
            ptr, nbytes = arr.ctypes.data, arr.nbytes
            self._blob_keep = arr
        h = ctypes.c_void_p()
        flags = (_abi.CREATE_PREFIX_INT8 if prefix_int8 else 0) | (_abi.CREATE_TRAIN if train else 0) | \
            (_abi.CREATE_EXPERT_INT8 if expert_int8 else 0)
        st = self.lib.svla_create_ex(ctypes.byref(self.cfg), ctypes.c_void_p(ptr), nbytes, device, flags,
                                     ctypes.byref(h))
        self._blob_keep = None
        _abi.check(st, None)
        self.h = h

    def close(self) -> None:
        if getattr(self, "h", None):
            self.lib.svla_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------
    def kv_cache_bytes(self, B: int, L: int) -> int:
        return int(self.lib.svla_kv_cache_bytes(self.h, B, L))

    def new_kv_cache(self, B: int, L: int) -> torch.Tensor:
        """A K/V cache buffer: bf16, [2, p_layers, B, L, p_kv_heads * head_dim]."""
        c = self.cfg
        return torch.empty((2, c.p_layers, B, L, c.p_kv_heads * c.head_dim), dtype=torch.bfloat16,
                           device=f"cuda:{self.device}")

    def prefill(self, embeds: torch.Tensor, pad_mask: torch.Tensor,
                kv_cache: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        B, L = pad_mask.shape
        if kv_cache is None:
            kv_cache = self.new_kv_cache(B, L)
        st = self.lib.svla_prefill(self.h, _ptr(embeds), _ptr(pad_mask), B, L, _ptr(kv_cache), _stream(stream))
        _abi.check(st, self.h)
        return kv_cache

    def denoise(self, kv_cache: torch.Tensor, pad_mask: torch.Tensor, noise: torch.Tensor, n_steps: int,
                actions: Optional[torch.Tensor] = None, trace: bool = False,
                stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
        B, H, A = noise.shape
        L = pad_mask.shape[1]
        if actions is None:
            actions = torch.empty_like(noise)
        tr = None
        if trace:
            tr = torch.empty((n_steps, 2, B, H, A), dtype=torch.float32, device=noise.device)
        st = self.lib.svla_denoise(self.h, _ptr(kv_cache), _ptr(pad_mask), B, L, _ptr(noise), H, n_steps,
                                   _ptr(actions), _ptr(tr), _stream(stream))
        _abi.check(st, self.h)
        return actions, tr

    def denoise_prefix(self, kv_cache: torch.Tensor, pad_mask: torch.Tensor, noise: torch.Tensor, n_steps: int,
                       prefix: torch.Tensor, actions: Optional[torch.Tensor] = None, trace: bool = False,
                       stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
        """Denoise with the first prefix.shape[1] actions of each query's chunk
        overwritten along the flow path of ``prefix`` ([B, d, A] fp32)."""
        B, H, A = noise.shape
        L = pad_mask.shape[1]
        d = prefix.shape[1]
        if actions is None:
            actions = torch.empty_like(noise)
        tr = None
        if trace:
            tr = torch.empty((n_steps, 2, B, H, A), dtype=torch.float32, device=noise.device)
        st = self.lib.svla_denoise_prefix(self.h, _ptr(kv_cache), _ptr(pad_mask), B, L, _ptr(noise), H, n_steps,
                                          _ptr(prefix), d, _ptr(actions), _ptr(tr), _stream(stream))
        _abi.check(st, self.h)
        return actions, tr

    def sample(self, embeds: torch.Tensor, pad_mask: torch.Tensor, seed: int, H: int, n_steps: int,
               kv_cache: Optional[torch.Tensor] = None, return_noise: bool = False, stream=None):
        B, L = pad_mask.shape
        if kv_cache is None:
            kv_cache = self.new_kv_cache(B, L)
        actions = torch.empty((B, H, self.action_dim), dtype=torch.float32, device=embeds.device)
        noise = torch.empty_like(actions) if return_noise else None
        st = self.lib.svla_sample(self.h, _ptr(embeds), _ptr(pad_mask), B, L, seed, H, n_steps,
                                  _ptr(kv_cache), _ptr(noise), _ptr(actions), _stream(stream))
        _abi.check(st, self.h)
        return (actions, kv_cache, noise) if return_noise else (actions, kv_cache)

    def set_assembly(self, blob, vis_width: int, grid: int, shuffle: int, state_dim: int, max_images: int) -> None:
        """Connector + state-projection weights (bf16 blob: W_c | W_s | b_s)."""
        import numpy as np
        if isinstance(blob, torch.Tensor):
            t = blob.contiguous()
            ptr, nbytes, keep = t.data_ptr(), t.numel() * t.element_size(), t
        else:
            keep = np.ascontiguousarray(blob)
            ptr, nbytes = keep.ctypes.data, keep.nbytes
        st = self.lib.svla_set_assembly(self.h, ctypes.c_void_p(ptr), nbytes, vis_width, grid, shuffle, state_dim,
                                        max_images)
        del keep
        _abi.check(st, self.h)
        self.asm = (grid, shuffle)

    def assemble_prefix(self, vis: torch.Tensor, text: torch.Tensor, text_valid: torch.Tensor, state: torch.Tensor,
                        stream=None):
        """vis bf16 [B, n_img, grid^2, C], text bf16 [B, T, p_width], text_valid u8 [B, T],
        state f32 [B, S] -> (embeds bf16 [B, L, p_width], pad u8 [B, L])."""
        B, n_img = vis.shape[0], vis.shape[1]
        T = text.shape[1]
        grid, r = self.asm
        L = n_img * (grid // r) ** 2 + T + 1
        embeds = torch.empty((B, L, self.cfg.p_width), dtype=torch.bfloat16, device=vis.device)
        pad = torch.empty((B, L), dtype=torch.uint8, device=vis.device)
        st = self.lib.svla_assemble_prefix(self.h, _ptr(vis), _ptr(text) if T else None,
                                           _ptr(text_valid) if T else None, _ptr(state), B, n_img, T,
                                           _ptr(embeds), _ptr(pad), _stream(stream))
        _abi.check(st, self.h)
        return embeds, pad

    def set_denoise_path(self, path: int) -> None:
        """_abi.DENOISE_AUTO (default), DENOISE_GRAPH or DENOISE_FUSED."""
        _abi.check(self.lib.svla_set_denoise_path(self.h, path), self.h)

    def train_step(self, kv_cache: torch.Tensor, pad_mask: torch.Tensor, actions: torch.Tensor,
                   noise: torch.Tensor, t: torch.Tensor, grads: Optional[torch.Tensor] = None, stream=None):
        """One training step of the expert: (loss [1] float32, gradients float32 in
        manifest order from the first expert tensor), both on the device."""
        B, H, _ = actions.shape
        L = pad_mask.shape[1]
        n = int(self.lib.svla_train_grad_elems(self.h))
        if grads is None:
            grads = torch.empty(n, dtype=torch.float32, device=actions.device)
        loss = torch.empty(1, dtype=torch.float32, device=actions.device)
        st = self.lib.svla_train_step(self.h, _ptr(kv_cache), _ptr(pad_mask), B, L, _ptr(actions), _ptr(noise),
                                      _ptr(t), H, _ptr(loss), _ptr(grads), _stream(stream))
        _abi.check(st, self.h)
        return loss, grads

    def set_prefix_weights(self, bits: int) -> None:
        """16 = dense bf16 prefix weights, 8 = the int8 copy (needs prefix_int8=True)."""
        _abi.check(self.lib.svla_set_prefix_weights(self.h, bits), self.h)

    @property
    def prefix_weights(self) -> int:
        return int(self.lib.svla_prefix_weights(self.h))

    def set_expert_weights(self, bits: int) -> None:
        """16 = dense bf16 expert weights, 8 = the int8 copy (needs expert_int8=True)."""
        _abi.check(self.lib.svla_set_expert_weights(self.h, bits), self.h)

    @property
    def expert_weights(self) -> int:
        return int(self.lib.svla_expert_weights(self.h))

    def fused_supported(self, B: int, H: int) -> bool:
        return bool(self.lib.svla_denoise_fused_supported(self.h, B, H))

    def device_status(self, stream=None) -> int:
        """Synchronise the stream; return (and clear) the device-side status."""
        return int(self.lib.svla_device_status(self.h, _stream(stream)))


# ----------------------------------------------------------------------
# single kernels (svla_op_*), for callers that compose their own schedule
# ----------------------------------------------------------------------
_EPI = {"f32": 0, "bf16": 1, "add_f32": 2, "silu_bf16": 3}


def op_gemm(epilogue: str, A: torch.Tensor, W: torch.Tensor, C: torch.Tensor, bias: Optional[torch.Tensor] = None,
            splits: int = 0, status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """svla_op_gemm: C = A W^T (+ bias) with the epilogue 'f32', 'bf16', 'add_f32' or 'silu_bf16'."""
    lib = _abi.load()
    M, K = A.shape
    N = W.shape[0]
    ws_bytes = int(lib.svla_op_gemm_workspace_bytes(M, N, K, splits))
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=A.device) if ws_bytes else None
    st = lib.svla_op_gemm(_EPI[epilogue], _ptr(A), A.stride(0), _ptr(W), W.stride(0), M, N, K, _ptr(C), C.stride(0),
                          _ptr(bias), splits, _ptr(ws), ws_bytes, _ptr(status), _stream(stream))
    _abi.check(st)
    return C


def op_quantize_affine8(W: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """svla_op_quantize_affine8: bf16 W [N, K] -> (codes uint8 [N, K], (alpha, beta) bf16 [G, N, 2]) with
    G = ceil(K / 64) groups (the last one holds the K mod 64 remaining inputs when K % 64 != 0)."""
    lib = _abi.load()
    N, K = W.shape
    q = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    ab = torch.empty(((K + 63) // 64, N, 2), dtype=torch.bfloat16, device=W.device)
    _abi.check(lib.svla_op_quantize_affine8(_ptr(W), W.stride(0), N, K, _ptr(q), q.stride(0), _ptr(ab),
                                            _stream(stream)))
    return q, ab


def op_gemm_w8(epilogue: str, A: torch.Tensor, q: torch.Tensor, ab: torch.Tensor, C: torch.Tensor,
               gain: Optional[torch.Tensor] = None, bias: Optional[torch.Tensor] = None, splits: int = 0,
               status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """svla_op_gemm_w8: C = A W^T with W = bf16(bf16(alpha q + beta) * gain) from op_quantize_affine8's output."""
    lib = _abi.load()
    M, K = A.shape
    N = q.shape[0]
    st = lib.svla_op_gemm_w8(_EPI[epilogue], _ptr(A), A.stride(0), _ptr(q), q.stride(0), _ptr(ab), _ptr(gain), M, N,
                             K, _ptr(C), C.stride(0), _ptr(bias), splits, _ptr(status), _stream(stream))
    _abi.check(st)
    return C


def op_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, n_q: int, n_kv: int,
                 head_dim: int, key_valid: Optional[torch.Tensor] = None, causal: bool = False,
                 stream=None) -> torch.Tensor:
    """svla_op_attention on [B, Lq, n_q * hd] queries and [B, Lk, n_kv * hd] keys / values."""
    lib = _abi.load()
    B, Lq, _ = q.shape
    Lk = k.shape[1]
    st = lib.svla_op_attention(_ptr(q), q.stride(1), _ptr(k), _ptr(v), k.stride(1), _ptr(key_valid), B, n_q, n_kv,
                               head_dim, Lq, Lk, int(causal), _ptr(out), out.stride(1), _stream(stream))
    _abi.check(st)
    return out


def op_rmsnorm(x: torch.Tensor, g: torch.Tensor, y: torch.Tensor, eps: float = 1e-5, stream=None) -> torch.Tensor:
    """svla_op_rmsnorm: y (bf16) = x (f32) / sqrt(mean(x^2) + eps) * g."""
    lib = _abi.load()
    M, D = x.shape
    _abi.check(lib.svla_op_rmsnorm(_ptr(x), _ptr(g), M, D, eps, _ptr(y), _stream(stream)))
    return y
