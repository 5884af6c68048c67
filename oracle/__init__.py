"""CPU oracle for SmolVLA action-chunk generation — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import or run anything in this package. The CUDA library
never calls it, and it shares no code with the CUDA library: both sides are
fed by the seeded generators in ``synth`` and nothing else.

The oracle is plain numpy in float64 (a matmul is the only library primitive
used), written step by step from the pages:

* "noeira docs, SmolVLA" §Architecture — SmolLM2 prefix LM (GQA 15/5 x 64,
  RoPE, SwiGLU, RMSNorm), per-layer K/V cache written once per query, action
  expert whose even layers self-attend and odd layers cross-attend to the
  cached K/V, flow-matching head with Euler steps from Gaussian noise at
  t = 1 toward t = 0, the block attention mask (the prefix cannot see the
  actions), and the flow-matching objective x_t = t*eps + (1-t)*a whose
  target eps - a fixes the sign of the velocity.
* "Paper vs hardware 11: SmolVLA" §claims — causal self-attention over the
  chunk, cross-attention to the VLM's keys/values.
* The CSDN precision post §2 (54 compared tensors: per-layer past K/V and,
  per Euler step, the velocity and the state x).

Every reading taken where the pages are silent is listed, numbered, in
``model.py``'s module docstring.

Parity pins (checked by ``tests/test_oracle_pins.py`` against things other
than the oracle itself): block mask / joint pass, constant velocity, GQA =
MHA with repeated heads, brute-force loops on the tiny shape, RoPE closed
form, L = 1 attention, padding and batch invariance, parameter counts, and
the Philox4x32-10 known-answer vectors. ``assembly.py`` (prefix assembly),
``quant.py`` (the weight-only int8 presets of the prefix and of the expert) and ``train.py`` (the expert's
training step) carry their own pins in ``tests/test_oracle_assembly.py``,
``tests/test_oracle_quant.py`` and ``tests/test_oracle_train.py``. Parity
against the real SmolVLA checkpoint is unpinned: no weights or activation
dumps exist here.
"""
from .model import (  # noqa: F401
    load_weights, rms_norm, rope, attention, silu, prefix_positions, prefill,
    time_embedding, velocity, denoise, denoise_prefix_overwrite, sample, oracle_joint, cross_kv,
)
from .philox import philox4x32_10, gaussian_noise  # noqa: F401
from .assembly import pixel_shuffle, connector, state_token, assemble_prefix  # noqa: F401
from .quant import quantize_affine8, dequantize_affine8, quantize_prefix, quantize_expert  # noqa: F401
from .train import train_step, trainable_names, loss_np  # noqa: F401
