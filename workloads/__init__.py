"""Seeded synthetic inputs for the Walsh-Hadamard adapter (WHA) layer.

This package is shared by the tests, the bench and the CPU oracle's callers.
It holds no arithmetic of the adapter itself (no Hadamard transform, no sparse
product, no AdaAlloc): only random tensors of the right shapes and value
distributions, the bf16 rounding used to store them, a round-to-nearest group
quantizer that manufactures the frozen quantized base weight W_Q together with
its error dW_Q = W0 - W_Q (the pages start from an already-quantized model,
see "QWHA" on papernotes.org, section 整体框架), and random sparsity patterns
for edge-case tests.
"""

from .synth import (  # noqa: F401
    CONFIGS,
    LayerSpec,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    layer_inputs,
    pack_codes,
    quantize_rtn,
    random_pattern,
    rank_rows,
    rng_for,
)
