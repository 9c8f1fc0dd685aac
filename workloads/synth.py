"""Seeded synthetic layers for the WHA adapter workloads.

Every tensor is drawn from its own numpy PCG64 stream, keyed by
(seed, workload, layer, tensor, row block), so that any block of token rows can
be regenerated on its own (the parity tests sample rows of the largest
workloads without building the whole activation matrix).

Shapes and value distributions follow the pages' setting (LLaMA-family linear
layers; weights whose quantization error is dominated by a few outliers, see
"QWHA" on papernotes.org, section 切入角度, and gist.science, section 1 item 3;
LoRA r=64 parameter budget, papernotes.org section 损失函数 / 训练策略).
No dataset content is used anywhere: the pages' models and corpora are not
available, and these seeded tensors stand in for them.
"""

from __future__ import annotations

import zlib
from dataclasses import dataclass

import numpy as np

ROW_BLOCK = 256  # token rows per independent random stream


# --------------------------------------------------------------------------
# workload table
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class LayerSpec:
    """One adapted linear layer: W0 is [d_out, d_in], activations are [T, d_in]."""

    name: str
    d_in: int
    d_out: int
    had_block: int  # Hadamard block length n (block-diagonal H when n < d_in)
    T: int  # tokens
    bits: int  # base-weight code width
    group: int  # quantization group length along d_in
    p: int  # adapter nonzeros
    dtype: str  # "f32" or "bf16" storage of W0, X, dY
    w_std: float = 0.02
    w_outlier_frac: float = 0.001
    w_outlier_scale: float = 20.0
    x_outlier_frac: float = 0.01
    x_outlier_scale: float = 20.0
    remainder: str = "fewest"  # "fewest" (pages) or "largest"
    x_stream: str = ""  # layers with the same x_stream read the same X
    min_per_row: int = 2
    w_stream: str = ""  # layers with the same w_stream share W0 (the init sweep over r)


def _llama8b_block(T: int, bits: int, group: int, r: int, dtype: str) -> list[LayerSpec]:
    shapes = [
        ("q", 4096, 4096, 4096, "x_attn"),
        ("k", 4096, 1024, 4096, "x_attn"),
        ("v", 4096, 1024, 4096, "x_attn"),
        ("o", 4096, 4096, 4096, "x_o"),
        ("gate", 4096, 14336, 4096, "x_mlp"),
        ("up", 4096, 14336, 4096, "x_mlp"),
        ("down", 14336, 4096, 2048, "x_down"),
    ]
    return [
        LayerSpec(n, di, do, hb, T, bits, group, r * (di + do), dtype, x_stream=xs)
        for (n, di, do, hb, xs) in shapes
    ]


def _init_sweep() -> list[LayerSpec]:
    out = []
    for r in (16, 64, 128):
        for s in _llama8b_block(0, 2, 64, r, "f32"):
            out.append(
                LayerSpec(
                    f"{s.name}_r{r}", s.d_in, s.d_out, s.had_block, 0, 2, 64, s.p, "f32",
                    remainder="largest", w_stream=s.name,
                )
            )
    return out


CONFIGS: dict[str, list[LayerSpec]] = {
    # 256x256 layer, 64 tokens, fp32, 4-bit g64, p=1024, outliers 0.5% x10,
    # remainder of the budget to the largest-error rows.
    "tiny": [
        LayerSpec(
            "tiny", 256, 256, 256, 64, 4, 64, 1024, "f32",
            w_outlier_frac=0.005, w_outlier_scale=10.0,
            x_outlier_frac=0.0, x_outlier_scale=1.0, remainder="largest",
        )
    ],
    # LLaMA-7B q_proj shape, 16 x 512 tokens, 4-bit g128, p = LoRA r=64 count.
    "q_proj": [LayerSpec("q_proj", 4096, 4096, 4096, 8192, 4, 128, 524288, "bf16")],
    # LLaMA-3-8B MLP: gate/up 4096->14336, down 14336->4096 (7 blocks of 2048).
    "mlp": [
        s for s in _llama8b_block(16384, 3, 128, 64, "bf16") if s.name in ("gate", "up", "down")
    ],
    # AdaAlloc over the seven LLaMA-3-8B linear shapes, 2-bit g64, r in {16,64,128}.
    "init_sweep": _init_sweep(),
    # Whole LLaMA-3-8B-shaped decoder block, 8 x 4096 tokens, 4-bit g128, r=64.
    "block": _llama8b_block(32768, 4, 128, 64, "bf16"),
}


# --------------------------------------------------------------------------
# streams and storage types
# --------------------------------------------------------------------------


def _h(s: str) -> int:
    return zlib.crc32(s.encode())


def rng_for(seed: int, *keys) -> np.random.Generator:
    """An independent PCG64 stream for (seed, *keys); keys are str or int."""
    ent = [int(seed)] + [(_h(k) if isinstance(k, str) else int(k)) for k in keys]
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(ent)))


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# base weight and its round-to-nearest quantization
# --------------------------------------------------------------------------


def _weights(spec: LayerSpec, seed: int, workload: str) -> np.ndarray:
    """W0 [d_out, d_in] as float32 values (bf16-representable for bf16 layers)."""
    key = spec.w_stream or spec.name
    g = rng_for(seed, workload, key, "W0")
    w = g.standard_normal((spec.d_out, spec.d_in), dtype=np.float32) * np.float32(spec.w_std)
    if spec.w_outlier_frac > 0:
        m = rng_for(seed, workload, key, "W0_outliers").random((spec.d_out, spec.d_in)) < spec.w_outlier_frac
        w[m] *= np.float32(spec.w_outlier_scale)
    if spec.dtype == "bf16":
        w = bf16_bits_to_f32(f32_to_bf16_bits(w))
    return w


def quantize_rtn(w: np.ndarray, bits: int, group: int):
    """Asymmetric round-to-nearest group quantization along d_in, in float32.

    Per group of `group` consecutive inputs of one output row:
      s = (max - min) / (2^b - 1)   (s = 1 for a constant group)
      z = clamp(rint(-min / s), 0, 2^b - 1)
      q = clamp(rint(w / s) + z, 0, 2^b - 1)
      W_Q = s * (q - z),   dW_Q = w - W_Q
    rint rounds half to even. The pages quantize with GPTQ+MagR (papernotes.org,
    section 局限与展望); this plain quantizer only manufactures a frozen W_Q and
    its error for the synthetic layers.
    Returns (q codes uint8 [d_out, d_in], scales f32 [d_out, d_in/group],
    zeros uint8 [d_out, d_in/group], W_Q f32, dW_Q f32).
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    d_out, d_in = w.shape
    assert d_in % group == 0
    qmax = np.float32(2**bits - 1)
    wg = w.reshape(d_out, d_in // group, group)
    mn = wg.min(axis=2)
    mx = wg.max(axis=2)
    s = ((mx - mn) / qmax).astype(np.float32)
    s[s == 0] = np.float32(1.0)
    z = np.clip(np.rint(-mn / s), 0, qmax).astype(np.float32)
    q = np.clip(np.rint(wg / s[..., None]) + z[..., None], 0, qmax).astype(np.float32)
    wq = (s[..., None] * (q - z[..., None])).astype(np.float32)
    dwq = (wg - wq).astype(np.float32)
    return (
        q.astype(np.uint8).reshape(d_out, d_in),
        s,
        z.astype(np.uint8),
        wq.reshape(d_out, d_in),
        dwq.reshape(d_out, d_in),
    )


def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    """Pack b-bit codes row by row as a little-endian bit stream.

    Code k of a row occupies bits [b*k, b*k + b) of that row's stream; bit i of
    the stream is bit (i mod 8) of byte i // 8. A row takes d_in*b/8 bytes
    (int4: two codes per byte, low nibble first; int2: four per byte; int3: 128
    codes per 48 bytes).
    """
    d_out, d_in = q.shape
    assert (d_in * bits) % 8 == 0
    bitsarr = ((q[..., None].astype(np.uint8) >> np.arange(bits, dtype=np.uint8)) & 1).astype(np.uint8)
    return np.packbits(bitsarr.reshape(d_out, d_in * bits), axis=1, bitorder="little")


# --------------------------------------------------------------------------
# activations and output gradients
# --------------------------------------------------------------------------


def _x_channels(spec: LayerSpec, seed: int, workload: str) -> np.ndarray:
    cnt = int(round(spec.x_outlier_frac * spec.d_in))
    if cnt == 0:
        return np.zeros(0, dtype=np.int64)
    key = spec.x_stream or spec.name
    return np.sort(rng_for(seed, workload, key, "X_channels").permutation(spec.d_in)[:cnt])


def _rows(spec: LayerSpec, seed: int, workload: str, tensor: str, width: int, rows) -> np.ndarray:
    """float32 values of `tensor` at the given token rows, block-streamed."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, width), dtype=np.float32)
    key = (spec.x_stream or spec.name) if tensor == "X" else spec.name
    blocks = np.unique(rows // ROW_BLOCK)
    for b in blocks:
        g = rng_for(seed, workload, key, tensor, int(b))
        blk = g.standard_normal((ROW_BLOCK, width), dtype=np.float32)
        sel = np.nonzero(rows // ROW_BLOCK == b)[0]
        out[sel] = blk[rows[sel] - b * ROW_BLOCK]
    if tensor == "X":
        ch = _x_channels(spec, seed, workload)
        if ch.size:
            out[:, ch] *= np.float32(spec.x_outlier_scale)
    return out


def layer_inputs(
    spec: LayerSpec,
    seed: int = 0,
    workload: str = "",
    parts=("W", "X", "dY"),
    rows=None,
) -> dict:
    """Inputs of one layer.

    parts: "W" gives W0, the packed codes, scales, zeros, W_Q and dW_Q;
    "X" and "dY" give activations and output gradients for `rows` (all T rows
    when None). bf16 layers return X/dY as uint16 bit patterns (`X_bits`,
    `dY_bits`) plus their exact float32 values (`X`, `dY`); f32 layers return
    float32 arrays only.
    """
    out: dict = {"spec": spec}
    if "W" in parts:
        w0 = _weights(spec, seed, workload)
        q, s, z, wq, dwq = quantize_rtn(w0, spec.bits, spec.group)
        out.update(W0=w0, codes=q, qweight=pack_codes(q, spec.bits), scales=s, zeros=z, Wq=wq, dWq=dwq)
    if rows is None:
        rows = np.arange(spec.T)
    for t, width in (("X", spec.d_in), ("dY", spec.d_out)):
        if t not in parts:
            continue
        v = _rows(spec, seed, workload, t, width, rows)
        if spec.dtype == "bf16":
            b = f32_to_bf16_bits(v)
            out[t + "_bits"] = b
            out[t] = bf16_bits_to_f32(b)
        else:
            out[t] = v
    return out


# --------------------------------------------------------------------------
# sparsity patterns for edge-case tests
# --------------------------------------------------------------------------


def random_pattern(
    d_out: int,
    d_in: int,
    counts=None,
    p: int | None = None,
    rng: np.random.Generator | None = None,
    coef_scale: float = 1.0,
):
    """A random CSR pattern by output row: (row_ptr int32 [d_out+1], col_idx int32 [p], coef f32 [p]).

    `counts` fixes the nonzeros of each row (0 gives an empty row, d_in a full
    row); otherwise `p` nonzeros are spread uniformly over the rows (capped at
    d_in per row). Column indices are unique and ascending within a row.
    """
    rng = rng or rng_for(0, "pattern")
    if counts is None:
        assert p is not None and p <= d_in * d_out
        counts = np.zeros(d_out, dtype=np.int64)
        left = p
        while left > 0:
            add = np.bincount(rng.integers(0, d_out, size=left), minlength=d_out)
            counts = np.minimum(counts + add, d_in)
            left = p - int(counts.sum())
    counts = np.asarray(counts, dtype=np.int64)
    row_ptr = np.zeros(d_out + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    col = np.empty(int(row_ptr[-1]), dtype=np.int32)
    for i in range(d_out):
        c = int(counts[i])
        if c:
            col[row_ptr[i] : row_ptr[i + 1]] = np.sort(rng.choice(d_in, size=c, replace=False))
    coef = (rng.standard_normal(col.size, dtype=np.float32) * np.float32(coef_scale)).astype(np.float32)
    return row_ptr.astype(np.int32), col, coef


__all__ = [
    "CONFIGS",
    "LayerSpec",
    "ROW_BLOCK",
    "bf16_bits_to_f32",
    "f32_to_bf16_bits",
    "layer_inputs",
    "pack_codes",
    "quantize_rtn",
    "random_pattern",
    "rng_for",
]


def rank_rows(rank: int, tokens_per_rank: int) -> np.ndarray:
    """Token rows of the seeded stream that data-parallel rank `rank` processes."""
    return np.arange(rank * tokens_per_rank, (rank + 1) * tokens_per_rank)
