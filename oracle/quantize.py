"""Per-tile dynamic-scale e4m3 quantisation of Q and K (TEST INFRASTRUCTURE ONLY).

Follows "从理论到实现：基于Triton剖析FlashAttention三代的演进与优化" §4.1: each
operand gets a dynamic scale from its absolute maximum, the QK^T product is
taken on the quantised values, and the product is multiplied by
1 / (q_scale * k_scale) to undo the scaling.  The page's constant is int8's
127 with a garbled epsilon term; for e4m3 the constant is 448 (the largest
finite value), and an all-zero tile gets scale 1 (the epsilon's role: no
division by zero).

Granularity: one scale per (batch, head, 128-row tile) of the sequence; the
last tile holds the ragged remainder.  Decisions that produce integer codes are
taken in fp32, the precision the GPU quantiser uses:
    amax  = max |x| over the tile          (exact in fp32 for bf16 inputs)
    scale = fp32(448) / amax                (one IEEE fp32 division, RNE)
    code  = e4m3_rne_satfinite(fp32(x * scale))   (one fp32 multiply, RNE)
"""

from __future__ import annotations

import numpy as np

from .e4m3 import E4M3_MAX, e4m3_decode, e4m3_encode_rne_satfinite

TILE_ROWS = 128


def _as_f32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        import torch

        x = x.detach().to("cpu", torch.float32).numpy()
    return np.asarray(x, dtype=np.float32)


def quantize_e4m3_tiles(x, tile_rows: int = TILE_ROWS):
    """x: [B, H, N, d] (bf16 values).  Returns (codes uint8 [B,H,N,d], scales fp32 [B,H,T])."""
    x = _as_f32(x)
    B, H, N, d = x.shape
    T = (N + tile_rows - 1) // tile_rows
    codes = np.empty((B, H, N, d), dtype=np.uint8)
    scales = np.empty((B, H, T), dtype=np.float32)
    for t in range(T):
        r0, r1 = t * tile_rows, min(N, (t + 1) * tile_rows)
        blk = x[:, :, r0:r1, :]
        amax = np.abs(blk).max(axis=(2, 3)).astype(np.float32)        # [B, H]
        with np.errstate(divide="ignore"):
            sc = np.where(amax > 0, np.float32(E4M3_MAX) / amax, np.float32(1.0)).astype(np.float32)
        scaled = (blk * sc[:, :, None, None]).astype(np.float32)      # fp32 multiply
        codes[:, :, r0:r1, :] = e4m3_encode_rne_satfinite(scaled)
        scales[:, :, t] = sc
    return codes, scales


def dequantize_e4m3_tiles(codes, scales, tile_rows: int = TILE_ROWS) -> np.ndarray:
    """Exact fp64 values code / scale, per tile."""
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.float32).astype(np.float64)
    B, H, N, d = codes.shape
    rows_tile = np.arange(N) // tile_rows
    return e4m3_decode(codes) / scales[:, :, rows_tile][..., None]
