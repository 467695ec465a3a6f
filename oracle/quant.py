"""Symmetric INT8 quantiser for cache rows (oracle).

Test infrastructure: only tests/, the smoke check and the CPU-baseline legs of
bench.py import this module.

The CONF-KV abstract and post store older retained tokens in INT8 while the
recent window stays FP16; the post's implementation note mentions dequantising
INT8 inside the attention kernel. The pages leave the granularity open. The
reading taken here: one fp32 scale per token, per KV head, for K and for V
separately.

* amax = max |x| over the head dimension, with fp16 widened exactly to fp32.
* scale = amax / 127, one IEEE fp32 division.
* code = clamp(round_half_even(x / scale), -127, 127), with x / scale an IEEE
  fp32 division.
* An all-zero row gets scale 0 and codes 0.
* Dequantised value: float(code) * scale in fp32.

Pins (tests/test_oracle_quant.py): a row with amax = 127 has scale exactly 1,
so 2.5 -> 2, 3.5 -> 4, -2.5 -> -2 and +-127 stay; a zero row; the error bound
|x - x_hat| <= scale / 2; codes lie in [-127, 127] and the amax element maps
to +-127.
"""
from __future__ import annotations

import numpy as np

_127 = np.float32(127.0)


def quantize_row(x16) -> tuple[np.ndarray, np.float32]:
    """Quantise one fp16 row. Returns (int8 codes, fp32 scale)."""
    x = np.asarray(x16, dtype=np.float16).astype(np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0.0)
    scale = np.float32(amax / _127)
    if scale == np.float32(0.0):
        return np.zeros(x.shape, dtype=np.int8), np.float32(0.0)
    ratio = (x / scale).astype(np.float32)      # IEEE fp32 division, elementwise
    codes = np.clip(np.rint(ratio), -127.0, 127.0).astype(np.int8)
    return codes, scale


def quantize_rows(x16) -> tuple[np.ndarray, np.ndarray]:
    """Quantise each row of an [n, D] fp16 array independently: the same
    formula as quantize_row, evaluated for all rows at once."""
    x = np.asarray(x16, dtype=np.float16).astype(np.float32)
    n = x.shape[0]
    if n == 0:
        return np.zeros(x.shape, dtype=np.int8), np.zeros(0, dtype=np.float32)
    amax = np.max(np.abs(x), axis=1).astype(np.float32)
    scales = (amax / _127).astype(np.float32)
    safe = np.where(scales == np.float32(0.0), np.float32(1.0), scales).astype(np.float32)
    ratio = (x / safe[:, None]).astype(np.float32)       # IEEE fp32 division, elementwise
    codes = np.clip(np.rint(ratio), -127.0, 127.0).astype(np.int8)
    codes[scales == np.float32(0.0)] = 0
    return codes, scales


def dequantize_rows(codes, scales) -> np.ndarray:
    """float(code) * scale in fp32 for every row; returns fp32 [n, D]."""
    codes = np.asarray(codes, dtype=np.int8)
    scales = np.asarray(scales, dtype=np.float32)
    return (codes.astype(np.float32) * scales[:, None]).astype(np.float32)
