"""FP8 (e4m3) block quantization and the reference for FP8 attention.

TEST INFRASTRUCTURE ONLY, like the rest of this package.

Source: polydesk.ai glossary "FlashAttention", section on FlashAttention-3: FP8 inputs
with block quantization (one scale per block of the tensor) bring H100 close to
1.2 PFLOPS with a smaller numerical error than per-tensor quantization.  The pages fix
neither the FP8 format nor the block shape; readings:

* format: e4m3 of the OCP 8-bit floating-point specification (1 sign, 4 exponent bits
  with bias 7, 3 mantissa bits; exponent 0 holds the subnormals m 2^-9; no infinities;
  S.1111.111 is NaN; the largest finite value is 448), the format Blackwell's tensor
  cores take;
* blocks: 128 consecutive rows (tokens) of one (batch, head), every d column, one fp32
  scale each: scale = amax / 448 (1 when the block is all zero), code = x / scale
  rounded to the nearest e4m3 value, ties to the even code, magnitudes above 448
  saturated, the sign kept when a value rounds to zero (as IEEE conversions do).  The
  two divisions are done in fp32 with round-to-nearest, on both sides: they decide
  integer codes, which must then agree bit for bit;
* FP8 attention: the exact attention (the fp64 routine of ``attention.py``) of the
  dequantized inputs code * scale.  What the tensor cores add beyond that (the
  probabilities rounded to e4m3 before P V) is the kernel's own error, bounded in the
  tests.
"""

from __future__ import annotations

import numpy as np

from .attention import as_f64, attention

E4M3_MAX = 448.0
BLOCK = 128


def e4m3_value(code: int) -> float:
    """The value of an e4m3 code (NaN for S.1111.111)."""
    code = int(code) & 0xFF
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_TABLE = np.array([e4m3_value(c) for c in range(256)])
_POS_CODES = np.array([c for c in range(0x7F)], dtype=np.int64)  # 0x00 .. 0x7E: finite, >= 0
_POS_VALUES = _TABLE[_POS_CODES]                                    # increasing


def quantize_e4m3(y) -> np.ndarray:
    """Nearest e4m3 code of each value (fp32 inputs), ties to the even code, saturating."""
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), E4M3_MAX)
    hi = np.searchsorted(_POS_VALUES, a, side="left")       # first value >= a
    hi = np.minimum(hi, len(_POS_VALUES) - 1)
    lo = np.maximum(hi - 1, 0)
    vlo, vhi = _POS_VALUES[lo], _POS_VALUES[hi]
    dlo, dhi = a - vlo, vhi - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (_POS_CODES[hi] % 2 == 0))
    pick_hi &= vhi >= a
    code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo])
    code = np.where(a == vhi, _POS_CODES[hi], code)
    sign = np.signbit(y).astype(np.int64) << 7  # the sign survives rounding to zero (-0 = 0x80)
    return (code | sign).astype(np.uint8)


def block_quantize(x, block: int = BLOCK):
    """x [..., N, d] (bf16 tensor or array) -> (codes uint8 [..., N, d], scales float32
    [..., ceil(N/block)])."""
    x32 = np.asarray(as_f64(x), dtype=np.float32)
    *lead, N, d = x32.shape
    nb = (N + block - 1) // block
    codes = np.zeros(x32.shape, dtype=np.uint8)
    scales = np.ones((*lead, nb), dtype=np.float32)
    for idx in np.ndindex(*lead):
        for j in range(nb):
            blk = x32[idx][j * block:(j + 1) * block]
            amax = np.float32(np.abs(blk).max()) if blk.size else np.float32(0)
            sc = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1)
            scales[idx + (j,)] = sc
            codes[idx][j * block:(j + 1) * block] = quantize_e4m3((blk / sc).astype(np.float32))
    return codes, scales


def dequantize(codes, scales, block: int = BLOCK) -> np.ndarray:
    """codes [..., N, d] and scales [..., ceil(N/block)] back to float64 values."""
    vals = _TABLE[np.asarray(codes, dtype=np.int64)]
    sc = np.repeat(np.asarray(scales, dtype=np.float64), block, axis=-1)[..., : vals.shape[-2]]
    return vals * sc[..., None]


def attention_fp8_reference(q8, qs, k8, ks, v8, vs, scale: float, causal: bool, **kw):
    """Exact attention of the dequantized FP8 inputs: (O, LSE) in float64."""
    return attention(dequantize(q8, qs), dequantize(k8, ks), dequantize(v8, vs), scale, causal, **kw)
