"""MXFP8 (E4M3 elements, one UE8M0 scale per 32-element block) by its published definition.

TEST INFRASTRUCTURE ONLY (see `oracle/moe.py`).

The pages name the format only ("MXFP8", noticiarioia.com "Otimizacoes e testes em escala de
trilhoes"; bytechap.com "Como funciona"; unite.ai "Parallelismo, precisione e tecniche di memoria").
The element and scale encodings follow the OCP Microscaling Formats (MX) v1.0 specification:

  E4M3 (the "fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; no infinities; the
  only NaN is S.1111.111; largest finite 448 = 1.75 * 2^8; smallest normal 2^-6; subnormals
  m * 2^-9, m = 1..7.
  UE8M0 scale: an unsigned 8-bit biased exponent, value 2^(byte - 127); 0xFF is NaN (never produced).
  Block scale: X = 2^(floor(log2(amax)) - emax_elem), emax_elem = 8 for E4M3; each element is
  v / X rounded to nearest (ties to even) and saturated to +-448.

Readings where the specification leaves a choice (each also stated in the design notes):
  * amax == 0: scale byte 0 (2^-127) and every code 0.
  * the block exponent is clamped to [-127, 127].
  * rounding of v / X to E4M3 is round-to-nearest-even, then saturate to 448 (no NaN from overflow).

All arithmetic is exact in float64 (inputs are bf16 values; scaling is by powers of two).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_EMAX = 8
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_MIN_SUBNORMAL = 2.0 ** -9
BLOCK = 32


def floor_log2(a: np.ndarray) -> np.ndarray:
    """floor(log2(a)) for a > 0, exact (frexp gives a = m 2^e with m in [0.5, 1))."""
    _, e = np.frexp(a)
    return e.astype(np.int64) - 1


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Round float64 values to E4M3 (nearest, ties to even), saturating to +-448. Returns uint8 codes."""
    v = np.asarray(v, dtype=np.float64)
    sign = (np.signbit(v)).astype(np.uint8) << 7
    a = np.abs(v)
    code = np.zeros(a.shape, dtype=np.int64)
    nz = a > 0
    e = np.where(nz, floor_log2(np.where(nz, a, 1.0)), 0)
    sub = nz & (e < -6)
    # subnormal range: integer multiple of 2^-9, rounded half-even; q == 8 is exactly the min normal
    q_sub = np.rint(np.where(sub, a, 0.0) / E4M3_MIN_SUBNORMAL).astype(np.int64)
    code = np.where(sub, q_sub, code)
    nrm = nz & ~sub
    m = np.where(nrm, a, 1.0) / np.power(2.0, np.where(nrm, e, 0).astype(np.float64))  # [1,2)
    q = np.rint((m - 1.0) * 8.0).astype(np.int64)
    e_n = np.where(q == 8, e + 1, e)
    q = np.where(q == 8, 0, q)
    ncode = ((e_n + 7) << 3) | q
    sat = (e_n > 8) | ((e_n == 8) & (q == 7))
    ncode = np.where(sat, 0x7E, ncode)
    code = np.where(nrm, ncode, code)
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(code & 0x80, -1.0, 1.0)
    ex = (code >> 3) & 0xF
    mt = code & 0x7
    val = np.where(ex == 0, mt * E4M3_MIN_SUBNORMAL,
                   (1.0 + mt / 8.0) * np.power(2.0, (ex - 7).astype(np.float64)))
    nan = (ex == 15) & (mt == 7)
    return np.where(nan, np.nan, s * val)


def ue8m0_decode(b: np.ndarray) -> np.ndarray:
    return np.power(2.0, np.asarray(b, dtype=np.int64).astype(np.float64) - 127.0)


def quantize_rows(a: np.ndarray, block: int = BLOCK):
    """Quantise along the last axis in blocks of `block`. a [..., K] with K % block == 0.
    Returns (codes uint8 [..., K], scales uint8 [..., K/block])."""
    a = np.asarray(a, dtype=np.float64)
    K = a.shape[-1]
    assert K % block == 0
    blk = a.reshape(a.shape[:-1] + (K // block, block))
    amax = np.max(np.abs(blk), axis=-1)
    pos = amax > 0
    ex = np.where(pos, floor_log2(np.where(pos, amax, 1.0)) - E4M3_EMAX, -127)
    ex = np.clip(ex, -127, 127)
    scales = (ex + 127).astype(np.uint8)
    scaled = blk / np.power(2.0, ex.astype(np.float64))[..., None]
    codes = e4m3_encode(scaled)
    codes = np.where(pos[..., None], codes, 0).astype(np.uint8)
    return codes.reshape(a.shape), scales


def dequantize_rows(codes: np.ndarray, scales: np.ndarray, block: int = BLOCK) -> np.ndarray:
    K = codes.shape[-1]
    v = e4m3_decode(codes).reshape(codes.shape[:-1] + (K // block, block))
    return (v * ue8m0_decode(scales)[..., None]).reshape(codes.shape)


def quantize_cols(a: np.ndarray, block: int = BLOCK):
    """Quantise a [R, C] along its rows axis (blocks of `block` consecutive rows per column).
    Returns codes [R, C] and scales [R/block, C]."""
    c, s = quantize_rows(np.asarray(a).T, block)
    return c.T.copy(), s.T.copy()


def dequantize_cols(codes, scales, block: int = BLOCK):
    return dequantize_rows(codes.T, scales.T, block).T.copy()


def fake_quant_rows(a, block: int = BLOCK):
    return dequantize_rows(*quantize_rows(a, block), block)


def fake_quant_cols(a, block: int = BLOCK):
    return dequantize_cols(*quantize_cols(a, block), block)
