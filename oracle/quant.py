"""Per-group symmetric absmax quantisation, fp16 scales, code packing.

Source: Hadamard-Int4-Accuracy wiki, Method: ``q_dequant_vec(x, out, K, G, bits)``
is per-group symmetric integer quantise -> dequantise for any bit-width; Hypothesis:
outliers blow out the per-group absmax scale.

Decision precision: the pages fix no precision for the quantiser's decisions (the
wiki's "exactly in fp32" is said of the identity A.B = (A.Q)(Q.B), not of the
quantiser). Where floating point decides an integer, this oracle takes the decision in
the precision the CUDA kernels compute in, fp32: the fp64 rotated value is rounded
once to fp32, the scale is fp32(absmax / qmax) rounded to binary16, and the quotient
y / s is an fp32 division. Against an all-fp64 decision this moves |y/s| by about
1e-6 (relative 2^-24 per rounding) and absmax/qmax by about 1e-7 relative, so the two
readings differ only inside the 1e-5 boundary windows that ``boundary_flags`` marks.

Readings where the pages are silent:
* levels are symmetric: qmax = 2^(bits-1) - 1 (int4: -7..7, int2: -1..1, int8:
  -127..127); the code -2^(bits-1) is never produced;
* scale s = fp16_rn(fp32(absmax / qmax)); codes use that stored fp16 value, so
  dequantisation q*s reproduces exactly what the codes mean;
* q = clamp(round_half_away_from_zero(fp32(y / s)), -qmax, qmax); s == 0 gives q = 0;
* groups are G contiguous coordinates of the rotated row;
* packing: int4 row j-th byte = (q[2j] & 0xF) | (q[2j+1] & 0xF) << 4; int2 row j-th
  byte holds q[4j+i] in bits 2i..2i+1; two's complement; int8 one code per byte.
"""
from __future__ import annotations

import numpy as np


def qmax_of(bits: int) -> int:
    if bits not in (2, 4, 8):
        raise ValueError("bits must be 2, 4 or 8")
    return (1 << (bits - 1)) - 1


def round_half_away(v: np.ndarray) -> np.ndarray:
    """sign(v) * floor(|v| + 1/2), evaluated exactly in fp64 (v holds fp32 values)."""
    v = np.asarray(v, dtype=np.float64)
    return np.sign(v) * np.floor(np.abs(v) + 0.5)


def scales_fp16(absmax32: np.ndarray, bits: int) -> np.ndarray:
    """s = fp16_rn(fp32(absmax / qmax)) (fp32 IEEE division, then RNE to binary16)."""
    q = np.float32(qmax_of(bits))
    with np.errstate(over="ignore"):
        return (absmax32.astype(np.float32) / q).astype(np.float32).astype(np.float16)


def quantize(y: np.ndarray, bits: int, G: int):
    """Quantise rows of y (fp64 rotated values) in groups of G.

    Returns (codes int8 [M,K], scales fp16 [M,K/G]).
    """
    y32 = np.asarray(y).astype(np.float32)
    M, K = y32.shape
    if K % G:
        raise ValueError("G must divide K")
    qm = qmax_of(bits)
    g = y32.reshape(M, K // G, G)
    m = np.abs(g).max(axis=2)
    s16 = scales_fp16(m, bits)
    s32 = s16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = g / s32[..., None]                      # fp32 IEEE division
    v = np.where((s32 == 0)[..., None], np.float32(0), v)
    q = np.clip(round_half_away(v), -qm, qm).astype(np.int8)
    return q.reshape(M, K), s16


def dequantize(codes: np.ndarray, scales16: np.ndarray, G: int) -> np.ndarray:
    """x_hat = q * s (exact in fp32: |q| <= 127 and s is a binary16 value)."""
    M, K = codes.shape
    s = scales16.astype(np.float32)
    x = codes.reshape(M, K // G, G).astype(np.float32) * s[..., None]
    return x.reshape(M, K)


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack int codes along rows (layout in the module docstring)."""
    c = np.asarray(codes).astype(np.int64)
    M, K = c.shape
    if bits == 8:
        return (c & 0xFF).astype(np.uint8)
    per = 8 // bits
    if K % per:
        raise ValueError("K must be a multiple of the codes per byte")
    mask = (1 << bits) - 1
    c = (c & mask).reshape(M, K // per, per)
    out = np.zeros((M, K // per), dtype=np.int64)
    for i in range(per):
        out |= c[:, :, i] << (bits * i)
    return out.astype(np.uint8)


def unpack(packed: np.ndarray, bits: int, K: int) -> np.ndarray:
    """Inverse of ``pack``: sign-extended int8 codes [M, K]."""
    p = np.asarray(packed).astype(np.int64)
    M = p.shape[0]
    if bits == 8:
        v = p & 0xFF
        return np.where(v >= 128, v - 256, v).astype(np.int8)
    per = 8 // bits
    mask = (1 << bits) - 1
    out = np.empty((M, K // per, per), dtype=np.int64)
    for i in range(per):
        v = (p >> (bits * i)) & mask
        out[:, :, i] = np.where(v >= (1 << (bits - 1)), v - (1 << bits), v)
    return out.reshape(M, K).astype(np.int8)


def _fp16_midpoint_distance(x: np.ndarray) -> np.ndarray:
    """Relative distance of x (> 0, fp64) to the nearest binary16 rounding midpoint."""
    x = np.asarray(x, dtype=np.float64)
    lo = x.astype(np.float16)
    lo = np.where(lo.astype(np.float64) > x, np.nextafter(lo, np.float16(0)), lo)
    hi = np.nextafter(lo, np.float16(np.inf))
    mid = (lo.astype(np.float64) + hi.astype(np.float64)) / 2.0
    with np.errstate(divide="ignore", invalid="ignore"):
        d = np.abs(x - mid) / x
    return np.where(x > 0, d, np.inf)


def boundary_flags(y: np.ndarray, bits: int, G: int, eps: float = 1e-5):
    """Elements whose decision lies within ``eps`` of a rounding boundary.

    * code flag: with the oracle's scale s, v = y / s (fp64) lies within eps * max(1, |v|) of a
      half-integer (the rounding boundary of round-to-nearest): the window is relative to the
      pre-rounding value, as the rotated values it is computed from are known to 1e-5 relative
      (absolute 1e-5 below |v| = 1; up to 7.5e-5 for int4 and 1.3e-3 for int8 codes);
    * scale flag: absmax/qmax (fp64) lies within eps (relative) of a binary16
      rounding midpoint, so an fp32 computation of the scale may round the other
      way; every code of such a group is flagged.

    Returns (code_flags bool [M,K], group_flags bool [M,K/G]).
    """
    y = np.asarray(y, dtype=np.float64)
    M, K = y.shape
    qm = qmax_of(bits)
    g = y.reshape(M, K // G, G)
    m = np.abs(g).max(axis=2)
    _, s16 = quantize(y, bits, G)
    s = s16.astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.abs(g) / s[..., None]
    v = np.where((s == 0)[..., None], 0.0, v)
    frac = v - np.floor(v)
    code_flag = np.abs(frac - 0.5) < eps * np.maximum(1.0, v)
    group_flag = _fp16_midpoint_distance(m / qm) < eps
    code_flag |= group_flag[..., None]
    return code_flag.reshape(M, K), group_flag
