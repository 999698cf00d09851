"""Microscaling (MX) number formats, fp64 reference.  TEST INFRASTRUCTURE ONLY.

What the pages fix:
  * "Kimi K3, previewed" (embedl blog): the specifications figure caption says
    MXFP4 weights with MXFP8 activations.
  * "kimi-k3-2" (open-llm-radar), About section: same statement.
  * "Kimi K3" (llm-atlas), Key facts table, Dtype row: the experts are MXFP4,
    and attention / shared expert / dense MLP / LM head stay high precision.

The pages do not define the formats.  The definitions below are those of the
OCP Microscaling Formats (MX) v1.0 specification and the OCP 8-bit floating
point specification (E4M3 "FN" variant):
  * E2M1 element: 1 sign, 2 exponent (bias 1), 1 mantissa bit; no inf/NaN;
    largest magnitude 6.
  * E4M3 element: 1 sign, 4 exponent (bias 7), 3 mantissa bits; S.1111.111 is
    NaN, no infinities; largest magnitude 448.
  * E8M0 scale: unsigned biased exponent, value 2^(b-127); 0xFF is NaN.
  * A block is 32 consecutive elements sharing one E8M0 scale.
  * Scale exponent of a block: floor(log2(amax)) - emax_elem (emax = 2 for
    E2M1, 8 for E4M3), where amax is the largest magnitude in the block.

Readings, for the places where the spec leaves a choice to the implementation:
  R1 Element conversion of V/2^e is round-to-nearest, ties to even mantissa,
     saturating to the largest finite magnitude.  Saturation matters because
     amax/2^e lies in [2^emax, 2^(emax+1)), which exceeds 6 (E2M1) or 448 (E4M3).
  R2 The sign of a value that rounds to zero is kept: -0 encodes as 0x8 / 0x80.
  R3 An all-zero block (amax = 0) takes the smallest scale exponent, -127
     (scale byte 0x00).  Its elements then encode +0 or -0 by R2.
  R4 The scale exponent is clamped to [-127, 127].
  R5 For E2M1 storage, element 2j of a row sits in the low nibble of byte j and
     element 2j+1 in the high nibble.
NaN and infinite inputs are outside the contract.
"""
import math

import numpy as np

BLOCK = 32
E2M1_EMAX = 2
E4M3_EMAX = 8
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def _e2m1_value(code):
    """Closed-form value of a 4-bit E2M1 code (exponent bias 1, 1 mantissa bit)."""
    s = -1.0 if (code >> 3) & 1 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        return s * (m / 2.0)                      # subnormal: 2^(1-1) * 0.m
    return s * (2.0 ** (e - 1)) * (1.0 + m / 2.0)


def _e4m3_value(code):
    """Closed-form value of an 8-bit E4M3 (FN) code (exponent bias 7, 3 mantissa bits)."""
    s = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 15
    m = code & 7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        return s * (2.0 ** -6) * (m / 8.0)        # subnormal
    return s * (2.0 ** (e - 7)) * (1.0 + m / 8.0)


E2M1_TABLE = np.array([_e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)

# Positive finite codes in increasing value order (code order == value order).
_E2M1_POS = E2M1_TABLE[:8]                         # codes 0..7
_E4M3_POS = E4M3_TABLE[:127]                       # codes 0..126 (127 is NaN)


def e8m0_value(byte):
    """2^(b-127) for a scale byte; NaN for 0xFF."""
    b = np.asarray(byte, dtype=np.int64)
    out = np.ldexp(1.0, (b - 127).astype(np.int64)).astype(np.float64)
    return np.where(b == 255, np.nan, out)


def decode_e2m1(codes):
    return E2M1_TABLE[np.asarray(codes, dtype=np.int64) & 15]


def decode_e4m3(codes):
    return E4M3_TABLE[np.asarray(codes, dtype=np.int64) & 255]


def _round_to_format(q, pos_values, max_mag):
    """RNE of q onto the positive value list, saturating; returns (codes, sign) (R1, R2).

    pos_values[i] is the value of code i (sign bit clear), increasing in i, so the
    mantissa LSB of code i is i & 1 and "ties to even" means the even index wins.
    Magnitudes at or above the largest value land on it (saturation).  Works through the
    array in chunks of 2^20 elements to stay in cache.
    """
    q = np.asarray(q, dtype=np.float64)
    flat = q.reshape(-1)
    idx = np.empty(flat.shape, dtype=np.int64)
    top = len(pos_values) - 1
    for s0 in range(0, flat.size, 1 << 20):
        a = np.minimum(np.abs(flat[s0:s0 + (1 << 20)]), max_mag)
        lo = np.searchsorted(pos_values, a, side="right") - 1      # value[lo] <= a
        hi = np.minimum(lo + 1, top)
        d_lo = a - pos_values[lo]
        d_hi = pos_values[hi] - a
        idx[s0:s0 + a.size] = np.where((d_hi < d_lo) | ((d_hi == d_lo) & ((hi & 1) == 0)), hi, lo)
    return idx.reshape(q.shape), np.signbit(q)


def block_scale_exponent(amax, emax):
    """floor(log2(amax)) - emax, clamped to [-127, 127]; -127 when amax == 0 (R3, R4)."""
    amax = np.asarray(amax, dtype=np.float64)
    out = np.full(amax.shape, -127, dtype=np.int64)
    nz = amax > 0
    if np.any(nz):
        _, ex = np.frexp(amax[nz])                 # amax = m * 2^ex, m in [0.5, 1)
        out[nz] = (ex.astype(np.int64) - 1) - emax
    return np.clip(out, -127, 127)


def quantize_mx(values, fmt):
    """MX-quantise along the last axis in blocks of 32.

    values: float array [..., K] with K % 32 == 0 (read as exact fp64).
    fmt:    "e4m3" (MXFP8) or "e2m1" (MXFP4).
    Returns (codes uint8 [..., K], scale bytes uint8 [..., K/32]).
    """
    v = np.asarray(values, dtype=np.float64)
    K = v.shape[-1]
    if K % BLOCK:
        raise ValueError("last dimension must be a multiple of 32")
    if fmt == "e4m3":
        emax, pos, mx, sign_bit = E4M3_EMAX, _E4M3_POS, E4M3_MAX, 0x80
    elif fmt == "e2m1":
        emax, pos, mx, sign_bit = E2M1_EMAX, _E2M1_POS, E2M1_MAX, 0x8
    else:
        raise ValueError(fmt)
    blocks = v.reshape(v.shape[:-1] + (K // BLOCK, BLOCK))
    amax = np.max(np.abs(blocks), axis=-1)
    e = block_scale_exponent(amax, emax)
    q = blocks / np.ldexp(1.0, e)[..., None]      # exact: division by a power of two
    idx, sign = _round_to_format(q, pos, mx)
    codes = (idx | np.where(sign, sign_bit, 0)).astype(np.uint8)
    return codes.reshape(v.shape), (e + 127).astype(np.uint8)


def dequantize_mx(codes, scales, fmt):
    """Exact fp64 value of MX data: decode(code) * 2^(scale-127) per block of 32."""
    c = np.asarray(codes)
    K = c.shape[-1]
    dec = decode_e4m3(c) if fmt == "e4m3" else decode_e2m1(c)
    s = e8m0_value(scales)
    dec = dec.reshape(c.shape[:-1] + (K // BLOCK, BLOCK)) * s[..., None]
    return dec.reshape(c.shape)


def pack_e2m1(codes):
    """Two E2M1 codes per byte along the last axis; element 2j in the low nibble (R5)."""
    c = np.asarray(codes, dtype=np.uint8) & 15
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_e2m1(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 15
    out[..., 1::2] = p >> 4
    return out


def bf16_round(x):
    """Round fp64 values to the nearest bfloat16 (ties to even), returned as fp64.

    bfloat16 has 8 exponent bits (bias 127) and 7 stored mantissa bits; below
    2^-126 the spacing stays 2^-133 (subnormals).  Overflow is outside the contract.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    if np.any(nz):
        _, ex = np.frexp(np.abs(x[nz]))            # |x| = m * 2^ex, floor(log2|x|) = ex-1
        e = np.maximum(ex.astype(np.int64) - 1, -126)
        ulp = np.ldexp(1.0, e - 7)
        out[nz] = np.round(x[nz] / ulp) * ulp      # np.round is round-half-even
    out[~nz] = x[~nz]
    return out


def log2_floor(x):
    """floor(log2(x)) for a positive finite scalar, exact."""
    _, ex = math.frexp(x)
    return ex - 1
