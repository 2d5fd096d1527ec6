"""MX (OCP microscaling) FP8 quantiser, fp64 oracle.

TEST INFRASTRUCTURE ONLY.  [OC3-ja] "MXFP8による精度最適化" names MXFP8 as the
low-precision format of the expert GEMMs; the format used here is the OCP MX
rule of the layer definition: E4M3 elements, one E8M0 scale per 32
contiguous elements along the GEMM's K axis,

    X = 2^(floor(log2(amax)) - 8)        (8 = exponent of E4M3's largest
                                          power of two, 448 = 1.75 * 2^8)
    code = round-to-nearest-even E4M3(v / X), saturating at +-448.

Readings where the rule is silent: an all-zero block gets the smallest scale
2^-127 (byte 0) and zero codes; the scale exponent is clamped to [-127, 127];
a negative value that rounds to zero keeps its sign (code 0x80); NaN and Inf
inputs are outside the domain.

The encoder works from the binary exponent and significand (frexp, then an
integer round-half-even of the significand); the pins compare it with a
brute-force nearest search over the 256-entry decode table, which is written
from the E4M3 bit layout (1 sign, 4 exponent with bias 7, 3 mantissa bits;
exponent field 0 = subnormal; S.1111.111 = NaN).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_EMAX = 8            # 448 = 1.75 * 2^8
SCALE_BIAS = 127
BLOCK = 32


def e4m3_decode_table():
    """Value of every E4M3FN code 0..255 (NaN for the two NaN codes)."""
    vals = np.zeros(256)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        ef = (c >> 3) & 0xF
        mf = c & 0x7
        if ef == 0xF and mf == 0x7:
            vals[c] = np.nan
        elif ef == 0:
            vals[c] = s * mf * 2.0 ** -9          # (m/8) * 2^(1-7)
        else:
            vals[c] = s * (1.0 + mf / 8.0) * 2.0 ** (ef - 7)
    return vals


def e4m3_encode(q):
    """E4M3FN codes of exact values q: round to nearest, ties to even,
    magnitudes above 448 saturate to 448; the sign bit follows q's sign
    (so -0 and negative values rounding to zero give 0x80)."""
    q = np.asarray(q, np.float64)
    neg = np.signbit(q)
    a = np.abs(q)
    code = np.zeros(q.shape, np.int64)

    sat = a >= E4M3_MAX
    sub = a < 2.0 ** -6                       # below the smallest normal
    nor = ~sat & ~sub

    # subnormals: steps of 2^-9; a count of 8 steps is the smallest normal
    code[sub] = np.rint(a[sub] * 2.0 ** 9).astype(np.int64)

    # normals: a = m * 2^ex with 0.5 <= m < 1, i.e. 1.mmm * 2^(ex-1)
    m, ex = np.frexp(a[nor])
    e = ex - 1
    steps = np.rint(m * 16.0).astype(np.int64)   # 8..16 eighths of 2^e
    carry = steps == 16
    e = e + carry
    steps = np.where(carry, 8, steps)
    ncode = ((e + 7) << 3) | (steps - 8)
    code[nor] = ncode
    code[sat] = 0x7E
    # 1.111 * 2^8 (480) would be the NaN pattern; values >= 464 are caught by
    # `sat` above (464 itself ties to the even 448)
    code = np.where(code == 0x7F, 0x7E, code)
    code = code | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


def mx_scale_exponent(amax):
    """Shared exponent s of a block: floor(log2(amax)) - 8, clamped to
    [-127, 127]; an all-zero block gets -127."""
    amax = np.asarray(amax, np.float64)
    _, ex = np.frexp(amax)                    # amax = m * 2^ex, m in [0.5, 1)
    s = (ex - 1) - E4M3_EMAX
    s = np.where(amax == 0.0, -SCALE_BIAS, s)
    return np.clip(s, -SCALE_BIAS, SCALE_BIAS).astype(np.int64)


def _quantize_blocks(blocks):
    """blocks [..., 32] -> (codes [..., 32] uint8, scale bytes [...] uint8)."""
    amax = np.max(np.abs(blocks), axis=-1)
    s = mx_scale_exponent(amax)
    q = blocks * np.ldexp(1.0, -s)[..., None]     # exact: power-of-two scaling
    return e4m3_encode(q), (s + SCALE_BIAS).astype(np.uint8)


def mx_quantize_rows(v):
    """Blocks of 32 contiguous elements along the last axis of v [R, C].
    Returns codes [R, C] uint8 and scales [R, C/32] uint8."""
    v = np.asarray(v, np.float64)
    R, C = v.shape
    assert C % BLOCK == 0
    codes, scales = _quantize_blocks(v.reshape(R, C // BLOCK, BLOCK))
    return codes.reshape(R, C), scales


def mx_quantize_cols_grouped(v, group_offsets):
    """Blocks of 32 consecutive rows of v [R, C], column by column; blocks
    start at each group's first row and never cross a group (every group
    offset must be a multiple of 32).  Returns codes [R, C] and scales
    [R/32, C] (block b covers rows 32b .. 32b+31)."""
    v = np.asarray(v, np.float64)
    R, C = v.shape
    go = np.asarray(group_offsets)
    assert R % BLOCK == 0 and np.all(go % BLOCK == 0)
    # the blocks of 32 rows from row 0 are exactly the in-group blocks
    # because every group starts on a multiple of 32
    blocks = v.reshape(R // BLOCK, BLOCK, C).transpose(0, 2, 1)   # [R/32, C, 32]
    codes, scales = _quantize_blocks(blocks)
    return codes.transpose(0, 2, 1).reshape(R, C), scales


_TABLE = None


def _decode(codes):
    global _TABLE
    if _TABLE is None:
        _TABLE = e4m3_decode_table()
    return _TABLE[np.asarray(codes, np.int64)]


def mx_dequantize_rows(codes, scales):
    R, C = codes.shape
    f = np.ldexp(1.0, scales.astype(np.int64) - SCALE_BIAS)     # [R, C/32]
    return (_decode(codes).reshape(R, C // BLOCK, BLOCK) * f[..., None]).reshape(R, C)


def mx_dequantize_cols(codes, scales):
    R, C = codes.shape
    f = np.ldexp(1.0, scales.astype(np.int64) - SCALE_BIAS)     # [R/32, C]
    return (_decode(codes).reshape(R // BLOCK, BLOCK, C) * f[:, None, :]).reshape(R, C)
