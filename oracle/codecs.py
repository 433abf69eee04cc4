"""Number formats used on the CSA path, written out from their published definitions.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

* bfloat16: IEEE-754 binary32 truncated to 8 significant bits, round to
  nearest, ties to even.
* FP8 E4M3 ("E4M3FN" of the OCP 8-bit floating point specification): 1 sign,
  4 exponent (bias 7), 3 mantissa bits; no infinities; S.1111.111 is NaN, so
  the largest finite value is 448; subnormals step by 2^-9.
* FP4 E2M1 (OCP Microscaling formats specification): 1 sign, 2 exponent
  (bias 1), 1 mantissa bit; values {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
* UE4M3: an E4M3 code with the sign bit zero, used as the per-16-element
  block scale of NVFP4.

Encoders round to nearest, ties to even, and saturate to the largest finite
value (the indexer quantiser of "DeepSeek V4 结构速览", section
"Lightning Indexer", caches keys in FP4; the 64K decode workload caches them
in FP8 with a per-row scale).  Pinned against ml_dtypes and torch
casts in ``tests/test_oracle_pins.py``.
"""

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0


def round_to_bf16(x):
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64.

    Rounds the float64 value directly (no intermediate float32), so a result is
    the correctly rounded bf16 of the exact input.  Overflow goes to +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    finite = np.isfinite(x) & (x != 0)
    xf = x[finite]
    _, ex = np.frexp(xf)                 # xf = f * 2^ex, 0.5 <= |f| < 1
    e = np.maximum(ex - 1, -126)         # unbiased exponent, clamped at bf16's min normal
    ulp = np.ldexp(1.0, e - 7)           # 8 significant bits
    r = np.rint(xf / ulp) * ulp          # np.rint: half to even; exact in float64
    r[np.abs(r) > 3.3895313892515355e38] = np.inf * np.sign(r[np.abs(r) > 3.3895313892515355e38])
    out[finite] = r
    return out


def bf16_bits(x):
    """uint16 bit patterns of bf16 values given as float64 already on the bf16 grid."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    return (x32.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(bits):
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def e4m3_decode(codes):
    """Value of each E4M3FN code (uint8) as float64; S.1111.111 decodes to NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    mant = c & 0x7
    sub = mant * 2.0 ** -9
    norm = (1.0 + mant / 8.0) * np.ldexp(1.0, e - 7)
    val = np.where(e == 0, sub, norm)
    val = np.where((e == 15) & (mant == 7), np.nan, val)
    return sign * val


def e4m3_encode(y):
    """E4M3FN code of each float32 value: round to nearest even, saturate at +-448."""
    y = np.asarray(y, dtype=np.float32).astype(np.float64)
    sign = (np.signbit(y)).astype(np.int64)
    a = np.minimum(np.abs(y), E4M3_MAX)
    code = np.zeros(a.shape, dtype=np.int64)
    small = a < 2.0 ** -6
    # subnormal range: multiples of 2^-9; a carry to 8 is the smallest normal (code 8)
    code[small] = np.rint(a[small] / 2.0 ** -9).astype(np.int64)
    big = ~small
    if np.any(big):
        _, ex = np.frexp(a[big])
        e = ex - 1                                   # a in [2^e, 2^(e+1))
        q = np.rint(a[big] / np.ldexp(1.0, e - 3)).astype(np.int64)   # in [8, 16]
        carry = q == 16
        e = np.where(carry, e + 1, e)
        q = np.where(carry, 8, q)
        code[big] = ((e + 7) << 3) | (q - 8)
    return ((sign << 7) | code).astype(np.uint8)


def e2m1_decode(codes):
    """Value of each E2M1 code (low 4 bits of a uint8) as float64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    mant = c & 0x1
    sub = mant * 0.5
    norm = (1.0 + mant / 2.0) * np.ldexp(1.0, e - 1)
    return sign * np.where(e == 0, sub, norm)


def e2m1_encode(y):
    """E2M1 code (0..15) of each float32 value: round to nearest even, saturate at +-6."""
    y = np.asarray(y, dtype=np.float32).astype(np.float64)
    sign = (np.signbit(y)).astype(np.int64)
    a = np.minimum(np.abs(y), E2M1_MAX)
    code = np.zeros(a.shape, dtype=np.int64)
    small = a < 1.0
    # subnormal range: multiples of 0.5; a carry to 2 is the smallest normal (code 2 = 1.0)
    code[small] = np.rint(a[small] / 0.5).astype(np.int64)
    big = ~small
    if np.any(big):
        _, ex = np.frexp(a[big])
        e = ex - 1                                   # 0, 1 or 2
        q = np.rint(a[big] / np.ldexp(1.0, e - 1)).astype(np.int64)   # in [2, 4]
        carry = q == 4
        e = np.where(carry, e + 1, e)
        q = np.where(carry, 2, q)
        code[big] = ((e + 1) << 1) | (q - 2)
    return ((sign << 3) | code).astype(np.uint8)


def pack_e2m1(codes):
    """Pack E2M1 codes two per byte along the last axis: element 2j in bits 0-3, 2j+1 in bits 4-7."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_e2m1(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


# ---------------------------------------------------------------------------
# Quantisers of the index path (FP8 per row, NVFP4 per 16 elements)
# ---------------------------------------------------------------------------

def quant_fp8_rows(x):
    """FP8 E4M3 with one float32 scale per row (last axis).

    scale = amax / 448 and code = e4m3(x / scale), both divisions in float32;
    a row whose amax is 0 gets scale 0 and all-zero codes.
    Returns (codes uint8 [..., d], scales float32 [...]).
    """
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=-1)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    y = (x32 / safe[..., None]).astype(np.float32)
    codes = e4m3_encode(y)
    codes[scale == 0] = 0
    return codes, scale


def dequant_fp8_rows(codes, scales):
    return e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[..., None]


def quant_nvfp4(x, block=16):
    """NVFP4: E2M1 codes with one UE4M3 scale per ``block`` consecutive elements.

    s = ue4m3(amax_block / 6) (float32 division, then E4M3 rounding), code =
    e2m1(x / s) in float32; a block whose scale rounds to 0 gets all-zero codes.
    Returns (packed codes uint8 [..., d/2], scale codes uint8 [..., d/block]).
    """
    x32 = np.asarray(x, dtype=np.float32)
    d = x32.shape[-1]
    xb = x32.reshape(x32.shape[:-1] + (d // block, block))
    amax = np.max(np.abs(xb), axis=-1)
    s_code = e4m3_encode((amax / np.float32(E2M1_MAX)).astype(np.float32))
    s = e4m3_decode(s_code).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    y = (xb / safe[..., None]).astype(np.float32)
    codes = e2m1_encode(y)
    codes[np.broadcast_to((s == 0)[..., None], codes.shape)] = 0
    codes = codes.reshape(x32.shape)
    return pack_e2m1(codes), s_code


def dequant_nvfp4(packed, s_codes, block=16):
    v = e2m1_decode(unpack_e2m1(packed))
    d = v.shape[-1]
    vb = v.reshape(v.shape[:-1] + (d // block, block))
    s = e4m3_decode(s_codes)
    return (vb * s[..., None]).reshape(v.shape)
