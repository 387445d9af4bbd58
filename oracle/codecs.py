"""Low-precision codecs and group-wise dequantisation (float64 oracle).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

What the pages fix: the frozen base stays in its deployment precision (INT4 for
Kimi-K2.6, FP4 for DeepSeek V4, FP8 named as the third option) and is
dequantised for the GEMM while the adapter is BF16 (m.xxlwj.com 771001,
sections "单节点 Kimi-K2.6 了局" and "单节点 DeepSeek V4 Flash 了局"; chooseai.io news
4086, section "技术原理：低精度基座 + BF16 适配器 + OFT").  The pages give no bit
formats; the code tables below follow the public OCP 8-bit floating point
specification (e4m3 "fn": bias 7, no infinities, S.1111.111 is NaN) and the OCP
Microscaling specification (e2m1 elements, e8m0 shared scales, block of 32).

Canonical dequantised value (the bit-exact target for the GPU):
  INT4  : w = bf16_rne(q * s)                  q in [-8,7], s a bf16 group scale
  FP8   : w = bf16_rne(f32_rne(v * s_n))       v an e4m3 value, s_n fp32 per channel
  MXFP4 : w = bf16_rne(v * 2^(e-127))          v an e2m1 value, e the e8m0 code
The FP8 chain rounds twice because that is what an fp32 multiply followed by a
bf16 conversion produces; q*s and v*2^k are exact in fp32, so INT4 and MXFP4 round
once (MXFP4 not at all).

Pins (tests/test_oracle_codecs.py): all 256 e4m3 codes against torch's
float8_e4m3fn decoder; the e2m1 grid against the OCP table values and the
e4m3 decoder on the codes both formats share; e8m0 against powers of two;
all 16 INT4 nibbles against int8 sign extension; bf16 rounding against torch's
fp32->bf16 conversion (random values, ties, overflow, NaN); whole dequantised
matrices against torch CPU arithmetic on the same codes.
"""

from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# bf16 <-> float
# ----------------------------------------------------------------------------


def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 values (exact)."""
    u = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f32_to_bf16_bits(x) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest, ties to even.

    NaN stays NaN (quietened); overflow past the largest bf16 goes to infinity.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    r = np.where(np.isnan(x), (u >> np.uint64(16)) | np.uint64(0x40), r)
    return (r & np.uint64(0xFFFF)).astype(np.uint16)


def f64_to_bf16_bits_via_f32(x) -> np.ndarray:
    """float64 -> float32 (RNE) -> bf16 (RNE): the rounding chain of an fp32
    product converted to bf16."""
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float64).astype(np.float32))


# ----------------------------------------------------------------------------
# element codecs
# ----------------------------------------------------------------------------


def e4m3_value(code: int) -> float:
    """OCP FP8 E4M3 ("fn"): 1 sign, 4 exponent (bias 7), 3 mantissa bits;
    exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e2m1_value(code: int) -> float:
    """OCP MX FP4 E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit;
    exponent 0 is subnormal (m * 0.5); no NaN or infinity encodings."""
    sign = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return sign * m * 0.5
    return sign * (1.0 + m / 2.0) * 2.0 ** (e - 1)


def e8m0_value(code: int) -> float:
    """OCP MX E8M0 scale: 2^(code-127); code 255 is NaN."""
    if code == 255:
        return float("nan")
    return 2.0 ** (code - 127)


def int4_value(nibble: int) -> int:
    """Two's complement 4-bit integer."""
    nibble &= 0xF
    return nibble - 16 if nibble >= 8 else nibble


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E8M0_TABLE = np.array([e8m0_value(c) for c in range(256)], dtype=np.float64)
INT4_TABLE = np.array([int4_value(c) for c in range(16)], dtype=np.float64)


def unpack_nibbles(codes, k0: int = 0, k1=None) -> np.ndarray:
    """uint8 [N][K/2] -> uint8 nibbles [N][k1-k0]; element k sits in byte k//2,
    low nibble for even k.  k0 must be even."""
    codes = np.asarray(codes, dtype=np.uint8)
    K = codes.shape[-1] * 2
    k1 = K if k1 is None else k1
    assert k0 % 2 == 0
    c = codes[..., k0 // 2:(k1 + 1) // 2]
    out = np.empty(c.shape[:-1] + (2 * c.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = c & 0xF
    out[..., 1::2] = c >> 4
    return out[..., : k1 - k0]


# ----------------------------------------------------------------------------
# dequantisation of a stored weight W^T [N][K]
# ----------------------------------------------------------------------------


def dequant_bits(fmt: str, codes, scales, K: int, group: int, rows=None, k0: int = 0, k1=None) -> np.ndarray:
    """Canonical bf16 bit patterns of the dequantised weight, rows x [k0, k1).

    codes/scales use the stored layouts: INT4 codes [N][K/2] with bf16 scales
    [K/G][N]; FP8 codes [N][K] with fp32 scales [N]; MXFP4 codes [N][K/2] with
    e8m0 scales [K/32][N].
    """
    k1 = K if k1 is None else k1
    codes = np.asarray(codes)
    scales = np.asarray(scales)
    N = codes.shape[0]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    ks = np.arange(k0, k1)
    if fmt == "int4":
        q = INT4_TABLE[unpack_nibbles(codes[rows], k0, k1)]
        s = bf16_bits_to_f64(scales.view(np.uint16) if scales.dtype != np.uint16 else scales)
        s_nk = s[ks // group][:, rows].T                          # [rows][k]
        prod = q * s_nk                                           # exact (<= 12 significant bits)
        return f64_to_bf16_bits_via_f32(prod)
    if fmt == "fp8":
        v = E4M3_TABLE[codes[rows][:, k0:k1]]
        s = np.asarray(scales, dtype=np.float32).astype(np.float64)[rows]
        prod = v * s[:, None]                                     # exact in float64 (4 x 24 bits)
        return f64_to_bf16_bits_via_f32(prod)                     # fp32 RNE, then bf16 RNE
    if fmt == "mxfp4":
        v = E2M1_TABLE[unpack_nibbles(codes[rows], k0, k1)]
        x = E8M0_TABLE[np.asarray(scales, dtype=np.uint8)[ks // 32][:, rows].T]
        return f64_to_bf16_bits_via_f32(v * x)                    # exact: power-of-two scale
    raise ValueError(fmt)


def dequant(fmt: str, codes, scales, K: int, group: int, rows=None, k0: int = 0, k1=None) -> np.ndarray:
    """Dequantised weight values (float64, each exactly a bf16 value)."""
    return bf16_bits_to_f64(dequant_bits(fmt, codes, scales, K, group, rows, k0, k1))
