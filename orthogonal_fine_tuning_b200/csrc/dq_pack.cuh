// Packed register-level decoding of the frozen low-precision base weight into
// bf16 pairs, for the dequantising producer warps of the fused GEMM and for the
// standalone dequant kernels.  The base stays INT4 / FP8 / FP4 and is turned
// into BF16 only for the product ("Orbit", chooseai.io news 4086, section
// "技术原理：低精度基座 + BF16 适配器 + OFT").  Element formats follow the OCP FP8
// (e4m3fn) and OCP MX (e2m1 + e8m0) specifications.
//
// Every routine maps 32 bits of codes to bf16x2 words, element 2i in the low
// half of word i.  All results are exact (see each routine), so INT4 and MXFP4
// reproduce the canonical bf16 dequantised value bit for bit.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace oftk {
namespace dq {

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t bf2_splat(uint16_t v) { return static_cast<uint32_t>(v) * 0x10001u; }

// INT4, two's complement nibbles (element 0 in bits 0..3), one bf16 group scale
// s2 = {s, s}.  Flipping bit 3 turns q into n = q + 8 in [0, 15]; the bf16
// pattern 0x4300 | n is exactly 128 + n, so (128 + n) - 136 = q exactly, and the
// final multiply rounds q * s once: bf16_rne(q * s).
__device__ __forceinline__ void int4x8(uint32_t w, uint32_t s2, uint32_t out[4]) {
  const uint32_t t = w ^ 0x88888888u;
  const uint32_t x0 = t & 0x0F0F0F0Fu;         // elements 0, 2, 4, 6
  const uint32_t x1 = (t >> 4) & 0x0F0F0F0Fu;  // elements 1, 3, 5, 7
  const uint32_t lo = prmt(x0, x1, 0x5140u);   // bytes: e0 e1 e2 e3
  const uint32_t hi = prmt(x0, x1, 0x7362u);   // bytes: e4 e5 e6 e7
  const uint32_t C = 0x43434343u;
  const uint32_t one2 = 0x3F803F80u, m136 = 0xC308C308u;  // 1.0, -136.0
  out[0] = bf2_mul(bf2_fma(prmt(lo, C, 0x5140u), one2, m136), s2);
  out[1] = bf2_mul(bf2_fma(prmt(lo, C, 0x5342u), one2, m136), s2);
  out[2] = bf2_mul(bf2_fma(prmt(hi, C, 0x5140u), one2, m136), s2);
  out[3] = bf2_mul(bf2_fma(prmt(hi, C, 0x5342u), one2, m136), s2);
}

// The same without the scale: the exact bf16 value q of each nibble.
__device__ __forceinline__ void int4x8_q(uint32_t w, uint32_t out[4]) {
  const uint32_t t = w ^ 0x88888888u;
  const uint32_t x0 = t & 0x0F0F0F0Fu;
  const uint32_t x1 = (t >> 4) & 0x0F0F0F0Fu;
  const uint32_t lo = prmt(x0, x1, 0x5140u);
  const uint32_t hi = prmt(x0, x1, 0x7362u);
  const uint32_t C = 0x43434343u;
  const uint32_t one2 = 0x3F803F80u, m136 = 0xC308C308u;
  out[0] = bf2_fma(prmt(lo, C, 0x5140u), one2, m136);
  out[1] = bf2_fma(prmt(lo, C, 0x5342u), one2, m136);
  out[2] = bf2_fma(prmt(hi, C, 0x5140u), one2, m136);
  out[3] = bf2_fma(prmt(hi, C, 0x5342u), one2, m136);
}

// Two e4m3 codes (bytes 0 and 1 of `u`, already moved to the high byte of each
// 16-bit lane) -> exact bf16 pair.  With c = S.EEEE.MMM, the bf16 pattern
// S.0000EEEE.MMM0000 is v * 2^-120 for normal and subnormal c alike, so one
// multiply by 2^120 is exact.  (S.1111.111 is NaN in e4m3 and lands on 480;
// weights never hold it.)
__device__ __forceinline__ uint32_t e4m3x2_hi_lanes(uint32_t u) {
  const uint32_t mag = (u >> 4) & 0x07F007F0u;
  const uint32_t v = mag | (u & 0x80008000u);
  return bf2_mul(v, 0x7B807B80u);  // 2^120
}

// The same pair without the final multiply: bf16 bits of v * 2^-120 (exact).
__device__ __forceinline__ uint32_t e4m3x2_bits(uint32_t u) {
  return ((u >> 4) & 0x07F007F0u) | (u & 0x80008000u);
}

// FP8 e4m3, four codes (byte i = element i) -> four exact fp32 values.  e4m3 is a
// subset of f16 (subnormals included), so the hardware pair conversion is exact.
__device__ __forceinline__ void e4m3x4_f32(uint32_t w, float (&out)[4]) {
  uint32_t h0, h1;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h0) : "h"(static_cast<uint16_t>(w & 0xFFFFu)));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h1) : "h"(static_cast<uint16_t>(w >> 16)));
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h0));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&h1));
  out[0] = a.x, out[1] = a.y, out[2] = b.x, out[3] = b.y;
}

// FP8 e4m3, four codes (byte i = element i) -> 2 exact bf16 pairs (no scale).
__device__ __forceinline__ void e4m3x4(uint32_t w, uint32_t out[2]) {
  out[0] = e4m3x2_hi_lanes(prmt(w, 0u, 0x1404u));  // bytes 0, 1 -> high byte of each lane
  out[1] = e4m3x2_hi_lanes(prmt(w, 0u, 0x3424u));  // bytes 2, 3
}

// MXFP4, e2m1 nibbles (element 0 in bits 0..3), e8m0 scale e.
// The bf16 pattern S.00000EE.M000000 (the three magnitude bits of c = S.EE.M in
// bits 8..6) is v * 2^-126 for every e2m1 value v (EE = 0 is the subnormal
// 0.5 * M), so multiplying by 2^(e - 1) gives v * 2^(e - 127) exactly; for
// e > 128 the factor is applied in two exact steps.
__device__ __forceinline__ uint32_t e2m1x2_lanes(uint32_t p, uint32_t f2, uint32_t g2, bool two_step) {
  // p: codes in the low nibble of each 16-bit lane
  const uint32_t v = ((p << 6) & 0x01C001C0u) | ((p << 12) & 0x80008000u);
  const uint32_t r = bf2_mul(v, f2);
  return two_step ? bf2_mul(r, g2) : r;
}

__device__ __forceinline__ void mxfp4x8(uint32_t w, uint32_t e, uint32_t out[4]) {
  const uint32_t x0 = w & 0x0F0F0F0Fu;
  const uint32_t x1 = (w >> 4) & 0x0F0F0F0Fu;
  const uint32_t lo = prmt(x0, x1, 0x5140u);
  const uint32_t hi = prmt(x0, x1, 0x7362u);
  const bool two_step = e > 128u;
  // factor 2^(e-1) (bf16 exponent field e + 126), or 2^126 followed by 2^(e-127)
  const uint32_t f = two_step ? 0x7E80u : ((e + 126u) << 7);
  const uint32_t g = (e == 255u) ? 0x7FC0u : ((e - 127u + 127u) << 7);  // 2^(e-127), only used when e > 128
  const uint32_t f2 = f * 0x10001u, g2 = g * 0x10001u;
  out[0] = e2m1x2_lanes(prmt(lo, 0u, 0x4140u), f2, g2, two_step);
  out[1] = e2m1x2_lanes(prmt(lo, 0u, 0x4342u), f2, g2, two_step);
  out[2] = e2m1x2_lanes(prmt(hi, 0u, 0x4140u), f2, g2, two_step);
  out[3] = e2m1x2_lanes(prmt(hi, 0u, 0x4342u), f2, g2, two_step);
}

// The same result as mxfp4x8 with fewer instructions per pair: one multiply places
// the nibble at both bit 6 (magnitude) and bit 12 (so the sign lands on bit 15),
// and one mask keeps bits 6..8 and 15.  (p * 0x1040 = p << 6 | p << 12: the two
// copies do not overlap, and neither crosses into the other 16-bit lane.)
__device__ __forceinline__ uint32_t e2m1x2_lanes_mul(uint32_t p, uint32_t f2, uint32_t g2, bool two_step) {
  const uint32_t v = (p * 0x1040u) & 0x81C081C0u;
  const uint32_t r = bf2_mul(v, f2);
  return two_step ? bf2_mul(r, g2) : r;
}

__device__ __forceinline__ void mxfp4x8_mul(uint32_t w, uint32_t e, uint32_t out[4]) {
  const uint32_t x0 = w & 0x0F0F0F0Fu;
  const uint32_t x1 = (w >> 4) & 0x0F0F0F0Fu;
  const uint32_t lo = prmt(x0, x1, 0x5140u);
  const uint32_t hi = prmt(x0, x1, 0x7362u);
  const bool two_step = e > 128u;
  const uint32_t f = two_step ? 0x7E80u : ((e + 126u) << 7);
  const uint32_t g = (e == 255u) ? 0x7FC0u : (e << 7);
  const uint32_t f2 = f * 0x10001u, g2 = g * 0x10001u;
  out[0] = e2m1x2_lanes_mul(prmt(lo, 0u, 0x4140u), f2, g2, two_step);
  out[1] = e2m1x2_lanes_mul(prmt(lo, 0u, 0x4342u), f2, g2, two_step);
  out[2] = e2m1x2_lanes_mul(prmt(hi, 0u, 0x4140u), f2, g2, two_step);
  out[3] = e2m1x2_lanes_mul(prmt(hi, 0u, 0x4342u), f2, g2, two_step);
}

// mxfp4x8_mul for four words sharing one e8m0 scale (a 32-element group), with the
// choice between the one-step factor (e <= 128, every realistic weight) and the
// two-step one taken once for the group rather than per pair.
__device__ __forceinline__ void mxfp4x32_mul(const uint32_t (&w)[4], uint32_t e, uint32_t (&out)[16]) {
  if (e <= 128u) {
    const uint32_t f2 = ((e + 126u) << 7) * 0x10001u;  // 2^(e-1)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t x0 = w[i] & 0x0F0F0F0Fu;
      const uint32_t x1 = (w[i] >> 4) & 0x0F0F0F0Fu;
      const uint32_t lo = prmt(x0, x1, 0x5140u);
      const uint32_t hi = prmt(x0, x1, 0x7362u);
      out[4 * i] = bf2_mul((prmt(lo, 0u, 0x4140u) * 0x1040u) & 0x81C081C0u, f2);
      out[4 * i + 1] = bf2_mul((prmt(lo, 0u, 0x4342u) * 0x1040u) & 0x81C081C0u, f2);
      out[4 * i + 2] = bf2_mul((prmt(hi, 0u, 0x4140u) * 0x1040u) & 0x81C081C0u, f2);
      out[4 * i + 3] = bf2_mul((prmt(hi, 0u, 0x4342u) * 0x1040u) & 0x81C081C0u, f2);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t t[4];
      mxfp4x8_mul(w[i], e, t);
      out[4 * i] = t[0], out[4 * i + 1] = t[1], out[4 * i + 2] = t[2], out[4 * i + 3] = t[3];
    }
  }
}

}  // namespace dq
}  // namespace oftk
