// Group-wise dequantisation of the frozen base weight to bf16 (bit-exact).
//
// The frozen base stays in its deployment precision -- INT4, FP4 or FP8 -- and
// is turned into BF16 only for the product with the BF16-adapted activations
// ("Orbit", chooseai.io news 4086, section "技术原理：低精度基座 + BF16 适配器 + OFT").
// Element formats follow the OCP FP8 (e4m3fn) and OCP MX (e2m1 + e8m0) specs.
//
//   INT4  : w = bf16_rne(q * s)              q two's complement nibble, s bf16 per (k/G, n)
//   FP8   : w = bf16_rne(f32_rne(v * s_n))   v e4m3 value, s_n fp32 per output channel
//   MXFP4 : w = bf16(v * 2^(e-127))          v e2m1 value, e e8m0 per (k/32, n); exact
#pragma once

#include "common.cuh"

namespace oftk {

enum : int { kFmtInt4 = 1, kFmtFp8 = 2, kFmtMxfp4 = 3 };

struct WeightView {
  int fmt;
  const uint8_t* codes;   // [N][K/2] or [N][K]
  const void* scales;     // see fmt
  int N, K, group;
  long long codes_expert_stride;   // bytes between experts (bank only)
  long long scales_expert_stride;  // bytes between experts (bank only)
};

// OCP e4m3fn -> fp32, from the format definition (bias 7, subnormal m * 2^-9,
// S.1111.111 = NaN).  Exact.
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  const uint32_t s = (c & 0x80u) << 24;
  const uint32_t e = (c >> 3) & 0xFu;
  const uint32_t m = c & 0x7u;
  if (e == 0xFu && m == 0x7u) return __uint_as_float(s | 0x7FC00000u);
  if (e == 0u) {
    const float v = static_cast<float>(m) * 0.001953125f;  // m * 2^-9, exact
    return s ? -v : v;
  }
  return __uint_as_float(s | ((e + 120u) << 23) | (m << 20));
}

// OCP e2m1 -> fp32 (bias 1, subnormal m * 0.5).  Exact.
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
  const uint32_t s = (c & 0x8u) << 28;
  const uint32_t e = (c >> 1) & 0x3u;
  const uint32_t m = c & 0x1u;
  if (e == 0u) return __uint_as_float(s | (m ? 0x3F000000u : 0u));
  return __uint_as_float(s | ((e + 126u) << 23) | (m << 22));
}

// OCP e8m0 -> fp32: 2^(e-127); 0 is the subnormal 2^-127; 255 is NaN.
__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
  if (e == 255u) return __uint_as_float(0x7FC00000u);
  if (e == 0u) return __uint_as_float(0x00400000u);
  return __uint_as_float(e << 23);
}

__device__ __forceinline__ float int4_to_f32(uint32_t nib) {
  return static_cast<float>(static_cast<int>(nib ^ 8u) - 8);
}

// Dequantise 8 consecutive elements k0..k0+7 (k0 % 8 == 0) of stored row n into
// four packed bf16x2 words (element k0 in the low half of out[0]).
__device__ __forceinline__ void dequant8(const WeightView& w, const uint8_t* codes, const void* scales, int n, int k0,
                                         uint32_t out[4]) {
  if (w.fmt == kFmtFp8) {
    const uint2 c = *reinterpret_cast<const uint2*>(codes + static_cast<size_t>(n) * w.K + k0);
    const float s = static_cast<const float*>(scales)[n];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t word = i < 2 ? c.x : c.y;
      const uint32_t sh = (i & 1) * 16;
      const float a = __fmul_rn(e4m3_to_f32((word >> sh) & 0xFFu), s);
      const float b = __fmul_rn(e4m3_to_f32((word >> (sh + 8)) & 0xFFu), s);
      out[i] = pack_bf16x2(a, b);
    }
    return;
  }
  const uint32_t word = *reinterpret_cast<const uint32_t*>(codes + static_cast<size_t>(n) * (w.K / 2) + k0 / 2);
  if (w.fmt == kFmtInt4) {
    const uint16_t sb = static_cast<const uint16_t*>(scales)[static_cast<size_t>(k0 / w.group) * w.N + n];
    const float s = bf16_bits_to_f32(sb);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = __fmul_rn(int4_to_f32((word >> (8 * i)) & 0xFu), s);  // exact in fp32
      const float b = __fmul_rn(int4_to_f32((word >> (8 * i + 4)) & 0xFu), s);
      out[i] = pack_bf16x2(a, b);
    }
    return;
  }
  // MXFP4
  const uint8_t eb = static_cast<const uint8_t*>(scales)[static_cast<size_t>(k0 / 32) * w.N + n];
  const float x = e8m0_to_f32(eb);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = e2m1_to_f32((word >> (8 * i)) & 0xFu) * x;          // exact
    const float b = e2m1_to_f32((word >> (8 * i + 4)) & 0xFu) * x;
    out[i] = pack_bf16x2(a, b);
  }
}

// out[n][k] = deq(W)[n][k] for all n < N, k < K.  One thread per 8 elements.
__global__ void __launch_bounds__(256) dequant_rows_kernel(WeightView w, uint16_t* __restrict__ out) {
  const long long units = static_cast<long long>(w.N) * (w.K / 8);
  for (long long u = blockIdx.x * 256ll + threadIdx.x; u < units; u += static_cast<long long>(gridDim.x) * 256) {
    const int n = static_cast<int>(u / (w.K / 8));
    const int k0 = static_cast<int>(u % (w.K / 8)) * 8;
    uint32_t v[4];
    dequant8(w, w.codes, w.scales, n, k0, v);
    *reinterpret_cast<uint4*>(out + static_cast<size_t>(n) * w.K + k0) = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

// out[k][n] = deq(W)[n][k]: 64 x 64 tiles transposed through shared memory.
__global__ void __launch_bounds__(256) dequant_transposed_kernel(WeightView w, uint16_t* __restrict__ out) {
  __shared__ uint16_t tile[64][64 + 8];
  const int n0 = blockIdx.y * 64;
  const int k0 = blockIdx.x * 64;
  // load: 64 rows (n) x 8 chunks of 8 k
  for (int it = threadIdx.x; it < 512; it += 256) {
    const int r = it >> 3, c = it & 7;
    const int n = n0 + r, k = k0 + c * 8;
    uint32_t v[4] = {0, 0, 0, 0};
    if (n < w.N && k < w.K) dequant8(w, w.codes, w.scales, n, k, v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      tile[r][c * 8 + 2 * i] = static_cast<uint16_t>(v[i] & 0xFFFFu);
      tile[r][c * 8 + 2 * i + 1] = static_cast<uint16_t>(v[i] >> 16);
    }
  }
  __syncthreads();
  // store: 64 rows (k) x 8 chunks of 8 n
  for (int it = threadIdx.x; it < 512; it += 256) {
    const int r = it >> 3, c = it & 7;
    const int k = k0 + r, n = n0 + c * 8;
    if (k >= w.K || n >= w.N) continue;
    uint32_t v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      v[i] = static_cast<uint32_t>(tile[c * 8 + 2 * i][r]) | (static_cast<uint32_t>(tile[c * 8 + 2 * i + 1][r]) << 16);
    if (n + 8 <= w.N) {
      *reinterpret_cast<uint4*>(out + static_cast<size_t>(k) * w.N + n) = make_uint4(v[0], v[1], v[2], v[3]);
    } else {
      for (int i = 0; i < 8 && n + i < w.N; ++i)
        out[static_cast<size_t>(k) * w.N + n + i] = static_cast<uint16_t>((v[i / 2] >> (16 * (i & 1))) & 0xFFFFu);
    }
  }
}

// MoE: dequantise the experts of chunk `chunk_idx` into buf[slot][N][K].
// grid = (blocks per expert, chunk slots).  Slots without an expert (-1) do nothing.
__global__ void __launch_bounds__(256) moe_chunk_dequant_kernel(WeightView bank, const int* __restrict__ chunk_table,
                                                                int chunk_idx, int chunk, uint16_t* __restrict__ buf) {
  const int slot = blockIdx.y;
  const int e = chunk_table[chunk_idx * chunk + slot];
  if (e < 0) return;
  const uint8_t* codes = bank.codes + static_cast<long long>(e) * bank.codes_expert_stride;
  const void* scales = static_cast<const uint8_t*>(bank.scales) + static_cast<long long>(e) * bank.scales_expert_stride;
  uint16_t* out = buf + static_cast<size_t>(slot) * bank.N * bank.K;
  const long long units = static_cast<long long>(bank.N) * (bank.K / 8);
  for (long long u = blockIdx.x * 256ll + threadIdx.x; u < units; u += static_cast<long long>(gridDim.x) * 256) {
    const int n = static_cast<int>(u / (bank.K / 8));
    const int k0 = static_cast<int>(u % (bank.K / 8)) * 8;
    uint32_t v[4];
    dequant8(bank, codes, scales, n, k0, v);
    *reinterpret_cast<uint4*>(out + static_cast<size_t>(n) * bank.K + k0) = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

}  // namespace oftk
