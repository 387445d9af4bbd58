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
#include "dq_pack.cuh"

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

// Dequantise 8 consecutive elements k0..k0+7 (k0 % 8 == 0) of stored row n into
// four packed bf16x2 words (element k0 in the low half of out[0]), with the same
// packed decoders the fused GEMM's producer warps use (dq_pack.cuh).
__device__ __forceinline__ void dequant8(const WeightView& w, const uint8_t* codes, const void* scales, int n, int k0,
                                         uint32_t out[4]) {
  if (w.fmt == kFmtFp8) {
    const uint2 c = *reinterpret_cast<const uint2*>(codes + static_cast<size_t>(n) * w.K + k0);
    const float s = static_cast<const float*>(scales)[n];
    uint32_t v[4];
    dq::e4m3x4(c.x, v);      // exact bf16 codes
    dq::e4m3x4(c.y, v + 2);
#pragma unroll
    for (int i = 0; i < 4; ++i)  // canonical chain: fp32 product, then bf16
      out[i] = pack_bf16x2(__fmul_rn(__uint_as_float(v[i] << 16), s), __fmul_rn(__uint_as_float(v[i] & 0xFFFF0000u), s));
    return;
  }
  const uint32_t word = *reinterpret_cast<const uint32_t*>(codes + static_cast<size_t>(n) * (w.K / 2) + k0 / 2);
  if (w.fmt == kFmtInt4) {
    const uint16_t sb = static_cast<const uint16_t*>(scales)[static_cast<size_t>(k0 / w.group) * w.N + n];
    dq::int4x8(word, dq::bf2_splat(sb), out);
    return;
  }
  const uint8_t eb = static_cast<const uint8_t*>(scales)[static_cast<size_t>(k0 / 32) * w.N + n];
  dq::mxfp4x8(word, eb, out);
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

// MXFP4 e8m0 scales -> bf16 factors 2^(e-127) (exact: e = 0 is the bf16 subnormal
// 2^-127, e = 255 is NaN), so the backward's producers apply a per-element scale
// with one multiply.
__global__ void e8m0_factor_kernel(const uint8_t* __restrict__ e, long long n, uint16_t* __restrict__ out) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t v = e[i];
  out[i] = static_cast<uint16_t>(v == 255u ? 0x7FC0u : (v == 0u ? 0x0040u : (v << 7)));
}

// Transposed copy of the codes for the backward's dequant producers:
// nibbles [N][K/2] -> [K][N/2] (NIB), or bytes [N][K] -> [K][N].  64 x 64 code tiles.
template <bool NIB>
__global__ void __launch_bounds__(256) transpose_codes_kernel(const uint8_t* __restrict__ in, int N, int K,
                                                              uint8_t* __restrict__ out) {
  __shared__ uint8_t t[64][64 + 4];  // [n][k], one code per byte
  const int n0 = blockIdx.y * 64, k0 = blockIdx.x * 64;
  const int kv = min(64, K - k0);
  constexpr int WPR = NIB ? 8 : 16;  // 32-bit words per 64 codes of a row
  for (int it = threadIdx.x; it < 64 * WPR; it += 256) {
    const int r = it / WPR, wi = it % WPR;
    const int n = n0 + r;
    uint32_t w = 0;
    if (n < N && wi * (NIB ? 8 : 4) < kv)
      w = NIB ? *reinterpret_cast<const uint32_t*>(in + static_cast<size_t>(n) * (K / 2) + k0 / 2 + 4 * wi)
              : *reinterpret_cast<const uint32_t*>(in + static_cast<size_t>(n) * K + k0 + 4 * wi);
    if (NIB) {
#pragma unroll
      for (int i = 0; i < 8; ++i) t[r][8 * wi + i] = (w >> (4 * i)) & 0xFu;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) t[r][4 * wi + i] = (w >> (8 * i)) & 0xFFu;
    }
  }
  __syncthreads();
  const int nv = min(64, N - n0);
  for (int it = threadIdx.x; it < 64 * WPR; it += 256) {
    const int kk = it / WPR, wi = it % WPR;
    const int k = k0 + kk;
    if (kk >= kv || wi * (NIB ? 8 : 4) >= nv) continue;
    uint32_t w = 0;
    if (NIB) {
#pragma unroll
      for (int i = 0; i < 8; ++i) w |= static_cast<uint32_t>(t[8 * wi + i][kk]) << (4 * i);
      *reinterpret_cast<uint32_t*>(out + static_cast<size_t>(k) * (N / 2) + n0 / 2 + 4 * wi) = w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) w |= static_cast<uint32_t>(t[4 * wi + i][kk]) << (8 * i);
      *reinterpret_cast<uint32_t*>(out + static_cast<size_t>(k) * N + n0 + 4 * wi) = w;
    }
  }
}

}  // namespace oftk
