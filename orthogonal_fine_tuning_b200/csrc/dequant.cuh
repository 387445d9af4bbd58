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

// The codes and scale of 8 consecutive elements k0..k0+7 (k0 % 8 == 0) of stored row
// n, loaded ahead of their decode.
struct Raw8 {
  uint32_t c0, c1;  // FP8: 8 codes; INT4 / MXFP4: c0 holds 8 nibbles
  uint32_t s;       // FP8: fp32 bits; INT4: bf16 bits; MXFP4: e8m0
};

__device__ __forceinline__ Raw8 load8(const WeightView& w, const uint8_t* codes, const void* scales, int n, int k0) {
  Raw8 r;
  if (w.fmt == kFmtFp8) {
    const uint2 c = *reinterpret_cast<const uint2*>(codes + static_cast<size_t>(n) * w.K + k0);
    r.c0 = c.x;
    r.c1 = c.y;
    r.s = __float_as_uint(static_cast<const float*>(scales)[n]);
    return r;
  }
  r.c0 = *reinterpret_cast<const uint32_t*>(codes + static_cast<size_t>(n) * (w.K / 2) + k0 / 2);
  r.c1 = 0;
  r.s = w.fmt == kFmtInt4 ? static_cast<const uint16_t*>(scales)[static_cast<size_t>(k0 / w.group) * w.N + n]
                          : static_cast<const uint8_t*>(scales)[static_cast<size_t>(k0 / 32) * w.N + n];
  return r;
}

// The 8 elements as four packed bf16x2 words (element k0 in the low half of out[0]),
// with the same packed decoders the fused GEMM's producer warps use (dq_pack.cuh).
__device__ __forceinline__ void decode8(int fmt, const Raw8& r, uint32_t out[4]) {
  if (fmt == kFmtFp8) {
    const float s = __uint_as_float(r.s);
    uint32_t v[4];
    dq::e4m3x4(r.c0, v);      // exact bf16 codes
    dq::e4m3x4(r.c1, v + 2);
#pragma unroll
    for (int i = 0; i < 4; ++i)  // canonical chain: fp32 product, then bf16
      out[i] = pack_bf16x2(__fmul_rn(__uint_as_float(v[i] << 16), s), __fmul_rn(__uint_as_float(v[i] & 0xFFFF0000u), s));
    return;
  }
  if (fmt == kFmtInt4) {
    dq::int4x8(r.c0, dq::bf2_splat(static_cast<uint16_t>(r.s)), out);
    return;
  }
  dq::mxfp4x8(r.c0, r.s, out);
}

// Dequantise 8 consecutive elements k0..k0+7 (k0 % 8 == 0) of stored row n into
// four packed bf16x2 words.
__device__ __forceinline__ void dequant8(const WeightView& w, const uint8_t* codes, const void* scales, int n, int k0,
                                         uint32_t out[4]) {
  decode8(w.fmt, load8(w, codes, scales, n, k0), out);
}

// out[n][k] = deq(W)[n][k] for all n < N, k < K.  A unit is 8 consecutive elements
// of a row; each thread takes four units a stride apart per pass, so four code
// loads are in flight before the first decode.  N * K / 8 < 2^31 (checked on the host).
__global__ void __launch_bounds__(256) dequant_rows_kernel(WeightView w, uint16_t* __restrict__ out) {
  pdl_wait();
  const int per_row = w.K / 8;
  const int units = w.N * per_row;
  const int stride = gridDim.x * 256;
  for (int u0 = blockIdx.x * 256 + threadIdx.x; u0 < units; u0 += 4 * stride) {
    uint32_t v[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int u = u0 + j * stride;
      if (u < units) dequant8(w, w.codes, w.scales, u / per_row, (u % per_row) * 8, v[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int u = u0 + j * stride;
      if (u < units)
        *reinterpret_cast<uint4*>(out + static_cast<size_t>(u) * 8) = make_uint4(v[j][0], v[j][1], v[j][2], v[j][3]);
    }
  }
}

// out[k][n] = deq(W)[n][k]: 64 x 64 tiles transposed through shared memory as
// 32-bit words (two k per word, rows padded to 33 words), so neither the decode
// side nor the transposed side has bank conflicts; each warp stores 64-byte runs of
// 8 k-rows.  A CTA walks a strip of kDeqTStrip tiles along K with every code and
// scale load of the strip issued before the first decode.
// grid = (ceil(K / (64 * kDeqTStrip)), ceil(N / 64)).
constexpr int kDeqTStrip = 4;

__global__ void __launch_bounds__(256) dequant_transposed_kernel(WeightView w, uint16_t* __restrict__ out) {
  __shared__ uint32_t tile[64][33];  // [row n][k pair]
  pdl_wait();
  const int n0 = blockIdx.y * 64;
  const int kb = blockIdx.x * 64 * kDeqTStrip;
  Raw8 raw[kDeqTStrip][2];
#pragma unroll
  for (int t = 0; t < kDeqTStrip; ++t)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int it = threadIdx.x + 256 * h;
      const int n = n0 + (it >> 3), k = kb + t * 64 + (it & 7) * 8;
      raw[t][h] = (n < w.N && k < w.K) ? load8(w, w.codes, w.scales, n, k) : Raw8{0u, 0u, 0u};
    }
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int t = 0; t < kDeqTStrip; ++t) {
    const int k0 = kb + t * 64;
    if (k0 >= w.K) break;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int it = threadIdx.x + 256 * h;
      const int r = it >> 3, c = it & 7;  // row n0 + r, k = k0 + 8c .. +7
      uint32_t v[4] = {0, 0, 0, 0};
      if (n0 + r < w.N && k0 + c * 8 < w.K) decode8(w.fmt, raw[t][h], v);
#pragma unroll
      for (int i = 0; i < 4; ++i) tile[r][c * 4 + i] = v[i];
    }
    __syncthreads();
    for (int it = threadIdx.x; it < 512; it += 256) {
      const int q = it >> 5;
      const int r = (lane & 7) + 8 * (q & 7);    // k row
      const int c = (lane >> 3) + 4 * (q >> 3);  // 8 consecutive n
      const int k = k0 + r, n = n0 + c * 8;
      if (k >= w.K || n >= w.N) continue;
      const int sh = (r & 1) * 16;
      uint32_t v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        v[i] = ((tile[c * 8 + 2 * i][r >> 1] >> sh) & 0xFFFFu) | (((tile[c * 8 + 2 * i + 1][r >> 1] >> sh) & 0xFFFFu) << 16);
      if (n + 8 <= w.N) {
        *reinterpret_cast<uint4*>(out + static_cast<size_t>(k) * w.N + n) = make_uint4(v[0], v[1], v[2], v[3]);
      } else {
        for (int i = 0; i < 8 && n + i < w.N; ++i)
          out[static_cast<size_t>(k) * w.N + n + i] = static_cast<uint16_t>((v[i / 2] >> (16 * (i & 1))) & 0xFFFFu);
      }
    }
    __syncthreads();  // the tile is free for the next
  }
}

// MoE: dequantise the experts of chunk `chunk_idx` into buf[slot][N][K] (INT4 bank).
// grid = (ceil(N / 32) row tiles, chunk slots); slots without an expert (-1) do
// nothing.  A CTA takes 32 rows of one expert: their K/G group scales are staged
// in shared memory row-major, then each warp walks whole rows, lane l decoding
// the 8 codes of word l + 32 i, so every load and store instruction of a warp
// covers contiguous memory (128 B of codes in, 512 B of bf16 out).
constexpr int kChunkRows = 32;  // small enough (staged scales ~14 KB) to co-reside with the grouped GEMM

__host__ __device__ constexpr int chunk_scale_ld(int groups) { return groups + 2; }

__global__ void __launch_bounds__(256) moe_chunk_dequant_kernel(WeightView bank, const int* __restrict__ chunk_table,
                                                                int chunk_idx, int chunk, uint16_t* __restrict__ buf) {
  extern __shared__ uint16_t s_scale[];  // [kChunkRows][K/G + 2]
  const int slot = blockIdx.y;
  const int e = chunk_table[chunk_idx * chunk + slot];
  if (e < 0) return;
  const int N = bank.N, K = bank.K, G = bank.group;
  const int ng = K / G, ld = chunk_scale_ld(ng);
  const int n0 = blockIdx.x * kChunkRows, rows = min(kChunkRows, N - n0);
  const uint32_t* codes = reinterpret_cast<const uint32_t*>(bank.codes + static_cast<long long>(e) * bank.codes_expert_stride);
  const uint16_t* S = reinterpret_cast<const uint16_t*>(static_cast<const uint8_t*>(bank.scales) +
                                                        static_cast<long long>(e) * bank.scales_expert_stride);
  for (int it = threadIdx.x; it < ng * kChunkRows; it += 256) {
    const int j = it / kChunkRows, r = it % kChunkRows;
    if (r < rows) s_scale[r * ld + j] = S[static_cast<size_t>(j) * N + n0 + r];
  }
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int words = K / 8;  // 8 codes per 32-bit word
  uint16_t* out = buf + (static_cast<size_t>(slot) * N + n0) * K;
  for (int r = warp; r < rows; r += 8) {
    const uint32_t* crow = codes + static_cast<size_t>(n0 + r) * words;
    const uint16_t* srow = s_scale + r * ld;
    uint4* orow = reinterpret_cast<uint4*>(out + static_cast<size_t>(r) * K);
    int w = lane;
    for (; w + 96 < words; w += 128) {  // four independent loads in flight per lane
      uint32_t c[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) c[u] = crow[w + 32 * u];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int wu = w + 32 * u;
        uint32_t v[4];
        dq::int4x8(c[u], dq::bf2_splat(srow[(wu * 8) / G]), v);
        orow[wu] = make_uint4(v[0], v[1], v[2], v[3]);
      }
    }
    for (; w < words; w += 32) {
      uint32_t v[4];
      dq::int4x8(crow[w], dq::bf2_splat(srow[(w * 8) / G]), v);
      orow[w] = make_uint4(v[0], v[1], v[2], v[3]);
    }
  }
}

// MXFP4 e8m0 scales -> bf16 factors 2^(e-127) (exact: e = 0 is the bf16 subnormal
// 2^-127, e = 255 is NaN), so the backward's producers apply a per-element scale
// with one multiply.
__global__ void e8m0_factor_kernel(const uint8_t* __restrict__ e, long long n, uint16_t* __restrict__ out) {
  pdl_wait();
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t v = e[i];
  out[i] = static_cast<uint16_t>(v == 255u ? 0x7FC0u : (v == 0u ? 0x0040u : (v << 7)));
}

// Code layout for the backward's dequant producers.  In the dX' product the weight
// rows are input features k and the reduction runs over the output channels n of
// one sub-projection.  For sub-projection g, row tile tw (128 features) and k-step
// ks (64 channels from the sub-projection's first), one block holds 128 rows x 64
// codes as [16-byte vector v][row r]: the 32 rows of a warp read 512 contiguous
// bytes per load.  Features past K and channels past the sub-projection's end
// are zero codes, so the producers never test bounds.
struct PackBwdParams {
  int num_groups;
  int blk0[5];          // first CTA (block) of each group; blk0[num_groups] = total
  int n0[4], np[4];     // channel range of each group
  int nk[4];            // k-steps of each group: ceil(np / 64)
  long long off[4];     // byte offset of each group's first block
};

template <bool NIB>
__global__ void __launch_bounds__(256) pack_codes_bwd_kernel(const uint8_t* __restrict__ in, int N, int K,
                                                             PackBwdParams pp, uint8_t* __restrict__ out) {
  __shared__ uint8_t t[64][128 + 4];  // [channel][feature], one code per byte
  pdl_wait();
  int g = 0;
  while (g + 1 < pp.num_groups && static_cast<int>(blockIdx.x) >= pp.blk0[g + 1]) ++g;
  const int local = static_cast<int>(blockIdx.x) - pp.blk0[g];
  const int tw = local / pp.nk[g], ks = local % pp.nk[g];
  const int k0 = tw * 128;
  const int nbeg = pp.n0[g] + ks * 64;
  const int nv = min(64, pp.n0[g] + pp.np[g] - nbeg);  // channels present
  const int kv = min(128, K - k0);                      // features present
  constexpr int WPR = NIB ? 16 : 32;                    // 32-bit input words per 128 features
  constexpr int CPW = NIB ? 8 : 4;                      // codes per word
  for (int it = threadIdx.x; it < 64 * WPR; it += 256) {
    const int r = it / WPR, wi = it % WPR;
    uint32_t w = 0;
    if (r < nv && wi * CPW < kv) {
      const size_t row = static_cast<size_t>(nbeg + r);
      w = NIB ? *reinterpret_cast<const uint32_t*>(in + row * (K / 2) + k0 / 2 + 4 * wi)
              : *reinterpret_cast<const uint32_t*>(in + row * K + k0 + 4 * wi);
    }
#pragma unroll
    for (int i = 0; i < CPW; ++i) t[r][CPW * wi + i] = NIB ? ((w >> (4 * i)) & 0xFu) : ((w >> (8 * i)) & 0xFFu);
  }
  __syncthreads();
  constexpr int NV4 = NIB ? 2 : 4;   // 16-byte vectors per row (64 codes)
  constexpr int CPV = 64 / NV4;      // codes per vector
  uint4* dst = reinterpret_cast<uint4*>(out + pp.off[g] + static_cast<size_t>(local) * (NV4 * 128 * 16));
  for (int it = threadIdx.x; it < NV4 * 128; it += 256) {
    const int v = it / 128, r = it % 128;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t x = 0;
#pragma unroll
      for (int i = 0; i < CPW; ++i) {
        const uint32_t c = t[v * CPV + q * CPW + i][r];
        x |= NIB ? (c << (4 * i)) : (c << (8 * i));
      }
      w[q] = x;
    }
    dst[v * 128 + r] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace oftk
