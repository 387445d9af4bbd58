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

// out[k][n] = deq(W)[n][k], transposed in registers: lane (ro, kw) of a warp decodes
// the 8-element units of rows 8 ro .. 8 ro + 7 at unit kw of the warp's 64-column
// block, then packs each column's 8 row values into one 16-byte store with byte
// permutes.  Per warp that is 32 rows x 64 columns; for a fixed row the 8 lanes of one
// ro read contiguous codes, and for a fixed column the 4 lanes of one kw write 64
// contiguous bytes.  A CTA's 8 warps take 8 consecutive column blocks of the same 32
// rows.  N % 8 == 0 (sub-projection sizes are multiples of 8) and K % 32 == 0, so
// every octet is whole.
constexpr int kDeqTRows = 32;    // rows per CTA
constexpr int kDeqTCols = 512;   // columns (k) per CTA: 8 warps x 64

__global__ void __launch_bounds__(256) dequant_transposed_kernel(WeightView w, uint16_t* __restrict__ out) {
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ro = lane >> 3, kw = lane & 7;
  const int row0 = blockIdx.y * kDeqTRows + ro * 8;          // this lane's 8 rows
  const int k = blockIdx.x * kDeqTCols + warp * 64 + kw * 8;  // and 8 columns
  if (row0 >= w.N || k >= w.K) return;
  Raw8 raw[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) raw[m] = load8(w, w.codes, w.scales, row0 + m, k);
  uint32_t v[8][4];  // v[m][q]: row row0 + m, columns k + 2q (low half) and k + 2q + 1
#pragma unroll
  for (int m = 0; m < 8; ++m) decode8(w.fmt, raw[m], v[m]);
  uint16_t* dst = out + static_cast<size_t>(k) * w.N + row0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {  // column k + i: rows row0 .. row0 + 7
    const uint32_t sel = (i & 1) ? 0x7632u : 0x5410u;
    *reinterpret_cast<uint4*>(dst + static_cast<size_t>(i) * w.N) =
        make_uint4(__byte_perm(v[0][i >> 1], v[1][i >> 1], sel), __byte_perm(v[2][i >> 1], v[3][i >> 1], sel),
                   __byte_perm(v[4][i >> 1], v[5][i >> 1], sel), __byte_perm(v[6][i >> 1], v[7][i >> 1], sel));
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
