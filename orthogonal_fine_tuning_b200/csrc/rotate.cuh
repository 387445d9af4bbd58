// Block-diagonal rotations of the OFT adapter on CUDA cores.
//
//   forward : X'_p[:, blk] = X[:, blk] R_p,blk                  (R^T applied to each token)
//   dX      : dX[:, blk]  = sum_p dX'_p[:, blk] R_p,blk^T
//   dR      : G_p,blk     = X[:, blk]^T dX'_p[:, blk]          (reduction over tokens)
//
// One independent rotation per sub-projection of a fused weight is the
// split-projection adapter (chooseai.io news 4086, item "自定义适配器核函数" and item
// "分投影适配器支持").  All three are blocked b x b products with fp32
// accumulation; tiles of 64 tokens x one block are staged in shared memory as
// fp32, rows padded to keep 16-byte alignment for vector loads.
#pragma once

#include "common.cuh"

namespace oftk {

constexpr int kRotTokens = 64;
constexpr int kRotThreads = 256;

template <int B>
struct RotCfg {
  static constexpr int LD = B + 4;                   // padded row (floats), multiple of 4
  static constexpr int TPT = kRotTokens * B / kRotThreads;  // tokens per thread (B/4)
};

// Load a [64 x B] fp32 tile (rows m0.., cols col0..) into shared memory.
template <int B>
__device__ __forceinline__ void load_tile_f32(const float* __restrict__ src, int M, int ld_src, int m0, int col0,
                                              float* __restrict__ dst) {
  constexpr int CH = B / 4;  // 16-byte chunks per row
  for (int it = threadIdx.x; it < kRotTokens * CH; it += kRotThreads) {
    const int r = it / CH, c = it % CH;
    const int m = m0 + r;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (m < M) v = *reinterpret_cast<const float4*>(src + static_cast<size_t>(m) * ld_src + col0 + c * 4);
    *reinterpret_cast<float4*>(dst + r * RotCfg<B>::LD + c * 4) = v;
  }
}

// Load a [64 x B] bf16 tile (rows m0.., cols col0..) into fp32 shared memory.
template <int B>
__device__ __forceinline__ void load_tile_bf16(const uint16_t* __restrict__ src, int M, int ld_src, int m0, int col0,
                                               float* __restrict__ dst) {
  constexpr int CH = B / 8;  // 16-byte chunks per row
  for (int it = threadIdx.x; it < kRotTokens * CH; it += kRotThreads) {
    const int r = it / CH, c = it % CH;
    const int m = m0 + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (m < M) v = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(m) * ld_src + col0 + c * 8);
    float* d = dst + r * RotCfg<B>::LD + c * 8;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      d[2 * i] = __uint_as_float(w[i] << 16);
      d[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// Xr[p][m][j*B + c] = sum_i X[m][j*B + i] R[p][j][i][c]
// grid = (K/B, ceil(M/64)).  One column per thread, TPT tokens per thread.
template <int B>
__global__ void __launch_bounds__(kRotThreads) rotate_fwd_kernel(const uint16_t* __restrict__ X, int M, int K, int P,
                                                                 const float* __restrict__ R,
                                                                 uint16_t* __restrict__ Xr) {
  constexpr int LD = RotCfg<B>::LD, TPT = RotCfg<B>::TPT;
  __shared__ __align__(16) float xs[kRotTokens * LD];
  __shared__ __align__(16) float rs[B * B];
  const int j = blockIdx.x, m0 = blockIdx.y * kRotTokens, nb = K / B;
  const int c = threadIdx.x % B, tg = threadIdx.x / B;
  load_tile_bf16<B>(X, M, K, m0, j * B, xs);
  for (int p = 0; p < P; ++p) {
    const float* Rb = R + (static_cast<size_t>(p) * nb + j) * B * B;
    for (int idx = threadIdx.x; idx < B * B / 4; idx += kRotThreads)
      reinterpret_cast<float4*>(rs)[idx] = reinterpret_cast<const float4*>(Rb)[idx];
    __syncthreads();
    float acc[TPT];
#pragma unroll
    for (int t = 0; t < TPT; ++t) acc[t] = 0.f;
#pragma unroll 4
    for (int i = 0; i < B; i += 4) {
      const float r0 = rs[(i + 0) * B + c], r1 = rs[(i + 1) * B + c];
      const float r2 = rs[(i + 2) * B + c], r3 = rs[(i + 3) * B + c];
#pragma unroll
      for (int t = 0; t < TPT; ++t) {
        const float4 x = *reinterpret_cast<const float4*>(xs + (tg * TPT + t) * LD + i);
        acc[t] = fmaf(x.x, r0, acc[t]);
        acc[t] = fmaf(x.y, r1, acc[t]);
        acc[t] = fmaf(x.z, r2, acc[t]);
        acc[t] = fmaf(x.w, r3, acc[t]);
      }
    }
    uint16_t* out = Xr + static_cast<size_t>(p) * M * K;
#pragma unroll
    for (int t = 0; t < TPT; ++t) {
      const int m = m0 + tg * TPT + t;
      if (m < M) out[static_cast<size_t>(m) * K + j * B + c] = f32_to_bf16_bits(acc[t]);
    }
    __syncthreads();
  }
}

// dX[m][j*B + i] = sum_p sum_l D[p][m][j*B + l] R[p][j][i][l]     (D = dX' in fp32)
template <int B>
__global__ void __launch_bounds__(kRotThreads) rotate_bwd_kernel(const float* __restrict__ D, int M, int K, int P,
                                                                 const float* __restrict__ R,
                                                                 uint16_t* __restrict__ dX) {
  constexpr int LD = RotCfg<B>::LD, TPT = RotCfg<B>::TPT;
  __shared__ __align__(16) float ds[kRotTokens * LD];
  __shared__ __align__(16) float rt[B * B];  // rt[l][i] = R[i][l]
  const int j = blockIdx.x, m0 = blockIdx.y * kRotTokens, nb = K / B;
  const int c = threadIdx.x % B, tg = threadIdx.x / B;
  float acc[TPT];
#pragma unroll
  for (int t = 0; t < TPT; ++t) acc[t] = 0.f;
  for (int p = 0; p < P; ++p) {
    load_tile_f32<B>(D + static_cast<size_t>(p) * M * K, M, K, m0, j * B, ds);
    const float* Rb = R + (static_cast<size_t>(p) * nb + j) * B * B;
    for (int idx = threadIdx.x; idx < B * B; idx += kRotThreads) {
      const int i = idx / B, l = idx % B;
      rt[l * B + i] = Rb[idx];
    }
    __syncthreads();
#pragma unroll 4
    for (int l = 0; l < B; l += 4) {
      const float r0 = rt[(l + 0) * B + c], r1 = rt[(l + 1) * B + c];
      const float r2 = rt[(l + 2) * B + c], r3 = rt[(l + 3) * B + c];
#pragma unroll
      for (int t = 0; t < TPT; ++t) {
        const float4 x = *reinterpret_cast<const float4*>(ds + (tg * TPT + t) * LD + l);
        acc[t] = fmaf(x.x, r0, acc[t]);
        acc[t] = fmaf(x.y, r1, acc[t]);
        acc[t] = fmaf(x.z, r2, acc[t]);
        acc[t] = fmaf(x.w, r3, acc[t]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int t = 0; t < TPT; ++t) {
    const int m = m0 + tg * TPT + t;
    if (m < M) dX[static_cast<size_t>(m) * K + j * B + c] = f32_to_bf16_bits(acc[t]);
  }
}

// Partial G: Gp[(p*nb + j)][part][i][l] = sum_{m in part} X[m][j*B+i] D[p][m][j*B+l]
// grid = (nb, P, nparts).  Each thread owns a TI x TL sub-block of the B x B result.
template <int B>
struct GCfg {
  static constexpr int TI = (B == 64) ? 4 : (B == 32 ? 2 : 1);
  static constexpr int TL = TI;
  static constexpr int NI = B / TI;  // threads along i
  static constexpr int NL = B / TL;  // threads along l
  static_assert(NI * NL == kRotThreads, "G tiling must use all threads");
};

constexpr int kGTok = 32;

template <int B>
__global__ void __launch_bounds__(kRotThreads) rot_grad_partial_kernel(const uint16_t* __restrict__ X,
                                                                       const float* __restrict__ D, int M, int K,
                                                                       int tokens_per_part, float* __restrict__ Gp) {
  constexpr int TI = GCfg<B>::TI, TL = GCfg<B>::TL, NL = GCfg<B>::NL;
  constexpr int LD = B + 4;
  __shared__ __align__(16) float xs[kGTok * LD];
  __shared__ __align__(16) float ds[kGTok * LD];
  const int j = blockIdx.x, p = blockIdx.y, part = blockIdx.z;
  const int nb = K / B, nparts = gridDim.z;
  const int ib = (threadIdx.x / NL) * TI, lb = (threadIdx.x % NL) * TL;
  const float* Dp = D + static_cast<size_t>(p) * M * K;
  float acc[TI][TL];
#pragma unroll
  for (int a = 0; a < TI; ++a)
#pragma unroll
    for (int c = 0; c < TL; ++c) acc[a][c] = 0.f;
  const int mbeg = part * tokens_per_part;
  const int mend = min(M, mbeg + tokens_per_part);
  constexpr int CH = B / 8;   // 16-byte bf16 chunks per X row
  constexpr int CF = B / 4;   // 16-byte fp32 chunks per dX' row
  for (int m0 = mbeg; m0 < mend; m0 += kGTok) {
    for (int it = threadIdx.x; it < kGTok * CH; it += kRotThreads) {
      const int r = it / CH, c = it % CH;
      const int m = m0 + r;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (m < mend) v = *reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + j * B + c * 8);
      float* d = xs + r * LD + c * 8;
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        d[2 * i] = __uint_as_float(w[i] << 16);
        d[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
    for (int it = threadIdx.x; it < kGTok * CF; it += kRotThreads) {
      const int r = it / CF, c = it % CF;
      const int m = m0 + r;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m < mend) v = *reinterpret_cast<const float4*>(Dp + static_cast<size_t>(m) * K + j * B + c * 4);
      *reinterpret_cast<float4*>(ds + r * LD + c * 4) = v;
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < kGTok; ++t) {
      float xv[TI], dv[TL];
#pragma unroll
      for (int a = 0; a < TI; ++a) xv[a] = xs[t * LD + ib + a];
#pragma unroll
      for (int c = 0; c < TL; ++c) dv[c] = ds[t * LD + lb + c];
#pragma unroll
      for (int a = 0; a < TI; ++a)
#pragma unroll
        for (int c = 0; c < TL; ++c) acc[a][c] = fmaf(xv[a], dv[c], acc[a][c]);
    }
    __syncthreads();
  }
  float* out = Gp + ((static_cast<size_t>(p) * nb + j) * nparts + part) * B * B;
#pragma unroll
  for (int a = 0; a < TI; ++a)
#pragma unroll
    for (int c = 0; c < TL; ++c) out[(ib + a) * B + lb + c] = acc[a][c];
}

}  // namespace oftk
