// Cayley map of the OFT adapter and its backward, one CTA per b x b block.
//
// OFT parameterises each block of the orthogonal rotation by a skew-symmetric Q
// (the pages name OFT as Orbit's default adapter: chooseai.io news 4086, section
// "技术原理：低精度基座 + BF16 适配器 + OFT"):
//     R = (I + Q)(I - Q)^-1 = (I - Q)^-1 (I + Q)
// Forward: solve (I - Q) R = (I + Q) by Gauss-Jordan elimination in shared
// memory, fp32, without pivoting.  I - Q has symmetric part I, so x^T (I-Q) x =
// |x|^2 > 0: every leading minor is non-zero, every pivot stays >= 1 in exact
// arithmetic, and sigma_min(I - Q) >= 1 (the solve is well conditioned for any Q).
// Backward: with G = dL/dR, dL/dQ = 1/2 (I + R)^T G (I + R)^T, projected onto the
// packed strict-upper parameters as dq_ij = D_ij - D_ji.
#pragma once

#include "common.cuh"

namespace oftk {

constexpr int kCayleyThreads = 256;

__device__ __forceinline__ int tri_index(int i, int j, int b) {  // i < j, row-major strict upper
  return i * b - i * (i + 1) / 2 + (j - i - 1);
}

// Q: bf16 [nblocks][b(b-1)/2]; R: fp32 [nblocks][b][b].
// Optional MoE filter: when `counts` is given, block `blk` belongs to expert
// blk / blocks_per_expert and is skipped when that expert has no tokens.
__global__ void __launch_bounds__(kCayleyThreads) cayley_fwd_kernel(const uint16_t* __restrict__ Q, int nblocks, int b,
                                                                    float* __restrict__ R, const int* __restrict__ offsets,
                                                                    int blocks_per_expert) {
  extern __shared__ float sm[];
  const int ld = b + 1;
  float* A = sm;               // I - Q, reduced to I
  float* B = sm + b * ld;      // I + Q, becomes R
  float* f = sm + 2 * b * ld;  // elimination factors of the current pivot column
  const int tid = threadIdx.x;
  for (int blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
    if (offsets != nullptr) {
      const int e = blk / blocks_per_expert;
      if (offsets[e + 1] == offsets[e]) continue;
    }
    const uint16_t* q = Q + static_cast<size_t>(blk) * (b * (b - 1) / 2);
    for (int idx = tid; idx < b * b; idx += kCayleyThreads) {
      const int i = idx / b, j = idx % b;
      float v = 0.f;
      if (i < j) v = bf16_bits_to_f32(q[tri_index(i, j, b)]);
      else if (i > j) v = -bf16_bits_to_f32(q[tri_index(j, i, b)]);
      const float d = (i == j) ? 1.f : 0.f;
      A[i * ld + j] = d - v;
      B[i * ld + j] = d + v;
    }
    __syncthreads();
    for (int c = 0; c < b; ++c) {
      const float inv = 1.0f / A[c * ld + c];
      __syncthreads();
      for (int j = tid; j < b; j += kCayleyThreads) {
        A[c * ld + j] *= inv;
        B[c * ld + j] *= inv;
      }
      for (int r = tid; r < b; r += kCayleyThreads) f[r] = (r == c) ? 0.f : A[r * ld + c];
      __syncthreads();
      for (int idx = tid; idx < b * b; idx += kCayleyThreads) {
        const int r = idx / b, j = idx % b;
        const float fr = f[r];
        if (fr != 0.f) {
          A[r * ld + j] -= fr * A[c * ld + j];
          B[r * ld + j] -= fr * B[c * ld + j];
        }
      }
      __syncthreads();
    }
    float* out = R + static_cast<size_t>(blk) * b * b;
    for (int idx = tid; idx < b * b; idx += kCayleyThreads) out[idx] = B[(idx / b) * ld + idx % b];
    __syncthreads();
  }
}

// dQ[blk] = pack(D - D^T), D = 1/2 (I+R)^T G (I+R)^T.
// G is read either directly ([nblocks][b][b]) or as `nparts` partial sums laid
// out [nblocks][nparts][b][b], summed in part order (deterministic).
__global__ void __launch_bounds__(kCayleyThreads) cayley_bwd_kernel(const float* __restrict__ R,
                                                                    const float* __restrict__ G, int nparts,
                                                                    int nblocks, int b, float* __restrict__ dQ) {
  extern __shared__ float sm[];
  const int ld = b + 1;
  float* T = sm;               // (I + R)^T, stored as T[i][j] = (I+R)[j][i]
  float* Gs = sm + b * ld;     // G
  float* U = sm + 2 * b * ld;  // T G, then D
  const int tid = threadIdx.x;
  for (int blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
    const float* r = R + static_cast<size_t>(blk) * b * b;
    for (int idx = tid; idx < b * b; idx += kCayleyThreads) {
      const int i = idx / b, j = idx % b;
      T[j * ld + i] = r[idx] + (i == j ? 1.f : 0.f);
      const float* g = G + static_cast<size_t>(blk) * nparts * b * b + idx;
      float acc = 0.f;
      for (int p = 0; p < nparts; ++p) acc += g[static_cast<size_t>(p) * b * b];
      Gs[i * ld + j] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < b * b; idx += kCayleyThreads) {  // U = T G
      const int i = idx / b, j = idx % b;
      float acc = 0.f;
      for (int l = 0; l < b; ++l) acc = fmaf(T[i * ld + l], Gs[l * ld + j], acc);
      U[i * ld + j] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < b * b; idx += kCayleyThreads) {  // Gs = U T = D * 2
      const int i = idx / b, j = idx % b;
      float acc = 0.f;
      for (int l = 0; l < b; ++l) acc = fmaf(U[i * ld + l], T[l * ld + j], acc);
      Gs[i * ld + j] = acc;
    }
    __syncthreads();
    float* out = dQ + static_cast<size_t>(blk) * (b * (b - 1) / 2);
    for (int idx = tid; idx < b * b; idx += kCayleyThreads) {
      const int i = idx / b, j = idx % b;
      if (i < j) out[tri_index(i, j, b)] = 0.5f * (Gs[i * ld + j] - Gs[j * ld + i]);
    }
    __syncthreads();
  }
}

}  // namespace oftk
