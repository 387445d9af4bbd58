// Shared-memory tile helpers for the CUDA-core block rotation used by the MoE
// rotated gather (rows of one tile may belong to different experts, each with
// its own R): tiles of 64 tokens x one b-wide block, staged as fp32 with rows
// padded to keep 16-byte alignment for vector loads.
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

}  // namespace oftk
