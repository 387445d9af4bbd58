// Full MoE expert layer: SwiGLU between the gate/up projections and a down
// projection that carries its own OFT adapter.
//
// The pages fine-tune whole low-precision MoE models through BF16 OFT adapters
// ("Orbit", chooseai.io news 4086, sections "技术原理：低精度基座 + BF16 适配器 + OFT"
// and "对低精度 MoE 模型的专门优化"; m.xxlwj.com 771001, section "技术细节", paragraph
// "Active-expert-chunked dequantization").  For every routed (t, k) with expert e:
//
//   h_tk = silu(g_tk) * u_tk,   [g_tk | u_tk] = Y_tk (the gate/up outputs, fp32)
//   Z_tk = (h_tk R_e,down) W_e,down
//   Y_t  = sum_k w_tk Z_tk
//
// The gate/up part and the combine are those of the chunked forward; the down
// projection runs through the same chunk dequant and grouped GEMM.  This file holds
// the step between them.
#pragma once

#include "common.cuh"

namespace oftk {

template <int B>
struct SwigluCfg {
  static constexpr int PT = 1024 / B;  // positions per tile: PT x B/4 column quads = 256 threads
  static constexpr int LDH = B + 4;    // padded fp32 rows (float4-aligned)
};

// Hg[pos][blk] = bf16( h[pos][blk] R_e,down,blk ) with h = silu(g) * u in fp32 and
// e = pos_expert[pos], for positions in bucket order.  Units are (tile of PT
// positions, block), grid-stride.  The R block of the tile's first expert is
// staged in shared memory; rows of another expert (a tile that crosses an expert
// boundary) read their block through the read-only cache.
// Ytk fp32 [TK][2n] (gate columns, then up); Rd fp32 [E][n/B][B][B]; Hg bf16 [TK][n].
template <int B>
__global__ void __launch_bounds__(256) moe_swiglu_rot_kernel(const float* __restrict__ Ytk,
                                                             const int* __restrict__ pos_expert, int TK, int n,
                                                             const float* __restrict__ Rd, uint16_t* __restrict__ Hg) {
  using C = SwigluCfg<B>;
  constexpr int PT = C::PT, LDH = C::LDH;
  __shared__ __align__(16) float Hs[PT * LDH];
  __shared__ __align__(16) float Rs[B * LDH];
  __shared__ int es[PT];
  const int tid = threadIdx.x;
  const int nbd = n / B;
  const int tiles = (TK + PT - 1) / PT;
  const int r = tid / (B / 4), c4 = (tid % (B / 4)) * 4;  // this thread's output quad
  for (int u = blockIdx.x; u < tiles * nbd; u += gridDim.x) {
    const int t0 = (u / nbd) * PT, blk = u % nbd;
    const int np = min(PT, TK - t0);
    const int e0 = pos_expert[t0];
    const float* r0 = Rd + (static_cast<size_t>(e0) * nbd + blk) * B * B;
    for (int i = tid; i < B * B / 4; i += 256) {
      const int row = (i * 4) / B, col = (i * 4) % B;
      *reinterpret_cast<float4*>(Rs + row * LDH + col) = *reinterpret_cast<const float4*>(r0 + i * 4);
    }
    {
      float4 h = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < np) {
        const float* row = Ytk + static_cast<size_t>(t0 + r) * 2 * n + blk * B + c4;
        const float4 g = *reinterpret_cast<const float4*>(row);
        const float4 v = *reinterpret_cast<const float4*>(row + n);
        h.x = g.x / (1.f + expf(-g.x)) * v.x;
        h.y = g.y / (1.f + expf(-g.y)) * v.y;
        h.z = g.z / (1.f + expf(-g.z)) * v.z;
        h.w = g.w / (1.f + expf(-g.w)) * v.w;
      }
      *reinterpret_cast<float4*>(Hs + r * LDH + c4) = h;
      if (c4 == 0) es[r] = r < np ? pos_expert[t0 + r] : e0;
    }
    __syncthreads();
    if (r < np) {
      const int e = es[r];
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const float* hrow = Hs + r * LDH;
      if (e == e0) {
#pragma unroll 8
        for (int i = 0; i < B; ++i) {
          const float hv = hrow[i];
          const float4 rv = *reinterpret_cast<const float4*>(Rs + i * LDH + c4);
          acc[0] = fmaf(hv, rv.x, acc[0]);
          acc[1] = fmaf(hv, rv.y, acc[1]);
          acc[2] = fmaf(hv, rv.z, acc[2]);
          acc[3] = fmaf(hv, rv.w, acc[3]);
        }
      } else {
        const float* re = Rd + (static_cast<size_t>(e) * nbd + blk) * B * B + c4;
#pragma unroll 8
        for (int i = 0; i < B; ++i) {
          const float hv = hrow[i];
          const float4 rv = __ldg(reinterpret_cast<const float4*>(re + i * B));
          acc[0] = fmaf(hv, rv.x, acc[0]);
          acc[1] = fmaf(hv, rv.y, acc[1]);
          acc[2] = fmaf(hv, rv.z, acc[2]);
          acc[3] = fmaf(hv, rv.w, acc[3]);
        }
      }
      *reinterpret_cast<uint2*>(Hg + static_cast<size_t>(t0 + r) * n + blk * B + c4) =
          make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
    }
    __syncthreads();
  }
}

}  // namespace oftk
