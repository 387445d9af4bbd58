// Active-expert MoE forward with the dequant fused into the grouped GEMM: the
// experts' INT4 weights are decoded straight into the tensor-core operand
// (gemm_dq.cuh, MoE mode) instead of into a transient bf16 chunk buffer.  The
// pages dequantise the router-selected experts chunk by chunk into a buffer that
// feeds a grouped GEMM (m.xxlwj.com 771001, section "技术细节"; chooseai.io news
// 4086, "对低精度 MoE 模型的专门优化"); this variant keeps their routing, rotation and
// combine and removes the buffer, so each active expert's weight crosses HBM once,
// as 4-bit codes.
#pragma once

#include "common.cuh"
#include "gemm_dq.cuh"

namespace oftk {

// One group per (active expert a, projection p), expert-major: rows = n_proj weight
// rows of projection p, tokens = the expert's bucket rows, activations at map row
// p * TK + offsets[e].  One warp builds them with a running scan of the unit counts.
// meta[0] = total units, meta[1] = groups.
__global__ void __launch_bounds__(32) moe_groups_kernel(const int* __restrict__ active, const int* __restrict__ n_active,
                                                        const int* __restrict__ offsets, int TK, int n_proj, int K,
                                                        long long code_stride, long long scale_stride,
                                                        gdq::Group* __restrict__ groups, int* __restrict__ meta) {
  const int lane = threadIdx.x;
  const int ng = 2 * *n_active;
  const int tiles_w = (n_proj + gdq::WM - 1) / gdq::WM;
  int carry = 0;
  for (int g0 = 0; g0 < ng; g0 += 32) {
    const int g = g0 + lane;
    gdq::Group G;
    memset(&G, 0, sizeof(G));
    int units = 0;
    if (g < ng) {
      const int e = active[g >> 1], pr = g & 1;
      const int off = offsets[e], n_e = offsets[e + 1] - off;
      G.rows = n_proj;
      G.tokens = n_e;
      G.kred = K;
      G.b_map = 0;
      G.b_row0 = pr * TK + off;
      G.w_row0 = pr * n_proj;
      G.w_k0 = 0;
      G.y_map = 0;
      G.tiles_w = tiles_w;
      G.tiles_t = ((n_e + gdq::TN - 1) / gdq::TN + gdq::TP - 1) / gdq::TP;
      G.code_off = static_cast<long long>(e) * code_stride;
      G.scale_off = static_cast<long long>(e) * scale_stride;
      G.out_row0 = off;
      G.out_col0 = pr * n_proj;
      units = G.tiles_w * G.tiles_t;
    }
    int x = units;  // inclusive scan over the warp
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, x, d);
      if (lane >= d) x += y;
    }
    if (g < ng) {
      G.tile0 = carry + x - units;
      groups[g] = G;
    }
    carry += __shfl_sync(0xFFFFFFFFu, x, 31);
  }
  if (lane == 0) {
    meta[0] = carry;
    meta[1] = ng;
  }
}

}  // namespace oftk
