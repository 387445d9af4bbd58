// Backward of the active-expert-chunked MoE OFT layer.
//
// The pages fine-tune low-precision MoE models through BF16 OFT adapters whose
// gradients never touch the frozen expert weights ("Orbit", chooseai.io news
// 4086, sections "技术原理：低精度基座 + BF16 适配器 + OFT" and "对低精度 MoE 模型的专门优化";
// m.xxlwj.com 771001, section "技术细节", DeepSeek V4 paragraph: the GEMM
// backward skips the base weight's gradient).  Every (token t, slot k) routed to
// expert e = idx[t, k] with gating weight w_tk contributes, for p = gate, up:
//
//   D_p       = dY_p[t] W_e,p^T                    (grouped GEMM over the chunk's experts)
//   U         = sum_p D_p R_e,p^T                  (blockwise)
//   dX[t]    += w_tk U
//   G_e,p,blk += X[t]_blk^T (w_tk D_p,blk)
//   dw_tk     = <U, X[t]>  (= sum_p <D_p, X[t] R_e,p> = <dY[t], Y_tk>), with dX[t] in one pass over U
//
// then dq_e,p = Cayley backward of G_e,p and, through the softmax over the k
// selected logits, dlogit[t, e_k] = w_tk (dw_tk - sum_j w_tj dw_tj).
//
// Everything below works in bucket order (positions sorted by expert, stable in
// (t, k)), the order the forward's grouped GEMM uses.  The rotations back, G and
// the Cayley backward run on the tensor cores in moe_bwd_tc.cuh.
#pragma once

#include "cayley.cuh"
#include "common.cuh"
#include "dequant.cuh"
#include "moe.cuh"

namespace oftk {

// dYg[p][pos][j] = dY[bucket[pos] / k][p * n + j]   (n % 8 == 0), and each position's
// routed token and gating weight: row_t[pos] = bucket[pos] / k, row_w[pos] = w[bucket[pos]].
__global__ void __launch_bounds__(256) moe_gather_dy_kernel(const uint16_t* __restrict__ dY,
                                                            const int* __restrict__ bucket, const float* __restrict__ w,
                                                            int TK, int k, int n, uint16_t* __restrict__ dYg,
                                                            int* __restrict__ row_t, float* __restrict__ row_w) {
  const int per_row = (2 * n) / 8;
  const long long units = static_cast<long long>(TK) * per_row;
  for (long long u = blockIdx.x * 256ll + threadIdx.x; u < units; u += static_cast<long long>(gridDim.x) * 256) {
    const int pos = static_cast<int>(u / per_row);
    const int col = static_cast<int>(u % per_row) * 8;
    const int p = col / n, j = col - p * n;
    const int ent = bucket[pos];
    const int t = ent / k;
    const uint4 v = *reinterpret_cast<const uint4*>(dY + static_cast<size_t>(t) * 2 * n + col);
    *reinterpret_cast<uint4*>(dYg + (static_cast<size_t>(p) * TK + pos) * n + j) = v;
    if (col == 0) {
      row_t[pos] = t;
      row_w[pos] = w[ent];
    }
  }
}

// Transposed chunk dequant: buf[slot][p][k][j] = deq(W_e)[p * n + j][k] for the
// experts of chunk `chunk_idx` (INT4 bank), bit-exact like every other decode.
// The transpose happens in registers: lane (ro, kw) of a warp decodes the 8 code
// words of rows 8 ro .. 8 ro + 7 at word kw of the warp's 64-column block (64
// elements), then packs each k's 8 row values into one 16-byte store with byte
// permutes.  Per warp that is 32 rows x 64 columns; for a fixed row the 8 lanes of one
// ro read 32 contiguous bytes of codes, and for a fixed k the 4 lanes of one kw write
// 64 contiguous bytes.  A CTA's 8 warps take 8 consecutive column blocks of the same
// 32 rows.  Requires n % 8 == 0 (8 consecutive rows never straddle gate / up).
constexpr int kDqtRows = 32;    // rows per CTA
constexpr int kDqtCols = 512;   // columns (k) per CTA: 8 warps x 64

inline dim3 dqt_grid(int K, int N, int chunk) {
  return dim3((K + kDqtCols - 1) / kDqtCols, (N + kDqtRows - 1) / kDqtRows, chunk);
}

__global__ void __launch_bounds__(256) moe_chunk_dequant_t_kernel(WeightView bank, const int* __restrict__ chunk_table,
                                                                  int chunk_idx, int chunk, int n,
                                                                  uint16_t* __restrict__ buf) {
  const int slot = blockIdx.z;
  const int e = chunk_table[chunk_idx * chunk + slot];
  if (e < 0) return;
  const uint8_t* codes = bank.codes + static_cast<long long>(e) * bank.codes_expert_stride;
  const uint16_t* scales = reinterpret_cast<const uint16_t*>(static_cast<const uint8_t*>(bank.scales) +
                                                             static_cast<long long>(e) * bank.scales_expert_stride);
  const int N = bank.N, K = bank.K, G = bank.group;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ro = lane >> 3, kw = lane & 7;
  const int row0 = blockIdx.y * kDqtRows + ro * 8;           // this lane's 8 rows
  const int k = blockIdx.x * kDqtCols + warp * 64 + kw * 8;  // and 8 columns
  if (row0 >= N || k >= K) return;                          // N % 8 == 0, K % 8 == 0: whole octets
  uint32_t w[8];
  uint16_t sc[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    w[m] = __ldg(reinterpret_cast<const uint32_t*>(codes + static_cast<size_t>(row0 + m) * (K / 2) + k / 2));
    sc[m] = __ldg(scales + static_cast<size_t>(k / G) * N + row0 + m);
  }
  uint32_t v[8][4];  // v[m][q]: row row0 + m, columns k + 2q (low half) and k + 2q + 1
#pragma unroll
  for (int m = 0; m < 8; ++m) dq::int4x8(w[m], dq::bf2_splat(sc[m]), v[m]);
  const int p = row0 / n, j = row0 - p * n;
  uint16_t* dst = buf + ((static_cast<size_t>(slot) * 2 + p) * K + k) * n + j;
#pragma unroll
  for (int i = 0; i < 8; ++i) {  // column k + i: rows row0 .. row0 + 7
    const uint32_t sel = (i & 1) ? 0x7632u : 0x5410u;
    *reinterpret_cast<uint4*>(dst + static_cast<size_t>(i) * n) =
        make_uint4(__byte_perm(v[0][i >> 1], v[1][i >> 1], sel), __byte_perm(v[2][i >> 1], v[3][i >> 1], sel),
                   __byte_perm(v[4][i >> 1], v[5][i >> 1], sel), __byte_perm(v[6][i >> 1], v[7][i >> 1], sel));
  }
}

// Active experts ordered by bucket size, largest first (ties: lower id first),
// so that the per-(expert, column group) units of the backward's rotation kernels
// (moe_bwd_tc.cuh) start with the longest ones.  One CTA; n_active <= E <= kMaxExperts.
__global__ void __launch_bounds__(1024) moe_order_kernel(const int* __restrict__ offsets,
                                                         const int* __restrict__ active, const int* __restrict__ n_active,
                                                         int* __restrict__ order) {
  __shared__ int cnt[kMaxExperts];
  const int na = *n_active;
  for (int a = threadIdx.x; a < na; a += 1024) cnt[a] = offsets[active[a] + 1] - offsets[active[a]];
  __syncthreads();
  for (int a = threadIdx.x; a < na; a += 1024) {
    int rank = 0;
    for (int b = 0; b < na; ++b) rank += (cnt[b] > cnt[a]) || (cnt[b] == cnt[a] && b < a);
    order[rank] = active[a];
  }
}

// dX[t] = sum_s w_ts U[pos(t, s)] (fp32 in slot order, stored as bf16) and
// dw_ts = <U[pos(t, s)], X[t]> (each lane sums its columns in order, then a fixed
// xor-shuffle tree).  One warp per token; K % 256 == 0 is not required (K % 8 == 0).
__global__ void __launch_bounds__(256) moe_combine_bwd_kernel(const float* __restrict__ U, const float* __restrict__ w,
                                                              const int* __restrict__ inv_pos,
                                                              const uint16_t* __restrict__ X, int T, int K, int k,
                                                              uint16_t* __restrict__ dX, float* __restrict__ dw) {
  const int lane = threadIdx.x % 32;
  for (int t = (blockIdx.x * 256 + threadIdx.x) / 32; t < T; t += gridDim.x * 8) {
    int pos[kMaxTopK];
    float ws[kMaxTopK], dws[kMaxTopK];
#pragma unroll
    for (int s = 0; s < kMaxTopK; ++s) {
      pos[s] = s < k ? inv_pos[static_cast<size_t>(t) * k + s] : 0;
      ws[s] = s < k ? w[static_cast<size_t>(t) * k + s] : 0.f;
      dws[s] = 0.f;
    }
    for (int c = lane * 8; c < K; c += 256) {
      const uint4 xq = *reinterpret_cast<const uint4*>(X + static_cast<size_t>(t) * K + c);
      const float x[8] = {__uint_as_float(xq.x << 16), __uint_as_float(xq.x & 0xFFFF0000u),
                          __uint_as_float(xq.y << 16), __uint_as_float(xq.y & 0xFFFF0000u),
                          __uint_as_float(xq.z << 16), __uint_as_float(xq.z & 0xFFFF0000u),
                          __uint_as_float(xq.w << 16), __uint_as_float(xq.w & 0xFFFF0000u)};
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float4 ua[kMaxTopK], ub[kMaxTopK];  // every slot's loads in flight before the first FMA
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s) {
        ua[s] = s < k ? *reinterpret_cast<const float4*>(U + static_cast<size_t>(pos[s]) * K + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        ub[s] = s < k ? *reinterpret_cast<const float4*>(U + static_cast<size_t>(pos[s]) * K + c + 4)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s) {
        const float u[8] = {ua[s].x, ua[s].y, ua[s].z, ua[s].w, ub[s].x, ub[s].y, ub[s].z, ub[s].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          acc[e] = fmaf(ws[s], u[e], acc[e]);
          dws[s] = fmaf(u[e], x[e], dws[s]);
        }
      }
      *reinterpret_cast<uint4*>(dX + static_cast<size_t>(t) * K + c) =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                     pack_bf16x2(acc[6], acc[7]));
    }
#pragma unroll
    for (int s = 0; s < kMaxTopK; ++s) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dws[s] += __shfl_xor_sync(0xFFFFFFFFu, dws[s], o);
      if (lane == 0 && s < k) dw[static_cast<size_t>(t) * k + s] = dws[s];
    }
  }
}

// dlogits[t][:] = 0 except dlogits[t][idx[t,s]] = w_ts (dw_ts - sum_j w_tj dw_tj)
// (the sum in slot order).  One warp per token.
__global__ void __launch_bounds__(256) moe_dlogits_kernel(const float* __restrict__ dw, const int* __restrict__ idx,
                                                          const float* __restrict__ w, int T, int E, int k,
                                                          float* __restrict__ dlogits) {
  const int warp = (blockIdx.x * 256 + threadIdx.x) / 32, lane = threadIdx.x % 32;
  if (warp >= T) return;
  const int t = warp;
  float s = 0.f;
  for (int j = 0; j < k; ++j) s = fmaf(w[static_cast<size_t>(t) * k + j], dw[static_cast<size_t>(t) * k + j], s);
  float* out = dlogits + static_cast<size_t>(t) * E;
  for (int e = lane; e < E; e += 32) out[e] = 0.f;
  __syncwarp();
  if (lane < k) {
    const size_t tk = static_cast<size_t>(t) * k + lane;
    out[idx[tk]] = w[tk] * (dw[tk] - s);
  }
}

}  // namespace oftk
