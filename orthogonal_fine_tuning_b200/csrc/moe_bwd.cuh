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
//   dw_tk     = <U, X[t]>  (= sum_p <D_p, X[t] R_e,p> = <dY[t], Y_tk>)
//
// then dq_e,p = Cayley backward of G_e,p and, through the softmax over the k
// selected logits, dlogit[t, e_k] = w_tk (dw_tk - sum_j w_tj dw_tj).
//
// Everything below works in bucket order (positions sorted by expert, stable in
// (t, k)), the order the forward's grouped GEMM uses.
#pragma once

#include "cayley.cuh"
#include "common.cuh"
#include "dequant.cuh"
#include "moe.cuh"

namespace oftk {

// dYg[p][pos][j] = dY[bucket[pos] / k][p * n + j]   (n % 8 == 0).
__global__ void __launch_bounds__(256) moe_gather_dy_kernel(const uint16_t* __restrict__ dY,
                                                            const int* __restrict__ bucket, int TK, int k, int n,
                                                            uint16_t* __restrict__ dYg) {
  const int per_row = (2 * n) / 8;
  const long long units = static_cast<long long>(TK) * per_row;
  for (long long u = blockIdx.x * 256ll + threadIdx.x; u < units; u += static_cast<long long>(gridDim.x) * 256) {
    const int pos = static_cast<int>(u / per_row);
    const int col = static_cast<int>(u % per_row) * 8;
    const int p = col / n, j = col - p * n;
    const int t = bucket[pos] / k;
    const uint4 v = *reinterpret_cast<const uint4*>(dY + static_cast<size_t>(t) * 2 * n + col);
    *reinterpret_cast<uint4*>(dYg + (static_cast<size_t>(p) * TK + pos) * n + j) = v;
  }
}

// Transposed chunk dequant: buf[slot][p][k][j] = deq(W_e)[p * n + j][k] for the
// experts of chunk `chunk_idx` (INT4 bank), bit-exact like every other decode.
// grid = (ceil(K / 64), ceil(2n / 64), chunk slots); 64 x 64 tiles transposed
// through shared memory so that both the code reads and the bf16 writes are
// contiguous.  Requires n % 8 == 0 (8 consecutive rows never straddle gate/up).
__global__ void __launch_bounds__(256) moe_chunk_dequant_t_kernel(WeightView bank, const int* __restrict__ chunk_table,
                                                                  int chunk_idx, int chunk, int n,
                                                                  uint16_t* __restrict__ buf) {
  __shared__ uint16_t tile[64][64 + 8];
  const int slot = blockIdx.z;
  const int e = chunk_table[chunk_idx * chunk + slot];
  if (e < 0) return;
  const uint8_t* codes = bank.codes + static_cast<long long>(e) * bank.codes_expert_stride;
  const void* scales = static_cast<const uint8_t*>(bank.scales) + static_cast<long long>(e) * bank.scales_expert_stride;
  const int N = bank.N, K = bank.K;
  const int n0 = blockIdx.y * 64, k0 = blockIdx.x * 64;
  for (int it = threadIdx.x; it < 512; it += 256) {
    const int r = it >> 3, c = it & 7;
    const int row = n0 + r, k = k0 + c * 8;
    uint32_t v[4] = {0, 0, 0, 0};
    if (row < N && k < K) dequant8(bank, codes, scales, row, k, v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      tile[r][c * 8 + 2 * i] = static_cast<uint16_t>(v[i] & 0xFFFFu);
      tile[r][c * 8 + 2 * i + 1] = static_cast<uint16_t>(v[i] >> 16);
    }
  }
  __syncthreads();
  for (int it = threadIdx.x; it < 512; it += 256) {
    const int r = it >> 3, c = it & 7;
    const int k = k0 + r, row = n0 + c * 8;
    if (k >= K || row >= N) continue;
    const int p = row / n, j = row - p * n;
    uint32_t v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      v[i] = static_cast<uint32_t>(tile[c * 8 + 2 * i][r]) | (static_cast<uint32_t>(tile[c * 8 + 2 * i + 1][r]) << 16);
    *reinterpret_cast<uint4*>(buf + ((static_cast<size_t>(slot) * 2 + p) * K + k) * n + j) =
        make_uint4(v[0], v[1], v[2], v[3]);
  }
}

// Active experts ordered by bucket size, largest first (ties: lower id first),
// so that the per-(expert, block) units below start with the longest ones; also
// resets the units' work counter.  One CTA; n_active <= E <= kMaxExperts.
__global__ void __launch_bounds__(1024) moe_order_kernel(const int* __restrict__ offsets,
                                                         const int* __restrict__ active, const int* __restrict__ n_active,
                                                         int* __restrict__ order, int* __restrict__ counter) {
  __shared__ int cnt[kMaxExperts];
  const int na = *n_active;
  for (int a = threadIdx.x; a < na; a += 1024) cnt[a] = offsets[active[a] + 1] - offsets[active[a]];
  __syncthreads();
  for (int a = threadIdx.x; a < na; a += 1024) {
    int rank = 0;
    for (int b = 0; b < na; ++b) rank += (cnt[b] > cnt[a]) || (cnt[b] == cnt[a] && b < a);
    order[rank] = active[a];
  }
  if (threadIdx.x == 0) *counter = 0;
}

template <int B>
struct MoeBwdCfg {
  static constexpr int PT = 1024 / B;   // positions per tile (PT x B = 4 U outputs per thread)
  static constexpr int LD = B + 4;      // padded row of R^T and of the staged tiles (float4-aligned)
  static constexpr int JG = B * B / 256;  // G columns per thread and projection
  static constexpr int TPI = 256 / B;     // threads per G row
  static constexpr int LDC = B + 1;       // Cayley scratch rows
  static constexpr int TILE_FLOATS = 3 * PT * LD + PT;  // X, D_gate, D_up, w
  static constexpr int SCRATCH_FLOATS = 2 * B * LDC;    // G, then T G
  static constexpr int REGION = TILE_FLOATS > SCRATCH_FLOATS ? TILE_FLOATS : SCRATCH_FLOATS;
  static constexpr size_t SMEM = sizeof(float) * (2 * B * LD + REGION);
  static constexpr int TI = (B == 64) ? 4 : (B == 32 ? 2 : 1);  // Cayley thread tile
  static constexpr int NT = B / TI;
};

// One unit = (active expert e, rotation block blk), taken heaviest expert first
// from a work counter.  The unit walks e's bucket range in tiles of PT positions:
//   U[pos][blk]   = sum_p D_p[pos][blk] R_e,p,blk^T       -> U (fp32, bucket order)
//   dwp[pos][blk] = <U[pos][blk], X[t][blk]>               (partial of dw over blocks)
//   G_p          += X[t][blk]^T (w D_p[pos][blk])          (registers)
// and finally the Cayley backward of G_gate, G_up -> dq_e,p,blk.  256 threads.
// D is fp32 [2][TK][K]; R fp32 [E][2][nb][B][B]; dQ fp32 [E][2][nb][B(B-1)/2].
template <int B>
__global__ void __launch_bounds__(256) moe_bwd_rot_kernel(const float* __restrict__ D, const uint16_t* __restrict__ X,
                                                          int K, int TK, int top_k, const int* __restrict__ bucket,
                                                          const int* __restrict__ offsets, const float* __restrict__ topk_w,
                                                          const int* __restrict__ order,
                                                          const int* __restrict__ n_active, int* __restrict__ counter,
                                                          const float* __restrict__ R, float* __restrict__ U,
                                                          float* __restrict__ dwp, float* __restrict__ dQ) {
  using C = MoeBwdCfg<B>;
  constexpr int PT = C::PT, LD = C::LD, JG = C::JG, TPI = C::TPI, LDC = C::LDC, TI = C::TI, NT = C::NT;
  extern __shared__ float4 msm4[];
  float* sm = reinterpret_cast<float*>(msm4);
  float* Rt = sm;                  // [2][B][LD]   R_p^T, later (I + R_p)^T
  float* region = sm + 2 * B * LD;
  float* Xs = region;              // [PT][LD]
  float* Ds = region + PT * LD;    // [2][PT][LD]
  float* ws = region + 3 * PT * LD;  // [PT]
  float* Gs = region;              // [B][LDC]  (after the tile loop)
  float* Us = region + B * LDC;    // [B][LDC]
  __shared__ int s_unit;
  const int tid = threadIdx.x;
  const int nb = K / B;
  const int total = *n_active * nb;
  const int gi = tid / TPI, gj = (tid % TPI) * JG;  // G row and first column
  const int up = tid / (B / 4), uj = (tid % (B / 4)) * 4;  // U position (in tile) and first column
  const int ti = (tid / NT) * TI, tj = (tid % NT) * TI;
  for (;;) {
    if (tid == 0) s_unit = atomicAdd(counter, 1);
    __syncthreads();
    const int u = s_unit;
    if (u >= total) break;
    const int e = order[u / nb], blk = u % nb;
    const int o0 = offsets[e], o1 = offsets[e + 1];
    for (int idx = tid; idx < 2 * B * B; idx += 256) {
      const int p = idx / (B * B), r = (idx / B) % B, c = idx % B;  // R_p[r][c]
      Rt[(p * B + c) * LD + r] = R[((static_cast<size_t>(e) * 2 + p) * nb + blk) * B * B + r * B + c];
    }
    float g0[JG], g1[JG];
#pragma unroll
    for (int c = 0; c < JG; ++c) g0[c] = g1[c] = 0.f;
    for (int t0 = o0; t0 < o1; t0 += PT) {
      const int np = min(PT, o1 - t0);
      __syncthreads();  // previous tile consumed (and R^T written, on the first tile)
      for (int it = tid; it < PT * (B / 8); it += 256) {
        const int r = it / (B / 8), c8 = (it % (B / 8)) * 8;
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (r < np) {
          const int tok = bucket[t0 + r] / top_k;
          const uint4 q = *reinterpret_cast<const uint4*>(X + static_cast<size_t>(tok) * K + blk * B + c8);
          const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(qw[i] << 16);
            v[2 * i + 1] = __uint_as_float(qw[i] & 0xFFFF0000u);
          }
        }
        *reinterpret_cast<float4*>(Xs + r * LD + c8) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4*>(Xs + r * LD + c8 + 4) = make_float4(v[4], v[5], v[6], v[7]);
      }
      for (int it = tid; it < 2 * PT * (B / 4); it += 256) {
        const int p = it / (PT * (B / 4)), r = (it / (B / 4)) % PT, c4 = (it % (B / 4)) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < np) v = *reinterpret_cast<const float4*>(D + (static_cast<size_t>(p) * TK + t0 + r) * K + blk * B + c4);
        *reinterpret_cast<float4*>(Ds + (p * PT + r) * LD + c4) = v;
      }
      for (int r = tid; r < PT; r += 256) ws[r] = r < np ? topk_w[bucket[t0 + r]] : 0.f;
      __syncthreads();
      // U and the partial dw of this block
      {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          const float* drow = Ds + (p * PT + up) * LD;
          const float* rt = Rt + p * B * LD;
#pragma unroll 8
          for (int i = 0; i < B; ++i) {
            const float d = drow[i];
            const float4 rr = *reinterpret_cast<const float4*>(rt + i * LD + uj);
            acc[0] = fmaf(d, rr.x, acc[0]);
            acc[1] = fmaf(d, rr.y, acc[1]);
            acc[2] = fmaf(d, rr.z, acc[2]);
            acc[3] = fmaf(d, rr.w, acc[3]);
          }
        }
        const float4 xv = *reinterpret_cast<const float4*>(Xs + up * LD + uj);
        float s = acc[0] * xv.x + acc[1] * xv.y + acc[2] * xv.z + acc[3] * xv.w;
#pragma unroll
        for (int o = 1; o < B / 4; o <<= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
        if (up < np) {
          *reinterpret_cast<float4*>(U + static_cast<size_t>(t0 + up) * K + blk * B + uj) =
              make_float4(acc[0], acc[1], acc[2], acc[3]);
          if (uj == 0) dwp[static_cast<size_t>(t0 + up) * nb + blk] = s;
        }
      }
      // G_p += X^T (w D_p)
      for (int r = 0; r < np; ++r) {
        const float xw = Xs[r * LD + gi] * ws[r];
        const float* d0 = Ds + r * LD + gj;
        const float* d1 = Ds + (PT + r) * LD + gj;
#pragma unroll
        for (int c = 0; c < JG; ++c) {
          g0[c] = fmaf(xw, d0[c], g0[c]);
          g1[c] = fmaf(xw, d1[c], g1[c]);
        }
      }
    }
    __syncthreads();  // tiles consumed: the region becomes Cayley scratch
    for (int idx = tid; idx < 2 * B; idx += 256) Rt[(idx / B) * B * LD + (idx % B) * (LD + 1)] += 1.f;  // T_p = (I + R_p)^T
#pragma unroll
    for (int p = 0; p < 2; ++p) {
#pragma unroll
      for (int c = 0; c < JG; ++c) Gs[gi * LDC + gj + c] = p == 0 ? g0[c] : g1[c];
      __syncthreads();
      const float* T = Rt + p * B * LD;
      float o[TI][TI];
#pragma unroll
      for (int x = 0; x < TI; ++x)
#pragma unroll
        for (int y = 0; y < TI; ++y) o[x][y] = 0.f;
#pragma unroll 4
      for (int l = 0; l < B; ++l) {  // U = T G
        float tv[TI], gv[TI];
#pragma unroll
        for (int x = 0; x < TI; ++x) tv[x] = T[(ti + x) * LD + l];
#pragma unroll
        for (int y = 0; y < TI; ++y) gv[y] = Gs[l * LDC + tj + y];
#pragma unroll
        for (int x = 0; x < TI; ++x)
#pragma unroll
          for (int y = 0; y < TI; ++y) o[x][y] = fmaf(tv[x], gv[y], o[x][y]);
      }
#pragma unroll
      for (int x = 0; x < TI; ++x)
#pragma unroll
        for (int y = 0; y < TI; ++y) Us[(ti + x) * LDC + tj + y] = o[x][y];
      __syncthreads();
#pragma unroll
      for (int x = 0; x < TI; ++x)
#pragma unroll
        for (int y = 0; y < TI; ++y) o[x][y] = 0.f;
#pragma unroll 4
      for (int l = 0; l < B; ++l) {  // 2 dQ_full = (T G) T
        float uv[TI], tv[TI];
#pragma unroll
        for (int x = 0; x < TI; ++x) uv[x] = Us[(ti + x) * LDC + l];
#pragma unroll
        for (int y = 0; y < TI; ++y) tv[y] = T[l * LD + tj + y];
#pragma unroll
        for (int x = 0; x < TI; ++x)
#pragma unroll
          for (int y = 0; y < TI; ++y) o[x][y] = fmaf(uv[x], tv[y], o[x][y]);
      }
#pragma unroll
      for (int x = 0; x < TI; ++x)
#pragma unroll
        for (int y = 0; y < TI; ++y) Gs[(ti + x) * LDC + tj + y] = o[x][y];
      __syncthreads();
      float* out = dQ + ((static_cast<size_t>(e) * 2 + p) * nb + blk) * (B * (B - 1) / 2);
      for (int idx = tid; idx < B * B; idx += 256) {
        const int i = idx / B, j = idx % B;
        if (i < j) out[tri_index(i, j, B)] = 0.5f * (Gs[i * LDC + j] - Gs[j * LDC + i]);
      }
      __syncthreads();
    }
  }
}

// dlogits[t][:] = 0 except dlogits[t][idx[t,s]] = w_ts (dw_ts - sum_j w_tj dw_tj),
// dw_ts = sum over blocks of dwp[pos(t, s)][blk] (fixed order).  One warp per token.
__global__ void __launch_bounds__(256) moe_dlogits_kernel(const float* __restrict__ dwp, int nb,
                                                          const int* __restrict__ idx, const float* __restrict__ w,
                                                          const int* __restrict__ inv_pos, int T, int E, int k,
                                                          float* __restrict__ dlogits) {
  const int warp = (blockIdx.x * 256 + threadIdx.x) / 32, lane = threadIdx.x % 32;
  if (warp >= T) return;
  const int t = warp;
  float mine = 0.f, s = 0.f;
  for (int j = 0; j < k; ++j) {
    const float* row = dwp + static_cast<size_t>(inv_pos[static_cast<size_t>(t) * k + j]) * nb;
    float acc = 0.f;
    for (int b = lane; b < nb; b += 32) acc += row[b];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    const float wj = w[static_cast<size_t>(t) * k + j];
    s = fmaf(wj, acc, s);
    if (lane == j) mine = acc;
  }
  float* out = dlogits + static_cast<size_t>(t) * E;
  for (int e = lane; e < E; e += 32) out[e] = 0.f;
  __syncwarp();
  if (lane < k) {
    const float wl = w[static_cast<size_t>(t) * k + lane];
    out[idx[static_cast<size_t>(t) * k + lane]] = wl * (mine - s);
  }
}

}  // namespace oftk
