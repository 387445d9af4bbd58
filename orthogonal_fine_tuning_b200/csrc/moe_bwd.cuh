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
// grid = (ceil(K / 256), ceil(2n / 64), chunk slots): a CTA walks a 64-row x
// 256-column strip as four 64 x 64 tiles, with the next tile's codes and scales
// already loaded into registers while the current one is transposed.  A tile goes
// through shared memory as 32-bit words (two k per word, rows padded to 33
// words), so neither side has bank conflicts; the code reads and the bf16 writes
// are contiguous.  Requires n % 8 == 0 (8 consecutive rows never straddle gate / up).
constexpr int kDqtStrip = 4;  // 64 x 64 tiles per CTA along K

__global__ void __launch_bounds__(256) moe_chunk_dequant_t_kernel(WeightView bank, const int* __restrict__ chunk_table,
                                                                  int chunk_idx, int chunk, int n,
                                                                  uint16_t* __restrict__ buf) {
  __shared__ uint32_t tile[64][33];  // [row n][k pair]
  const int slot = blockIdx.z;
  const int e = chunk_table[chunk_idx * chunk + slot];
  if (e < 0) return;
  const uint8_t* codes = bank.codes + static_cast<long long>(e) * bank.codes_expert_stride;
  const uint16_t* scales = reinterpret_cast<const uint16_t*>(static_cast<const uint8_t*>(bank.scales) +
                                                             static_cast<long long>(e) * bank.scales_expert_stride);
  const int N = bank.N, K = bank.K, G = bank.group;
  const int n0 = blockIdx.y * 64;
  const int lane = threadIdx.x & 31;
  // this thread's two decode items of a tile: row r, k = 8c .. 8c+7 (it = tid, tid + 256)
  uint32_t word[2];
  uint16_t sc[2];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int it = threadIdx.x + 256 * h;
      const int row = n0 + (it >> 3), k = k0 + (it & 7) * 8;
      const bool ok = row < N && k < K;
      word[h] = ok ? *reinterpret_cast<const uint32_t*>(codes + static_cast<size_t>(row) * (K / 2) + k / 2) : 0u;
      sc[h] = ok ? scales[static_cast<size_t>(k / G) * N + row] : uint16_t(0);
    }
  };
  fetch(blockIdx.x * 64 * kDqtStrip);
  for (int t = 0; t < kDqtStrip; ++t) {
    const int k0 = (blockIdx.x * kDqtStrip + t) * 64;
    if (k0 >= K) break;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int it = threadIdx.x + 256 * h;
      uint32_t v[4];
      dq::int4x8(word[h], dq::bf2_splat(sc[h]), v);
#pragma unroll
      for (int i = 0; i < 4; ++i) tile[it >> 3][(it & 7) * 4 + i] = v[i];
    }
    __syncthreads();
    if (t + 1 < kDqtStrip && k0 + 64 < K) fetch(k0 + 64);
    for (int it = threadIdx.x; it < 512; it += 256) {
      const int q = it >> 5;
      const int r = (lane & 7) + 8 * (q & 7);  // k row
      const int c = (lane >> 3) + 4 * (q >> 3);  // 8 consecutive n
      const int k = k0 + r, row = n0 + c * 8;
      if (k >= K || row >= N) continue;
      const int p = row / n, j = row - p * n;
      const int sh = (r & 1) * 16;
      uint32_t v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        v[i] = ((tile[c * 8 + 2 * i][r >> 1] >> sh) & 0xFFFFu) | (((tile[c * 8 + 2 * i + 1][r >> 1] >> sh) & 0xFFFFu) << 16);
      *reinterpret_cast<uint4*>(buf + ((static_cast<size_t>(slot) * 2 + p) * K + k) * n + j) =
          make_uint4(v[0], v[1], v[2], v[3]);
    }
    __syncthreads();
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
  static constexpr int PT = 2048 / B;   // positions per tile (128 U threads x 4 positions x 4 columns)
  static constexpr int LDT = PT + 4;    // transposed tile rows [column][position] (float4-aligned)
  static constexpr int LDR = B + 4;     // rows of the stacked [R_gate^T; R_up^T]
  static constexpr int GI = B / 16, GJ = B / 8;  // G thread tile: rows gi + 16 ii, columns gj + 8 jj
  static constexpr int LDC = B + 1;     // Cayley scratch rows
  static constexpr int TILE_FLOATS = 3 * B * LDT + PT;  // D_gate^T, D_up^T, X^T, w
  static constexpr int SCRATCH_FLOATS = 2 * B * LDC;    // G, then T G
  static constexpr int REGION = TILE_FLOATS > SCRATCH_FLOATS ? TILE_FLOATS : SCRATCH_FLOATS;
  static constexpr size_t SMEM = sizeof(float) * (2 * B * LDR + REGION);
  static constexpr int TI = (B == 64) ? 4 : (B == 32 ? 2 : 1);  // Cayley thread tile
  static constexpr int NT = B / TI;
  static constexpr int D_VEC = 2 * PT * (B / 4) / 256;  // float4 of D per thread and tile
  static constexpr int X_VEC = PT * (B / 8) / 256;      // 8 x bf16 of X per thread and tile
  static_assert(D_VEC * 256 == 2 * PT * (B / 4) && X_VEC * 256 == PT * (B / 8), "tile loads must cover the CTA");
};

// Position swizzle of the transposed tiles: element (row, pos) lives at
// row * LDT + (pos ^ moe_swz(row)).  XOR with a multiple of 4 keeps every aligned
// group of four positions together (float4 reads stay whole), and it spreads the
// transposing stores over all banks; the G and U reads stay conflict-free.
__device__ __forceinline__ int moe_swz(int row) { return ((row >> 3) & 7) << 2; }

// One unit = (active expert e, rotation block blk), taken heaviest expert first
// from a work counter.  The unit walks e's bucket range in tiles of PT positions,
// staged transposed in shared memory (the next tile's loads are in flight, in
// registers, while the current one is computed):
//   warps 0-3:  U[pos][blk]   = sum_p D_p[pos][blk] R_e,p,blk^T    -> U (fp32, bucket order)
//               dwp[pos][blk] = <U[pos][blk], X[t][blk]>            (partial of dw over blocks)
//   warps 4-7:  G_p          += X[t][blk]^T (w D_p[pos][blk])       (registers)
// and finally all warps run the Cayley backward of G_gate, G_up -> dq_e,p,blk.
// D is fp32 [2][TK][K]; R fp32 [E][2][nb][B][B]; dQ fp32 [E][2][nb][B(B-1)/2].
template <int B>
__global__ void __launch_bounds__(256, (B == 64 ? 2 : 3)) moe_bwd_rot_kernel(const float* __restrict__ D, const uint16_t* __restrict__ X,
                                                          int K, int TK, int top_k, const int* __restrict__ bucket,
                                                          const int* __restrict__ offsets, const float* __restrict__ topk_w,
                                                          const int* __restrict__ order,
                                                          const int* __restrict__ n_active, int* __restrict__ counter,
                                                          const float* __restrict__ R, float* __restrict__ U,
                                                          float* __restrict__ dwp, float* __restrict__ dQ) {
  using C = MoeBwdCfg<B>;
  constexpr int PT = C::PT, LDT = C::LDT, LDR = C::LDR, GI = C::GI, GJ = C::GJ, LDC = C::LDC, TI = C::TI, NT = C::NT;
  constexpr int D_VEC = C::D_VEC, X_VEC = C::X_VEC;
  extern __shared__ float4 msm4[];
  float* sm = reinterpret_cast<float*>(msm4);
  float* Rc = sm;                   // [2B][LDR]: row p*B + i holds column i of R_p (R_p^T), later (I + R_p)^T
  float* region = sm + 2 * B * LDR;
  float* Dt = region;               // [2][B][LDT]
  float* Xt = region + 2 * B * LDT;  // [B][LDT]
  float* ws = region + 3 * B * LDT;  // [PT]
  float* Gs = region;               // [B][LDC]  (after the tile loop)
  float* Us = region + B * LDC;     // [B][LDC]
  __shared__ int s_unit;
  const int tid = threadIdx.x, warp = tid / 32;
  const int nb = K / B;
  const int total = *n_active * nb;
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
      Rc[(p * B + c) * LDR + r] = R[((static_cast<size_t>(e) * 2 + p) * nb + blk) * B * B + r * B + c];
    }
    // tile loads into registers (zeros past the end of e's range)
    float4 dreg[D_VEC];
    uint4 xreg[X_VEC];
    float wreg = 0.f;
    auto fetch = [&](int t0) {
      const int np = min(PT, o1 - t0);
#pragma unroll
      for (int v = 0; v < D_VEC; ++v) {
        const int it = tid + 256 * v;
        const int p = it / (PT * (B / 4)), rem = it % (PT * (B / 4));
        const int r = rem / (B / 4), c4 = (rem % (B / 4)) * 4;
        dreg[v] = r < np ? *reinterpret_cast<const float4*>(D + (static_cast<size_t>(p) * TK + t0 + r) * K + blk * B + c4)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int v = 0; v < X_VEC; ++v) {
        const int it = tid + 256 * v;
        const int r = it / (B / 8), c8 = (it % (B / 8)) * 8;
        xreg[v] = r < np ? *reinterpret_cast<const uint4*>(X + static_cast<size_t>(bucket[t0 + r] / top_k) * K + blk * B + c8)
                         : make_uint4(0u, 0u, 0u, 0u);
      }
      if (tid < PT) wreg = tid < np ? topk_w[bucket[t0 + tid]] : 0.f;
    };
    auto stage = [&]() {
#pragma unroll
      for (int v = 0; v < D_VEC; ++v) {
        const int it = tid + 256 * v;
        const int p = it / (PT * (B / 4)), rem = it % (PT * (B / 4));
        const int r = rem / (B / 4), c4 = (rem % (B / 4)) * 4;
        const int row = p * B + c4;
        Dt[row * LDT + (r ^ moe_swz(row))] = dreg[v].x;
        Dt[(row + 1) * LDT + (r ^ moe_swz(row + 1))] = dreg[v].y;
        Dt[(row + 2) * LDT + (r ^ moe_swz(row + 2))] = dreg[v].z;
        Dt[(row + 3) * LDT + (r ^ moe_swz(row + 3))] = dreg[v].w;
      }
#pragma unroll
      for (int v = 0; v < X_VEC; ++v) {
        const int it = tid + 256 * v;
        const int r = it / (B / 8), c8 = (it % (B / 8)) * 8;
        const uint32_t q[4] = {xreg[v].x, xreg[v].y, xreg[v].z, xreg[v].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = c8 + 2 * i;
          Xt[row * LDT + (r ^ moe_swz(row))] = __uint_as_float(q[i] << 16);
          Xt[(row + 1) * LDT + (r ^ moe_swz(row + 1))] = __uint_as_float(q[i] & 0xFFFF0000u);
        }
      }
      if (tid < PT) ws[tid] = wreg;
    };
    float g[2][GI][GJ];
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
      for (int ii = 0; ii < GI; ++ii)
#pragma unroll
        for (int jj = 0; jj < GJ; ++jj) g[p][ii][jj] = 0.f;
    fetch(o0);
    for (int t0 = o0; t0 < o1; t0 += PT) {
      const int np = min(PT, o1 - t0);
      __syncthreads();  // previous tile consumed (and R^T written, on the first tile)
      stage();
      __syncthreads();
      if (t0 + PT < o1) fetch(t0 + PT);
      if (warp < 4) {
        // U: 4 positions x 4 columns per thread, and the partial dw of this block
        const int jg = tid % (B / 4), pos0 = (tid / (B / 4)) * 4;
        float acc[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        if (pos0 < np) {
#pragma unroll 8
          for (int i2 = 0; i2 < 2 * B; ++i2) {
            const float4 dv = *reinterpret_cast<const float4*>(Dt + i2 * LDT + (pos0 ^ moe_swz(i2)));
            const float4 rv = *reinterpret_cast<const float4*>(Rc + i2 * LDR + jg * 4);
            const float d4[4] = {dv.x, dv.y, dv.z, dv.w}, r4[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
              for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(d4[a], r4[c], acc[a][c]);
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int row = jg * 4 + c;
            const float4 xv = *reinterpret_cast<const float4*>(Xt + row * LDT + (pos0 ^ moe_swz(row)));
            s[0] = fmaf(acc[0][c], xv.x, s[0]);
            s[1] = fmaf(acc[1][c], xv.y, s[1]);
            s[2] = fmaf(acc[2][c], xv.z, s[2]);
            s[3] = fmaf(acc[3][c], xv.w, s[3]);
          }
        }
#pragma unroll
        for (int o = 1; o < B / 4; o <<= 1)
#pragma unroll
          for (int a = 0; a < 4; ++a) s[a] += __shfl_xor_sync(0xFFFFFFFFu, s[a], o);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          if (pos0 + a < np) {
            *reinterpret_cast<float4*>(U + static_cast<size_t>(t0 + pos0 + a) * K + blk * B + jg * 4) =
                make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
            if (jg == 0) dwp[static_cast<size_t>(t0 + pos0 + a) * nb + blk] = s[a];
          }
        }
      } else {
        // G_p += X^T (w D_p): rows gi + 16 ii, columns gj + 8 jj, four positions per step
        const int gt = tid - 128, gj = gt % 8, gi = gt / 8;
        for (int pos0 = 0; pos0 < np; pos0 += 4) {
          const float4 w4 = *reinterpret_cast<const float4*>(ws + pos0);
          float4 xv[GI];
#pragma unroll
          for (int ii = 0; ii < GI; ++ii) {
            const int row = gi + 16 * ii;
            const float4 x = *reinterpret_cast<const float4*>(Xt + row * LDT + (pos0 ^ moe_swz(row)));
            xv[ii] = make_float4(x.x * w4.x, x.y * w4.y, x.z * w4.z, x.w * w4.w);
          }
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int jj = 0; jj < GJ; ++jj) {
              const int row = p * B + gj + 8 * jj;
              const float4 dv = *reinterpret_cast<const float4*>(Dt + row * LDT + (pos0 ^ moe_swz(row)));
#pragma unroll
              for (int ii = 0; ii < GI; ++ii) {
                float a = g[p][ii][jj];
                a = fmaf(xv[ii].x, dv.x, a);
                a = fmaf(xv[ii].y, dv.y, a);
                a = fmaf(xv[ii].z, dv.z, a);
                a = fmaf(xv[ii].w, dv.w, a);
                g[p][ii][jj] = a;
              }
            }
        }
      }
    }
    __syncthreads();  // tiles consumed: the region becomes Cayley scratch
    for (int idx = tid; idx < 2 * B; idx += 256) Rc[(idx / B) * B * LDR + (idx % B) * (LDR + 1)] += 1.f;  // (I + R_p)^T
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      if (warp >= 4) {
        const int gt = tid - 128, gj = gt % 8, gi = gt / 8;
#pragma unroll
        for (int ii = 0; ii < GI; ++ii)
#pragma unroll
          for (int jj = 0; jj < GJ; ++jj) Gs[(gi + 16 * ii) * LDC + gj + 8 * jj] = g[p][ii][jj];
      }
      __syncthreads();
      const float* T = Rc + p * B * LDR;
      float o[TI][TI];
#pragma unroll
      for (int x = 0; x < TI; ++x)
#pragma unroll
        for (int y = 0; y < TI; ++y) o[x][y] = 0.f;
#pragma unroll 4
      for (int l = 0; l < B; ++l) {  // U = T G
        float tv[TI], gv[TI];
#pragma unroll
        for (int x = 0; x < TI; ++x) tv[x] = T[(ti + x) * LDR + l];
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
        for (int y = 0; y < TI; ++y) tv[y] = T[l * LDR + tj + y];
#pragma unroll
        for (int x = 0; x < TI; ++x)
#pragma unroll
          for (int y = 0; y < TI; ++y) o[x][y] = fmaf(uv[x], tv[y], o[x][y]);
      }
      __syncthreads();  // every thread is done reading G before it is overwritten
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
