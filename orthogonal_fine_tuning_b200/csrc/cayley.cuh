// Cayley map of the OFT adapter and its backward.
//
// OFT parameterises each block of the orthogonal rotation by a skew-symmetric Q
// (the pages name OFT as Orbit's default adapter: chooseai.io news 4086, section
// "技术原理：低精度基座 + BF16 适配器 + OFT"):
//     R = (I + Q)(I - Q)^-1 = (I - Q)^-1 (I + Q)
// Forward: solve (I - Q) R = (I + Q) by Gauss-Jordan elimination in fp32
// without pivoting.  I - Q has symmetric part I, so x^T (I-Q) x = |x|^2 > 0:
// every leading minor is non-zero, every pivot stays >= 1 in exact arithmetic,
// and sigma_min(I - Q) >= 1 (the solve is well conditioned for any Q).
// Backward: with G = dL/dR, dL/dQ = 1/2 (I + R)^T G (I + R)^T, projected onto the
// packed strict-upper parameters as dq_ij = D_ij - D_ji.
#pragma once

#include "common.cuh"

namespace oftk {

constexpr int kCayleyThreads = 256;
constexpr int kCayleyUnrollBlocks = 4096;  // forward launches at least this large use the unrolled pivots

__host__ __device__ __forceinline__ int tri_index(int i, int j, int b) {  // i < j, row-major strict upper
  return i * b - i * (i + 1) / 2 + (j - i - 1);
}

// Forward, one thread per matrix row: thread r keeps row r of A = I - Q and of
// the right-hand side I + Q in registers.  At pivot c the pivot row is published
// through shared memory (double-buffered, so one barrier per pivot).  UNROLL = true unrolls the pivot loop, so every register index is
// static and only the columns right of c are updated: the fastest form when
// many blocks share each SM's instruction cache (the MoE build of every active
// expert).  UNROLL = false keeps a small rolled loop over a sliding window of
// the uneliminated columns, for launches of a few hundred blocks, where the
// unrolled code would mostly miss in the instruction cache.  CTAs are one warp (B = 16: two blocks; B = 32: one) or two warps
// (B = 64, one block, block-wide barrier), so the serial pivot chains of many
// blocks interleave on every SM.
// Q: bf16 [nblocks][B(B-1)/2]; R: fp32 [nblocks][B][B].  The grid is persistent:
// each CTA walks blocks with a stride of the whole grid.  With an active-expert
// list (MoE), only the blocks of the first *n_active experts of `active` are
// built: linear block i is block i % blocks_per_expert of expert
// active[i / blocks_per_expert].
// Stage one block's packed Q (B(B-1)/2 bf16 = B(B-1)/16 16-byte vectors; blocks
// are 16-byte aligned for B = 16, 32, 64) in shared memory with coalesced vector
// loads by the block's `nthr` threads, so each thread then gathers its row's
// entries from shared memory instead of with scattered 2-byte global loads.
template <int B>
__device__ __forceinline__ void stage_q(const uint16_t* __restrict__ q, uint16_t* qs, int t, int nthr) {
  constexpr int NV = B * (B - 1) / 16;
  for (int v = t; v < NV; v += nthr)
    reinterpret_cast<uint4*>(qs)[v] = reinterpret_cast<const uint4*>(q)[v];
}

// Second output form of the forward (lo_off > 0): R^T of each block as bf16 hi and lo
// parts, hi = bf16_rne(R[r][c]) at element [c][r] of the block's B x B slice of
// (uint16_t*)R, and lo = bf16_rne(R[r][c] - hi) lo_off elements further.  This is the
// operand the MoE rotated gather feeds to its bf16 MMAs (R = hi + lo to about 2^-16),
// laid out so that 8 consecutive reduction indices are one 16-byte load.
__device__ __forceinline__ void store_r_hl_t(float* R, long long lo_off, int blk, int B, int r, int c, float v) {
  uint16_t* hi = reinterpret_cast<uint16_t*>(R) + (static_cast<long long>(blk) * B + c) * B + r;
  const uint16_t h = f32_to_bf16_bits(v);
  hi[0] = h;
  hi[lo_off] = f32_to_bf16_bits(v - bf16_bits_to_f32(h));
}

template <int B>
struct CayleyFwdCfg {
  static constexpr int THREADS = B < 32 ? 32 : B;
  static constexpr int BPC = THREADS / B;  // blocks per CTA
  static constexpr int MIN_CTAS = B == 64 ? 8 : 24;  // resident CTAs per SM the register budget allows
};

template <int B, bool UNROLL>
__device__ __forceinline__ void cayley_fwd_block(const uint16_t* __restrict__ Q, float* __restrict__ R, int lin,
                                                 int total, const int* __restrict__ active_list,
                                                 int blocks_per_expert, long long lo_off) {
  constexpr int BPC = CayleyFwdCfg<B>::BPC;
  __shared__ __align__(16) float piv[2][BPC][2 * B + 4];  // pivot row, right-hand side, 1 / pivot
  __shared__ __align__(16) uint16_t qsh[BPC][B * (B - 1) / 2];
  const int sub = threadIdx.x / B, r = threadIdx.x % B;
  const bool active = lin < total;  // B = 16: the CTA's second block may run past the end
  int blk = lin;
  if (active && active_list != nullptr)
    blk = active_list[lin / blocks_per_expert] * blocks_per_expert + lin % blocks_per_expert;
  auto block_sync = [&]() {
    if constexpr (B <= 32) {
      __syncwarp();
    } else {
      __syncthreads();
    }
  };

  float a[B], rhs[B];
  const uint16_t* q = qsh[sub];
  block_sync();  // the previous block of this CTA is done with qsh and piv
  if (active) stage_q<B>(Q + static_cast<size_t>(blk) * (B * (B - 1) / 2), qsh[sub], r, B);
  block_sync();
#pragma unroll
  for (int j = 0; j < B; ++j) {
    float v = 0.f;
    if (active && j != r) {
      const float t = bf16_bits_to_f32(q[j > r ? tri_index(r, j, B) : tri_index(j, r, B)]);
      v = j > r ? t : -t;  // Q[r][j]
    }
    const float d = (j == r) ? 1.f : 0.f;
    a[j] = d - v;
    rhs[j] = d + v;
  }

  // Rows are never normalised during the sweep: the pivot row stays as it is and
  // every other row subtracts f = A[r][c] / A[c][c] times it, so all threads run
  // the same instructions (the pivot row with f = 0).  The pivot thread computes
  // 1 / A[c][c] once and publishes it with its row; at the end each row divides
  // by its own pivot.
  float my_inv = 1.f;
  if constexpr (UNROLL) {
#pragma unroll
    for (int c = 0; c < B; ++c) {
      float* pr = piv[c & 1][sub];
      const int k0 = c & ~3;  // first float4 holding a column >= c
      if (r == c) {
        my_inv = __frcp_rn(a[c]);  // >= 1 in exact arithmetic, so never a zero pivot; correctly rounded
        pr[2 * B] = my_inv;
#pragma unroll
        for (int k = k0; k < B; k += 4)
          *reinterpret_cast<float4*>(pr + k) = make_float4(a[k], a[k + 1], a[k + 2], a[k + 3]);
#pragma unroll
        for (int k = 0; k < B; k += 4)
          *reinterpret_cast<float4*>(pr + B + k) = make_float4(rhs[k], rhs[k + 1], rhs[k + 2], rhs[k + 3]);
      }
      block_sync();
      const float f = (r == c) ? 0.f : a[c] * pr[2 * B];
#pragma unroll
      for (int k = k0; k < B; k += 4) {
        if (k + 3 <= c) continue;
        const float4 v = *reinterpret_cast<const float4*>(pr + k);
        if (k + 0 > c) a[k + 0] = fmaf(-f, v.x, a[k + 0]);
        if (k + 1 > c) a[k + 1] = fmaf(-f, v.y, a[k + 1]);
        if (k + 2 > c) a[k + 2] = fmaf(-f, v.z, a[k + 2]);
        a[k + 3] = fmaf(-f, v.w, a[k + 3]);
      }
#pragma unroll
      for (int k = 0; k < B; k += 4) {
        const float4 v = *reinterpret_cast<const float4*>(pr + B + k);
        rhs[k] = fmaf(-f, v.x, rhs[k]);
        rhs[k + 1] = fmaf(-f, v.y, rhs[k + 1]);
        rhs[k + 2] = fmaf(-f, v.z, rhs[k + 2]);
        rhs[k + 3] = fmaf(-f, v.w, rhs[k + 3]);
      }
    }
  } else {
    // rolled: a[k] = A[r][c + k] is a window over the columns not yet eliminated,
    // shifted left after each pivot, so the pivot element is always a[0]
#pragma unroll 1
    for (int c = 0; c < B; ++c) {
      float* pr = piv[c & 1][sub];
      if (r == c) {
        my_inv = __frcp_rn(a[0]);
        pr[2 * B] = my_inv;
#pragma unroll
        for (int k = 0; k < B; k += 4) {
          *reinterpret_cast<float4*>(pr + k) = make_float4(a[k], a[k + 1], a[k + 2], a[k + 3]);
          *reinterpret_cast<float4*>(pr + B + k) = make_float4(rhs[k], rhs[k + 1], rhs[k + 2], rhs[k + 3]);
        }
      }
      block_sync();
      const float f = (r == c) ? 0.f : a[0] * pr[2 * B];
#pragma unroll
      for (int k = 0; k < B; k += 4) {
        const float4 v = *reinterpret_cast<const float4*>(pr + k);
        const float4 w = *reinterpret_cast<const float4*>(pr + B + k);
        a[k] = fmaf(-f, v.x, a[k]);
        a[k + 1] = fmaf(-f, v.y, a[k + 1]);
        a[k + 2] = fmaf(-f, v.z, a[k + 2]);
        a[k + 3] = fmaf(-f, v.w, a[k + 3]);
        rhs[k] = fmaf(-f, w.x, rhs[k]);
        rhs[k + 1] = fmaf(-f, w.y, rhs[k + 1]);
        rhs[k + 2] = fmaf(-f, w.z, rhs[k + 2]);
        rhs[k + 3] = fmaf(-f, w.w, rhs[k + 3]);
      }
      // drop the eliminated column c: the window moves one column right
#pragma unroll
      for (int k = 0; k < B - 1; ++k) a[k] = a[k + 1];
      a[B - 1] = 0.f;
    }
  }
#pragma unroll
  for (int k = 0; k < B; ++k) rhs[k] *= my_inv;
  if (active && lo_off > 0) {
#pragma unroll
    for (int j = 0; j < B; ++j) store_r_hl_t(R, lo_off, blk, B, r, j, rhs[j]);
  } else if (active) {
    float* out = R + (static_cast<size_t>(blk) * B + r) * B;
#pragma unroll
    for (int j = 0; j < B; j += 4)
      *reinterpret_cast<float4*>(out + j) = make_float4(rhs[j], rhs[j + 1], rhs[j + 2], rhs[j + 3]);
  }
}

// Many-block form (UNROLL = true): in-place Gauss-Jordan inversion of A = I - Q with
// one thread per row, then R = 2 A^-1 - I, since I + R = 2 (I - Q)^-1.  Each pivot
// publishes one row of B values and every other row updates B entries, against 2B
// of each for elimination on [A | I + Q]; with half the row state in registers more
// blocks stay resident per SM.  The pivot loop is fully unrolled, so every register
// index is static.  No pivoting: every pivot is >= 1 in exact arithmetic.
template <int B>
__device__ __forceinline__ void cayley_fwd_block_inv(const uint16_t* __restrict__ Q, float* __restrict__ R, int lin,
                                                     int total, const int* __restrict__ active_list,
                                                     int blocks_per_expert, long long lo_off) {
  constexpr int BPC = CayleyFwdCfg<B>::BPC;
  __shared__ __align__(16) float piv[2][BPC][B + 4];  // pivot row, then its reciprocal
  __shared__ __align__(16) uint16_t qsh[BPC][B * (B - 1) / 2];
  const int sub = threadIdx.x / B, r = threadIdx.x % B;
  const bool active = lin < total;  // B = 16: the CTA's second block may run past the end
  int blk = lin;
  if (active && active_list != nullptr)
    blk = active_list[lin / blocks_per_expert] * blocks_per_expert + lin % blocks_per_expert;
  auto block_sync = [&]() {
    if constexpr (B <= 32) {
      __syncwarp();
    } else {
      __syncthreads();
    }
  };
  block_sync();  // the previous block of this CTA is done with qsh and piv
  if (active) stage_q<B>(Q + static_cast<size_t>(blk) * (B * (B - 1) / 2), qsh[sub], r, B);
  block_sync();
  const uint16_t* q = qsh[sub];
  float a[B];
#pragma unroll
  for (int j = 0; j < B; ++j) {
    float v = 0.f;
    if (active && j != r) {
      const float t = bf16_bits_to_f32(q[j > r ? tri_index(r, j, B) : tri_index(j, r, B)]);
      v = j > r ? t : -t;  // Q[r][j]
    }
    a[j] = ((j == r) ? 1.f : 0.f) - v;
  }
  // Pivot c in one uniform update for every row: with p = 1 / A[c][c] and the pivot row
  // P = A[c][:] published as it is, each row r takes f = (A[r][c] - [r == c]) p and
  // A[r][j] -= f P[j] for j != c, then A[r][c] = -f (r != c) or p (r = c).  For r != c
  // this is the elimination step of the in-place inverse; for r = c it scales the row
  // by p (A[c][j] - (A[c][c] - 1) p A[c][j] = A[c][j] p).  Only the publication (one
  // reciprocal and B / 4 vector stores) runs on the pivot row's thread alone.
#pragma unroll
  for (int c = 0; c < B; ++c) {
    float* pr = piv[c & 1][sub];
    if (r == c) {
      pr[B] = __frcp_rn(a[c]);  // correctly rounded; A[c][c] >= 1 in exact arithmetic
#pragma unroll
      for (int j = 0; j < B; j += 4) *reinterpret_cast<float4*>(pr + j) = make_float4(a[j], a[j + 1], a[j + 2], a[j + 3]);
    }
    block_sync();
    const float pinv = pr[B];
    const float f = (a[c] - (r == c ? 1.f : 0.f)) * pinv;
#pragma unroll
    for (int j = 0; j < B; j += 4) {
      const float4 v = *reinterpret_cast<const float4*>(pr + j);
      const float w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (j + t != c) a[j + t] = fmaf(-f, w[t], a[j + t]);
    }
    a[c] = (r == c) ? pinv : -f;
  }
  if (active && lo_off > 0) {
#pragma unroll
    for (int j = 0; j < B; ++j) store_r_hl_t(R, lo_off, blk, B, r, j, 2.f * a[j] - (j == r ? 1.f : 0.f));
  } else if (active) {
    float* out = R + (static_cast<size_t>(blk) * B + r) * B;
#pragma unroll
    for (int j = 0; j < B; j += 4)
      *reinterpret_cast<float4*>(out + j) =
          make_float4(2.f * a[j] - (j == r ? 1.f : 0.f), 2.f * a[j + 1] - (j + 1 == r ? 1.f : 0.f),
                      2.f * a[j + 2] - (j + 2 == r ? 1.f : 0.f), 2.f * a[j + 3] - (j + 3 == r ? 1.f : 0.f));
  }
}

template <int B, bool UNROLL>
__global__ void __launch_bounds__(CayleyFwdCfg<B>::THREADS, CayleyFwdCfg<B>::MIN_CTAS) cayley_fwd_kernel(const uint16_t* __restrict__ Q,
                                                                               int nblocks, float* __restrict__ R,
                                                                               const int* __restrict__ active_list,
                                                                               const int* __restrict__ n_active,
                                                                               int blocks_per_expert, long long lo_off) {
  constexpr int BPC = CayleyFwdCfg<B>::BPC;
  pdl_wait();
  const int total = active_list != nullptr ? min(nblocks, *n_active * blocks_per_expert) : nblocks;
  for (int base = blockIdx.x * BPC; base < total; base += gridDim.x * BPC) {
    if constexpr (UNROLL) {
      cayley_fwd_block_inv<B>(Q, R, base + threadIdx.x / B, total, active_list, blocks_per_expert, lo_off);
    } else {
      cayley_fwd_block<B, UNROLL>(Q, R, base + threadIdx.x / B, total, active_list, blocks_per_expert, lo_off);
    }
  }
}

// Forward for launches of a few hundred blocks (b = 32, 64), where each block's
// serial pivot chain sets the time: the in-place inversion of the many-block form
// (R = 2 (I - Q)^-1 - I, one uniform update per pivot), with each row split over TPR
// threads that hold H = B / TPR consecutive columns each, so a pivot costs each
// thread H FMAs and H / 4 vector loads.  The row's pivot-column element comes from
// the thread holding it by one shuffle; the pivot row's TPR threads publish it
// through double-buffered shared memory (one barrier per pivot).  The pivot loop is
// unrolled, so every register index is static.
template <int B, int TPR>
__global__ void __launch_bounds__(TPR * B) cayley_fwd_inv_split_kernel(const uint16_t* __restrict__ Q, int nblocks,
                                                                     float* __restrict__ R,
                                                                     const int* __restrict__ active_list,
                                                                     const int* __restrict__ n_active,
                                                                     int blocks_per_expert, long long lo_off) {
  constexpr int H = B / TPR;  // columns per thread
  static_assert(H % 4 == 0 && (TPR & (TPR - 1)) == 0 && 32 % TPR == 0, "slices of whole float4s");
  __shared__ __align__(16) float piv[2][B + 4];  // pivot row, then its reciprocal
  __shared__ __align__(16) uint16_t qsh[B * (B - 1) / 2];
  const int r = threadIdx.x / TPR, h = threadIdx.x % TPR;
  const int lane0 = (threadIdx.x & 31) & ~(TPR - 1);  // this row's first lane in the warp
  const unsigned full = 0xFFFFFFFFu;
  pdl_wait();
  const int total = active_list != nullptr ? min(nblocks, *n_active * blocks_per_expert) : nblocks;
  for (int lin = blockIdx.x; lin < total; lin += gridDim.x) {
    int blk = lin;
    if (active_list != nullptr) blk = active_list[lin / blocks_per_expert] * blocks_per_expert + lin % blocks_per_expert;
    __syncthreads();  // the previous block is done with qsh and piv
    stage_q<B>(Q + static_cast<size_t>(blk) * (B * (B - 1) / 2), qsh, threadIdx.x, TPR * B);
    __syncthreads();
    float a[H];
#pragma unroll
    for (int k = 0; k < H; ++k) {
      const int j = h * H + k;
      float v = 0.f;
      if (j != r) {
        const float t = bf16_bits_to_f32(qsh[j > r ? tri_index(r, j, B) : tri_index(j, r, B)]);
        v = j > r ? t : -t;  // Q[r][j]
      }
      a[k] = (j == r ? 1.f : 0.f) - v;
    }
#pragma unroll
    for (int c = 0; c < B; ++c) {
      const int owner = c / H, kc = c % H;
      float* pr = piv[c & 1];
      const float arc = __shfl_sync(full, a[kc], lane0 + owner);  // A[r][c]
      if (r == c) {
#pragma unroll
        for (int k = 0; k < H; k += 4)
          *reinterpret_cast<float4*>(pr + h * H + k) = make_float4(a[k], a[k + 1], a[k + 2], a[k + 3]);
        if (h == owner) pr[B] = __frcp_rn(arc);  // correctly rounded; A[c][c] >= 1 in exact arithmetic
      }
      __syncthreads();
      const float pinv = pr[B];
      const float f = (arc - (r == c ? 1.f : 0.f)) * pinv;
#pragma unroll
      for (int k = 0; k < H; k += 4) {
        const float4 v = *reinterpret_cast<const float4*>(pr + h * H + k);
        a[k] = fmaf(-f, v.x, a[k]);
        a[k + 1] = fmaf(-f, v.y, a[k + 1]);
        a[k + 2] = fmaf(-f, v.z, a[k + 2]);
        a[k + 3] = fmaf(-f, v.w, a[k + 3]);
      }
      if (h == owner) a[kc] = (r == c) ? pinv : -f;  // column c of the inverse
    }
    if (lo_off > 0) {
#pragma unroll
      for (int k = 0; k < H; ++k) {
        const int j = h * H + k;
        store_r_hl_t(R, lo_off, blk, B, r, j, 2.f * a[k] - (j == r ? 1.f : 0.f));
      }
    } else {
      float* out = R + (static_cast<size_t>(blk) * B + r) * B + h * H;
#pragma unroll
      for (int k = 0; k < H; k += 4) {
        const int j = h * H + k;
        *reinterpret_cast<float4*>(out + k) =
            make_float4(2.f * a[k] - (j == r ? 1.f : 0.f), 2.f * a[k + 1] - (j + 1 == r ? 1.f : 0.f),
                        2.f * a[k + 2] - (j + 2 == r ? 1.f : 0.f), 2.f * a[k + 3] - (j + 3 == r ? 1.f : 0.f));
      }
    }
  }
}


// dQ[blk] = pack(D - D^T), D = 1/2 (I+R)^T G (I+R)^T.
// G is read either directly ([nblocks][b][b], nparts = 1) or as `nparts` partial
// sums laid out [nblocks][nparts][b][b], summed in part order (deterministic).
// With a map (the MoE's active experts), only the blocks map[i] * per + r for
// i < *n_map and r < per are computed; the others are left as they are.
// Each thread owns a 4 x 4 tile of the two b x b products, so a CTA of blockDim.x
// threads works on blockDim.x / (b/4)^2 blocks at once (up to 16, 4, 1 for b = 16,
// 32, 64; the host takes fewer when the launch has few blocks).  Per block
// the shared memory holds I + R, its transpose T, G (later 2D) and (T G)^T, rows
// padded to b + 4 floats, so that both operands of every product step are float4
// reads: 2 vector loads per 16 FMAs.
template <int B>
struct CayleyBwdCfg {
  static constexpr int NT = (B / 4) * (B / 4);        // threads per block
  static constexpr int BPC = kCayleyThreads / NT;     // most blocks per CTA
  static constexpr int LD = B + 4;
  static constexpr int SZ = B * LD;                   // floats per array
  static constexpr size_t SMEM_PER_BLOCK = sizeof(float) * 4 * SZ;
};

template <int B>
__global__ void __launch_bounds__(kCayleyThreads) cayley_bwd_kernel(const float* __restrict__ R,
                                                                    const float* __restrict__ G, int nparts,
                                                                    int nblocks, float* __restrict__ dQ,
                                                                    const int* __restrict__ map,
                                                                    const int* __restrict__ n_map, int per) {
  using C = CayleyBwdCfg<B>;
  constexpr int NT = C::NT, LD = C::LD, SZ = C::SZ;
  const int BPC = blockDim.x / NT;
  constexpr int V = B * B / 4 / NT;  // float4s of a block per thread (4)
  extern __shared__ float4 cbw_smem[];
  const int sub = threadIdx.x / NT, t = threadIdx.x % NT;
  float* Tt = reinterpret_cast<float*>(cbw_smem) + sub * 4 * SZ;  // I + R: Tt[l][i] = T[i][l]
  float* T = Tt + SZ;                                              // T = (I + R)^T
  float* Gs = T + SZ;                                              // G, then 2D
  float* Mt = Gs + SZ;                                             // (T G)^T
  const int ti = (t / (B / 4)) * 4, tj = (t % (B / 4)) * 4;
  pdl_wait();
  const int count = map != nullptr ? *n_map * per : nblocks;
  for (int base = blockIdx.x * BPC; base < count; base += gridDim.x * BPC) {
    const int it = base + sub;
    const bool act = it < count;
    const int blk = !act ? 0 : (map != nullptr ? map[it / per] * per + it % per : it);
    __syncthreads();  // the previous blocks are done with shared memory
    if (act) {
      const float4* rb = reinterpret_cast<const float4*>(R + static_cast<size_t>(blk) * B * B);
      const float4* gb = reinterpret_cast<const float4*>(G + static_cast<size_t>(blk) * nparts * B * B);
      float4 rv[V], acc[V];
#pragma unroll
      for (int v = 0; v < V; ++v) {
        rv[v] = rb[t + v * NT];
        acc[v] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      for (int q = 0; q < nparts; q += 2) {  // two parts' loads in flight, summed in part order
        float4 g0[V], g1[V];
#pragma unroll
        for (int v = 0; v < V; ++v) {
          g0[v] = gb[static_cast<size_t>(q) * (B * B / 4) + t + v * NT];
          g1[v] = q + 1 < nparts ? gb[static_cast<size_t>(q + 1) * (B * B / 4) + t + v * NT]
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int v = 0; v < V; ++v) {
          acc[v] = make_float4(acc[v].x + g0[v].x, acc[v].y + g0[v].y, acc[v].z + g0[v].z, acc[v].w + g0[v].w);
          acc[v] = make_float4(acc[v].x + g1[v].x, acc[v].y + g1[v].y, acc[v].z + g1[v].z, acc[v].w + g1[v].w);
        }
      }
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int idx = (t + v * NT) * 4;
        const int i = idx / B, j0 = idx % B;
        const float e[4] = {rv[v].x + (i == j0 ? 1.f : 0.f), rv[v].y + (i == j0 + 1 ? 1.f : 0.f),
                            rv[v].z + (i == j0 + 2 ? 1.f : 0.f), rv[v].w + (i == j0 + 3 ? 1.f : 0.f)};
        *reinterpret_cast<float4*>(Tt + i * LD + j0) = make_float4(e[0], e[1], e[2], e[3]);
#pragma unroll
        for (int c = 0; c < 4; ++c) T[(j0 + c) * LD + i] = e[c];
        *reinterpret_cast<float4*>(Gs + i * LD + j0) = acc[v];
      }
    }
    __syncthreads();
    float o[4][4];
    if (act) {  // M = T G
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) o[x][y] = 0.f;
#pragma unroll 8
      for (int l = 0; l < B; ++l) {
        const float4 tv = *reinterpret_cast<const float4*>(Tt + l * LD + ti);  // T[ti + x][l]
        const float4 gv = *reinterpret_cast<const float4*>(Gs + l * LD + tj);  // G[l][tj + y]
        const float a4[4] = {tv.x, tv.y, tv.z, tv.w}, b4[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) o[x][y] = fmaf(a4[x], b4[y], o[x][y]);
      }
#pragma unroll
      for (int y = 0; y < 4; ++y)
        *reinterpret_cast<float4*>(Mt + (tj + y) * LD + ti) = make_float4(o[0][y], o[1][y], o[2][y], o[3][y]);
    }
    __syncthreads();
    if (act) {  // 2D = M T, over G's rows (G is no longer read)
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) o[x][y] = 0.f;
#pragma unroll 8
      for (int l = 0; l < B; ++l) {
        const float4 mv = *reinterpret_cast<const float4*>(Mt + l * LD + ti);  // M[ti + x][l]
        const float4 tv = *reinterpret_cast<const float4*>(T + l * LD + tj);   // T[l][tj + y]
        const float a4[4] = {mv.x, mv.y, mv.z, mv.w}, b4[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) o[x][y] = fmaf(a4[x], b4[y], o[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
        *reinterpret_cast<float4*>(Gs + (ti + x) * LD + tj) = make_float4(o[x][0], o[x][1], o[x][2], o[x][3]);
    }
    __syncthreads();
    if (act) {
      float* out = dQ + static_cast<size_t>(blk) * (B * (B - 1) / 2);
      for (int idx = t; idx < B * B; idx += NT) {
        const int i = idx / B, j = idx % B;
        if (i < j) out[tri_index(i, j, B)] = 0.5f * (Gs[i * LD + j] - Gs[j * LD + i]);
      }
    }
  }
}

}  // namespace oftk
