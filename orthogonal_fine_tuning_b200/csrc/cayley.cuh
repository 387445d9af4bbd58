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
  __shared__ __align__(16) float piv[2][BPC][B];
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
#pragma unroll
  for (int c = 0; c < B; ++c) {
    float* pr = piv[c & 1][sub];
    if (r == c) {
      const float p = __frcp_rn(a[c]);  // correctly rounded
#pragma unroll
      for (int j = 0; j < B; ++j) a[j] = (j == c) ? p : a[j] * p;
#pragma unroll
      for (int j = 0; j < B; j += 4) *reinterpret_cast<float4*>(pr + j) = make_float4(a[j], a[j + 1], a[j + 2], a[j + 3]);
    }
    block_sync();
    if (r != c) {
      const float f = a[c];
#pragma unroll
      for (int j = 0; j < B; j += 4) {
        const float4 v = *reinterpret_cast<const float4*>(pr + j);
        const float w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) a[j + t] = (j + t == c) ? -f * w[t] : fmaf(-f, w[t], a[j + t]);
      }
    }
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
// serial pivot chain sets the time: TPR threads per row, each holding a 1/TPR
// slice of the row's sliding window over the uneliminated columns of A and of the
// right-hand side, so every pivot costs each thread 1/TPR of the loads and FMAs.
// Per pivot, one shuffle brings the row's pivot-column element (held by the
// group's first thread) to the others, and one carries the element that crosses
// from each slice to the previous one when the window shifts.  Same sweep as the one-thread-per-row kernel: the
// pivot row is published through double-buffered shared memory, rows are never
// normalised during the sweep, and each row divides by its own pivot at the end.
template <int B, int TPR>
__global__ void __launch_bounds__(TPR * B) cayley_fwd_split_kernel(const uint16_t* __restrict__ Q, int nblocks,
                                                                 float* __restrict__ R,
                                                                 const int* __restrict__ active_list,
                                                                 const int* __restrict__ n_active,
                                                                 int blocks_per_expert, long long lo_off) {
  constexpr int H = B / TPR;  // columns per thread
  static_assert(H % 4 == 0 && (TPR & (TPR - 1)) == 0, "slices of whole float4s");
  __shared__ __align__(16) float piv[2][2 * B + 4];
  __shared__ __align__(16) uint16_t qsh[B * (B - 1) / 2];
  const int r = threadIdx.x / TPR, h = threadIdx.x % TPR;
  const unsigned full = 0xFFFFFFFFu;
  pdl_wait();
  const int total = active_list != nullptr ? min(nblocks, *n_active * blocks_per_expert) : nblocks;
  for (int lin = blockIdx.x; lin < total; lin += gridDim.x) {
    int blk = lin;
    if (active_list != nullptr) blk = active_list[lin / blocks_per_expert] * blocks_per_expert + lin % blocks_per_expert;
    __syncthreads();  // the previous block is done with qsh and piv
    stage_q<B>(Q + static_cast<size_t>(blk) * (B * (B - 1) / 2), qsh, threadIdx.x, TPR * B);
    __syncthreads();
    const uint16_t* q = qsh;
    float a[H], rhs[H];
#pragma unroll
    for (int k = 0; k < H; ++k) {
      const int j = h * H + k;
      float v = 0.f;
      if (j != r) {
        const float t = bf16_bits_to_f32(q[j > r ? tri_index(r, j, B) : tri_index(j, r, B)]);
        v = j > r ? t : -t;  // Q[r][j]
      }
      const float d = (j == r) ? 1.f : 0.f;
      a[k] = d - v;
      rhs[k] = d + v;
    }
    float my_inv = 1.f;
#pragma unroll 1
    for (int c = 0; c < B; ++c) {
      float* pr = piv[c & 1];
      // the row's pivot-column element A[r][c] is the first thread's a[0]
      const float arc = __shfl_sync(full, a[0], threadIdx.x & ~(TPR - 1));
      if (r == c) {
        if (h == 0) pr[2 * B] = __frcp_rn(a[0]);  // >= 1 in exact arithmetic; correctly rounded
#pragma unroll
        for (int k = 0; k < H; k += 4) {
          *reinterpret_cast<float4*>(pr + h * H + k) = make_float4(a[k], a[k + 1], a[k + 2], a[k + 3]);
          *reinterpret_cast<float4*>(pr + B + h * H + k) = make_float4(rhs[k], rhs[k + 1], rhs[k + 2], rhs[k + 3]);
        }
      }
      __syncthreads();
      const float inv = pr[2 * B];
      if (r == c) my_inv = inv;
      const float f = (r == c) ? 0.f : arc * inv;
#pragma unroll
      for (int k = 0; k < H; k += 4) {
        const float4 v = *reinterpret_cast<const float4*>(pr + h * H + k);
        const float4 w = *reinterpret_cast<const float4*>(pr + B + h * H + k);
        a[k] = fmaf(-f, v.x, a[k]);
        a[k + 1] = fmaf(-f, v.y, a[k + 1]);
        a[k + 2] = fmaf(-f, v.z, a[k + 2]);
        a[k + 3] = fmaf(-f, v.w, a[k + 3]);
        rhs[k] = fmaf(-f, w.x, rhs[k]);
        rhs[k + 1] = fmaf(-f, w.y, rhs[k + 1]);
        rhs[k + 2] = fmaf(-f, w.z, rhs[k + 2]);
        rhs[k + 3] = fmaf(-f, w.w, rhs[k + 3]);
      }
      // drop column c: the window moves one column right across the pair
      const float nxt = __shfl_down_sync(full, a[0], 1);  // the next slice's first element
#pragma unroll
      for (int k = 0; k < H - 1; ++k) a[k] = a[k + 1];
      a[H - 1] = h < TPR - 1 ? nxt : 0.f;
    }
    if (lo_off > 0) {
#pragma unroll
      for (int k = 0; k < H; ++k) store_r_hl_t(R, lo_off, blk, B, r, h * H + k, rhs[k] * my_inv);
    } else {
      float* out = R + (static_cast<size_t>(blk) * B + r) * B + h * H;
#pragma unroll
      for (int k = 0; k < H; k += 4)
        *reinterpret_cast<float4*>(out + k) =
            make_float4(rhs[k] * my_inv, rhs[k + 1] * my_inv, rhs[k + 2] * my_inv, rhs[k + 3] * my_inv);
    }
  }
}

// dQ[blk] = pack(D - D^T), D = 1/2 (I+R)^T G (I+R)^T.
// G is read either directly ([nblocks][b][b], nparts = 1) or as `nparts` partial
// sums laid out [nblocks][nparts][b][b], summed in part order (deterministic).
// With a map (the MoE's active experts), only the blocks map[i] * per + r for
// i < *n_map and r < per are computed; the others are left as they are.
// One CTA per block; each thread owns a TI x TI tile of the two b x b products.
// Dynamic shared memory: 3 * B * (B + 1) floats.
template <int B>
__global__ void __launch_bounds__(kCayleyThreads) cayley_bwd_kernel(const float* __restrict__ R,
                                                                    const float* __restrict__ G, int nparts,
                                                                    int nblocks, float* __restrict__ dQ,
                                                                    const int* __restrict__ map,
                                                                    const int* __restrict__ n_map, int per) {
  constexpr int TI = (B == 64) ? 4 : (B == 32 ? 2 : 1);
  constexpr int NT = B / TI;  // threads per output row of tiles
  static_assert(NT * NT == kCayleyThreads, "tile grid must cover the CTA");
  constexpr int LD = B + 1;
  extern __shared__ float csm[];
  float* T = csm;               // (I + R)^T
  float* Gs = csm + B * LD;     // G, then D * 2
  float* U = csm + 2 * B * LD;  // T G
  const int tid = threadIdx.x;
  const int ti = (tid / NT) * TI, tj = (tid % NT) * TI;
  pdl_wait();
  const int count = map != nullptr ? *n_map * per : nblocks;
  for (int it = blockIdx.x; it < count; it += gridDim.x) {
    const int blk = map != nullptr ? map[it / per] * per + it % per : it;
    const float* rb = R + static_cast<size_t>(blk) * B * B;
    const float* gb = G + static_cast<size_t>(blk) * nparts * B * B;
    constexpr int EPT = B * B / kCayleyThreads;  // elements per thread
    float acc[EPT], rv[EPT];
#pragma unroll
    for (int k = 0; k < EPT; ++k) {
      rv[k] = rb[tid + k * kCayleyThreads];
      acc[k] = 0.f;
    }
    for (int p = 0; p < nparts; p += 4) {  // 4 * EPT independent loads in flight, summed in part order
      float t[4][EPT];
#pragma unroll
      for (int pp = 0; pp < 4; ++pp)
#pragma unroll
        for (int k = 0; k < EPT; ++k)
          t[pp][k] = (p + pp < nparts) ? gb[static_cast<size_t>(p + pp) * B * B + tid + k * kCayleyThreads] : 0.f;
#pragma unroll
      for (int pp = 0; pp < 4; ++pp)
#pragma unroll
        for (int k = 0; k < EPT; ++k) acc[k] += t[pp][k];
    }
#pragma unroll
    for (int k = 0; k < EPT; ++k) {
      const int idx = tid + k * kCayleyThreads;
      const int i = idx / B, j = idx % B;
      T[j * LD + i] = rv[k] + (i == j ? 1.f : 0.f);
      Gs[i * LD + j] = acc[k];
    }
    __syncthreads();
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
      for (int y = 0; y < TI; ++y) gv[y] = Gs[l * LD + tj + y];
#pragma unroll
      for (int x = 0; x < TI; ++x)
#pragma unroll
        for (int y = 0; y < TI; ++y) o[x][y] = fmaf(tv[x], gv[y], o[x][y]);
    }
#pragma unroll
    for (int x = 0; x < TI; ++x)
#pragma unroll
      for (int y = 0; y < TI; ++y) U[(ti + x) * LD + tj + y] = o[x][y];
    __syncthreads();
#pragma unroll
    for (int x = 0; x < TI; ++x)
#pragma unroll
      for (int y = 0; y < TI; ++y) o[x][y] = 0.f;
#pragma unroll 4
    for (int l = 0; l < B; ++l) {  // 2D = U T
      float uv[TI], tv[TI];
#pragma unroll
      for (int x = 0; x < TI; ++x) uv[x] = U[(ti + x) * LD + l];
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
      for (int y = 0; y < TI; ++y) Gs[(ti + x) * LD + tj + y] = o[x][y];
    __syncthreads();
    float* out = dQ + static_cast<size_t>(blk) * (B * (B - 1) / 2);
    for (int idx = tid; idx < B * B; idx += kCayleyThreads) {
      const int i = idx / B, j = idx % B;
      if (i < j) out[tri_index(i, j, B)] = 0.5f * (Gs[i * LD + j] - Gs[j * LD + i]);
    }
    __syncthreads();
  }
}

}  // namespace oftk
