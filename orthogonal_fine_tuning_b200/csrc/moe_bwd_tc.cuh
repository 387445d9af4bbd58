// MoE backward rotations on the tcgen05 tensor cores (kind::tf32).
//
// The expert rows of D_p = dY_p W_e,p^T (fp32, bucket order: positions sorted by
// expert) go back through each expert's own rotations and into its adapter
// gradient, the contractions of the dense backward with a rotation and a gating
// weight per routed row ("Orbit", chooseai.io news 4086, section
// "对低精度 MoE 模型的专门优化"; the OFT backward itself is the standard one):
//
//   moe_rotb_tc_kernel: U[pos] = sum_p D_p[pos] R_e,p^T        (blockwise; R as tf32 hi + lo)
//   moe_grad_tc_kernel: G_e,p,blk = sum over e's positions of (w_pos X[t, blk])^T D_p[pos, blk]
//
// followed by the Cayley backward of every active expert's G (cayley_bwd_kernel
// with an expert map); dw_tk = <U[pos], X[t]> is formed by the combine pass over U.
// t = bucket[pos] / top_k is the routed token, w_pos its gating weight.
//
// Units are (active expert, column group), taken heaviest expert first and dealt
// round-robin to the CTAs, so each CTA's share is within one unit of the mean; a
// unit walks all of its expert's rows in tiles.  The last tile of an expert runs
// into the next expert's rows (or past the end, read as zeros): their U rows are
// computed with the wrong rotation but never written, and their X rows are staged
// as zeros so that they add nothing to G.
//
// Both kernels keep the dense kernels' roles (192 threads, one CTA per SM):
//   warp 0      TMA producer of the D tiles
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warps 2..5  build the per-unit operand (R tiles / weighted X tiles) in shared
//               memory and drain TMEM in the epilogue
// The two kernels read D in the two layouts its two contractions need: U reduces
// over D's columns (K-major, 128B swizzle), G over its rows (MN-major, the
// 32-byte-atom variant of the swizzle).
#pragma once

#include "common.cuh"
#include "rot_tc.cuh"

namespace oftk {
namespace rtc {

struct MoeUnit {
  int e, g, r0, r1;  // expert, column group, its bucket range [r0, r1)
};

// The k-th unit of this CTA; false past the last one.
__device__ __forceinline__ bool moe_unit(const int* order, const int* offsets, int n_units, int groups, int k,
                                         MoeUnit& u) {
  const int id = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
  if (id >= n_units) return false;
  u.e = order[id / groups];
  u.g = id % groups;
  u.r0 = offsets[u.e];
  u.r1 = offsets[u.e + 1];
  return true;
}

// ===========================================================================
// U = sum_p D_p R_e,p^T
// ===========================================================================
struct MoeRotbParams {
  CUtensorMap tmD;          // D fp32 3-D {K, TK, 2}, box {32, 128, 1}, 128B swizzle
  const float* R;           // [E][2][nb][b][b]
  const int* offsets;       // [E + 1]
  const int* order;         // active experts, heaviest first
  const int* n_active;
  float* U;                 // [TK][K], bucket order
  int K, TK, nb, groups;    // groups of 64 columns
};

constexpr int MRB_A_BYTES = TM * 64 * 4;  // one split's 128-row x 64-column fp32 tile (two 32-column boxes)
constexpr int MRB_STAGES = 3;
constexpr int MRB_ACC = 4;                // 64-column accumulators in TMEM
constexpr int MRB_B_BYTES = 2 * 2 * BWD_BP_BYTES;  // one unit's R tiles, both splits, tf32 hi then lo
constexpr size_t kMoeRotbSmem = 1024 + MRB_STAGES * MRB_A_BYTES + 2 * MRB_B_BYTES + 256;

// The diagonal R blocks of one (expert, 64-column group) unit, both splits: 2 (64/b) b^2
// floats, 32 b / 128 float4s per builder thread, loaded one unit ahead of their store.
template <int B>
struct RbRegs {
  static constexpr int N = 2 * 16 * B / 128;
  float4 v[N];
};

template <int B>
__device__ __forceinline__ void rb_load(const float* Re, int nb, int K, int g, int tid, RbRegs<B>& r) {
#pragma unroll
  for (int u = 0; u < RbRegs<B>::N; ++u) {
    const int f = u * 128 + tid;  // float4 index over both splits' diagonal blocks
    const int sp = f / (16 * B), rem = f % (16 * B);
    const int jb = rem / (B * B / 4), w = rem % (B * B / 4);
    const int i = w / (B / 4), l4 = (w % (B / 4)) * 4;
    const int j = (g * 64) / B + jb;
    r.v[u] = (j + 1) * B <= K ? *reinterpret_cast<const float4*>(Re + ((static_cast<size_t>(sp) * nb + j) * B + i) * B + l4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Into one unit buffer (hi tiles of both splits, then lo tiles), K-major in two 32-wide
// chunks as the dense dX rotation lays them out.  Positions off the diagonal blocks are
// never written: they stay zero from the kernel's start.
template <int B>
__device__ __forceinline__ void rb_store(const RbRegs<B>& r, uint8_t* buf, int tid) {
#pragma unroll
  for (int u = 0; u < RbRegs<B>::N; ++u) {
    const int f = u * 128 + tid;
    const int sp = f / (16 * B), rem = f % (16 * B);
    const int jb = rem / (B * B / 4), w = rem % (B * B / 4);
    const int i = w / (B / 4), l4 = (w % (B / 4)) * 4;
    const int row = jb * B + i, k = jb * B + l4;
    const uint32_t off = sp * BWD_BP_BYTES + (k >> 5) * 8192 + swz(row, (k & 31) >> 2);
    const float4 v = r.v[u];
    const float4 hi = make_float4(tf32_rn(v.x), tf32_rn(v.y), tf32_rn(v.z), tf32_rn(v.w));
    *reinterpret_cast<float4*>(buf + off) = hi;
    *reinterpret_cast<float4*>(buf + 2 * BWD_BP_BYTES + off) =
        make_float4(tf32_rn(v.x - hi.x), tf32_rn(v.y - hi.y), tf32_rn(v.z - hi.z), tf32_rn(v.w - hi.w));
  }
}

template <int B>
__global__ void __launch_bounds__(NUM_THREADS, 1) moe_rotb_tc_kernel(const __grid_constant__ MoeRotbParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + MRB_STAGES * MRB_A_BYTES;  // two unit buffers
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + 2 * MRB_B_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = full + MRB_STAGES;
  uint64_t* acc_full = empty + MRB_STAGES;
  uint64_t* acc_empty = acc_full + MRB_ACC;
  uint64_t* b_full = acc_empty + MRB_ACC;
  uint64_t* b_empty = b_full + 2;
  uint64_t* drain = b_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < MRB_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < MRB_ACC; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&b_full[h], 128);
      mbar_init(&b_empty[h], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&p.tmD);
  if (warp == 1) {
    tmem_alloc(tmem_slot, MRB_ACC * 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const int n_units = *p.n_active * p.groups;
  const size_t r_expert = 2ull * p.nb * B * B;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      MoeUnit u;
      for (int k = 0; ok && moe_unit(p.order, p.offsets, n_units, p.groups, k, u); ++k) {
        const int nt = (u.r1 - u.r0 + TM - 1) / TM;
        for (int mt = 0; mt < nt && ok; ++mt)
          for (int sp = 0; sp < 2; ++sp) {
            if (!mbar_wait(&empty[stage], ph ^ 1, abort_flag, kErrWaitEmpty)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[stage], MRB_A_BYTES);
            uint8_t* dst = sA + stage * MRB_A_BYTES;
            tma_load_3d(dst, &p.tmD, &full[stage], u.g * 64, u.r0 + mt * TM, sp);
            tma_load_3d(dst + 16384, &p.tmD, &full[stage], u.g * 64 + 32, u.r0 + mt * TM, sp);
            ++issued;
            if (++stage == MRB_STAGES) {
              stage = 0;
              ph ^= 1;
            }
          }
      }
      if (*abort_flag)
        for (long long i = (issued > MRB_STAGES ? issued - MRB_STAGES : 0); i < issued; ++i)
          gemm_drain_wait(&full[i % MRB_STAGES], static_cast<uint32_t>((i / MRB_STAGES) & 1));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t ph = 0, acc_ph = 0;
      const uint32_t idesc = idesc_tf32_f32(TM, 64, false, false);
      bool ok = true;
      MoeUnit u;
      for (int k = 0; ok && moe_unit(p.order, p.offsets, n_units, p.groups, k, u); ++k) {
        const int bb = k & 1;
        if (!mbar_wait(&b_full[bb], static_cast<uint32_t>((k >> 1) & 1), abort_flag, kErrWaitFull)) break;
        tc_fence_after();
        const int nt = (u.r1 - u.r0 + TM - 1) / TM;
        for (int mt = 0; mt < nt && ok; ++mt) {
          if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1, abort_flag, kErrWaitAccEmpty)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + static_cast<uint32_t>(acc * 64);
          for (int sp = 0; sp < 2; ++sp) {
            if (!mbar_wait(&full[stage], ph, abort_flag, kErrWaitFull)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(sA + stage * MRB_A_BYTES);
            const uint32_t b0 = smem_u32(sB + bb * MRB_B_BYTES + sp * BWD_BP_BYTES);
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                for (int lo = 0; lo < 2; ++lo)  // R = R_hi + R_lo
                  mma_tf32_ss(d, sdesc_sw128(a0 + h * 16384 + kk * 32, 16, 1024),
                              sdesc_sw128(b0 + lo * 2 * BWD_BP_BYTES + h * 8192 + kk * 32, 16, 1024), idesc,
                              (sp | h | kk | lo) ? 1u : 0u);
            mma_commit(&empty[stage]);
            if (++stage == MRB_STAGES) {
              stage = 0;
              ph ^= 1;
            }
          }
          if (!ok) break;
          mma_commit(&acc_full[acc]);
          if (++acc == MRB_ACC) {
            acc = 0;
            acc_ph ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(&b_empty[bb]);
      }
      mma_commit(drain);
      gemm_drain_wait(drain, 0);
    }
  } else {
    const int q = warp & 3, tid = threadIdx.x - 64;
    const int r = q * 32 + lane;  // this thread's row of every tile
    for (int v = tid; v < 2 * MRB_B_BYTES / 16; v += 128) reinterpret_cast<uint4*>(sB)[v] = make_uint4(0, 0, 0, 0);
    builders_sync();
    int acc = 0;
    uint32_t acc_ph = 0;
    RbRegs<B> rv;
    MoeUnit u, un, un2;
    bool have = moe_unit(p.order, p.offsets, n_units, p.groups, 0, u);
    if (have) {
      rb_load<B>(p.R + u.e * r_expert, p.nb, p.K, u.g, tid, rv);
      rb_store<B>(rv, sB, tid);
      fence_proxy_async_smem();
      mbar_arrive(&b_full[0]);
    }
    bool next = have && moe_unit(p.order, p.offsets, n_units, p.groups, 1, un);
    if (next) rb_load<B>(p.R + un.e * r_expert, p.nb, p.K, un.g, tid, rv);
    for (int k = 0; have; ++k) {
      // the next unit's R tiles (loaded during this unit's predecessor) go into the other
      // buffer, and the loads of the one after start, while this unit's MMAs run
      bool next2 = false;
      if (next) {
        const int bb = (k + 1) & 1;
        if (k + 1 >= 2 &&
            !warp_wait(&b_empty[bb], static_cast<uint32_t>((((k + 1) >> 1) - 1) & 1), abort_flag, kErrWaitEmpty))
          break;
        rb_store<B>(rv, sB + bb * MRB_B_BYTES, tid);
        fence_proxy_async_smem();
        mbar_arrive(&b_full[bb]);
        next2 = moe_unit(p.order, p.offsets, n_units, p.groups, k + 2, un2);
        if (next2) rb_load<B>(p.R + un2.e * r_expert, p.nb, p.K, un2.g, tid, rv);
      }
      const int nt = (u.r1 - u.r0 + TM - 1) / TM;
      bool ok = true;
      for (int mt = 0; mt < nt; ++mt) {
        const int pos = u.r0 + mt * TM + r;
        if (!warp_wait(&acc_full[acc], acc_ph, abort_flag, kErrWaitAccFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t rr[32];
          __syncwarp();
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * 64 + h * 32), rr);
          tmem_ld_wait();
          const int col = u.g * 64 + h * 32;
          if (pos < u.r1 && col < p.K) {
            float4* dst = reinterpret_cast<float4*>(p.U + static_cast<size_t>(pos) * p.K + col);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(__uint_as_float(rr[4 * v]), __uint_as_float(rr[4 * v + 1]),
                                   __uint_as_float(rr[4 * v + 2]), __uint_as_float(rr[4 * v + 3]));
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[acc]);
        if (++acc == MRB_ACC) {
          acc = 0;
          acc_ph ^= 1;
        }
      }
      if (!ok) break;
      u = un;
      un = un2;
      have = next;
      next = next2;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, MRB_ACC * 64);
  }
}

// ===========================================================================
// G_e,p,blk = sum over the expert's positions of (w X[t, blk])^T D_p[pos, blk]
// ===========================================================================
constexpr int MG_TP = 64;                        // positions per tile (8 MMAs of K = 8)
constexpr int MG_REGION = MG_TP * 128;           // 8 KB: 64 positions x 32 fp32 columns
constexpr int MG_D_BYTES = 2 * 4 * MG_REGION;    // both splits, 128 columns: the N = 256 B operand
constexpr int MG_X_BYTES = 4 * MG_REGION;        // 128 weighted X columns: the M = 128 A operand
constexpr int MG_STAGES = 2;
constexpr size_t kMoeGradSmem = 1024 + MG_STAGES * (MG_D_BYTES + MG_X_BYTES) + 256;

struct MoeGradParams {
  CUtensorMap tmD;          // D fp32 3-D {K, TK, 2}, box {32, 64, 1}, 128B swizzle with 32-byte atoms
  const uint16_t* X;        // [T][K]
  const int* row_t;         // [TK] routed token of each position
  const float* row_w;       // [TK] gating weight of each position
  const int* offsets;
  const int* order;
  const int* n_active;
  float* G;                 // [E][2][nb][b][b]
  int K, TK, b, nb, groups;  // groups of 128 columns
};

// Position in a CTA's sequence of (unit, 64-row tile) steps.
struct TileCursor {
  MoeUnit u;
  int k, mt, nt;
  bool valid;
};

__device__ __forceinline__ void cursor_init(TileCursor& c, const int* order, const int* offsets, int n_units,
                                            int groups) {
  c.k = 0;
  c.mt = 0;
  c.valid = moe_unit(order, offsets, n_units, groups, 0, c.u);
  c.nt = c.valid ? (c.u.r1 - c.u.r0 + MG_TP - 1) / MG_TP : 0;
}

__device__ __forceinline__ void cursor_next(TileCursor& c, const int* order, const int* offsets, int n_units,
                                            int groups) {
  if (!c.valid) return;
  if (++c.mt < c.nt) return;
  c.mt = 0;
  c.valid = moe_unit(order, offsets, n_units, groups, ++c.k, c.u);
  c.nt = c.valid ? (c.u.r1 - c.u.r0 + MG_TP - 1) / MG_TP : 0;
}


__global__ void __launch_bounds__(NUM_THREADS, 1) moe_grad_tc_kernel(const __grid_constant__ MoeGradParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sD = smem;
  uint8_t* sX = sD + MG_STAGES * MG_D_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + MG_STAGES * MG_X_BYTES);
  uint64_t* d_full = bars;
  uint64_t* d_empty = d_full + MG_STAGES;
  uint64_t* x_full = d_empty + MG_STAGES;
  uint64_t* x_empty = x_full + MG_STAGES;
  uint64_t* acc_full = x_empty + MG_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < MG_STAGES; ++s) {
      mbar_init(&d_full[s], 1);
      mbar_init(&d_empty[s], 1);
      mbar_init(&x_full[s], 128);
      mbar_init(&x_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&p.tmD);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const int n_units = *p.n_active * p.groups;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      MoeUnit u;
      for (int k = 0; ok && moe_unit(p.order, p.offsets, n_units, p.groups, k, u); ++k) {
        const int nt = (u.r1 - u.r0 + MG_TP - 1) / MG_TP;
        for (int mt = 0; mt < nt; ++mt) {
          if (!mbar_wait(&d_empty[stage], ph ^ 1, abort_flag, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&d_full[stage], MG_D_BYTES);
          uint8_t* dst = sD + stage * MG_D_BYTES;
#pragma unroll
          for (int sp = 0; sp < 2; ++sp)
#pragma unroll
            for (int a = 0; a < 4; ++a)
              tma_load_3d(dst + (sp * 4 + a) * MG_REGION, &p.tmD, &d_full[stage], u.g * 128 + a * 32,
                          u.r0 + mt * MG_TP, sp);
          ++issued;
          if (++stage == MG_STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      if (*abort_flag)
        for (long long i = (issued > MG_STAGES ? issued - MG_STAGES : 0); i < issued; ++i)
          gemm_drain_wait(&d_full[i % MG_STAGES], static_cast<uint32_t>((i / MG_STAGES) & 1));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      const uint32_t idesc = idesc_tf32_f32(128, 256, true, true);
      bool ok = true;
      MoeUnit u;
      for (int k = 0; ok && moe_unit(p.order, p.offsets, n_units, p.groups, k, u); ++k) {
        const int acc = k & 1;
        if (!mbar_wait(&acc_empty[acc], static_cast<uint32_t>(((k >> 1) & 1) ^ 1), abort_flag, kErrWaitAccEmpty)) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * 256);
        const int nt = (u.r1 - u.r0 + MG_TP - 1) / MG_TP;
        for (int mt = 0; mt < nt; ++mt) {
          if (!mbar_wait(&x_full[stage], ph, abort_flag, kErrWaitFull) ||
              !mbar_wait(&d_full[stage], ph, abort_flag, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t x0 = smem_u32(sX + stage * MG_X_BYTES);
          const uint32_t d0 = smem_u32(sD + stage * MG_D_BYTES);
#pragma unroll
          for (int ks = 0; ks < MG_TP / 8; ++ks)
            mma_tf32_ss(d, sdesc_mn_sw128_32b(x0 + ks * 1024, MG_REGION, 512),
                        sdesc_mn_sw128_32b(d0 + ks * 1024, MG_REGION, 512), idesc, (mt | ks) ? 1u : 0u);
          mma_commit(&d_empty[stage]);
          mma_commit(&x_empty[stage]);
          if (++stage == MG_STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
      }
      mma_commit(drain);
      gemm_drain_wait(drain, 0);
    }
  } else {
    const int q = warp & 3, tid = threadIdx.x - 64;
    const int ci = tid & 15;  // this thread's 8-column chunk of every staged row
    const int b = p.b;
    // epilogue of unit k (accumulator k & 1): this warp's 32 rows i = 32q + lane of the
    // 128 x 256 product hold the diagonal b x b blocks of G_gate (columns 0..127) and G_up
    auto epilogue = [&](int k, const MoeUnit& v) -> bool {
      const int acc = k & 1;
      if (!warp_wait(&acc_full[acc], static_cast<uint32_t>((k >> 1) & 1), abort_flag, kErrWaitAccFull)) return false;
      tc_fence_after();
      const int i = q * 32 + lane;
      for (int sp = 0; sp < 2; ++sp) {
        float* Ge = p.G + (static_cast<size_t>(v.e) * 2 + sp) * p.nb * b * b;
        if (b >= 32) {
          const int blk_col0 = ((q * 32) / b) * b;
#pragma unroll 1
          for (int h = 0; h < b / 32; ++h) {
            uint32_t rr[32];
            __syncwarp();
            tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(acc * 256 + sp * 128 + blk_col0 + h * 32), rr);
            tmem_ld_wait();
            const int gcol = v.g * 128 + blk_col0;
            if (gcol < p.K) {
              uint4* dst = reinterpret_cast<uint4*>(Ge + (static_cast<size_t>(gcol / b) * b + (i % b)) * b + h * 32);
#pragma unroll
              for (int c = 0; c < 8; ++c) dst[c] = make_uint4(rr[4 * c], rr[4 * c + 1], rr[4 * c + 2], rr[4 * c + 3]);
            }
          }
        } else {  // b == 16: the warp's 32 rows hold two diagonal blocks
          uint32_t rr[32];
          __syncwarp();
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>(acc * 256 + sp * 128 + q * 32), rr);
          tmem_ld_wait();
          const int half = lane >> 4;
          const int gcol = v.g * 128 + q * 32 + half * 16;
          if (gcol < p.K) {
            uint4* dst = reinterpret_cast<uint4*>(Ge + (static_cast<size_t>(gcol / 16) * 16 + (lane & 15)) * 16);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              dst[c] = half ? make_uint4(rr[16 + 4 * c], rr[17 + 4 * c], rr[18 + 4 * c], rr[19 + 4 * c])
                            : make_uint4(rr[4 * c], rr[4 * c + 1], rr[4 * c + 2], rr[4 * c + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      return true;
    };
    // Weighted X rows of one tile: thread chunk ci of rows (tid >> 4) + 8 it.  Three tiles
    // are in flight: the X rows of tile i + 1 and the token ids / weights of tile i + 2
    // load while tile i is converted and stored.
    uint4 xr[8];    // X chunks of the next tile to stage
    float xw[8];    // their weights
    int mt_[8];     // token ids of the tile after (then of the one after that)
    float mw[8];    // its weights
    auto load_meta = [&](const TileCursor& c) {
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int pos = c.u.r0 + c.mt * MG_TP + (tid >> 4) + 8 * it;
        const bool ok = c.valid && pos < c.u.r1;
        mt_[it] = ok ? p.row_t[pos] : -1;
        mw[it] = ok ? p.row_w[pos] : 0.f;
      }
    };
    auto load_x = [&](const TileCursor& c) {  // from the meta registers, which then free up
      const int col = c.u.g * 128 + ci * 8;
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        xr[it] = (mt_[it] >= 0 && col < p.K)
                     ? __ldg(reinterpret_cast<const uint4*>(p.X + static_cast<size_t>(mt_[it]) * p.K + col))
                     : make_uint4(0u, 0u, 0u, 0u);
        xw[it] = mw[it];
      }
    };
    int stage = 0;
    uint32_t ph = 0;
    TileCursor c0, c1;  // the tile being staged, the tile after the next one
    cursor_init(c0, p.order, p.offsets, n_units, p.groups);
    c1 = c0;
    if (c0.valid) {
      load_meta(c0);
      load_x(c0);
      cursor_next(c1, p.order, p.offsets, n_units, p.groups);
      load_meta(c1);
      cursor_next(c1, p.order, p.offsets, n_units, p.groups);
    }
    MoeUnit prev;
    while (c0.valid) {
      if (!warp_wait(&x_empty[stage], ph ^ 1, abort_flag, kErrWaitEmpty)) break;
      uint8_t* base = sX + stage * MG_X_BYTES + (ci >> 2) * MG_REGION;
      const uint32_t c16 = (ci & 3) * 2;
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int row = (tid >> 4) + 8 * it;
        const uint4 v = xr[it];
        const float s = xw[it];
        *reinterpret_cast<float4*>(base + swz32(row, c16)) =
            make_float4(tf32_rn(__uint_as_float(v.x << 16) * s), tf32_rn(__uint_as_float(v.x & 0xFFFF0000u) * s),
                        tf32_rn(__uint_as_float(v.y << 16) * s), tf32_rn(__uint_as_float(v.y & 0xFFFF0000u) * s));
        *reinterpret_cast<float4*>(base + swz32(row, c16 + 1)) =
            make_float4(tf32_rn(__uint_as_float(v.z << 16) * s), tf32_rn(__uint_as_float(v.z & 0xFFFF0000u) * s),
                        tf32_rn(__uint_as_float(v.w << 16) * s), tf32_rn(__uint_as_float(v.w & 0xFFFF0000u) * s));
      }
      fence_proxy_async_smem();
      mbar_arrive(&x_full[stage]);
      if (++stage == MG_STAGES) {
        stage = 0;
        ph ^= 1;
      }
      const TileCursor done = c0;
      cursor_next(c0, p.order, p.offsets, n_units, p.groups);
      if (c0.valid) load_x(c0);  // the meta registers hold c0's tile
      load_meta(c1);
      cursor_next(c1, p.order, p.offsets, n_units, p.groups);
      // once a unit's first tile is staged, drain the unit before it (its MMAs keep the
      // tensor pipe busy meanwhile); after the last tile, drain the last unit
      if (done.mt == 0) {
        if (done.k > 0 && !epilogue(done.k - 1, prev)) break;
        prev = done.u;
      }
      if (!c0.valid) epilogue(done.k, done.u);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace rtc
}  // namespace oftk
