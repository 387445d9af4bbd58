// Block-diagonal OFT rotations on the tcgen05 tensor cores.
//
//   forward : X'_p[:, blk] = X[:, blk] R_p,blk           (kind::f16, R split hi+lo in bf16)
//   dX      : dX[:, blk]  = sum_p dX'_p[:, blk] R_p,blk^T (kind::tf32, dX' read as fp32)
//   dR      : G_p,blk     = X[:, blk]^T dX'_p[:, blk]     (kind::tf32, MN-major operands,
//                                                          reduced over a token chunk in TMEM)
//
// One independent rotation per sub-projection of a fused weight is the
// split-projection adapter (chooseai.io news 4086, item "自定义适配器核函数" and item
// "分投影适配器支持"); the formulas are the standard OFT definition.  Each b x b
// rotation (b = 16, 32 or 64) is a small dense contraction, so the work is laid
// out as 64-column groups: within a group the rotation is a 64 x 64
// block-diagonal matrix (one, two or four blocks) that the kernel builds in
// shared memory straight from R, and one tcgen05.mma pass handles the group for
// 128 tokens.  The contraction is tiny next to the bytes moved, so all three
// kernels are bound by HBM: they read each activation tile once and write each
// output once.
//
// Roles (192 threads, one CTA per SM, persistent over a contiguous range of
// (group, token-tile) units so the resident R tiles are rebuilt only when the
// group changes):
//   warp 0      TMA producer of the activation tiles (128B swizzle)
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warps 2..5  build the R tiles (and, for dR, the fp32 X tiles) in shared
//               memory, then drain TMEM in the epilogue
#pragma once

#include "common.cuh"

namespace oftk {
namespace rtc {

constexpr int TM = 128;
constexpr int NUM_THREADS = 192;
constexpr int A_STAGES = 4;
constexpr int MAX_P = 4;

// Contiguous, balanced range of units for this CTA.
__device__ __forceinline__ void unit_range(int total, int& beg, int& end) {
  const int per = total / static_cast<int>(gridDim.x), rem = total % static_cast<int>(gridDim.x);
  const int bx = static_cast<int>(blockIdx.x);
  beg = bx * per + min(bx, rem);
  end = beg + per + (bx < rem ? 1 : 0);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, unsigned err) {
  return warp_wait_bounded(bar, parity, abort, err);
}

// Offset of 16-byte chunk `c` of row `r` in a 128B-swizzled region of 128-byte rows.
__device__ __forceinline__ uint32_t swz(uint32_t r, uint32_t c) { return (r >> 3) * 1024u + (r & 7u) * 128u + ((c ^ (r & 7u)) << 4); }

// Same for the 32-byte-atom variant (MN-major tf32 operands): granule = chunk / 2, XORed with (r & 3).
__device__ __forceinline__ uint32_t swz32(uint32_t r, uint32_t c) {
  return r * 128u + (((((c >> 1) ^ (r & 3u)) << 1) | (c & 1u)) << 4);
}

__device__ __forceinline__ uint16_t bf16_rn(float v) { return f32_to_bf16_bits(v); }

// ===========================================================================
// forward rotation: X'_p = X R_p
// ===========================================================================
struct FwdParams {
  CUtensorMap tmX;  // X bf16 [M][K], box {64, 128}
  CUtensorMap tmY;  // X' bf16 3-D {K, M, P}, box {64, 32, 1}, 128B swizzle (stores clip at M and K)
  const float* R;   // [P][nb][b][b]
  uint16_t* Xr;     // [P][M][K]
  int M, K, P, b, nb, groups, tiles_m;
  int transpose;    // 1: X'_p = X R_p^T (weight-side rotation of deq(W)^T rows)
  int* zero_ptr;    // optional: zero_n ints CTA 0 clears for the kernel that follows (its split-K counters)
  int zero_n;
};

constexpr int FWD_A_BYTES = TM * 64 * 2;           // 16 KB
constexpr int FWD_BP_BYTES = 64 * 64 * 2;          // one 64x64 bf16 tile
constexpr int FWD_OUT_BYTES = 32 * 64 * 2;           // one staged 32-token x 64-column bf16 box
constexpr int FWD_OUT_SLOTS = 2;                     // per epilogue warp
constexpr int FWD_EPI_WARPS = 8;                     // two per TMEM lane quarter, splits shared by parity
constexpr int FWD_THREADS = 64 + 32 * FWD_EPI_WARPS;
constexpr size_t kFwdSmem =
    1024 + A_STAGES * FWD_A_BYTES + 2 * MAX_P * FWD_BP_BYTES + FWD_EPI_WARPS * FWD_OUT_SLOTS * FWD_OUT_BYTES + 256;

// Named barrier over the 128 builder/epilogue threads (warps 2..5).
__device__ __forceinline__ void builders_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Named barrier over the forward rotation's FWD_EPI_WARPS epilogue warps.
__device__ __forceinline__ void fwd_epi_sync() { asm volatile("bar.sync 2, %0;" ::"n"(32 * FWD_EPI_WARPS) : "memory"); }

// B[r = p*64 + c][i] = R_p[i][c] restricted to group g (block-diagonal), split
// hi/lo (with p.transpose: B[r = p*64 + i][c] = R_p[i][c], i.e. R_p^T), by the
// forward's epilogue threads (tid < 32 * FWD_EPI_WARPS).  Zero the tiles, then stream
// each diagonal R block in with coalesced float4 loads (eight in flight per thread)
// and scatter it transposed.
__device__ void build_fwd_b(const FwdParams& p, int g, uint8_t* sBhi, uint8_t* sBlo, int tid) {
  constexpr int NT = 32 * FWD_EPI_WARPS;
  const int b = p.b;
  for (int v = tid; v < p.P * FWD_BP_BYTES / 16; v += NT) {
    reinterpret_cast<uint4*>(sBhi)[v] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4*>(sBlo)[v] = make_uint4(0, 0, 0, 0);
  }
  fwd_epi_sync();
  const int per_split = 16 * b;             // float4s of the group's diagonal blocks: (64/b) * b * b / 4
  const int total = p.P * per_split;
  for (int base = 0; base < total; base += NT * 8) {
    float4 v[8];
    int meta[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int f = base + u * NT + tid;
      meta[u] = -1;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (f < total) {
        const int sp = f / per_split, rem = f % per_split;
        const int jb = rem / (b * b / 4), w = rem % (b * b / 4);
        const int i = w / (b / 4), c4 = (w % (b / 4)) * 4;
        const int j = (g * 64) / b + jb;
        if ((j + 1) * b <= p.K) {
          v[u] = *reinterpret_cast<const float4*>(p.R + ((static_cast<size_t>(sp) * p.nb + j) * b + i) * b + c4);
          meta[u] = (sp << 16) | ((jb * b + i) << 8) | (jb * b + c4);  // split, k (= i in group), first c in group
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (meta[u] < 0) continue;
      const int sp = meta[u] >> 16, k = (meta[u] >> 8) & 255, c0 = meta[u] & 255;
      const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int r = sp * 64 + (p.transpose ? k : c0 + t);
        const int kk = p.transpose ? c0 + t : k;
        const uint32_t off = swz(r, kk >> 3) + (kk & 7) * 2;
        const uint16_t h = bf16_rn(e[t]);
        *reinterpret_cast<uint16_t*>(sBhi + off) = h;
        *reinterpret_cast<uint16_t*>(sBlo + off) = bf16_rn(e[t] - bf16_bits_to_f32(h));
      }
    }
  }
}

__global__ void __launch_bounds__(FWD_THREADS, 1) rot_fwd_tc_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sBhi = sA + A_STAGES * FWD_A_BYTES;
  uint8_t* sBlo = sBhi + MAX_P * FWD_BP_BYTES;
  uint8_t* sOut = sBlo + MAX_P * FWD_BP_BYTES;  // 1024-byte aligned: the store boxes are 128B-swizzled
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + FWD_EPI_WARPS * FWD_OUT_SLOTS * FWD_OUT_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + A_STAGES;
  uint64_t* acc_full = bars + 2 * A_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* b_full = acc_empty + 2;
  uint64_t* drain = b_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < A_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 32 * FWD_EPI_WARPS);
    }
    mbar_init(b_full, 32 * FWD_EPI_WARPS);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmX);
    tma_prefetch_desc(&p.tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < p.zero_n; i += blockDim.x) p.zero_ptr[i] = 0;
  const uint32_t tmem = *tmem_slot;
  int ubeg, uend;
  unit_range(p.groups * p.tiles_m, ubeg, uend);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      long long issued = 0;
      for (int u = ubeg; u < uend; ++u) {
        const int g = u / p.tiles_m, mt = u % p.tiles_m;
        if (!mbar_wait(&empty[stage], ph ^ 1, abort_flag, kErrWaitEmpty)) break;
        mbar_arrive_expect_tx(&full[stage], FWD_A_BYTES);
        tma_load_2d(sA + stage * FWD_A_BYTES, &p.tmX, &full[stage], g * 64, mt * TM);
        ++issued;
        if (++stage == A_STAGES) {
          stage = 0;
          ph ^= 1;
        }
      }
      if (*abort_flag)
        for (long long i = (issued > A_STAGES ? issued - A_STAGES : 0); i < issued; ++i)
          gemm_drain_wait(&full[i % A_STAGES], static_cast<uint32_t>((i / A_STAGES) & 1));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, acc = 0, cur_g = -1;
      uint32_t ph = 0, acc_ph = 0, b_ph = 0;
      const uint32_t idesc = idesc_bf16_f32(TM, 64 * p.P);
      for (int u = ubeg; u < uend; ++u) {
        const int g = u / p.tiles_m;
        if (g != cur_g) {
          if (!mbar_wait(b_full, b_ph, abort_flag, kErrWaitFull)) break;
          b_ph ^= 1;
          cur_g = g;
        }
        if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1, abort_flag, kErrWaitAccEmpty)) break;
        if (!mbar_wait(&full[stage], ph, abort_flag, kErrWaitFull)) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * 256);
        const uint32_t a0 = smem_u32(sA + stage * FWD_A_BYTES);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = sdesc_sw128(a0 + kk * 32, 16, 1024);
          mma_bf16_ss(d, ad, sdesc_sw128(smem_u32(sBhi) + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
          mma_bf16_ss(d, ad, sdesc_sw128(smem_u32(sBlo) + kk * 32, 16, 1024), idesc, 1u);
        }
        mma_commit(&empty[stage]);
        mma_commit(&acc_full[acc]);
        if (++stage == A_STAGES) {
          stage = 0;
          ph ^= 1;
        }
        acc ^= 1;
        if (acc == 0) acc_ph ^= 1;
      }
      mma_commit(drain);
      gemm_drain_wait(drain, 0);
    }
  } else {
    const int q = warp & 3, tid = threadIdx.x - 64, ew = warp - 2;
    const int half = ew / 4;  // splits half, half + 2, ... of every unit
    int acc = 0, cur_g = -1, out_slot = 0;
    uint32_t acc_ph = 0;
    for (int u = ubeg; u < uend; ++u) {
      const int g = u / p.tiles_m, mt = u % p.tiles_m;
      if (g != cur_g) {  // every MMA reading the previous group's tiles has completed (last epilogue)
        build_fwd_b(p, g, sBhi, sBlo, tid);
        fence_proxy_async_smem();
        mbar_arrive(b_full);
        cur_g = g;
      }
      if (!warp_wait(&acc_full[acc], acc_ph, abort_flag, kErrWaitAccFull)) break;
      tc_fence_after();
      // Each warp owns 32 tokens: per split, its 32 x 64 bf16 block is staged in a
      // 128B-swizzled slot (row = token, lane-private, conflict-free) and leaves by one
      // TMA store, which clips tokens past M and columns past K.
      for (int sp = half; sp < p.P; sp += 2) {
        uint8_t* slot = sOut + (ew * FWD_OUT_SLOTS + out_slot) * FWD_OUT_BYTES;
        if (lane == 0) bulk_wait_read<FWD_OUT_SLOTS - 1>();  // the store that last read this slot is done
        __syncwarp();
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>(acc * 256 + sp * 64 + h * 32), r);
          tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 4; ++v)
            *reinterpret_cast<uint4*>(slot + swz(lane, h * 4 + v)) =
                make_uint4(pack_bf16x2(__uint_as_float(r[8 * v]), __uint_as_float(r[8 * v + 1])),
                           pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                           pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                           pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&p.tmY, slot, g * 64, mt * TM + q * 32, sp);
          bulk_commit();
        }
        out_slot = (out_slot + 1) % FWD_OUT_SLOTS;
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      acc ^= 1;
      if (acc == 0) acc_ph ^= 1;
    }
    if (lane == 0) bulk_wait_all();  // the staged blocks are read (and written) before the CTA exits
    __syncwarp();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// dX rotation: dX = sum_p dX'_p R_p^T   (dX' fp32 -> tf32)
// ===========================================================================
struct BwdParams {
  CUtensorMap tmD;  // dX' fp32, 3-D {K, M, P}, box {32, 128, 1}
  const float* R;
  uint16_t* dX;     // [M][K]
  int M, K, P, b, nb, groups, tiles_m;
};

constexpr int BWD_A_BYTES = TM * 64 * 4;           // 32 KB: two 128 x 32 fp32 boxes
constexpr int BWD_BP_BYTES = 64 * 64 * 4;          // 16 KB: one 64 x 64 fp32 tile (two K chunks)
constexpr size_t kBwdSmem = 1024 + A_STAGES * BWD_A_BYTES + MAX_P * BWD_BP_BYTES + 256;

// B_p[i][l] = R_p[i][l] restricted to group g (block-diagonal), fp32, K-major in
// two 32-wide chunks, for the P rotations R[P][nb][b][b] of d_in = K.  Zero the
// tiles, then stream the diagonal blocks in with coalesced float4 loads (eight in
// flight per thread).  With sBlo, R is split into its nearest tf32 value (sB) and
// the nearest tf32 value of the remainder (sBlo): two tf32 MMAs then carry R to
// about 2^-22 of its size.
__device__ void build_bwd_b(const float* R, int P, int nb, int b, int K, int g, uint8_t* sB, int tid,
                            uint8_t* sBlo = nullptr) {
  for (int v = tid; v < P * BWD_BP_BYTES / 16; v += 128) {
    reinterpret_cast<uint4*>(sB)[v] = make_uint4(0, 0, 0, 0);
    if (sBlo != nullptr) reinterpret_cast<uint4*>(sBlo)[v] = make_uint4(0, 0, 0, 0);
  }
  builders_sync();
  const int per_split = 16 * b;
  const int total = P * per_split;
  for (int base = 0; base < total; base += 128 * 8) {
    float4 v[8];
    int meta[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int f = base + u * 128 + tid;
      meta[u] = -1;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (f < total) {
        const int sp = f / per_split, rem = f % per_split;
        const int jb = rem / (b * b / 4), w = rem % (b * b / 4);
        const int i = w / (b / 4), l4 = (w % (b / 4)) * 4;
        const int j = (g * 64) / b + jb;
        if ((j + 1) * b <= K) {
          v[u] = *reinterpret_cast<const float4*>(R + ((static_cast<size_t>(sp) * nb + j) * b + i) * b + l4);
          meta[u] = (sp << 16) | ((jb * b + i) << 8) | (jb * b + l4);  // split, row i in group, first l in group
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (meta[u] < 0) continue;
      const int sp = meta[u] >> 16, r = (meta[u] >> 8) & 255, k = meta[u] & 255;
      const uint32_t off = sp * BWD_BP_BYTES + (k >> 5) * 8192 + swz(r, (k & 31) >> 2);
      if (sBlo == nullptr) {
        *reinterpret_cast<float4*>(sB + off) = v[u];
      } else {
        const float4 hi = make_float4(tf32_rn(v[u].x), tf32_rn(v[u].y), tf32_rn(v[u].z), tf32_rn(v[u].w));
        *reinterpret_cast<float4*>(sB + off) = hi;
        *reinterpret_cast<float4*>(sBlo + off) = make_float4(tf32_rn(v[u].x - hi.x), tf32_rn(v[u].y - hi.y),
                                                             tf32_rn(v[u].z - hi.z), tf32_rn(v[u].w - hi.w));
      }
    }
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1) rot_bwd_tc_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + A_STAGES * BWD_A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + MAX_P * BWD_BP_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + A_STAGES;
  uint64_t* acc_full = bars + 2 * A_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* b_full = acc_empty + 2;
  uint64_t* drain = b_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < A_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    mbar_init(b_full, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&p.tmD);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  int ubeg, uend;
  unit_range(p.groups * p.tiles_m, ubeg, uend);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int u = ubeg; u < uend && ok; ++u) {
        const int g = u / p.tiles_m, mt = u % p.tiles_m;
        for (int sp = 0; sp < p.P; ++sp) {
          if (!mbar_wait(&empty[stage], ph ^ 1, abort_flag, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], BWD_A_BYTES);
          uint8_t* dst = sA + stage * BWD_A_BYTES;
          tma_load_3d(dst, &p.tmD, &full[stage], g * 64, mt * TM, sp);
          tma_load_3d(dst + 16384, &p.tmD, &full[stage], g * 64 + 32, mt * TM, sp);
          ++issued;
          if (++stage == A_STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      if (*abort_flag)
        for (long long i = (issued > A_STAGES ? issued - A_STAGES : 0); i < issued; ++i)
          gemm_drain_wait(&full[i % A_STAGES], static_cast<uint32_t>((i / A_STAGES) & 1));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, acc = 0, cur_g = -1;
      uint32_t ph = 0, acc_ph = 0, b_ph = 0;
      const uint32_t idesc = idesc_tf32_f32(TM, 64, false, false);
      bool ok = true;
      for (int u = ubeg; u < uend && ok; ++u) {
        const int g = u / p.tiles_m;
        if (g != cur_g) {
          if (!mbar_wait(b_full, b_ph, abort_flag, kErrWaitFull)) break;
          b_ph ^= 1;
          cur_g = g;
        }
        if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1, abort_flag, kErrWaitAccEmpty)) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * 64);
        for (int sp = 0; sp < p.P; ++sp) {
          if (!mbar_wait(&full[stage], ph, abort_flag, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * BWD_A_BYTES);
          const uint32_t b0 = smem_u32(sB + sp * BWD_BP_BYTES);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_tf32_ss(d, sdesc_sw128(a0 + h * 16384 + kk * 32, 16, 1024),
                          sdesc_sw128(b0 + h * 8192 + kk * 32, 16, 1024), idesc, (sp | h | kk) ? 1u : 0u);
          mma_commit(&empty[stage]);
          if (++stage == A_STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
        acc ^= 1;
        if (acc == 0) acc_ph ^= 1;
      }
      mma_commit(drain);
      gemm_drain_wait(drain, 0);
    }
  } else {
    const int q = warp & 3, tid = threadIdx.x - 64;
    int acc = 0, cur_g = -1;
    uint32_t acc_ph = 0;
    for (int u = ubeg; u < uend; ++u) {
      const int g = u / p.tiles_m, mt = u % p.tiles_m;
      if (g != cur_g) {
        build_bwd_b(p.R, p.P, p.nb, p.b, p.K, g, sB, tid);
        fence_proxy_async_smem();
        mbar_arrive(b_full);
        cur_g = g;
      }
      if (!warp_wait(&acc_full[acc], acc_ph, abort_flag, kErrWaitAccFull)) break;
      tc_fence_after();
      const int t = mt * TM + q * 32 + lane;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * 64 + h * 32), r);
        tmem_ld_wait();
        const int col = g * 64 + h * 32;
        if (t < p.M && col < p.K) {
          uint4* dst = reinterpret_cast<uint4*>(p.dX + static_cast<size_t>(t) * p.K + col);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * v]), __uint_as_float(r[8 * v + 1])),
                                pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                                pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                                pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      acc ^= 1;
      if (acc == 0) acc_ph ^= 1;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ===========================================================================
// dR: G_p,blk = X_blk^T dX'_p,blk, summed over a chunk of token tiles in TMEM.
// Units are (128-column group, token chunk); the 128 x 128 product holds the
// group's diagonal b x b blocks, which the epilogue writes as one partial per
// (block, chunk).  Partials are summed in chunk order by the Cayley backward.
// ===========================================================================
struct GradParams {
  CUtensorMap tmD;      // dX' fp32, 3-D {K, M, P}, box {32, 128, 1}, 128B swizzle with 32-byte atoms
  CUtensorMap tmX;      // X bf16 [M][K], box {64, 128}, 128B swizzle
  const uint16_t* X;    // [M][K]
  float* Gp;            // [(p*nb + j)][chunks][b][b]
  int M, K, P, b, nb, groups, chunks, tiles_per_chunk, tiles_m;
};

constexpr int GR_X_BYTES = 4 * 16384;   // 128 tokens x 128 columns fp32, MN-major (4 atom columns)
constexpr int GR_XS_BYTES = 2 * 16384;  // the same tile as staged by TMA: bf16, two 64-column boxes
constexpr int GR_B_BYTES = 4 * 16384;   // one dX' tile, same layout as the fp32 X tile
constexpr int GR_STAGES = 2;
constexpr int GR_BUILD_WARPS = 8;  // X-tile conversion and epilogue: two warps per TMEM lane quarter
constexpr int GR_THREADS = 64 + 32 * GR_BUILD_WARPS;
constexpr size_t kGradSmem = 1024 + GR_X_BYTES + GR_XS_BYTES + GR_STAGES * GR_B_BYTES + 256;

__global__ void __launch_bounds__(GR_THREADS, 1) grad_tc_kernel(const __grid_constant__ GradParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem;
  uint8_t* sXs = sX + GR_X_BYTES;
  uint8_t* sB = sXs + GR_XS_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + GR_STAGES * GR_B_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + GR_STAGES;
  uint64_t* x_full = bars + 2 * GR_STAGES;
  uint64_t* x_empty = x_full + 1;
  uint64_t* xs_full = x_empty + 1;
  uint64_t* xs_empty = xs_full + 1;
  uint64_t* acc_full = xs_empty + 1;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < GR_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(x_full, 32 * GR_BUILD_WARPS);
    mbar_init(x_empty, 1);
    mbar_init(xs_full, 1);
    mbar_init(xs_empty, 32 * GR_BUILD_WARPS);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 32 * GR_BUILD_WARPS);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmD);
    tma_prefetch_desc(&p.tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  int ubeg, uend;
  unit_range(p.groups * p.chunks, ubeg, uend);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0, xs_ph = 0;
      long long issued = 0, xs_issued = 0;
      bool ok = true;
      for (int u = ubeg; u < uend && ok; ++u) {
        const int g = u / p.chunks, c = u % p.chunks;
        const int mt0 = c * p.tiles_per_chunk, mt1 = min(p.tiles_m, mt0 + p.tiles_per_chunk);
        for (int mt = mt0; mt < mt1 && ok; ++mt) {
          if (!mbar_wait(xs_empty, xs_ph ^ 1, abort_flag, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          xs_ph ^= 1;
          mbar_arrive_expect_tx(xs_full, GR_XS_BYTES);
          tma_load_2d(sXs, &p.tmX, xs_full, g * 128, mt * TM);
          tma_load_2d(sXs + 16384, &p.tmX, xs_full, g * 128 + 64, mt * TM);
          ++xs_issued;
          for (int sp = 0; sp < p.P; ++sp) {
            if (!mbar_wait(&empty[stage], ph ^ 1, abort_flag, kErrWaitEmpty)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[stage], GR_B_BYTES);
            uint8_t* dst = sB + stage * GR_B_BYTES;
#pragma unroll
            for (int a = 0; a < 4; ++a) tma_load_3d(dst + a * 16384, &p.tmD, &full[stage], g * 128 + a * 32, mt * TM, sp);
            ++issued;
            if (++stage == GR_STAGES) {
              stage = 0;
              ph ^= 1;
            }
          }
        }
      }
      if (*abort_flag) {
        for (long long i = (issued > GR_STAGES ? issued - GR_STAGES : 0); i < issued; ++i)
          gemm_drain_wait(&full[i % GR_STAGES], static_cast<uint32_t>((i / GR_STAGES) & 1));
        if (xs_issued > 0) gemm_drain_wait(xs_full, static_cast<uint32_t>((xs_issued - 1) & 1));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0, x_ph = 0, acc_ph = 0;
      const uint32_t idesc = idesc_tf32_f32(TM, 128, true, true);
      bool ok = true;
      for (int u = ubeg; u < uend && ok; ++u) {
        const int c = u % p.chunks;
        const int mt0 = c * p.tiles_per_chunk, mt1 = min(p.tiles_m, mt0 + p.tiles_per_chunk);
        if (!mbar_wait(acc_empty, acc_ph ^ 1, abort_flag, kErrWaitAccEmpty)) break;
        tc_fence_after();
        for (int mt = mt0; mt < mt1 && ok; ++mt) {
          if (!mbar_wait(x_full, x_ph, abort_flag, kErrWaitFull)) {
            ok = false;
            break;
          }
          x_ph ^= 1;
          tc_fence_after();
          const uint32_t x0 = smem_u32(sX);
          for (int sp = 0; sp < p.P; ++sp) {
            if (!mbar_wait(&full[stage], ph, abort_flag, kErrWaitFull)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t b0 = smem_u32(sB + stage * GR_B_BYTES);
            const uint32_t d = tmem + static_cast<uint32_t>(sp * 128);
#pragma unroll 4
            for (int ks = 0; ks < TM / 8; ++ks)
              mma_tf32_ss(d, sdesc_mn_sw128_32b(x0 + ks * 1024, 16384, 512),
                          sdesc_mn_sw128_32b(b0 + ks * 1024, 16384, 512), idesc, (mt > mt0 || ks > 0) ? 1u : 0u);
            mma_commit(&empty[stage]);
            if (++stage == GR_STAGES) {
              stage = 0;
              ph ^= 1;
            }
          }
          mma_commit(x_empty);
        }
        if (!ok) break;
        mma_commit(acc_full);
        acc_ph ^= 1;
      }
      mma_commit(drain);
      gemm_drain_wait(drain, 0);
    }
  } else {
    const int q = warp & 3, tid = threadIdx.x - 64;
    const int half = (warp - 2) / 4;  // sub-projections half, half + 2, ... in the epilogue
    uint32_t x_ph = 0, xs_ph = 0, acc_ph = 0;
    const int b = p.b;
    for (int u = ubeg; u < uend; ++u) {
      const int g = u / p.chunks, c = u % p.chunks;
      const int mt0 = c * p.tiles_per_chunk, mt1 = min(p.tiles_m, mt0 + p.tiles_per_chunk);
      bool ok = true;
      for (int mt = mt0; mt < mt1; ++mt) {
        // the previous tile's MMAs are done with sX
        if (!warp_wait(x_empty, x_ph ^ 1, abort_flag, kErrWaitEmpty)) {
          ok = false;
          break;
        }
        x_ph ^= 1;
        if (!warp_wait(xs_full, xs_ph, abort_flag, kErrWaitFull)) {
          ok = false;
          break;
        }
        xs_ph ^= 1;
        // staged X tile (bf16, K-major 128B-swizzled) -> fp32, MN-major, 128B rows with 32-byte atoms
#pragma unroll 4
        for (int it = 0; it < 2048 / (32 * GR_BUILD_WARPS); ++it) {
          const int k = tid + 32 * GR_BUILD_WARPS * it;
          const int t = k >> 4, ci = k & 15;
          const uint4 v = *reinterpret_cast<const uint4*>(sXs + (ci >> 3) * 16384 + swz(t, ci & 7));
          uint8_t* base = sX + (ci >> 2) * 16384;
          const uint32_t c16 = (ci & 3) * 2;
          *reinterpret_cast<uint4*>(base + swz32(t, c16)) =
              make_uint4(v.x << 16, v.x & 0xFFFF0000u, v.y << 16, v.y & 0xFFFF0000u);
          *reinterpret_cast<uint4*>(base + swz32(t, c16 + 1)) =
              make_uint4(v.z << 16, v.z & 0xFFFF0000u, v.w << 16, v.w & 0xFFFF0000u);
        }
        mbar_arrive(xs_empty);
        fence_proxy_async_smem();
        mbar_arrive(x_full);
      }
      if (!ok) break;
      if (!warp_wait(acc_full, acc_ph, abort_flag, kErrWaitAccFull)) break;
      acc_ph ^= 1;
      tc_fence_after();
      // this warp's 32 rows i = 32q + lane of the group's 128 x 128 product
      const int i = q * 32 + lane;
      for (int sp = half; sp < p.P; sp += 2) {
        if (b >= 32) {
          const int blk_col0 = ((q * 32) / b) * b;  // first column of this warp's diagonal block
#pragma unroll 1
          for (int h = 0; h < b / 32; ++h) {
            uint32_t r[32];
            __syncwarp();
            tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(sp * 128 + blk_col0 + h * 32), r);
            tmem_ld_wait();
            const int gcol = g * 128 + blk_col0;
            if (gcol < p.K) {
              const int j = gcol / b;
              float* dst = p.Gp + ((static_cast<size_t>(sp) * p.nb + j) * p.chunks + c) * b * b + (i % b) * b + h * 32;
#pragma unroll
              for (int v = 0; v < 8; ++v)
                reinterpret_cast<uint4*>(dst)[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
            }
          }
        } else {  // b == 16: the warp's 32 rows hold two diagonal blocks
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(sp * 128 + q * 32), r);
          tmem_ld_wait();
          const int half = lane >> 4;
          const int gcol = g * 128 + q * 32 + half * 16;
          if (gcol < p.K) {
            const int j = gcol / 16;
            float* dst = p.Gp + ((static_cast<size_t>(sp) * p.nb + j) * p.chunks + c) * 256 + (lane & 15) * 16;
            uint32_t hv[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) hv[e] = half ? r[16 + e] : r[e];
#pragma unroll
            for (int v = 0; v < 4; ++v)
              reinterpret_cast<uint4*>(dst)[v] = make_uint4(hv[4 * v], hv[4 * v + 1], hv[4 * v + 2], hv[4 * v + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
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
