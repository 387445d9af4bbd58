// Small-M fused-dequant OFT GEMM (the decode / rollout shape: a few tokens against
// the whole frozen weight).  At M <= 128 tokens the product is bounded by streaming
// the low-precision weight and decoding it, not by the MMA: every weight element
// is used for only M multiply-adds.  So this kernel is built around the weight
// stream:
//
//   * TMA brings 128-row x 128-byte code tiles (256 INT4 / MXFP4 codes, or 128 FP8
//     codes, per row) into a 6-stage shared-memory ring with the 128-byte swizzle,
//     together with their scale tiles; about 100 KB per SM are in flight.
//   * 16 decode warps (four per TMEM lane quarter) each take every fourth 128-wide
//     k-chunk: one weight row per thread, its 64 or 128 code bytes read from the
//     swizzled tile without bank conflicts, decoded to bf16 in registers and
//     written with tcgen05.st into a ring of 64-column A slots in tensor memory
//     (4 to 7 slots, all of TMEM the accumulators do not use).
//   * Two threads issue tcgen05.mma (kind::f16, A = 128 weight rows from TMEM,
//     B = the M tokens of X' from a shared-memory TMA ring, N = M rounded up to 16),
//     the even chunks into one accumulator and the odd ones into another, and
//     release each A slot and X' stage by tcgen05.commit.  An MMA of this shape holds
//     the tensor pipe about 95 cycles for any N up to 128 and its issuer waits for
//     it, so one issuer alone leaves the pipe idle during its own waits.
//   * The reduction is split over the SMs when the weight has fewer 128-row tiles
//     than SMs (split-K): each split writes an fp32 partial tile, and the last
//     split of a tile to finish (an atomic counter per tile) sums the partials in
//     split order -- the result does not depend on which CTA finishes last -- and
//     writes Y in bf16.
//
// Every decoded value is the canonical bf16 dequantised weight (dq_pack.cuh), the
// same as the large-M kernels use; the frozen base stays in deployment precision
// and is dequantised for the product ("Orbit", chooseai.io news 4086, section
// "技术原理：低精度基座 + BF16 适配器 + OFT"), sub-projections are groups of one
// launch (split-projection, chooseai.io news 4086, item "自定义适配器核函数"), and the
// rollout side serves the same frozen base and adapter at small batch
// (m.xxlwj.com 771001, the Kimi-K2.6 and DeepSeek V4 Flash runs).
//
// Roles (640 threads, one CTA per SM, persistent over work units):
//   warp 0        TMA producer of code + scale tiles
//   warps 1, 19   MMA issuers (even / odd chunks into accumulators 0 / 1); warp 1 also
//                 allocates TMEM
//   warps 2..17   decode (128-wide chunk j goes to the warps with (j mod 4) == (warp - 2) / 4),
//                 then the epilogue of the unit
//   warp 18       TMA producer of X' tiles (apart from the codes, so the code ring runs
//                 as far ahead as its stages allow)
// TMEM: two accumulators of M rounded up to 32 columns, then the A slots.
// Ring positions advance by one with a phase flip on wrap-around (no divisions in the
// loops), and the long waits sleep in mbarrier.try_wait rather than spin.
// Every wait is bounded (common.cuh).
#pragma once

#include "common.cuh"
#include "dq_pack.cuh"

namespace oftk {
namespace gsm {

constexpr int WM = 128;                 // weight rows per tile (MMA M)
constexpr int MAX_TOKENS = 128;         // MMA N = tokens rounded up to 16
constexpr int SC = 6;                   // code stages
constexpr int CODE_BYTES = WM * 128;    // one code tile: 128 rows x 128 bytes, 128B swizzle
constexpr int SCALE_STAGE = 2304;       // INT4: <= 8 x 128 bf16; MXFP4: 8 x 144 e8m0
constexpr int MAX_SX = 12;              // X' stages (128 k each)
constexpr int NUM_THREADS = 640;
constexpr int X_WARP = 18;              // the X' producer
constexpr int MMA_WARP2 = 19;           // the second MMA issuer
constexpr int DEC_WARPS = 16;
constexpr int MAX_GROUPS = 4;
constexpr int MAX_SPLITS = 8;

enum : int { kInt4 = 1, kFp8 = 2, kMxfp4 = 3 };

struct Group {
  int rows;    // weight rows (output channels) of this sub-projection
  int w_row0;  // its first row in the codes / scales
  int b_row0;  // its first row in the X' map ([P][M][K] flattened)
  int tiles;   // ceil(rows / 128)
  int tile0;   // first global tile index of the group
};

struct Params {
  CUtensorMap tmC;  // codes uint8 [N][row bytes], box {128, 128}, 128B swizzle
  CUtensorMap tmS;  // INT4: bf16 [K/G][N], box {128, 256/G}; MXFP4: e8m0 [K/32][N], box {144, 8}
  CUtensorMap tmX;  // X' bf16 [P*M][K], box {64, MN}, 128B swizzle
  const float* fp8_scales;  // FP8: fp32 [N]
  uint16_t* Y;              // bf16 [M][N]
  float* part;              // [tiles][splits][MN][128] fp32 partial tiles (splits > 1)
  int* counters;            // [tiles], zero on entry (splits > 1)
  int M, MN, K, N, group;
  int splits, nkb;          // k-blocks of 128 code bytes over K
  int total_tiles, units;
  int sx;                   // X' stages in use
  int num_groups;
  Group groups[MAX_GROUPS];
};

// k elements per code tile row (128 bytes); a chunk (one A slot, one X' stage, one
// MMA hand-off) is KC = 128 of them: the fixed cost of each hand-off (barriers,
// tensor-memory stores, commits) is paid once per 128 x 128 weight elements
constexpr int KC = 128;
template <int FMT>
__host__ __device__ constexpr int kb_elems() { return FMT == kFp8 ? 128 : 256; }
template <int FMT>
__host__ __device__ constexpr int chunks_per_kb() { return kb_elems<FMT>() / KC; }

// one X' stage: two 64-column boxes of MN rows
__host__ __device__ inline size_t x_stage_bytes(int MN) { return static_cast<size_t>(MN) * 128 * 2; }

// dynamic shared memory: alignment slack, code + scale stages (padded to 1 KB), X' stages, barriers
__host__ __device__ inline size_t smem_bytes(int MN, int sx) {
  const size_t cs = (static_cast<size_t>(SC) * (CODE_BYTES + SCALE_STAGE) + 1023) / 1024 * 1024;
  return 1024 + cs + static_cast<size_t>(sx) * x_stage_bytes(MN) + 1024;
}

__device__ __forceinline__ void unit_of(const Params& p, int u, int& g, int& tile, int& s) {
  const int t = u / p.splits;
  s = u - t * p.splits;
  g = 0;
  while (g + 1 < p.num_groups && t >= p.groups[g + 1].tile0) ++g;
  tile = t - p.groups[g].tile0;
}

// k-blocks [kb0, kb1) of split s
__device__ __forceinline__ void split_range(const Params& p, int s, int& kb0, int& kb1) {
  kb0 = static_cast<int>((static_cast<long long>(s) * p.nkb) / p.splits);
  kb1 = static_cast<int>((static_cast<long long>(s + 1) * p.nkb) / p.splits);
}

// KC-wide chunks of k-blocks [kb0, kb1): the last block may be partial along K
template <int FMT>
__device__ __forceinline__ int chunks_in(const Params& p, int kb0, int kb1) {
  const int k0 = kb0 * kb_elems<FMT>();
  const int k1 = min(p.K, kb1 * kb_elems<FMT>());
  return k1 > k0 ? (k1 - k0 + KC - 1) / KC : 0;
}

// One 64-wide chunk of one weight row -> 32 bf16x2 words (element 2i in the low half of word i).
template <int FMT>
__device__ __forceinline__ void decode_chunk(const uint8_t* crow, int r, int c, const uint8_t* srow_base, int srem,
                                             int group, float fp8_scale, uint32_t (&o)[32]) {
  if (FMT == kFp8) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 w = *reinterpret_cast<const uint4*>(crow + (((4 * c + v) ^ (r & 7)) << 4));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float f[4];
        dq::e4m3x4_f32(ws[i], f);
        o[8 * v + 2 * i] = pack_bf16x2(f[0] * fp8_scale, f[1] * fp8_scale);
        o[8 * v + 2 * i + 1] = pack_bf16x2(f[2] * fp8_scale, f[3] * fp8_scale);
      }
    }
  } else {
    // two 16-byte pieces: elements 0..31 and 32..63 of the chunk
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 w = *reinterpret_cast<const uint4*>(crow + (((2 * c + h) ^ (r & 7)) << 4));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
      if (FMT == kInt4) {
        const uint16_t* S = reinterpret_cast<const uint16_t*>(srow_base);  // [group][128] bf16
        const int gi = (64 * c + 32 * h) / group;
        const uint32_t s2 = dq::bf2_splat(S[gi * WM + r]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t t[4];
          dq::int4x8(ws[i], s2, t);
          o[16 * h + 4 * i] = t[0], o[16 * h + 4 * i + 1] = t[1], o[16 * h + 4 * i + 2] = t[2], o[16 * h + 4 * i + 3] = t[3];
        }
      } else {
        const uint32_t e = srow_base[(2 * c + h) * 144 + srem + r];  // [32-group][144] e8m0
        uint32_t t[16];
        dq::mxfp4x32_mul(ws, e, t);
#pragma unroll
        for (int i = 0; i < 16; ++i) o[16 * h + i] = t[i];
      }
    }
  }
}

__device__ __forceinline__ void dec_sync() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

// warp_wait_bounded with the sleeping wait (lane 0 waits, the outcome is broadcast)
__device__ __forceinline__ bool warp_wait_bounded_sleep(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                        unsigned err) {
  bool ok = false;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait_sleep(bar, parity, abort, err, 5000u);
  return __shfl_sync(0xFFFFFFFFu, ok, 0);
}

// Advances a ring position and flips its phase parity on wrap-around.
__device__ __forceinline__ void ring_next(int& pos, uint32_t& ph, int n) {
  if (++pos == n) {
    pos = 0;
    ph ^= 1u;
  }
}

template <int FMT>
__global__ void __launch_bounds__(NUM_THREADS, 1) gemm_sm_kernel(const __grid_constant__ Params p) {
  constexpr int CPB = chunks_per_kb<FMT>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sC = smem;
  uint8_t* sS = sC + SC * CODE_BYTES;
  uint8_t* sX = smem + (static_cast<size_t>(SC) * (CODE_BYTES + SCALE_STAGE) + 1023) / 1024 * 1024;
  const int XB = static_cast<int>(x_stage_bytes(p.MN));  // one X' stage (two boxes)
  const int XH = XB / 2;                                  // one box
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + p.sx * XB);
  uint64_t* c_full = bars;
  uint64_t* c_empty = c_full + SC;
  uint64_t* x_full = c_empty + SC;
  uint64_t* chunk_empty = x_full + MAX_SX;
  uint64_t* a_full = chunk_empty + MAX_SX;  // up to 12 slots
  uint64_t* acc_full = a_full + MAX_SX;  // one per accumulator
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 1;       // one per issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_last = reinterpret_cast<int*>(tmem_slot + 2);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  const int AC = (p.MN + 31) / 32 * 32;          // columns of each of the two accumulators
  // One ring of chunk slots: slot s is A slot s in TMEM (64 columns after the
  // accumulators, KC bf16 each) and X' stage s in shared memory, released together by
  // one tcgen05.commit on chunk_empty[s] after the chunk's MMAs.
  const int NS = min(p.sx, min(15, (512 - 2 * AC) / 64));
  const uint32_t A_COL0 = static_cast<uint32_t>(2 * AC);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SC; ++s) {
      mbar_init(&c_full[s], 1);
      mbar_init(&c_empty[s], 4 * CPB);
    }
    for (int s = 0; s < MAX_SX; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&chunk_empty[s], 1);
      mbar_init(&a_full[s], 4);
    }
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_full[1], 1);
    mbar_init(acc_empty, DEC_WARPS);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmC);
    if (FMT != kFp8) tma_prefetch_desc(&p.tmS);
  }
  if (warp == X_WARP && lane == 0) tma_prefetch_desc(&p.tmX);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const int nu = static_cast<int>(blockIdx.x) < p.units
                     ? (p.units - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                     : 0;
  auto unit_at = [&](int i) { return static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x); };
  const uint32_t scale_tx = FMT == kInt4 ? static_cast<uint32_t>(WM * 2 * (kb_elems<FMT>() / p.group))
                                         : (FMT == kMxfp4 ? 144u * 8u : 0u);

  if (warp == 0) {
    // ---------------- code + scale tile producer ----------------
    if (lane == 0) {
      int st = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = 0; i < nu && ok; ++i) {
        int g, tile, s, kb0, kb1;
        unit_of(p, unit_at(i), g, tile, s);
        split_range(p, s, kb0, kb1);
        const int n_first = p.groups[g].w_row0 + tile * WM;
        // Code tiles go out in pairs of adjacent k-blocks: each row's two 128-byte pieces
        // then reach DRAM together (one page), instead of a stage period apart.
        for (int kb = kb0; kb < kb1 && ok; kb += 2) {
          const int nb = min(2, kb1 - kb);
          int st2 = st;
          uint32_t ph2 = ph;
          for (int t = 0; t < nb; ++t) {
            if (!mbar_wait_sleep(&c_empty[st2], ph2 ^ 1u, abort_flag, kErrWaitEmpty)) {
              ok = false;
              break;
            }
            ring_next(st2, ph2, SC);
          }
          if (!ok) break;
          for (int t = 0; t < nb; ++t) {
            const int k = kb + t;
            mbar_arrive_expect_tx(&c_full[st], CODE_BYTES + scale_tx);
            tma_load_2d(sC + st * CODE_BYTES, &p.tmC, &c_full[st], k * 128, n_first);
            if (FMT == kInt4) tma_load_2d(sS + st * SCALE_STAGE, &p.tmS, &c_full[st], n_first, k * kb_elems<FMT>() / p.group);
            if (FMT == kMxfp4) tma_load_2d(sS + st * SCALE_STAGE, &p.tmS, &c_full[st], n_first & ~15, k * 8);
            ++issued;
            ring_next(st, ph, SC);
          }
        }
      }
      if (*abort_flag)
        for (int i = (issued > SC ? issued - SC : 0); i < issued; ++i)
          gemm_drain_wait(&c_full[i % SC], static_cast<uint32_t>((i / SC) & 1));
    }
  } else if (warp == X_WARP) {
    // ---------------- X' tile producer ----------------
    if (lane == 0) {
      int xs = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = 0; i < nu && ok; ++i) {
        int g, tile, s, kb0, kb1;
        unit_of(p, unit_at(i), g, tile, s);
        split_range(p, s, kb0, kb1);
        const int nch = chunks_in<FMT>(p, kb0, kb1);
        const int k0 = kb0 * kb_elems<FMT>();
        for (int j = 0; j < nch; ++j) {
          if (!mbar_wait_sleep(&chunk_empty[xs], ph ^ 1u, abort_flag, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&x_full[xs], static_cast<uint32_t>(XB));
          tma_load_2d(sX + xs * XB, &p.tmX, &x_full[xs], k0 + j * KC, p.groups[g].b_row0);
          tma_load_2d(sX + xs * XB + XH, &p.tmX, &x_full[xs], k0 + j * KC + 64, p.groups[g].b_row0);
          ++issued;
          ring_next(xs, ph, NS);
        }
      }
      if (*abort_flag)
        for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i)
          gemm_drain_wait(&x_full[i % NS], static_cast<uint32_t>((i / NS) & 1));
    }
  } else if (warp == 1 || warp == MMA_WARP2) {
    // ---------------- MMA issuers ----------------
    // A tcgen05.mma of this shape occupies the tensor pipe for a fixed time whatever N,
    // and the issuing thread waits for it; two issuers on different SMSPs take the even
    // and the odd chunks into accumulators 0 and 1, so one issuer's waits and
    // bookkeeping overlap the other's products.  The epilogue adds the two.
    if (lane == 0) {
      const int h = warp == 1 ? 0 : 1;
      const uint32_t d_acc = tmem + static_cast<uint32_t>(h * AC);
      const uint32_t idesc = idesc_bf16_f32(WM, p.MN);
      int sl = 0;  // chunk slot: A slot and X' stage
      uint32_t aph = 0;
      bool ok = true;
      for (int i = 0; i < nu && ok; ++i) {
        int g, tile, s, kb0, kb1;
        unit_of(p, unit_at(i), g, tile, s);
        split_range(p, s, kb0, kb1);
        const int nch = chunks_in<FMT>(p, kb0, kb1);
        if (i > 0) {
          // the decode warps have read the previous unit's accumulator
          if (!mbar_wait_sleep(acc_empty, static_cast<uint32_t>((i - 1) & 1), abort_flag, kErrWaitAccEmpty)) break;
          tc_fence_after();
        }
        for (int j = 0; j < nch; ++j) {
          if ((j & 1) == h) {
            if (!mbar_wait_sleep(&a_full[sl], aph, abort_flag, kErrWaitDequant, 2000u) ||
                !mbar_wait_sleep(&x_full[sl], aph, abort_flag, kErrWaitFull, 2000u)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = tmem + A_COL0 + static_cast<uint32_t>(sl * 64);
            const uint64_t b0 = sdesc_sw128(smem_u32(sX + sl * XB), 16, 1024);
            const uint64_t b1 = sdesc_sw128(smem_u32(sX + sl * XB + XH), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // +32 bytes along K per 16 elements: +2 in the descriptor's address field
              mma_bf16_ts(d_acc, a0 + kk * 8, (kk < 4 ? b0 : b1) + static_cast<uint64_t>(2 * (kk & 3)), idesc,
                          (j >= 2 || kk) ? 1u : 0u);
            mma_commit(&chunk_empty[sl]);
          }
          ring_next(sl, aph, NS);
        }
        if (!ok) break;
        // (an accumulator that took no chunk -- nch <= h -- is committed unwritten: the
        // epilogue treats it as zero)
        mma_commit(&acc_full[h]);
      }
      mma_commit(&drain[h]);
      gemm_drain_wait(&drain[h], 0);
    }
  } else {
    // ---------------- decode, then the epilogue of each unit ----------------
    const int q = warp & 3;           // TMEM lane quarter
    const int u = (warp - 2) >> 2;    // chunk class
    const int r = q * 32 + lane;      // weight row within the tile = TMEM lane
    const uint32_t trow = static_cast<uint32_t>(q * 32) << 16;
    int cst = 0, sl = 0, vmod = 0;    // code stage of the current k-block, next A slot, position mod 4
    uint32_t cph = 0, aph = 0;
    bool ok = true;
    for (int i = 0; i < nu && ok; ++i) {
      int g, tile, s, kb0, kb1;
      unit_of(p, unit_at(i), g, tile, s);
      split_range(p, s, kb0, kb1);
      const Group& G = p.groups[g];
      const int nch = chunks_in<FMT>(p, kb0, kb1);
      const int n_first = G.w_row0 + tile * WM;
      float fp8_scale = 0.f;
      if (FMT == kFp8) {
        const int n = n_first + r;
        fp8_scale = n < p.N ? p.fp8_scales[n] : 0.f;
      }
      const int srem = FMT == kMxfp4 ? (n_first & 15) : 0;
      // Every k-block holds CPB chunk positions; its code stage is released after each
      // position has been visited by one warp of each lane quarter, also positions past
      // K in a partial last block (nothing decoded there).  Positions go round-robin to
      // the four warps of a quarter; real chunks (j < nch) take the A slots in order.
      int j = 0;
      for (int kb = kb0; kb < kb1 && ok; ++kb) {
        for (int c = 0; c < CPB; ++c, ++j) {
          const bool real = j < nch;
          if (vmod == u) {
            if (!warp_wait_bounded_sleep(&c_full[cst], cph, abort_flag, kErrWaitFull)) {
              ok = false;
              break;
            }
            mbar_try_wait(smem_u32(&c_full[cst]), cph);  // every lane acquires the tile
            if (real) {
              // two 64-wide halves: decode, store into the slot's 32-column halves
              const uint8_t* crow = sC + cst * CODE_BYTES + r * 128;
              const uint8_t* srow = sS + cst * SCALE_STAGE;
              uint32_t o[32];
              decode_chunk<FMT>(crow, r, 2 * c, srow, srem, p.group, fp8_scale, o);
              if (!warp_wait_bounded_sleep(&chunk_empty[sl], aph ^ 1u, abort_flag, kErrWaitEmpty)) {
                ok = false;
                break;
              }
              tc_fence_after();
              tmem_st_32x32b_x32(tmem + trow + A_COL0 + static_cast<uint32_t>(sl * 64), o);
              decode_chunk<FMT>(crow, r, 2 * c + 1, srow, srem, p.group, fp8_scale, o);
              __syncwarp();
              if (lane == 0) mbar_arrive(&c_empty[cst]);
              tmem_st_32x32b_x32(tmem + trow + A_COL0 + static_cast<uint32_t>(sl * 64 + 32), o);
              tmem_st_wait();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&a_full[sl]);
            } else {
              __syncwarp();
              if (lane == 0) mbar_arrive(&c_empty[cst]);
            }
          }
          if (real) ring_next(sl, aph, NS);
          vmod = (vmod + 1) & 3;
        }
        if (!ok) break;
        ring_next(cst, cph, SC);
      }
      if (!ok) break;

      // ---- epilogue: 32-column chunks of the accumulators, chunk c to the warp with u == c ----
      if (!warp_wait_bounded_sleep(&acc_full[0], static_cast<uint32_t>(i & 1), abort_flag, kErrWaitAccFull) ||
          !warp_wait_bounded_sleep(&acc_full[1], static_cast<uint32_t>(i & 1), abort_flag, kErrWaitAccFull)) {
        ok = false;
        break;
      }
      mbar_try_wait(smem_u32(&acc_full[0]), static_cast<uint32_t>(i & 1));
      mbar_try_wait(smem_u32(&acc_full[1]), static_cast<uint32_t>(i & 1));
      tc_fence_after();
      uint32_t acc[32];
      const int m0 = u * 32;
      const bool mine = m0 < p.MN;
      if (mine) {
        __syncwarp();
        tmem_ld_32x32b_x32(tmem + trow + static_cast<uint32_t>(m0), acc);
        tmem_ld_wait();
        if (nch >= 2) {  // accumulator 1 holds the odd chunks
          uint32_t acc1[32];
          tmem_ld_32x32b_x32(tmem + trow + static_cast<uint32_t>(AC + m0), acc1);
          tmem_ld_wait();
#pragma unroll
          for (int j2 = 0; j2 < 32; ++j2) acc[j2] = __float_as_uint(__uint_as_float(acc[j2]) + __uint_as_float(acc1[j2]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      const int row = tile * WM + r;      // row within the group
      const bool row_ok = row < G.rows;
      const int col = G.w_row0 + row;     // column of Y
      if (nch == 0 && mine) {
#pragma unroll
        for (int j2 = 0; j2 < 32; ++j2) acc[j2] = 0u;
      }
      if (p.splits == 1) {
        if (mine && row_ok) {
#pragma unroll
          for (int j2 = 0; j2 < 32; ++j2) {
            const int m = m0 + j2;
            if (m < p.M) p.Y[static_cast<size_t>(m) * p.N + col] = f32_to_bf16_bits(__uint_as_float(acc[j2]));
          }
        }
      } else {
        const int gt = G.tile0 + tile;    // global tile
        float* part = p.part + (static_cast<size_t>(gt) * p.splits) * p.MN * WM;
        if (mine) {
#pragma unroll
          for (int j2 = 0; j2 < 32; ++j2) {
            const int m = m0 + j2;
            if (m < p.M) __stcg(part + (static_cast<size_t>(s) * p.MN + m) * WM + r, __uint_as_float(acc[j2]));
          }
        }
        dec_sync();
        if (threadIdx.x == 64) {
          __threadfence();
          const int prev = atomicAdd(&p.counters[gt], 1);
          *s_last = prev == p.splits - 1 ? 1 : 0;
          if (prev == p.splits - 1) {
            __threadfence();
            p.counters[gt] = 0;  // ready for the next call
          }
        }
        dec_sync();
        if (*s_last && mine && row_ok) {
          __threadfence();
          // 16 tokens at a time, all loads of a split in flight together; the sum runs
          // over the splits in order
          const int mc = min(32, p.M - m0);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (hh * 16 >= mc) break;
            float sum[16];
#pragma unroll
            for (int j2 = 0; j2 < 16; ++j2) sum[j2] = 0.f;
            for (int s2 = 0; s2 < p.splits; ++s2) {
              const float* ps = part + (static_cast<size_t>(s2) * p.MN + m0 + hh * 16) * WM + r;
              float v[16];
#pragma unroll
              for (int j2 = 0; j2 < 16; ++j2) v[j2] = hh * 16 + j2 < mc ? __ldcg(ps + j2 * WM) : 0.f;
#pragma unroll
              for (int j2 = 0; j2 < 16; ++j2) sum[j2] += v[j2];
            }
#pragma unroll
            for (int j2 = 0; j2 < 16; ++j2)
              if (hh * 16 + j2 < mc)
                p.Y[static_cast<size_t>(m0 + hh * 16 + j2) * p.N + col] = f32_to_bf16_bits(sum[j2]);
          }
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace gsm
}  // namespace oftk
