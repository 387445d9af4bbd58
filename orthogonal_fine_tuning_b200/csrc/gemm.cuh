// Persistent tcgen05 / TMEM grouped GEMM, bf16 x bf16 -> fp32 -> bf16.
//
//   C[c_row0 + m][c_col0 + n] = sum_k A[a_row0 + m][k] * B[b_row0 + n][k]
//
// for every group (sub-projection p of a fused weight, or (expert, projection)
// pair of an MoE chunk).  The pages call for one independent adapter per
// sub-projection of a fused QKV / gate-up tensor (chooseai.io news 4086, item
// "自定义适配器核函数") and for a grouped GEMM over a chunk of transiently
// dequantised experts (m.xxlwj.com 771001, section "技术细节"); both map onto
// this one engine as groups.
//
// Roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: A tile 128x64 and B tile 256x64 per stage, SW128
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer (M=128, N=256, K=16)
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns -> bf16 -> global
// Two 256-column fp32 accumulators in TMEM let the epilogue of tile i overlap
// the main loop of tile i+1.  Every wait is bounded (see common.cuh).
//
// gemm_bf16_pair_kernel is the same engine on a 2-SM pair (tcgen05 cta_group::2)
// for the dense path: a 256 x 256 tile per pair, each CTA loading 128 rows of A
// and 128 rows of B per k-step, so an SM moves 32 KB of operands per k-step for the
// FLOPs that cost the one-CTA kernel 48 KB.
#pragma once

#include "common.cuh"

namespace oftk {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_TILE_BYTES = BM * BK * 2;
constexpr int B_TILE_BYTES = BN * BK * 2;
constexpr int NUM_THREADS = 192;
constexpr int MAX_GROUPS = 32;
constexpr int MAX_MAPS = 4;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int GM = 16;  // m-tiles per raster band (L2 reuse of the B tiles)
constexpr int MAX_SCHED_CTAS = 160;
constexpr int MAX_SCHED_TILES = 2048;

struct Group {
  int m, n, k;
  int a_map, b_map;
  int a_row0, b_row0;
  int c_row0, c_col0;
  int tiles_m, tiles_n, tile0;
};

// MoE chunk: groups are derived on the device from the routing results.
//   gate/up  (mode 0): Y_tk[pos][p n + j] = Xg[p][pos][:] . buf[slot][p n + j][:]   (contract over K)
//   backward (mode 1): D[p][pos][c]      = dYg[p][pos][:] . buft[slot][p][c][:]    (contract over n)
//   down     (mode 2): Z[pos][c]         = Hg[pos][:] . bufd[slot][c][:]           (contract over n)
enum : int { kMoeGateUp = 0, kMoeBwd = 1, kMoeDown = 2 };
struct MoESrc {
  const int* chunk_table;  // [n_chunks][chunk], -1 padded
  const int* offsets;      // [E+1]
  int chunk_idx, chunk, TK, n_proj, K;
  int mode;
};

struct Params {
  CUtensorMap tmA[MAX_MAPS];
  CUtensorMap tmB[MAX_MAPS];
  void* C;            // bf16 [..][ldc], or fp32 when c_f32 != 0
  long long ldc;
  int c_f32;
  int num_groups;
  int use_moe;
  Group groups[MAX_GROUPS];
  MoESrc moe;
  // Optional static schedule for groups of unequal depth (sub-projections of different
  // widths contracted in the backward): CTA c runs tiles sched[sched_off[c] .. sched_off[c+1])
  // in that order.  sched_ctas == 0 means round-robin over the tiles.
  int sched_ctas;
  uint16_t sched_off[MAX_SCHED_CTAS + 1];
  uint16_t sched[MAX_SCHED_TILES];
};

// The tiles of worker `id` of `count` (a CTA, or a pair): a slice of the static
// schedule, or every count-th tile.
struct TileIter {
  int i, end, step;
  bool tab;
  __device__ __forceinline__ TileIter(const Params& p, int total, int id, int count) {
    tab = p.sched_ctas == count;
    i = tab ? p.sched_off[id] : id;
    end = tab ? p.sched_off[id + 1] : total;
    step = tab ? 1 : count;
  }
  __device__ __forceinline__ int tile(const Params& p) const { return tab ? p.sched[i] : i; }
};

constexpr size_t kBarrierBytes = 256;
constexpr size_t kGroupBytes = sizeof(Group) * MAX_GROUPS;
constexpr int EPI_LD = 33;                                   // fp32 staging row: 32 columns + 1 (no bank conflicts)
constexpr size_t kEpiBytes = 4 * 32 * EPI_LD * sizeof(float);  // one 32 x 32 fp32 block per epilogue warp
constexpr size_t kSmemBytes = 1024 + STAGES * (A_TILE_BYTES + B_TILE_BYTES) + kBarrierBytes + kGroupBytes + kEpiBytes;

__device__ __forceinline__ void decode_tile(const Group* sg, int ng, int t, int& g, int& mt, int& nt) {
  g = 0;
  while (g + 1 < ng && t >= sg[g + 1].tile0) ++g;
  const int local = t - sg[g].tile0;
  const int tm = sg[g].tiles_m, tn = sg[g].tiles_n;
  const int band = local / (GM * tn);
  const int rem = local - band * GM * tn;
  const int rows = min(GM, tm - band * GM);
  mt = band * GM + rem % rows;
  nt = rem / rows;
}

// Group table in shared memory (one thread): tiles of bm rows x BN columns, numbered
// group by group; s_meta[0] = tiles, s_meta[1] = groups.
__device__ __forceinline__ void build_group_table(const Params& p, Group* sg, int* s_meta, int bm) {
  int ng = 0, tile = 0;
  auto add = [&](const Group& src) {
    Group g = src;
    g.tiles_m = (g.m + bm - 1) / bm;
    g.tiles_n = (g.n + BN - 1) / BN;
    g.tile0 = tile;
    tile += g.tiles_m * g.tiles_n;
    sg[ng++] = g;
  };
  if (!p.use_moe) {
    for (int g = 0; g < p.num_groups; ++g)
      if (p.groups[g].m > 0 && p.groups[g].n > 0) add(p.groups[g]);
  } else {
    const MoESrc& s = p.moe;
    for (int slot = 0; slot < s.chunk; ++slot) {
      const int e = s.chunk_table[s.chunk_idx * s.chunk + slot];
      if (e < 0) continue;
      const int cnt = s.offsets[e + 1] - s.offsets[e];
      if (cnt <= 0) continue;
      for (int proj = 0; proj < (s.mode == kMoeDown ? 1 : 2); ++proj) {
        Group g{};
        g.m = cnt;
        g.a_map = 0;
        g.b_map = 0;
        g.a_row0 = proj * s.TK + s.offsets[e];
        if (s.mode == kMoeDown) {
          g.n = s.K;
          g.k = s.n_proj;
          g.b_row0 = slot * s.K;
          g.c_row0 = s.offsets[e];
          g.c_col0 = 0;
        } else if (s.mode == kMoeBwd) {
          g.n = s.K;
          g.k = s.n_proj;
          g.b_row0 = (slot * 2 + proj) * s.K;
          g.c_row0 = proj * s.TK + s.offsets[e];
          g.c_col0 = 0;
        } else {
          g.n = s.n_proj;
          g.k = s.K;
          g.b_row0 = (slot * 2 + proj) * s.n_proj;
          g.c_row0 = s.offsets[e];
          g.c_col0 = proj * s.n_proj;
        }
        add(g);
      }
    }
  }
  s_meta[0] = tile;
  s_meta[1] = ng;
}

__device__ __forceinline__ uint32_t pack2(uint32_t lo, uint32_t hi) {
  return pack_bf16x2(__uint_as_float(lo), __uint_as_float(hi));
}

// Epilogue of one warp: the 32 accumulator lanes at `tacc` are rows row0 + lane of group
// G (row0 relative to the group), columns nt * BN + [0, BN).  bf16 rows are stored
// directly; fp32 goes through the warp's 32 x 32 staging block `stg`, so every store
// instruction writes four full 128-byte row segments.  fp32 outputs (dX', the MoE's
// D) are only ever read as tf32 MMA operands, so they are stored rounded to the
// nearest tf32 value.
__device__ __forceinline__ void store_rows(const Params& p, const Group& G, int row0, int nt, uint32_t tacc, float* stg,
                                           int lane) {
  const int row = row0 + lane;
  const bool row_ok = row < G.m;
  const long long crow_off = static_cast<long long>(G.c_row0 + (row_ok ? row : 0)) * p.ldc + G.c_col0;
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    uint32_t r[32];
    __syncwarp();
    tmem_ld_32x32b_x32(tacc + static_cast<uint32_t>(c), r);
    tmem_ld_wait();
    const int col = nt * BN + c;
    if (p.c_f32) {
#pragma unroll
      for (int j = 0; j < 32; ++j) stg[lane * EPI_LD + j] = tf32_rn(__uint_as_float(r[j]));
      __syncwarp();
      const int c4 = (lane & 7) * 4;
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int rr = it * 4 + (lane >> 3);
        const int grow = row0 + rr;
        const int gcol = col + c4;
        if (grow < G.m && gcol < G.n) {
          const float* sv = stg + rr * EPI_LD + c4;
          float* dst = static_cast<float*>(p.C) + static_cast<long long>(G.c_row0 + grow) * p.ldc + G.c_col0 + gcol;
          if (gcol + 4 <= G.n) {
            *reinterpret_cast<float4*>(dst) = make_float4(sv[0], sv[1], sv[2], sv[3]);
          } else {
            for (int e = 0; e < 4 && gcol + e < G.n; ++e) dst[e] = sv[e];
          }
        }
      }
      __syncwarp();
    } else if (row_ok && col < G.n) {
      uint16_t* crow = static_cast<uint16_t*>(p.C) + crow_off;
      if (col + 32 <= G.n) {
        uint4* dst = reinterpret_cast<uint4*>(crow + col);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          dst[v] = make_uint4(pack2(r[8 * v + 0], r[8 * v + 1]), pack2(r[8 * v + 2], r[8 * v + 3]),
                              pack2(r[8 * v + 4], r[8 * v + 5]), pack2(r[8 * v + 6], r[8 * v + 7]));
      } else {
        for (int i = 0; i < 32 && col + i < G.n; ++i) crow[col + i] = f32_to_bf16_bits(__uint_as_float(r[i]));
      }
    }
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1) gemm_bf16_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_TILE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_meta = reinterpret_cast<int*>(tmem_slot + 2);  // [0] total tiles, [1] groups
  Group* sg = reinterpret_cast<Group*>(reinterpret_cast<uint8_t*>(bars) + kBarrierBytes);
  float* s_epi = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sg) + kGroupBytes);  // [4 warps][32][EPI_LD]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (p.use_moe) {
    pdl_wait();  // the prologue reads the device-built routing tables
    // a chunk past the active experts (they fill the chunks in order) has no tiles:
    // leave before the barriers and the TMEM allocation
    if (p.moe.chunk_table[p.moe.chunk_idx * p.moe.chunk] < 0) return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    build_group_table(p, sg, s_meta, BM);
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < MAX_MAPS; ++i) {
      tma_prefetch_desc(&p.tmA[i]);
      tma_prefetch_desc(&p.tmB[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_meta[0];
  const int ng = s_meta[1];

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      long long issued = 0;
      for (TileIter it(p, total, blockIdx.x, gridDim.x); it.i < it.end; it.i += it.step) {
        const int t = it.tile(p);
        if (t >= total) continue;
        int g, mt, nt;
        decode_tile(sg, ng, t, g, mt, nt);
        const Group& G = sg[g];
        const int nk = (G.k + BK - 1) / BK;
        bool ok = true;
        for (int kt = 0; kt < nk; ++kt) {
          if (!mbar_wait(&empty[stage], ph ^ 1, abort_flag, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], A_TILE_BYTES + B_TILE_BYTES);
          tma_load_2d(sA + stage * A_TILE_BYTES, &p.tmA[G.a_map], &full[stage], kt * BK, G.a_row0 + mt * BM);
          tma_load_2d(sB + stage * B_TILE_BYTES, &p.tmB[G.b_map], &full[stage], kt * BK, G.b_row0 + nt * BN);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {  // let the copies already in flight land before the CTA exits
        for (long long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          gemm_drain_wait(&full[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
      for (TileIter it(p, total, blockIdx.x, gridDim.x); it.i < it.end; it.i += it.step) {
        const int t = it.tile(p);
        if (t >= total) continue;
        int g, mt, nt;
        decode_tile(sg, ng, t, g, mt, nt);
        const int nk = (sg[g].k + BK - 1) / BK;
        if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1, abort_flag, kErrWaitAccEmpty)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN);
        bool ok = true;
        for (int kt = 0; kt < nk; ++kt) {
          if (!mbar_wait(&full[stage], ph, abort_flag, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sdesc_kmajor_sw128(smem_u32(sA + stage * A_TILE_BYTES));
          const uint64_t bd = sdesc_kmajor_sw128(smem_u32(sB + stage * B_TILE_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ss(d, ad + static_cast<uint64_t>(kk * 2), bd + static_cast<uint64_t>(kk * 2), idesc,
                        (kt | kk) ? 1u : 0u);
          mma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
        acc ^= 1;
        if (acc == 0) acc_ph ^= 1;
      }
      // all MMAs issued by this thread have completed once `drain` flips
      mma_commit(drain);
      gemm_drain_wait(drain, 0);
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_ph = 0;
    for (TileIter it(p, total, blockIdx.x, gridDim.x); it.i < it.end; it.i += it.step) {
      const int t = it.tile(p);
      if (t >= total) continue;
      int g, mt, nt;
      decode_tile(sg, ng, t, g, mt, nt);
      const Group& G = sg[g];
      bool ok = false;
      if (lane == 0) ok = mbar_wait(&acc_full[acc], acc_ph, abort_flag, kErrWaitAccFull);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      store_rows(p, G, mt * BM + q * 32, nt, tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN),
                 s_epi + q * 32 * EPI_LD, lane);
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      acc ^= 1;
      if (acc == 0) acc_ph ^= 1;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// 2-SM pair variant for the dense path (no MoE groups).
//
// Synchronisation across the pair (all waits bounded):
//   full[s]      leader's; both CTAs' TMA loads count their bytes on it, the leader's
//                producer adds the one arrival with the expected byte count
//   empty[s]     in each CTA, completed by the leader's tcgen05.commit multicast
//   acc_full[a]  in each CTA, the same
//   acc_empty[a] leader's; both CTAs' 128 epilogue threads arrive
constexpr int PM = 256;                       // rows per pair tile (128 per CTA)
constexpr int P_STAGES = 6;
constexpr int P_HALF_BYTES = 128 * BK * 2;    // one CTA's 128 rows of A (or of B) per stage
constexpr size_t kPairSmemBytes = 1024 + P_STAGES * 2 * P_HALF_BYTES + kBarrierBytes + kGroupBytes + kEpiBytes;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    gemm_bf16_pair_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                                // [P_STAGES][128 x 64] bf16, 128B swizzle
  uint8_t* sB = smem + P_STAGES * P_HALF_BYTES;      // [P_STAGES][128 x 64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + P_STAGES * P_HALF_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + P_STAGES;
  uint64_t* acc_full = bars + 2 * P_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_meta = reinterpret_cast<int*>(tmem_slot + 2);
  Group* sg = reinterpret_cast<Group*>(reinterpret_cast<uint8_t*>(bars) + kBarrierBytes);
  float* s_epi = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sg) + kGroupBytes);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    build_group_table(p, sg, s_meta, PM);
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < MAX_MAPS; ++i) {
      tma_prefetch_desc(&p.tmA[i]);
      tma_prefetch_desc(&p.tmB[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_meta[0];
  const int ng = s_meta[1];
  const int cid = static_cast<int>(cluster_id_x()), ncl = static_cast<int>(cluster_count_x());

  if (warp == 0) {
    // TMA producer, both CTAs: this CTA's 128 rows of the A tile and of the B tile
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      for (TileIter it(p, total, cid, ncl); it.i < it.end; it.i += it.step) {
        const int t = it.tile(p);
        if (t >= total) continue;
        int g, mt, nt;
        decode_tile(sg, ng, t, g, mt, nt);
        const Group& G = sg[g];
        const int nk = (G.k + BK - 1) / BK;
        bool ok = true;
        for (int kt = 0; kt < nk; ++kt) {
          // the MMAs that last read this stage (in both CTAs) have completed
          if (!mbar_wait(&empty[stage], ph ^ 1, abort_flag, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], 4 * P_HALF_BYTES);  // both CTAs' A and B halves
          const uint32_t bar = mapa_u32(&full[stage], 0);
          const int half = static_cast<int>(rank) * 128;
          tma_load_2d_pair(sA + stage * P_HALF_BYTES, &p.tmA[G.a_map], bar, kt * BK, G.a_row0 + mt * PM + half);
          tma_load_2d_pair(sB + stage * P_HALF_BYTES, &p.tmB[G.b_map], bar, kt * BK, G.b_row0 + nt * BN + half);
          if (++stage == P_STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // MMA issuer, leader only: M = 256 (128 rows per CTA), N = 256 (128 columns per CTA)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      constexpr uint32_t idesc = idesc_bf16_f32(PM, BN);
      for (TileIter it(p, total, cid, ncl); it.i < it.end; it.i += it.step) {
        const int t = it.tile(p);
        if (t >= total) continue;
        int g, mt, nt;
        decode_tile(sg, ng, t, g, mt, nt);
        const int nk = (sg[g].k + BK - 1) / BK;
        if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1, abort_flag, kErrWaitAccEmpty)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN);
        bool ok = true;
        for (int kt = 0; kt < nk; ++kt) {
          if (!mbar_wait(&full[stage], ph, abort_flag, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sdesc_kmajor_sw128(smem_u32(sA + stage * P_HALF_BYTES));
          const uint64_t bd = sdesc_kmajor_sw128(smem_u32(sB + stage * P_HALF_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ss_pair(d, ad + static_cast<uint64_t>(kk * 2), bd + static_cast<uint64_t>(kk * 2), idesc,
                             (kt | kk) ? 1u : 0u);
          mma_commit_pair_both(&empty[stage]);
          if (++stage == P_STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        mma_commit_pair_both(&acc_full[acc]);
        acc ^= 1;
        if (acc == 0) acc_ph ^= 1;
      }
      // all MMAs issued by this thread have completed once `drain` flips
      mma_commit_pair_local(drain);
      gemm_drain_wait(drain, 0);
    }
  } else {
    // epilogue, both CTAs: this CTA's 128 rows of the 256-row tile
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_ph = 0;
    const uint32_t acc_empty_leader0 = mapa_u32(&acc_empty[0], 0), acc_empty_leader1 = mapa_u32(&acc_empty[1], 0);
    for (TileIter it(p, total, cid, ncl); it.i < it.end; it.i += it.step) {
      const int t = it.tile(p);
      if (t >= total) continue;
      int g, mt, nt;
      decode_tile(sg, ng, t, g, mt, nt);
      const Group& G = sg[g];
      bool ok = false;
      if (lane == 0) ok = mbar_wait(&acc_full[acc], acc_ph, abort_flag, kErrWaitAccFull);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      store_rows(p, G, mt * PM + static_cast<int>(rank) * 128 + q * 32, nt,
                 tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN), s_epi + q * 32 * EPI_LD,
                 lane);
      tc_fence_before();
      mbar_arrive_cluster(acc ? acc_empty_leader1 : acc_empty_leader0);
      acc ^= 1;
      if (acc == 0) acc_ph ^= 1;
    }
  }
  // In-flight copies: on an abort, give the loads this CTA issued (whose bytes count on
  // the leader's barrier) time to land before shared memory goes away.
  if (*abort_flag) {
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  tc_fence_before();
  cluster_sync_all();  // no remote arrival or MMA into this CTA is still pending
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemm
}  // namespace oftk
