// Fused-dequant OFT GEMM: the frozen INT4 / FP8 / MXFP4 weight is decoded by
// producer warps straight into tensor memory and consumed there by tcgen05.mma;
// the bf16 activations (rotated X', or dY in the backward) stream in through a
// TMA ring.  Neither a bf16 copy of the weight nor a bf16 weight tile in shared
// memory exists: codes go HBM -> registers -> TMEM.
//
// The frozen base stays in deployment precision and is dequantised for the
// product with the BF16-adapted activations ("Orbit", chooseai.io news 4086,
// section "技术原理：低精度基座 + BF16 适配器 + OFT"); the backward computes only the
// activation gradient, never the frozen weight's (m.xxlwj.com 771001, section
// "技术细节", DeepSeek V4 paragraph); sub-projections of a fused weight are groups
// of one launch (split-projection, chooseai.io news 4086, item "自定义适配器核函数").
//
// The weight is the MMA's A operand (M = 128 weight rows, from TMEM), the
// activations its B operand (N = 192 tokens, K-major from shared memory):
//   forward  D[n][m] = sum_k deq(W)[n][k] X'_p[m][k]        -> Y[m][n]      (bf16)
//   backward D[k][m] = sum_n deq(W)[n][k] dY_p[m][n]        -> dX'_p[m][k]  (fp32)
// The backward reads a transposed copy of the codes so that each producer thread
// decodes one contiguous row.
//
// A work unit is one 128-row weight tile against two 192-token activation tiles:
// every decoded weight k-step feeds two MMAs (N = 2 x 192), halving the decode
// work per FLOP; the two fp32 accumulators (columns 0..383) are single-buffered.
//
// Roles (448 threads, one CTA per SM):
//   warp 0       TMA producer: two 192 x 64 activation tiles per k-step (+ backward scale tiles)
//   warp 1       TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2..5   epilogue: TMEM -> registers -> shared memory -> TMA store
//   warps 6..13  dequant producers, two per TMEM lane quarter taking alternate
//                k-steps: one weight row per thread, codes prefetched two of its
//                k-steps ahead in registers (fixed ring slots, so no register moves
//                wait on a load), tcgen05.st into a TMEM A slot
// TMEM: two 192-column fp32 accumulators (columns 0..383) and four 32-column A
// slots (384..511).  Every wait is bounded (common.cuh).
#pragma once

#include "common.cuh"
#include "dq_pack.cuh"

namespace oftk {
namespace gdq {

constexpr int WM = 128;
constexpr int TN = 192;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int TP = 2;                         // token tiles per work unit
constexpr int BT_BYTES = TN * BK * 2;          // one token tile
constexpr int B_BYTES = TP * BT_BYTES;
constexpr int S_BYTES = 512;                  // backward scale tile per stage
constexpr int NUM_THREADS = 448;
constexpr uint32_t A_COL0 = 2 * TN;
constexpr int PREFETCH = 2;
constexpr int MAX_GROUPS = 4;

enum : int { kInt4 = 1, kFp8 = 2, kMxfp4 = 3 };

struct Group {
  int rows;      // weight rows of this group (MMA M extent)
  int tokens;    // tokens (MMA N extent)
  int kred;      // reduction length
  int b_map;     // activation tensor map
  int b_row0;    // first activation row in that map
  int w_row0;    // first weight row in the codes' row space
  int w_k0;      // first reduction index within a codes row
  int y_map;     // output tensor map (rows: tokens, columns: this group's weight rows)
  int tiles_w, tiles_t, tile0;
  long long code_off;   // byte offset of this group's codes (backward: packed blocks; MoE: the expert's codes)
  long long scale_off;  // byte offset of this group's scales (MoE: the expert's scales)
  int out_row0, out_col0;  // MoE: output row of the group's first token, column of its first weight row
};

struct Params {
  CUtensorMap tmB[MAX_GROUPS];  // activations, bf16, box {64, 192}, 128B swizzle
  CUtensorMap tmS;              // backward only: bf16 scales (INT4), bf16 factors (MXFP4), fp32 scales (FP8); box {64, rows}
  CUtensorMap tmY[MAX_GROUPS];  // outputs, box {32, 32}, no swizzle: forward Y_p bf16, backward dX'_p fp32
  // MoE mode: groups built on the device (one per active expert and projection), fp32 output
  const Group* moe_groups;      // [n_groups], tile0 ascending
  const int* moe_meta;          // [0] total units, [1] n_groups
  float* moe_out;               // [token slots][moe_ldo]: row out_row0 + token, column out_col0 + weight row
  int moe_ldo;
  const uint8_t* codes;         // forward: [N][K] codes; backward: blocks packed by pack_codes_bwd_kernel
  long long code_row_bytes;     // forward only
  const void* scales;           // INT4 bf16 [K/G][N]; FP8 fp32 [N]; MXFP4 e8m0 [K/32][N]
  int N, K, group;
  int num_groups;
  Group groups[MAX_GROUPS];
};

// Balanced static schedule for launches whose groups have different reduction
// lengths (the backward of a fused weight with unequal sub-projections): the host
// assigns units longest-first to the least-loaded CTA, and CTA b runs
// list[off[b] .. off[b+1]) in order.  Without it, CTA b runs units b, b + grid, ...
constexpr int kMaxSchedCtas = 160;
constexpr int kMaxSchedUnits = 12000;
struct Sched {
  uint16_t off[kMaxSchedCtas + 1];
  uint16_t list[kMaxSchedUnits];
};

template <bool SCHED>
struct KParams {
  Params p;
};
template <>
struct KParams<true> {
  Params p;
  Sched s;
};

constexpr size_t kBarBytes = 256;
constexpr int EP_BYTES = 16384;  // epilogue staging: 4 warps x 4 KB (two bf16 or one fp32 32 x 32 block)
constexpr size_t kSmemBytes = 1024 + STAGES * (B_BYTES + S_BYTES) + EP_BYTES + kBarBytes + sizeof(Group) * MAX_GROUPS;

__device__ __forceinline__ void decode(const Group* sg, int ng, int u, int& g, int& tw, int& tt) {
  if (ng > 8) {  // many groups (MoE, built on the device): binary search on tile0
    int lo = 0, hi = ng - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sg[mid].tile0 <= u) lo = mid; else hi = mid - 1;
    }
    g = lo;
  } else {
    g = 0;
    while (g + 1 < ng && u >= sg[g + 1].tile0) ++g;
  }
  const int local = u - sg[g].tile0;
  tt = local / sg[g].tiles_w;
  tw = local % sg[g].tiles_w;
}

// Raw codes of one k-step for one weight row, prefetched into registers.
struct Raw {
  uint32_t c[16];  // INT4 / MXFP4: 8 words (64 codes); FP8: 16 words
  uint32_t sc;     // forward: INT4 two bf16 group scales; MXFP4 two e8m0 exponents; FP8 the row's fp32 scale
};

template <int FMT, bool BWD>
__device__ __forceinline__ void load_raw(const Params& p, const Group& G, int tw, int r, int ks, Raw& raw) {
  constexpr int NW = (FMT == kFp8) ? 16 : 8;   // 32-bit words per k-step
  constexpr int PER = (FMT == kFp8) ? 4 : 8;   // codes per word
  const int k0 = ks * BK;
  if (BWD) {
    // packed blocks: zero codes pad every row and k-step of the existing row tiles;
    // the warp's 32 rows read 512 contiguous bytes per vector.  A 256-row pair unit
    // may reach one 128-row tile past the last: it decodes zeros.
    constexpr int NV4 = NW / 4;
    if (tw * WM >= G.rows) {
#pragma unroll
      for (int i = 0; i < NW; ++i) raw.c[i] = 0;
      raw.sc = 0;
      return;
    }
    const int nk = (G.kred + BK - 1) / BK;
    const uint4* src = reinterpret_cast<const uint4*>(p.codes + G.code_off) +
                       (static_cast<size_t>(tw) * nk + ks) * (NV4 * WM) + r;
#pragma unroll
    for (int i = 0; i < NV4; ++i) {
      const uint4 v = src[i * WM];
      raw.c[4 * i] = v.x, raw.c[4 * i + 1] = v.y, raw.c[4 * i + 2] = v.z, raw.c[4 * i + 3] = v.w;
    }
    raw.sc = 0;
    return;
  }
  const int row = tw * WM + r;
#pragma unroll
  for (int i = 0; i < NW; ++i) raw.c[i] = 0;
  raw.sc = 0;
  if (row >= G.rows || k0 >= G.kred) return;
  const int valid = min(BK, G.kred - k0);      // reduction elements present in this k-step
  const long long rbase = G.code_off + static_cast<long long>(G.w_row0 + row) * p.code_row_bytes;
  const int kk = G.w_k0 + k0;                  // first reduction index in the codes row
  // forward rows are 32/64-byte aligned; the reduction (d_in) is a multiple of 32
  const uint4* src = reinterpret_cast<const uint4*>(p.codes + rbase + (FMT == kFp8 ? kk : kk / 2));
  const uint8_t* scales = static_cast<const uint8_t*>(p.scales) + G.scale_off;
  constexpr int NV = NW / 4;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    if (i * 4 * PER < valid) {
      const uint4 v = src[i];
      raw.c[4 * i] = v.x, raw.c[4 * i + 1] = v.y, raw.c[4 * i + 2] = v.z, raw.c[4 * i + 3] = v.w;
    }
  }
  if (FMT == kFp8) {
    raw.sc = __float_as_uint(reinterpret_cast<const float*>(scales)[G.w_row0 + row]);  // fp32 channel scale
  } else {
    const int n = G.w_row0 + row;
    const bool second = valid > 32;
    if (FMT == kInt4) {
      const uint16_t* S = reinterpret_cast<const uint16_t*>(scales);
      const uint32_t s0 = S[static_cast<size_t>(kk / p.group) * p.N + n];
      const uint32_t s1 = second ? S[static_cast<size_t>((kk + 32) / p.group) * p.N + n] : 0u;
      raw.sc = s0 | (s1 << 16);
    } else {
      const uint8_t* E = scales;
      const uint32_t e0 = E[static_cast<size_t>(kk / 32) * p.N + n];
      const uint32_t e1 = second ? E[static_cast<size_t>(kk / 32 + 1) * p.N + n] : 127u;
      raw.sc = e0 | (e1 << 8);
    }
  }
}

// Decode one k-step (64 reduction elements) into 32 bf16x2 words.
template <int FMT, bool BWD>
__device__ __forceinline__ void convert(const Raw& raw, const uint8_t* sS, int srow, uint32_t (&o)[32]) {
  if (!BWD) {
    if (FMT == kInt4) {
      const uint32_t s0 = dq::bf2_splat(static_cast<uint16_t>(raw.sc & 0xFFFFu));
      const uint32_t s1 = dq::bf2_splat(static_cast<uint16_t>(raw.sc >> 16));
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        uint32_t t[4];
        dq::int4x8(raw.c[w], w < 4 ? s0 : s1, t);
        o[4 * w] = t[0], o[4 * w + 1] = t[1], o[4 * w + 2] = t[2], o[4 * w + 3] = t[3];
      }
    } else if (FMT == kMxfp4) {
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        uint32_t t[4];
        dq::mxfp4x8(raw.c[w], w < 4 ? (raw.sc & 0xFFu) : ((raw.sc >> 8) & 0xFFu), t);
        o[4 * w] = t[0], o[4 * w + 1] = t[1], o[4 * w + 2] = t[2], o[4 * w + 3] = t[3];
      }
    } else {
      // FP8: w = bf16(fp32(v * s)): exact v, one fp32 product, then the bf16 rounding
      const float sv = __uint_as_float(raw.sc);
#pragma unroll
      for (int w = 0; w < 16; ++w) {
        float f[4];
        dq::e4m3x4_f32(raw.c[w], f);
        o[2 * w] = pack_bf16x2(f[0] * sv, f[1] * sv);
        o[2 * w + 1] = pack_bf16x2(f[2] * sv, f[3] * sv);
      }
    }
  } else {
    // backward: the scale varies along the reduction (output channel) index; the
    // producer reads this row's 64 per-element bf16 scales (INT4) or factors 2^(e-127)
    // (MXFP4) from the staged tile
    const uint32_t* S = reinterpret_cast<const uint32_t*>(sS + srow * 128);
    if (FMT == kInt4) {
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        uint32_t t[4];
        dq::int4x8_q(raw.c[w], t);  // exact q as bf16
#pragma unroll
        for (int i = 0; i < 4; ++i) o[4 * w + i] = dq::bf2_mul(t[i], S[4 * w + i]);
      }
    } else if (FMT == kMxfp4) {
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        uint32_t t[4];
        dq::mxfp4x8(raw.c[w], 127u, t);  // exact e2m1 value (unit scale)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[4 * w + i] = dq::bf2_mul(t[i], S[4 * w + i]);
      }
    } else {
      // FP8: per-element fp32 channel scales; exact v, one fp32 product, the bf16 rounding
      const float4* S4 = reinterpret_cast<const float4*>(sS);
#pragma unroll
      for (int w = 0; w < 16; ++w) {
        float f[4];
        dq::e4m3x4_f32(raw.c[w], f);
        const float4 s4 = S4[w];
        o[2 * w] = pack_bf16x2(f[0] * s4.x, f[1] * s4.y);
        o[2 * w + 1] = pack_bf16x2(f[2] * s4.z, f[3] * s4.w);
      }
    }
  }
}

template <int FMT, bool BWD, bool SCHED, bool MOE = false>
__global__ void __launch_bounds__(NUM_THREADS, 1) gemm_dq_kernel(const __grid_constant__ KParams<SCHED> kp) {
  const Params& p = kp.p;
  if constexpr (MOE) pdl_wait();  // the prologue reads the device-built group list
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;
  uint8_t* sS = sB + STAGES * B_BYTES;
  uint8_t* sE = sS + STAGES * S_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sE + EP_BYTES);
  uint64_t* full_b = bars;
  uint64_t* full_a = bars + STAGES;
  uint64_t* empty = bars + 2 * STAGES;
  uint64_t* acc_full = bars + 3 * STAGES;  // one per 192-column accumulator half
  uint64_t* acc_empty = acc_full + TP;
  uint64_t* drain = acc_empty + TP;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_meta = reinterpret_cast<int*>(tmem_slot + 2);
  Group* sg = reinterpret_cast<Group*>(reinterpret_cast<uint8_t*>(bars) + kBarBytes);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_b[s], 1);
      mbar_init(&full_a[s], 128);
      mbar_init(&empty[s], 1);
    }
    for (int h = 0; h < TP; ++h) {
      mbar_init(&acc_full[h], 1);
      mbar_init(&acc_empty[h], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    int ng = 0, tile = 0;
    for (int g = 0; g < p.num_groups; ++g) {
      Group G = p.groups[g];
      if (G.rows <= 0 || G.tokens <= 0) continue;
      G.tiles_w = (G.rows + WM - 1) / WM;
      G.tiles_t = ((G.tokens + TN - 1) / TN + TP - 1) / TP;  // token-tile pairs
      G.tile0 = tile;
      tile += G.tiles_w * G.tiles_t;
      sg[ng++] = G;
    }
    s_meta[0] = tile;
    s_meta[1] = ng;
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < p.num_groups; ++i) {
      tma_prefetch_desc(&p.tmB[i]);
      tma_prefetch_desc(&p.tmY[i]);
    }
    if (MOE) tma_prefetch_desc(&p.tmB[0]);
    if (BWD) tma_prefetch_desc(&p.tmS);
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
  // groups: from the launch (shared memory copy), or built on the device (MoE)
  const Group* gsrc = MOE ? p.moe_groups : sg;
  const int total = MOE ? p.moe_meta[0] : s_meta[0], ng = MOE ? p.moe_meta[1] : s_meta[1];
  // this CTA's units: count, and the i-th one
  int nu;
  if constexpr (SCHED) {
    nu = kp.s.off[blockIdx.x + 1] - kp.s.off[blockIdx.x];
  } else {
    nu = static_cast<int>(blockIdx.x) < total ? (total - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1 : 0;
  }
  auto unit_at = [&](int i) -> int {
    if constexpr (SCHED) {
      return kp.s.list[kp.s.off[blockIdx.x] + i];
    } else {
      return static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    }
  };
  const int scale_rows = BWD ? (FMT == kFp8 ? 1 : (FMT == kInt4 ? WM / p.group : WM / 32)) : 0;
  const uint32_t s_tx = BWD ? static_cast<uint32_t>(FMT == kFp8 ? 64 * 4 : 64 * 2 * scale_rows) : 0u;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int i = 0; i < nu && ok; ++i) {
        int g, tw, tt;
        decode(gsrc, ng, unit_at(i), g, tw, tt);
        const Group& G = gsrc[g];
        const int nk = (G.kred + BK - 1) / BK;
        for (int ks = 0; ks < nk; ++ks) {
          if (!mbar_wait(&empty[stage], ph ^ 1, abort_flag, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_b[stage], B_BYTES + s_tx);
#pragma unroll
          for (int h = 0; h < TP; ++h)
            tma_load_2d(sB + stage * B_BYTES + h * BT_BYTES, &p.tmB[G.b_map], &full_b[stage], ks * BK,
                        G.b_row0 + (tt * TP + h) * TN);
          if (BWD) {
            // bf16 rows (fp32 for FP8): x is a multiple of 8 elements, so 16-byte aligned
            const int y = (FMT == kFp8) ? 0 : (tw * WM) / (FMT == kInt4 ? p.group : 32);
            tma_load_2d(sS + stage * S_BYTES, &p.tmS, &full_b[stage], G.w_k0 + ks * BK, y);
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      if (*abort_flag)
        for (long long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          gemm_drain_wait(&full_b[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1));
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t acc_ph = 0;
      bool ok = true;
      long long gk = 0;  // k-steps of this CTA's earlier units
      for (int i = 0; i < nu && ok; ++i) {
        int g, tw, tt;
        decode(gsrc, ng, unit_at(i), g, tw, tt);
        const int nk = (gsrc[g].kred + BK - 1) / BK;
        // Accumulator halves overlap with the epilogue at both ends of a unit: the first D
        // k-steps feed half 0 only while the epilogue still reads half 1 of the previous
        // unit, and the last D k-steps finish half 0 first, so the epilogue can drain it
        // while their half-1 products run.  Each A slot and B stage is released after its
        // half-1 products.
        const int D = nk < STAGES ? nk : STAGES;
        const int T0 = nk - D > D ? nk - D : D;  // tail [T0, nk); empty when nk <= D
        auto st_of = [&](int j) { return static_cast<int>((gk + j) % STAGES); };
        // each token tile's MMAs are only as wide as its tokens (a multiple of 16; none
        // for a tile past the group's end): small or ragged token counts do not pay for
        // the full 192 columns
        uint32_t idesc_h[TP];
        bool live_h[TP];
#pragma unroll
        for (int h = 0; h < TP; ++h) {
          const int tok = min(TN, max(0, gsrc[g].tokens - (tt * TP + h) * TN));
          live_h[h] = tok > 0;
          idesc_h[h] = idesc_bf16_f32(WM, live_h[h] ? (tok + 15) / 16 * 16 : TN);
        }
        auto issue = [&](int h, int j) {
          if (!live_h[h]) return;
          const int st = st_of(j);
          const uint32_t a0 = tmem + A_COL0 + static_cast<uint32_t>(st * 32);
          const uint32_t b0 = smem_u32(sB + st * B_BYTES + h * BT_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ts(tmem + static_cast<uint32_t>(h * TN), a0 + kk * 8, sdesc_sw128(b0 + kk * 32, 16, 1024),
                        idesc_h[h], (j | kk) ? 1u : 0u);
        };
        auto wait_full = [&](int j) {
          const int st = st_of(j);
          const uint32_t pj = static_cast<uint32_t>(((gk + j) / STAGES) & 1);
          if (!mbar_wait(&full_a[st], pj, abort_flag, kErrWaitDequant) ||
              !mbar_wait(&full_b[st], pj, abort_flag, kErrWaitFull))
            return false;
          tc_fence_after();
          return true;
        };
        auto wait_acc = [&](int h) {
          if (!mbar_wait(&acc_empty[h], acc_ph ^ 1, abort_flag, kErrWaitAccEmpty)) return false;
          tc_fence_after();
          return true;
        };
        auto release = [&](int j) { mma_commit(&empty[st_of(j)]); };
        if (!wait_acc(0)) break;
        for (int j = 0; j < D && ok; ++j) {
          ok = wait_full(j);
          if (ok) issue(0, j);
        }
        if (!ok) break;
        if (nk <= D) {
          mma_commit(&acc_full[0]);
          if (!wait_acc(1)) break;
          for (int j = 0; j < D; ++j) {
            issue(1, j);
            release(j);
          }
        } else {
          if (!wait_acc(1)) break;
          for (int j = 0; j < D; ++j) {
            issue(1, j);
            release(j);
          }
          for (int j = D; j < T0 && ok; ++j) {
            ok = wait_full(j);
            if (!ok) break;
            issue(0, j);
            issue(1, j);
            release(j);
          }
          for (int j = T0; j < nk && ok; ++j) {
            ok = wait_full(j);
            if (ok) issue(0, j);
          }
          if (!ok) break;
          mma_commit(&acc_full[0]);
          for (int j = T0; j < nk; ++j) {
            issue(1, j);
            release(j);
          }
        }
        mma_commit(&acc_full[1]);
        gk += nk;
        acc_ph ^= 1;
      }
      mma_commit(drain);
      gemm_drain_wait(drain, 0);
    }
  } else if (warp < 6) {
    // ---------------- epilogue ----------------
    // Lane n of warp q holds weight row tw*128 + 32q + n for 32 consecutive tokens per
    // TMEM load.  Each 32 x 32 block is written token-major into shared memory (one
    // conflict-free 64/128-byte row per register) and leaves by one TMA store, which
    // clips rows and tokens outside the group.  The load of the next 32 columns is in
    // flight while the current ones are staged; each 192-column half of the accumulator
    // is released to the MMA issuer as soon as it has been read.
    constexpr int ES = BWD ? 4 : 2;            // output element bytes
    constexpr int BLK = 32 * 32 * ES;          // one staged block
    constexpr int SLOTS = EP_BYTES / 4 / BLK;  // staging slots per warp (2 bf16, 1 fp32)
    static_assert(SLOTS >= 1 && SLOTS <= 2, "epilogue staging");
    const int q = warp & 3;
    uint8_t* ebuf = sE + q * (EP_BYTES / 4);
    int slot = 0;
    uint32_t acc_ph = 0;
    for (int i = 0; i < nu; ++i) {
      int g, tw, tt;
      decode(gsrc, ng, unit_at(i), g, tw, tt);
      const Group& G = gsrc[g];
      const int n0 = tw * WM + q * 32;  // first weight row of this warp's blocks
      const int m_base = tt * TP * TN;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      constexpr int NCH = TP * TN / 32;
      uint32_t ra[32], rb[32];
      auto stage_chunk = [&](const uint32_t (&r)[32], int c) {
        const int m0 = m_base + c * 32;
        if (n0 >= G.rows || m0 >= G.tokens) return;
        if constexpr (MOE) {
          // fp32 rows of the group's token slots: lane = weight row, so each of the 32
          // stores of the warp writes 128 contiguous bytes; tokens past the group's end
          // (the next expert's rows in the activation map) are not written
          if (n0 + lane < G.rows) {
            float* out = p.moe_out + static_cast<size_t>(G.out_row0 + m0) * p.moe_ldo + G.out_col0 + n0 + lane;
            const int jn = min(32, G.tokens - m0);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < jn) out[static_cast<size_t>(j) * p.moe_ldo] = __uint_as_float(r[j]);
          }
          return;
        }
        if (lane == 0) bulk_wait_read<SLOTS - 1>();  // the store that last read this slot is done
        __syncwarp();
        uint8_t* b = ebuf + slot * BLK;
        if (BWD) {
          float* f = reinterpret_cast<float*>(b);
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j * 32 + lane] = __uint_as_float(r[j]);
        } else {
          uint16_t* h = reinterpret_cast<uint16_t*>(b);
#pragma unroll
          for (int j = 0; j < 32; ++j) h[j * 32 + lane] = f32_to_bf16_bits(__uint_as_float(r[j]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&p.tmY[G.y_map], b, n0, m0);
          bulk_commit();
        }
        slot = (slot + 1) % SLOTS;
      };
      constexpr int HCH = NCH / TP;  // chunks per half
      static_assert(HCH % 2 == 0, "chunks are drained in pairs");
      bool ok = true;
      for (int h = 0; h < TP; ++h) {
        if (!warp_wait_bounded(&acc_full[h], acc_ph, abort_flag, kErrWaitAccFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int c0 = h * HCH;
        __syncwarp();
        tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c0 * 32), ra);
        tmem_ld_wait();
#pragma unroll 1
        for (int c = c0; c < c0 + HCH; c += 2) {
          // chunk c is in ra; fetch c + 1 into rb while ra is staged
          tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>((c + 1) * 32), rb);
          stage_chunk(ra, c);
          tmem_ld_wait();
          if (c + 1 == c0 + HCH - 1) {
            // every column of this half has been read into registers
            tc_fence_before();
            mbar_arrive(&acc_empty[h]);
          }
          if (c + 2 < c0 + HCH) tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>((c + 2) * 32), ra);
          stage_chunk(rb, c + 1);
          tmem_ld_wait();
        }
      }
      if (!ok) break;
      acc_ph ^= 1;
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else {
    // ---------------- dequant producers ----------------
    const int q = warp & 3;
    const int par = (warp - 6) >> 2;  // this warp takes the k-steps of parity `par`
    const int r = q * 32 + lane;      // TMEM lane = weight row within the tile
    // a cursor over this CTA's flattened (unit, k-step) sequence; the load cursor
    // runs PREFETCH of this warp's k-steps ahead of the decode cursor
    struct Cursor {
      int i, ks, step, g, tw, tt, nk;  // i: index into this CTA's units
    };
    auto set_unit = [&](Cursor& c) {
      if (c.i < nu) {
        decode(gsrc, ng, unit_at(c.i), c.g, c.tw, c.tt);
        c.nk = (gsrc[c.g].kred + BK - 1) / BK;
      }
    };
    auto advance = [&](Cursor& c) {
      ++c.step;
      if (++c.ks >= c.nk) {
        c.ks = 0;
        ++c.i;
        set_unit(c);
      }
    };
    auto to_parity = [&](Cursor& c) {
      if (c.i < nu && (c.step & 1) != par) advance(c);
    };
    Cursor ld{0, 0, 0, 0, 0, 0, 1};
    set_unit(ld);
    Cursor cv = ld;
    auto fetch = [&](Raw& raw) {
      to_parity(ld);
      if (ld.i < nu) {
        load_raw<FMT, BWD>(p, gsrc[ld.g], ld.tw, r, ld.ks, raw);
        advance(ld);
      }
    };
    // decode the k-step at `cv` from `cur`, store it to TMEM, publish the A slot, then
    // refill `cur`: the next loads stay off the path from a freed slot to a full one
    auto step_one = [&](Raw& cur) -> bool {
      to_parity(cv);
      if (cv.i >= nu) return false;
      const int stage = cv.step % STAGES;
      const uint32_t ph = static_cast<uint32_t>((cv.step / STAGES) & 1);
      // Forward: decode first, then wait for the MMA that last read this A slot and only
      // store.  Backward: the scale tile of this step lands after the slot is free
      // (same stage), so wait for it, then decode.
      uint32_t o[32];
      const int srow = BWD ? ((FMT == kFp8) ? 0 : r / (FMT == kInt4 ? p.group : 32)) : 0;
      if (BWD) {
        if (!warp_wait_bounded(&empty[stage], ph ^ 1, abort_flag, kErrWaitEmpty)) return false;
        if (!warp_wait_bounded(&full_b[stage], ph, abort_flag, kErrWaitFull)) return false;
        convert<FMT, BWD>(cur, sS + stage * S_BYTES, srow, o);
      } else {
        convert<FMT, BWD>(cur, sS + stage * S_BYTES, srow, o);
        if (!warp_wait_bounded(&empty[stage], ph ^ 1, abort_flag, kErrWaitEmpty)) return false;
      }
      __syncwarp();
      tmem_st_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + A_COL0 + static_cast<uint32_t>(stage * 32), o);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&full_a[stage]);
      fetch(cur);
      advance(cv);
      return true;
    };
    Raw ring[PREFETCH];
#pragma unroll
    for (int i = 0; i < PREFETCH; ++i) fetch(ring[i]);
    static_assert(PREFETCH == 2, "the loop below names the ring slots");
    while (step_one(ring[0]) && step_one(ring[1])) {
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace gdq
}  // namespace oftk
