// Fused-dequant OFT GEMM on a 2-SM pair (tcgen05 cta_group::2).
//
// Same product and roles as the one-CTA kernel in gemm_dq.cuh: the frozen INT4 /
// FP8 / MXFP4 weight is decoded by producer warps into tensor memory (the MMA's A
// operand) and the bf16 activations stream in through TMA (the B operand); the
// frozen base stays in deployment precision ("Orbit", chooseai.io news 4086,
// section "技术原理：低精度基座 + BF16 适配器 + OFT"), sub-projections of a fused weight
// are groups of one launch (item "自定义适配器核函数"), and the backward forms only
// the activation gradient (m.xxlwj.com 771001, section "技术细节").
//
// Here a cluster of two CTAs computes a 256-row weight tile against 384 tokens:
// each CTA decodes its own 128 weight rows into its own TMEM, and loads only its
// 96-token half of each 192-token activation tile.  The leader CTA issues
// tcgen05.mma.cta_group::2 (M = 256, N = 192): the tensor cores of both SMs work
// on one instruction, every activation byte a CTA loads feeds 256 weight rows, and
// each SM's L2 -> shared-memory traffic halves against the one-CTA kernel.
//
// Synchronisation across the pair (all waits bounded):
//   b_full[s]  leader's; both CTAs' activation loads count their bytes on it
//   a_full[j]  leader's; its 128 decode threads arrive, plus one relay arrival from
//              the peer: the peer's decode threads arrive on its own a_full[j] and its
//              otherwise idle MMA warp forwards one cluster-scope arrival per k-step
//              (a cluster-scope release by a decode thread would first wait for that
//              thread's prefetch loads still in flight)
//   b_empty[s], a_empty[j], acc_full[h]: in each CTA, completed by the leader's
//              tcgen05.commit multicast to both CTAs
//   acc_empty[h] leader's; both CTAs' epilogue threads arrive
//   s_full[s]  each CTA's own (backward scale tiles for its decode warps)
// Activation stages (6) and TMEM weight slots (4) are separate rings: the slot
// hand-off crosses both SMs, so the weight ring is as deep as TMEM allows.
#pragma once

#include "common.cuh"
#include "dq_pack.cuh"
#include "gemm_dq.cuh"

namespace oftk {
namespace gdq2 {

using gdq::Group;
using gdq::KParams;
using gdq::Params;
using gdq::Raw;
using gdq::kFp8;
using gdq::kInt4;
using gdq::kMxfp4;

constexpr int WM = 128;                  // weight rows per CTA
constexpr int UROWS = 256;               // weight rows per pair unit
constexpr int TN = 192;                  // tokens per MMA (per accumulator half)
constexpr int TNC = TN / 2;              // tokens per CTA per half
constexpr int BK = 64;
constexpr int TP = 2;                    // accumulator halves per unit
constexpr int SB = 6;                    // activation stages
constexpr int SA = 4;                    // TMEM weight slots (2 x 192 accumulator + 4 x 32 = 512 columns)
constexpr int BT_BYTES = TNC * BK * 2;   // one CTA's half-tile: 12 KB
constexpr int B_BYTES = TP * BT_BYTES;   // one stage
constexpr int S_BYTES = 512;             // backward scale tile per stage
constexpr int NUM_THREADS = 448;
constexpr uint32_t A_COL0 = 2 * TN;
constexpr int EP_BYTES = 16384;
constexpr size_t kBarBytes = 512;
constexpr size_t kSmemBytes = 1024 + SB * (B_BYTES + S_BYTES) + EP_BYTES + kBarBytes + sizeof(Group) * gdq::MAX_GROUPS;

__device__ __forceinline__ void decode_unit(const Group* sg, int ng, int u, int& g, int& tw, int& tt) {
  g = 0;
  while (g + 1 < ng && u >= sg[g + 1].tile0) ++g;
  const int local = u - sg[g].tile0;
  tt = local / sg[g].tiles_w;
  tw = local % sg[g].tiles_w;  // 256-row tile
}

template <int FMT, bool BWD, bool SCHED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    gemm_dq2_kernel(const __grid_constant__ KParams<SCHED> kp) {
  const Params& p = kp.p;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;                       // [SB][2 halves][96 tokens x 64] bf16, 128B swizzle
  uint8_t* sS = sB + SB * B_BYTES;          // [SB] backward scale tiles
  uint8_t* sE = sS + SB * S_BYTES;          // epilogue staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(sE + EP_BYTES);
  uint64_t* b_full = bars;
  uint64_t* b_empty = b_full + SB;
  uint64_t* s_full = b_empty + SB;
  uint64_t* a_full = s_full + SB;
  uint64_t* a_empty = a_full + SA;
  uint64_t* acc_full = a_empty + SA;
  uint64_t* acc_empty = acc_full + TP;
  uint64_t* drain = acc_empty + TP;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_meta = reinterpret_cast<int*>(tmem_slot + 2);
  Group* sg = reinterpret_cast<Group*>(reinterpret_cast<uint8_t*>(bars) + kBarBytes);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SB; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
      mbar_init(&s_full[s], 1);
    }
    for (int j = 0; j < SA; ++j) {
      mbar_init(&a_full[j], leader ? 128 + 1 : 128);
      mbar_init(&a_empty[j], 1);
    }
    for (int h = 0; h < TP; ++h) {
      mbar_init(&acc_full[h], 1);
      mbar_init(&acc_empty[h], 2 * 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    int ng = 0, tile = 0;
    for (int g = 0; g < p.num_groups; ++g) {
      Group G = p.groups[g];
      if (G.rows <= 0 || G.tokens <= 0) continue;
      G.tiles_w = (G.rows + UROWS - 1) / UROWS;
      G.tiles_t = ((G.tokens + TN - 1) / TN + TP - 1) / TP;
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
    if (BWD) tma_prefetch_desc(&p.tmS);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const int total = s_meta[0], ng = s_meta[1];
  const int cid = static_cast<int>(cluster_id_x()), ncl = static_cast<int>(cluster_count_x());
  int nu;
  if constexpr (SCHED) {
    nu = kp.s.off[cid + 1] - kp.s.off[cid];
  } else {
    nu = cid < total ? (total - 1 - cid) / ncl + 1 : 0;
  }
  auto unit_at = [&](int i) -> int {
    if constexpr (SCHED) {
      return kp.s.list[kp.s.off[cid] + i];
    } else {
      return cid + i * ncl;
    }
  };
  const int gsz = FMT == kInt4 ? p.group : 32;  // rows of weight per backward scale row
  const uint32_t s_tx = BWD ? static_cast<uint32_t>(FMT == kFp8 ? 64 * 4 : 64 * 2 * (WM / gsz)) : 0u;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs: own half of each activation tile) ----------------
    if (lane == 0) {
      int sb = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = 0; i < nu && ok; ++i) {
        int g, tw, tt;
        decode_unit(sg, ng, unit_at(i), g, tw, tt);
        const Group& G = sg[g];
        const int nk = (G.kred + BK - 1) / BK;
        for (int ks = 0; ks < nk; ++ks) {
          // the MMA that last read this stage (in both CTAs) has completed
          if (!mbar_wait(&b_empty[sb], ph ^ 1, abort_flag, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&b_full[sb], 2 * B_BYTES);  // both CTAs' bytes
          const uint32_t bar = mapa_u32(&b_full[sb], 0);
#pragma unroll
          for (int h = 0; h < TP; ++h)
            tma_load_2d_pair(sB + sb * B_BYTES + h * BT_BYTES, &p.tmB[G.b_map], bar, ks * BK,
                             G.b_row0 + (tt * TP + h) * TN + static_cast<int>(rank) * TNC);
          if (BWD) {
            // this CTA's scale rows for its own decode warps (bf16 rows, or fp32 for FP8:
            // x is a multiple of 8 elements, so 16-byte aligned)
            const int y = (FMT == kFp8) ? 0 : ((tw * 2 + static_cast<int>(rank)) * WM) / gsz;
            mbar_arrive_expect_tx(&s_full[sb], s_tx);
            tma_load_2d(sS + sb * S_BYTES, &p.tmS, &s_full[sb], G.w_k0 + ks * BK, y);
          }
          if (++sb == SB) {
            sb = 0;
            ph ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only) ----------------
    if (leader && lane == 0) {
      uint32_t acc_ph = 0;
      constexpr uint32_t idesc = idesc_bf16_f32(UROWS, TN);
      bool ok = true;
      long long gk = 0;  // k-steps of this pair's earlier units
      for (int i = 0; i < nu && ok; ++i) {
        int g, tw, tt;
        decode_unit(sg, ng, unit_at(i), g, tw, tt);
        const int nk = (sg[g].kred + BK - 1) / BK;
        // Accumulator halves overlap with the epilogue at both ends of a unit (as in the
        // one-CTA kernel): the first D k-steps feed half 0 only, the last D k-steps finish
        // half 0 first.  Those k-steps hold their weight slot and activation stage until
        // their half-1 products are issued, so D is at most the smaller ring.
        const int D = nk < SA ? nk : SA;
        const int T0 = nk - D > D ? nk - D : D;
        auto bst = [&](int j) { return static_cast<int>((gk + j) % SB); };
        auto ast = [&](int j) { return static_cast<int>((gk + j) % SA); };
        auto issue = [&](int h, int j) {
          const uint32_t a0 = tmem + A_COL0 + static_cast<uint32_t>(ast(j) * 32);
          const uint32_t b0 = smem_u32(sB + bst(j) * B_BYTES + h * BT_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ts_pair(tmem + static_cast<uint32_t>(h * TN), a0 + kk * 8, sdesc_sw128(b0 + kk * 32, 16, 1024),
                             idesc, (j | kk) ? 1u : 0u);
        };
        auto wait_full = [&](int j) {
          const uint32_t pb = static_cast<uint32_t>(((gk + j) / SB) & 1);
          const uint32_t pa = static_cast<uint32_t>(((gk + j) / SA) & 1);
          if (!mbar_wait(&b_full[bst(j)], pb, abort_flag, kErrWaitFull) ||
              !mbar_wait(&a_full[ast(j)], pa, abort_flag, kErrWaitDequant))
            return false;
          tc_fence_after();
          return true;
        };
        auto wait_acc = [&](int h) {
          if (!mbar_wait(&acc_empty[h], acc_ph ^ 1, abort_flag, kErrWaitAccEmpty)) return false;
          tc_fence_after();
          return true;
        };
        auto release = [&](int j) {
          mma_commit_pair_both(&b_empty[bst(j)]);
          mma_commit_pair_both(&a_empty[ast(j)]);
        };
        if (!wait_acc(0)) break;
        for (int j = 0; j < D && ok; ++j) {
          ok = wait_full(j);
          if (ok) issue(0, j);
        }
        if (!ok) break;
        if (nk <= D) {
          mma_commit_pair_both(&acc_full[0]);
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
          mma_commit_pair_both(&acc_full[0]);
          for (int j = T0; j < nk; ++j) {
            issue(1, j);
            release(j);
          }
        }
        mma_commit_pair_both(&acc_full[1]);
        gk += nk;
        acc_ph ^= 1;
      }
      mma_commit_pair_local(drain);
      gemm_drain_wait(drain, 0);
    } else if (!leader && lane == 0) {
      // relay: once this CTA's 128 decode threads have stored weight slot j, one
      // cluster-scope arrival tells the leader's MMA issuer
      uint32_t a_full_leader[SA];
#pragma unroll
      for (int j = 0; j < SA; ++j) a_full_leader[j] = mapa_u32(&a_full[j], 0);
      long long step = 0;
      bool ok = true;
      for (int i = 0; i < nu && ok; ++i) {
        int g, tw, tt;
        decode_unit(sg, ng, unit_at(i), g, tw, tt);
        const int nk = (sg[g].kred + BK - 1) / BK;
        for (int ks = 0; ks < nk; ++ks, ++step) {
          const int j = static_cast<int>(step % SA);
          if (!mbar_wait(&a_full[j], static_cast<uint32_t>((step / SA) & 1), abort_flag, kErrWaitDequant)) {
            ok = false;
            break;
          }
          tc_fence_after();
          tc_fence_before();
          mbar_arrive_cluster(a_full_leader[j]);
        }
      }
    }
  } else if (warp < 6) {
    // ---------------- epilogue (both CTAs: their own 128 weight rows) ----------------
    constexpr int ES = BWD ? 4 : 2;
    constexpr int BLK = 32 * 32 * ES;
    constexpr int SLOTS = EP_BYTES / 4 / BLK;
    static_assert(SLOTS >= 1 && SLOTS <= 2, "epilogue staging");
    const int q = warp & 3;
    uint8_t* ebuf = sE + q * (EP_BYTES / 4);
    int slot = 0;
    uint32_t acc_ph = 0;
    uint32_t acc_empty_leader[TP];
#pragma unroll
    for (int h = 0; h < TP; ++h) acc_empty_leader[h] = mapa_u32(&acc_empty[h], 0);
    for (int i = 0; i < nu; ++i) {
      int g, tw, tt;
      decode_unit(sg, ng, unit_at(i), g, tw, tt);
      const Group& G = sg[g];
      const int n0 = tw * UROWS + static_cast<int>(rank) * WM + q * 32;  // first weight row of this warp's blocks
      const int m_base = tt * TP * TN;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      constexpr int NCH = TP * TN / 32;
      uint32_t ra[32], rb[32];
      auto stage_chunk = [&](const uint32_t (&r)[32], int c) {
        const int m0 = m_base + c * 32;
        if (n0 >= G.rows || m0 >= G.tokens) return;
        if (lane == 0) bulk_wait_read<SLOTS - 1>();
        __syncwarp();
        uint8_t* b = ebuf + slot * BLK;
        if (BWD) {
          float* f = reinterpret_cast<float*>(b);
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j * 32 + lane] = __uint_as_float(r[j]);
        } else {
          uint16_t* hh = reinterpret_cast<uint16_t*>(b);
#pragma unroll
          for (int j = 0; j < 32; ++j) hh[j * 32 + lane] = f32_to_bf16_bits(__uint_as_float(r[j]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&p.tmY[G.y_map], b, n0, m0);
          bulk_commit();
        }
        slot = (slot + 1) % SLOTS;
      };
      constexpr int HCH = NCH / TP;  // 32-column chunks per half (5)
      bool ok = true;
      for (int h = 0; h < TP; ++h) {
        bool got = false;
        if (lane == 0) got = mbar_wait(&acc_full[h], acc_ph, abort_flag, kErrWaitAccFull);
        if (!__shfl_sync(0xFFFFFFFFu, got, 0)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int c0 = h * HCH, c1 = c0 + HCH;
        __syncwarp();
        tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c0 * 32), ra);
        tmem_ld_wait();
        // chunk c is in ra; the next load is in flight while a chunk is staged
#pragma unroll 1
        for (int c = c0; c + 1 < c1; c += 2) {
          tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>((c + 1) * 32), rb);
          stage_chunk(ra, c);
          tmem_ld_wait();
          if (c + 2 == c1) {  // every column of this half is in registers
            tc_fence_before();
            mbar_arrive_cluster(acc_empty_leader[h]);
          }
          if (c + 2 < c1) tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>((c + 2) * 32), ra);
          stage_chunk(rb, c + 1);
          tmem_ld_wait();
        }
        if (HCH % 2 == 1) {  // the last chunk is in ra
          tc_fence_before();
          mbar_arrive_cluster(acc_empty_leader[h]);
          stage_chunk(ra, c1 - 1);
        }
      }
      if (!ok) break;
      acc_ph ^= 1;
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else {
    // ---------------- dequant producers (both CTAs: their own 128 weight rows) ----------------
    const int q = warp & 3;
    const int par = (warp - 6) >> 2;
    const int r = q * 32 + lane;
    struct Cursor {
      int i, ks, step, g, tw, tt, nk;
    };
    auto set_unit = [&](Cursor& c) {
      if (c.i < nu) {
        decode_unit(sg, ng, unit_at(c.i), c.g, c.tw, c.tt);
        c.nk = (sg[c.g].kred + BK - 1) / BK;
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
        gdq::load_raw<FMT, BWD>(p, sg[ld.g], ld.tw * 2 + static_cast<int>(rank), r, ld.ks, raw);
        advance(ld);
      }
    };
    auto step_one = [&](Raw& cur) -> bool {
      to_parity(cv);
      if (cv.i >= nu) return false;
      const int slot_a = cv.step % SA;
      const uint32_t pa = static_cast<uint32_t>((cv.step / SA) & 1);
      const int sb = cv.step % SB;
      const uint32_t pb = static_cast<uint32_t>((cv.step / SB) & 1);
      // decode first (backward: once this step's scale tile has landed), then wait for
      // the MMA that last read this weight slot (in both CTAs) and only store
      if (BWD && !warp_wait_bounded(&s_full[sb], pb, abort_flag, kErrWaitFull)) return false;
      uint32_t o[32];
      const int srow = BWD ? ((FMT == kFp8) ? 0 : r / gsz) : 0;
      gdq::convert<FMT, BWD>(cur, sS + sb * S_BYTES, srow, o);
      bool ok = false;
      if (lane == 0) ok = mbar_wait(&a_empty[slot_a], pa ^ 1, abort_flag, kErrWaitEmpty);
      if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) return false;
      __syncwarp();
      tmem_st_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + A_COL0 + static_cast<uint32_t>(slot_a * 32), o);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&a_full[slot_a]);  // this CTA's barrier (the peer's is relayed to the leader)
      fetch(cur);
      advance(cv);
      return true;
    };
    Raw ring[2];
    fetch(ring[0]);
    fetch(ring[1]);
    while (step_one(ring[0]) && step_one(ring[1])) {
    }
  }
  // In-flight copies: on an abort, give the activation loads this CTA issued (whose
  // bytes count on the leader's barrier) time to land before shared memory goes away.
  if (*abort_flag) {
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  tc_fence_before();
  cluster_sync_all();  // no remote arrival or MMA into this CTA is still pending
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace gdq2
}  // namespace oftk
