// Routing, bucketing, chunking, rotated gather and combine for the
// active-expert-chunked MoE OFT forward.
//
// The pages: the experts the router selects are grouped into fixed-size chunks,
// each chunk is dequantised transiently and fed to a grouped GEMM, after which
// its high-precision copy is released, so peak transient memory stays bounded by
// one chunk (m.xxlwj.com 771001, section "技术细节", paragraph
// "Active-expert-chunked dequantization"; chooseai.io news 4086, section
// "对低精度 MoE 模型的专门优化").  Readings for what the pages leave open: top-k by
// logit with ties to the lower expert id, softmax over the selected logits,
// buckets stable in (token, slot), active experts ascending, combine in slot order.
#pragma once

#include "common.cuh"

namespace oftk {

constexpr int kMaxExperts = 512;
constexpr int kMaxTopK = 8;

// One warp per token: top_k by (logit desc, expert id asc), then softmax over
// the selected logits (fp32).
//
// Non-finite logits (a diverging router): NaN ranks as -inf.  Only lanes holding a
// real expert (e < E) are ever candidates and k <= E, so every emitted index is in
// [0, E) whatever the logits hold.  The weights are the softmax's limit where the
// selected values are infinite: if the largest is +inf, the +inf entries share the
// weight equally and the rest get 0; if it is -inf (every selected logit is -inf or
// NaN), each of the k gets 1/k.
__global__ void __launch_bounds__(256) moe_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                       int* __restrict__ idx_out, float* __restrict__ w_out) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (warp >= T) return;
  constexpr int PER = kMaxExperts / 32;
  float v[PER];
  uint32_t taken = 0;
  const float* row = logits + static_cast<size_t>(warp) * E;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    const float x = e < E ? row[e] : -INFINITY;
    v[i] = isnan(x) ? -INFINITY : x;
    if (e >= E) taken |= 1u << i;
  }
  float sel_v[kMaxTopK];
  int sel_e[kMaxTopK];
  for (int s = 0; s < k; ++s) {
    float bv = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      if (!(taken & (1u << i)) && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
      const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    // some lane with e < E is still free (k <= E), and it beats the (-inf, INT_MAX)
    // placeholder of lanes without a candidate, so be < E here
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    sel_v[s] = bv;
    sel_e[s] = be;
  }
  if (lane == 0) {
    const float mx = sel_v[0];
    float ex[kMaxTopK];
    float sum = 0.f;
    for (int s = 0; s < k; ++s) {
      if (mx == INFINITY)
        ex[s] = sel_v[s] == INFINITY ? 1.f : 0.f;
      else if (mx == -INFINITY)
        ex[s] = 1.f;
      else
        ex[s] = expf(sel_v[s] - mx);
      sum += ex[s];
    }
    for (int s = 0; s < k; ++s) {
      idx_out[static_cast<size_t>(warp) * k + s] = sel_e[s];
      w_out[static_cast<size_t>(warp) * k + s] = ex[s] / sum;
    }
  }
}

// Single CTA of 1024 threads (32 warps).  Each warp owns a contiguous range of
// the T*k entries; warp-private histograms give every (warp, expert) a base
// offset, and each warp then places its entries in order (match_any ranks
// equal experts within a 32-entry step), so the bucket is stable in (t, slot)
// and independent of scheduling.
// Outputs: offsets[E+1], bucket[TK], inv_pos[TK] (entry -> bucket position),
// pos_expert[TK], chunk_table[n_chunks_max * chunk] (-1 padded), n_active[1].
__global__ void __launch_bounds__(1024) moe_route_kernel(const int* __restrict__ idx, int TK, int E, int chunk,
                                                         int n_chunks_max, int* __restrict__ offsets,
                                                         int* __restrict__ bucket, int* __restrict__ inv_pos,
                                                         int* __restrict__ pos_expert, int* __restrict__ chunk_table,
                                                         int* __restrict__ n_active) {
  extern __shared__ int rsm[];
  int* hist = rsm;                // [32][E]
  int* off = rsm + 32 * E;        // [E + 1]
  int* act = off + E + 1;         // [E] exclusive rank among active experts
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int per = (TK + 31) / 32;
  const int beg = min(TK, warp * per), end = min(TK, beg + per);
  for (int i = threadIdx.x; i < 32 * E; i += 1024) hist[i] = 0;
  __syncthreads();
  for (int j = beg + lane; j < end; j += 32) atomicAdd(&hist[warp * E + idx[j]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += 1024) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    off[e] = run;  // total count for now
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0, na = 0;
    for (int e = 0; e < E; ++e) {
      const int c = off[e];
      off[e] = acc;
      acc += c;
      act[e] = c > 0 ? na++ : -1;
    }
    off[E] = acc;
    *n_active = na;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += 1024) offsets[e] = off[e];
  for (int i = threadIdx.x; i < n_chunks_max * chunk; i += 1024) chunk_table[i] = -1;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += 1024)
    if (act[e] >= 0) chunk_table[act[e]] = e;
  // stable fill
  for (int j0 = beg; j0 < end; j0 += 32) {
    const int j = j0 + lane;
    const bool valid = j < end;
    const int e = valid ? idx[j] : -1 - lane;  // distinct dummies for idle lanes
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int base = 0;
    if (valid) base = hist[warp * E + e];
    __syncwarp();
    if (valid) {
      const int pos = off[e] + base + rank;
      bucket[pos] = j;
      inv_pos[j] = pos;
      pos_expert[pos] = e;
      if (rank == 0) hist[warp * E + e] = base + __popc(peers);
    }
    __syncwarp();
  }
}

// Rotated gather on the tensor cores: Xg[proj][pos][:] = X[bucket[pos] / k] R_{e,proj}.
// Units are (active expert, 64-column group, 128-position tile of that expert's
// bucket rows), in that order with the tile fastest, so a tile never mixes experts
// and consecutive units of a CTA share the expert's rotation tiles.  A CTA (128
// threads, four resident per SM) walks a contiguous range of units:
//   gather the tile's 128 activation rows (64 bf16 columns) into a 128B-swizzled
//   K-major tile; on an (expert, group) change the B tiles B[p*64 + c][i] =
//   R_{e,p}[i][c] over the group's diagonal blocks for p = gate, up hold bf16 hi + lo
//   parts; one thread issues 8 tcgen05.mma (M = 128, N = 128, K = 64 as 4 x 16, hi
//   and lo) into TMEM; the epilogue writes the tile's valid rows.
// The rotations come from the Cayley build already split into hi / lo and
// transposed (Rhi / Rlo [e][p][block][c][i]), so each 8 reduction indices of a B row
// are one 16-byte cp.async; the tiles' off-diagonal zeros are written once, and the
// next unit's diagonal blocks are fetched while the current unit's epilogue runs.
// The rotation of activations in front of the frozen weight is the OFT adapter
// ("Orbit", chooseai.io news 4086, section "技术原理：低精度基座 + BF16 适配器 + OFT");
// the per-expert split into gate and up is its split-projection form (item
// "自定义适配器核函数").
constexpr int kMoeRotThreads = 128;
constexpr size_t kMoeRotSmem = 1024 + 3 * 16384 + 64;

template <int B>
__global__ void __launch_bounds__(kMoeRotThreads, 4) moe_rot_tc_kernel(
    const uint16_t* __restrict__ X, int K, int top_k, const int* __restrict__ bucket,
    const int* __restrict__ offsets, const int* __restrict__ active, const int* __restrict__ n_active_p,
    const uint16_t* __restrict__ Rhi, const uint16_t* __restrict__ Rlo, int TK, uint16_t* __restrict__ Xg) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                 // 128 positions x 64 columns, bf16, 128B swizzle
  uint8_t* sBhi = sA + 16384;         // 128 (gate|up output columns) x 64, bf16 hi
  uint8_t* sBlo = sBhi + 16384;       // lo
  uint64_t* bar = reinterpret_cast<uint64_t*>(sBlo + 16384);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ int s_pref[kMaxExperts + 1];  // units before active expert a
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int G = (K + 63) / 64, nb = K / B;
  const int na = *n_active_p;
  if (warp == 0) {
    // prefix over active experts of (position tiles x column groups), one warp
    int carry = 0;
    for (int a0 = 0; a0 < na; a0 += 32) {
      const int a = a0 + lane;
      int v = 0;
      if (a < na) {
        const int e = active[a];
        v = ((offsets[e + 1] - offsets[e] + 127) / 128) * G;
      }
      int x = v;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, x, d);
        if (lane >= d) x += y;
      }
      if (a < na) s_pref[a + 1] = carry + x;
      carry += __shfl_sync(0xFFFFFFFFu, x, 31);
    }
    if (lane == 0) s_pref[0] = 0;
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  // the B tiles' off-diagonal blocks stay zero for the whole launch
  for (int v = tid; v < 16384 / 16; v += kMoeRotThreads) {
    reinterpret_cast<uint4*>(sBhi)[v] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4*>(sBlo)[v] = make_uint4(0, 0, 0, 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total = s_pref[na];
  const int per = total / static_cast<int>(gridDim.x), rem = total % static_cast<int>(gridDim.x);
  const int ubeg = static_cast<int>(blockIdx.x) * per + min(static_cast<int>(blockIdx.x), rem);
  const int uend = ubeg + per + (static_cast<int>(blockIdx.x) < rem ? 1 : 0);
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
  constexpr int NIT = 128 * 8 / kMoeRotThreads;  // 16-byte activation loads per thread and unit
  struct Unit {
    int e, g, pos0, nrows;
  };
  // units are visited in increasing order; each cursor keeps its own active-expert index
  auto unit_at = [&](int u, int& acur) -> Unit {
    while (acur + 1 < na && s_pref[acur + 1] <= u) ++acur;
    const int e = active[acur];
    const int pos_beg = offsets[e], n_e = offsets[e + 1] - pos_beg;
    const int tiles = (n_e + 127) / 128;
    const int local = u - s_pref[acur];
    const int g = local / tiles, rt = local % tiles;
    return Unit{e, g, pos_beg + rt * 128, min(128, n_e - rt * 128)};
  };
  // Software pipeline: unit u's activation rows are loaded while unit u-1 is multiplied
  // and stored, and the bucket entries that give their token ids one unit earlier still,
  // so no load waits on another load.
  auto load_tokens = [&](const Unit& U, bool valid, int (&tok)[NIT]) {
#pragma unroll
    for (int q = 0; q < NIT; ++q) {
      const int r = (tid + q * kMoeRotThreads) >> 3;
      tok[q] = (valid && r < U.nrows) ? bucket[U.pos0 + r] : -1;
    }
  };
  auto load_rows = [&](const Unit& U, const int (&tok)[NIT], uint4 (&xv)[NIT]) {
#pragma unroll
    for (int q = 0; q < NIT; ++q) {
      const int col = U.g * 64 + ((tid + q * kMoeRotThreads) & 7) * 8;
      xv[q] = make_uint4(0, 0, 0, 0);
      if (tok[q] >= 0 && col < K) xv[q] = *reinterpret_cast<const uint4*>(X + static_cast<size_t>(tok[q] / top_k) * K + col);
    }
  };
  // the diagonal blocks of (e, g) into the B tiles: 16-byte cp.async per 8 reduction
  // indices of one output column, hi and lo (zeros for a block past K)
  auto issue_b = [&](int e, int g) {
    constexpr int NBG = 64 / B, CH = B / 8;
    constexpr int NCOPY = 2 * NBG * B * CH;
    for (int v = tid; v < NCOPY; v += kMoeRotThreads) {
      const int pr = v / (NBG * B * CH);
      int rem = v % (NBG * B * CH);
      const int jb = rem / (B * CH);
      rem %= B * CH;
      const int c = rem / CH, i8 = rem % CH;
      const int j = (g * 64) / B + jb;
      const uint32_t off = sw128_offset(static_cast<uint32_t>(pr * 64 + jb * B + c),
                                        static_cast<uint32_t>((jb * B + i8 * 8) >> 3));
      if ((j + 1) * B <= K) {
        const size_t src = (((static_cast<size_t>(e) * 2 + pr) * nb + j) * B + c) * B + i8 * 8;
        cp_async_16(sBhi + off, Rhi + src);
        cp_async_16(sBlo + off, Rlo + src);
      } else {
        *reinterpret_cast<uint4*>(sBhi + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(sBlo + off) = make_uint4(0, 0, 0, 0);
      }
    }
    cp_async_commit();
  };
  int cur_e = -1, cur_g = -1, pf_e = -1, pf_g = -1, a = 0, a1 = 0, a2 = 0, ab = 0;
  uint32_t phase = 0;
  uint4 xv[NIT];
  // token ids of the unit after next go to one of two buffers by unit parity (the loop
  // below is unrolled by two), so no instruction waits on loads still in flight
  int tokE[NIT], tokO[NIT];
  if (ubeg < uend) {
    const Unit u0 = unit_at(ubeg, a1);
    load_tokens(u0, true, tokE);
    load_rows(u0, tokE, xv);
    const bool v1 = ubeg + 1 < uend;
    load_tokens(v1 ? unit_at(ubeg + 1, a2) : u0, v1, tokO);
  }
  a1 = a2;
  // one unit: tok_next holds the token ids of unit u + 1; unit u + 2's are loaded into tok_dst
  auto run_unit = [&](int u, const int (&tok_next)[NIT], int (&tok_dst)[NIT]) -> bool {
    const Unit U = unit_at(u, a);
    const int e = U.e, g = U.g, pos0 = U.pos0, nrows = U.nrows;
    // 1. rotation tiles of (e, g), when they change (fetched during the previous unit's
    //    epilogue, after its MMAs had completed; the first unit's here)
    if (e != cur_e || g != cur_g) {
      if (e != pf_e || g != pf_g) issue_b(e, g);
      cp_async_wait_all();
      cur_e = e;
      cur_g = g;
      pf_e = pf_g = -1;
    }
    // 2. this unit's activation rows (loaded one unit ago) into the swizzled A tile
#pragma unroll
    for (int q = 0; q < NIT; ++q) {
      const int it = tid + q * kMoeRotThreads;
      *reinterpret_cast<uint4*>(sA + sw128_offset(static_cast<uint32_t>(it >> 3), static_cast<uint32_t>(it & 7))) = xv[q];
    }
    fence_proxy_async_smem();
    __syncthreads();
    // 3. the product
    if (tid == 0) {
      tc_fence_after();
      const uint32_t a0 = smem_u32(sA), bh = smem_u32(sBhi), bl = smem_u32(sBlo);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = sdesc_sw128(a0 + kk * 32, 16, 1024);
        mma_bf16_ss(tmem, ad, sdesc_sw128(bh + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        mma_bf16_ss(tmem, ad, sdesc_sw128(bl + kk * 32, 16, 1024), idesc, 1u);
      }
      mma_commit(bar);
    }
    // prefetch: unit u+1's rows (their token ids are already in tok_next), unit u+2's token ids
    if (u + 1 < uend) {
      load_rows(unit_at(u + 1, a1), tok_next, xv);
      const bool v2 = u + 2 < uend;
      load_tokens(v2 ? unit_at(u + 2, a2) : U, v2, tok_dst);
    }
    if (!warp_wait_bounded(bar, phase, abort_flag, kErrWaitAccFull)) return false;
    phase ^= 1;
    tc_fence_after();
    // the product has read the B tiles: start the next unit's, if they differ
    if (u + 1 < uend) {
      const Unit Un = unit_at(u + 1, ab);
      if (Un.e != cur_e || Un.g != cur_g) {
        issue_b(Un.e, Un.g);
        pf_e = Un.e;
        pf_g = Un.g;
      }
    }
    // 4. epilogue: TMEM lane = position row, 64 columns per projection
    const int r = warp * 32 + lane;
#pragma unroll 1
    for (int pr = 0; pr < 2; ++pr) {
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(pr * 64 + h * 32), v);
        tmem_ld_wait();
        const int col = g * 64 + h * 32;
        if (r < nrows) {
          uint4* dst = reinterpret_cast<uint4*>(Xg + (static_cast<size_t>(pr) * TK + pos0 + r) * K + col);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (col + 8 * q < K)  // K is a multiple of 16: 8-column chunks are whole
            dst[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                                pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                                pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                                pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // TMEM and the shared tiles are free for the next unit
    return true;
  };
  for (int u = ubeg; u < uend; u += 2) {
    if (!run_unit(u, tokO, tokE)) break;
    if (u + 1 < uend && !run_unit(u + 1, tokE, tokO)) break;
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// Y[t][n] = sum_{s < k} w[t][s] * Ytk[inv_pos[t*k + s]][n], fp32 in slot order (Ytk kept in fp32).
__global__ void __launch_bounds__(256) moe_combine_kernel(const float* __restrict__ Ytk, const float* __restrict__ w,
                                                          const int* __restrict__ inv_pos, int T, int N, int k,
                                                          uint16_t* __restrict__ Y) {
  const long long units = static_cast<long long>(T) * (N / 8);
  for (long long u = blockIdx.x * 256ll + threadIdx.x; u < units; u += static_cast<long long>(gridDim.x) * 256) {
    const int t = static_cast<int>(u / (N / 8));
    const int n = static_cast<int>(u % (N / 8)) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < k; ++s) {
      const float ws = w[static_cast<size_t>(t) * k + s];
      const int pos = inv_pos[static_cast<size_t>(t) * k + s];
      const float4 a = *reinterpret_cast<const float4*>(Ytk + static_cast<size_t>(pos) * N + n);
      const float4 b = *reinterpret_cast<const float4*>(Ytk + static_cast<size_t>(pos) * N + n + 4);
      acc[0] = fmaf(ws, a.x, acc[0]);
      acc[1] = fmaf(ws, a.y, acc[1]);
      acc[2] = fmaf(ws, a.z, acc[2]);
      acc[3] = fmaf(ws, a.w, acc[3]);
      acc[4] = fmaf(ws, b.x, acc[4]);
      acc[5] = fmaf(ws, b.y, acc[5]);
      acc[6] = fmaf(ws, b.z, acc[6]);
      acc[7] = fmaf(ws, b.w, acc[7]);
    }
    *reinterpret_cast<uint4*>(Y + static_cast<size_t>(t) * N + n) =
        make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                   pack_bf16x2(acc[6], acc[7]));
  }
}

}  // namespace oftk
