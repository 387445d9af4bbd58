// C ABI of the OFT hot path (declared in include/oft.h): argument checks,
// workspace carving, TMA descriptor encoding and kernel launches.  All the
// arithmetic runs in the kernels included below.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <memory>
#include <mutex>
#include <queue>
#include <vector>
#include <string>
#include <utility>

#include "oft.h"

#include "common.cuh"
#include "dequant.cuh"
#include "cayley.cuh"
#include "gemm.cuh"
#include "moe.cuh"
#include "rot_tc.cuh"
#include "gemm_dq.cuh"
#include "gemm_dq2.cuh"
#include "gemm_sm.cuh"
#include "moe_fused.cuh"
#include "moe_bwd.cuh"
#include "moe_bwd_tc.cuh"
#include "moe_layer.cuh"

using namespace oftk;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

#define OFT_CUDA(call)                                                                      \
  do {                                                                                      \
    cudaError_t e_ = (call);                                                                \
    if (e_ != cudaSuccess) return fail(OFT_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

#define OFT_LAUNCHED(what)                                                                     \
  do {                                                                                         \
    cudaError_t e_ = cudaGetLastError();                                                       \
    if (e_ != cudaSuccess) return fail(OFT_ERR_CUDA, "launch %s: %s", what, cudaGetErrorString(e_)); \
  } while (0)

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Launches with programmatic stream serialisation (the kernel may be scheduled while
// the previous kernel on the stream drains; it calls pdl_wait() before touching
// global memory).  OFT_PDL=0 in the environment turns it off.
bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("OFT_PDL");
    return v == nullptr || v[0] != '0';
  }();
  return on;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Per-device side stream and events for the MoE chunk pipeline (dequant of chunk
// c + 1 overlaps the grouped GEMM of chunk c).  Created on first use, kept until
// exit; they hold no device memory.
// The events are shared by every call on the device, so a call holds the pipe's lock
// from its first record to its last wait (host-side enqueue only): two host threads
// then never interleave their records and waits on the same event.
struct SidePipe {
  bool ready = false;
  cudaStream_t side = nullptr;
  cudaEvent_t start = nullptr, dq_done[2] = {nullptr, nullptr}, gemm_done[2] = {nullptr, nullptr};
  std::mutex mu;
};
SidePipe g_side[64];
std::mutex g_side_create_mu;

// On success *out is the device's pipe and *lock holds its mutex.
int side_pipe(SidePipe** out, std::unique_lock<std::mutex>* lock) {
  int dev = 0;
  OFT_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(OFT_ERR_UNSUPPORTED, "device index %d out of range", dev);
  SidePipe& sp = g_side[dev];
  std::lock_guard<std::mutex> create(g_side_create_mu);
  if (!sp.ready) {
    OFT_CUDA(cudaStreamCreateWithFlags(&sp.side, cudaStreamNonBlocking));
    OFT_CUDA(cudaEventCreateWithFlags(&sp.start, cudaEventDisableTiming));
    for (int i = 0; i < 2; ++i) {
      OFT_CUDA(cudaEventCreateWithFlags(&sp.dq_done[i], cudaEventDisableTiming));
      OFT_CUDA(cudaEventCreateWithFlags(&sp.gemm_done[i], cudaEventDisableTiming));
    }
    sp.ready = true;
  }
  *lock = std::unique_lock<std::mutex>(sp.mu);
  *out = &sp;
  return OFT_OK;
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return n;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  n = n > 0 ? n : 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

// ---- launch profiler: CUDA event pairs around launches, per kernel class ----
struct ProfState {
  bool on = false;
  int cap = 0, n = 0, dropped = 0;
  cudaEvent_t* ev = nullptr;  // 2 per slot
  int* kind = nullptr;
  int counts[OFT_K_NUM] = {0};
};
ProfState g_prof;

struct ProfScope {
  int idx = -1;
  cudaStream_t st;
  ProfScope(int k, cudaStream_t s) : st(s) {
    if (!g_prof.on) return;
    g_prof.counts[k]++;
    if (g_prof.n < g_prof.cap) {
      idx = g_prof.n++;
      g_prof.kind[idx] = k;
      cudaEventRecord(g_prof.ev[2 * idx], st);
    } else {
      g_prof.dropped++;
    }
  }
  ~ProfScope() {
    if (idx >= 0) cudaEventRecord(g_prof.ev[2 * idx + 1], st);
  }
};

// ---- driver entry point for TMA descriptors (no link-time libcuda dependency) ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor [outer][inner] with row pitch `pitch_elems`, box {64, box_rows}, 128B swizzle.
int make_map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch_elems,
                  uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(OFT_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(OFT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d): inner=%llu outer=%llu pitch=%llu", int(r),
                (unsigned long long)inner, (unsigned long long)outer, (unsigned long long)pitch_elems);
  return OFT_OK;
}

// 3-D fp32 tensor [P][M][K] (dX'), box {32, box_rows, 1}; rows past M read as zero.  `swizzle` is the
// 128B swizzle (K-major operands) or its 32-byte-atom variant (MN-major tf32 operands).
int make_map_f32_3d(CUtensorMap* m, const void* base, uint64_t K, uint64_t M, uint64_t P,
                    CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B, uint32_t box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(OFT_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {K, M, P};
  cuuint64_t strides[2] = {K * 4, M * K * 4};
  cuuint32_t box[3] = {32, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(OFT_ERR_CUDA, "cuTensorMapEncodeTiled (fp32 3-D) failed (%d)", int(r));
  return OFT_OK;
}

// 3-D bf16 tensor [P][M][K] for TMA stores of 32-row x 64-column boxes, 128B swizzle:
// stores clip at M within each split and at K.
int make_map_bf16_3d_store(CUtensorMap* m, void* base, uint64_t K, uint64_t M, uint64_t P) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(OFT_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {K, M, P};
  cuuint64_t strides[2] = {K * 2, M * K * 2};
  cuuint32_t box[3] = {64, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(OFT_ERR_CUDA, "cuTensorMapEncodeTiled (bf16 3-D store) failed (%d)", int(r));
  return OFT_OK;
}

// Generic 2-D map without swizzle (scale tiles of the backward's dequant producers).
int make_map_plain_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                      uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(OFT_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(OFT_ERR_CUDA, "cuTensorMapEncodeTiled (plain 2-D) failed (%d)", int(r));
  return OFT_OK;
}

// ---- argument checks ----
int check_weight(const oft_weight* W, bool bank_ok) {
  if (W == nullptr) return fail(OFT_ERR_INVALID_ARG, "weight descriptor is NULL");
  if (W->codes == nullptr || W->scales == nullptr) return fail(OFT_ERR_INVALID_ARG, "weight codes/scales NULL");
  if (!aligned16(W->codes) || !aligned16(W->scales))
    return fail(OFT_ERR_INVALID_ARG, "weight codes/scales must be 16-byte aligned");
  if (W->d_in <= 0 || W->d_out <= 0) return fail(OFT_ERR_INVALID_ARG, "d_in/d_out must be positive");
  if (W->d_in % 32 != 0) return fail(OFT_ERR_UNSUPPORTED, "d_in must be a multiple of 32 (got %d)", W->d_in);
  if (W->d_out % 8 != 0) return fail(OFT_ERR_UNSUPPORTED, "d_out must be a multiple of 8 (got %d)", W->d_out);
  if (!bank_ok && W->n_experts > 1) return fail(OFT_ERR_INVALID_ARG, "an expert bank is not accepted here");
  switch (W->fmt) {
    case OFT_W_INT4:
      if (W->group != 32 && W->group != 64 && W->group != 128)
        return fail(OFT_ERR_UNSUPPORTED, "INT4 group must be 32, 64 or 128 (got %d)", W->group);
      if (W->d_in % W->group != 0) return fail(OFT_ERR_UNSUPPORTED, "d_in %% group != 0");
      break;
    case OFT_W_FP8:
      break;
    case OFT_W_MXFP4:
      if (W->group != 32 && W->group != 0) return fail(OFT_ERR_UNSUPPORTED, "MXFP4 blocks are 32 wide");
      break;
    default:
      return fail(OFT_ERR_UNSUPPORTED, "unknown weight format %d", W->fmt);
  }
  return OFT_OK;
}

int check_b(int b, int K) {
  if (b != 16 && b != 32 && b != 64) return fail(OFT_ERR_UNSUPPORTED, "block size b must be 16, 32 or 64 (got %d)", b);
  if (K % b != 0) return fail(OFT_ERR_UNSUPPORTED, "d_in %d is not a multiple of b %d", K, b);
  return OFT_OK;
}

int check_split(const oft_split* S, int N) {
  if (S == nullptr) return fail(OFT_ERR_INVALID_ARG, "split descriptor is NULL");
  if (S->n < 1 || S->n > 4) return fail(OFT_ERR_UNSUPPORTED, "1..4 sub-projections supported (got %d)", S->n);
  int sum = 0;
  for (int i = 0; i < S->n; ++i) {
    if (S->sizes[i] <= 0 || S->sizes[i] % 8 != 0)
      return fail(OFT_ERR_UNSUPPORTED, "sub-projection sizes must be positive multiples of 8");
    sum += S->sizes[i];
  }
  if (sum != N) return fail(OFT_ERR_INVALID_ARG, "sub-projection sizes sum to %d, d_out is %d", sum, N);
  return OFT_OK;
}

WeightView view_of(const oft_weight* W) {
  WeightView v{};
  v.fmt = W->fmt;
  v.codes = static_cast<const uint8_t*>(W->codes);
  v.scales = W->scales;
  v.N = W->d_out;
  v.K = W->d_in;
  v.group = W->fmt == OFT_W_INT4 ? W->group : 32;
  const long long code_bytes = W->fmt == OFT_W_FP8 ? 1ll * W->d_out * W->d_in : 1ll * W->d_out * W->d_in / 2;
  long long scale_bytes = 0;
  if (W->fmt == OFT_W_INT4) scale_bytes = 2ll * (W->d_in / W->group) * W->d_out;
  if (W->fmt == OFT_W_FP8) scale_bytes = 4ll * W->d_out;
  if (W->fmt == OFT_W_MXFP4) scale_bytes = 1ll * (W->d_in / 32) * W->d_out;
  v.codes_expert_stride = code_bytes;
  v.scales_expert_stride = scale_bytes;
  return v;
}

int launch_dequant(const WeightView& v, uint16_t* out, bool transpose, cudaStream_t st) {
  if (1ll * v.N * v.K / 8 >= (1ll << 31)) return fail(OFT_ERR_UNSUPPORTED, "weight too large for one dequant launch");
  if (!transpose) {
    const long long units = 1ll * v.N * (v.K / 8);
    const int grid = static_cast<int>(std::min<long long>((units + 1023) / 1024, 148ll * 8));
    ProfScope ps(OFT_K_DEQUANT, st);
    OFT_CUDA(launch_pdl(dequant_rows_kernel, grid, 256, 0, st, v, out));
    OFT_LAUNCHED("dequant_rows_kernel");
  } else {
    dim3 grid((v.K + kDeqTCols - 1) / kDeqTCols, (v.N + kDeqTRows - 1) / kDeqTRows);
    ProfScope ps(OFT_K_DEQUANT, st);
    OFT_CUDA(launch_pdl(dequant_transposed_kernel, grid, 256, 0, st, v, out));
    OFT_LAUNCHED("dequant_transposed_kernel");
  }
  return OFT_OK;
}

// active_list / n_active (device): build only the blocks of the active experts.
// lo_off > 0: R is written as the bf16 hi / lo parts of each block's transpose, hi at
// (uint16_t*)R and lo lo_off elements further (the MoE rotated gather's operand).
int launch_cayley(const uint16_t* Q, int nblocks, int b, float* R, const int* active_list, const int* n_active,
                  int blocks_per_expert, cudaStream_t st, long long lo_off = 0) {
  ProfScope ps(OFT_K_CAYLEY, st);
  // unrolled pivots pay off once many blocks run from a warm instruction cache;
  // persistent grid of about 32 resident warps per SM
  const int bpc = b == 16 ? 2 : 1, warps = b == 64 ? 2 : 1;
  const int grid = std::max(1, std::min((nblocks + bpc - 1) / bpc, sm_count() * 32 / warps));
  const int* al = active_list;
  if (nblocks >= kCayleyUnrollBlocks) {
    if (b == 16) OFT_CUDA(launch_pdl(cayley_fwd_kernel<16, true>, grid, 32, 0, st, Q, nblocks, R, al, n_active, blocks_per_expert, lo_off));
    if (b == 32) OFT_CUDA(launch_pdl(cayley_fwd_kernel<32, true>, grid, 32, 0, st, Q, nblocks, R, al, n_active, blocks_per_expert, lo_off));
    if (b == 64) OFT_CUDA(launch_pdl(cayley_fwd_kernel<64, true>, grid, 64, 0, st, Q, nblocks, R, al, n_active, blocks_per_expert, lo_off));
  } else {
    if (b == 16) OFT_CUDA(launch_pdl(cayley_fwd_kernel<16, false>, grid, 32, 0, st, Q, nblocks, R, al, n_active, blocks_per_expert, lo_off));
    // few blocks: the per-block pivot chain is the time, so four threads share each row
    const int sgrid = std::max(1, std::min(nblocks, sm_count() * 8));
    if (b == 32) OFT_CUDA(launch_pdl(cayley_fwd_inv_split_kernel<32, 4>, sgrid, 128, 0, st, Q, nblocks, R, al, n_active, blocks_per_expert, lo_off));
    if (b == 64) OFT_CUDA(launch_pdl(cayley_fwd_inv_split_kernel<64, 4>, sgrid, 256, 0, st, Q, nblocks, R, al, n_active, blocks_per_expert, lo_off));
  }
  OFT_LAUNCHED("cayley_fwd_kernel");
  return OFT_OK;
}

int launch_cayley_bwd(const float* R, const float* G, int nparts, int nblocks, int b, float* dQ, cudaStream_t st,
                      const int* map = nullptr, const int* n_map = nullptr, int per = 1) {
  // blocks per CTA: as many as fit (up to 256 threads), but no fewer CTAs than about
  // two per SM while the launch has the blocks for it
  const int nt = (b / 4) * (b / 4);
  const int bpc_max = kCayleyThreads / nt;
  int bpc = 1;
  while (bpc * 2 <= bpc_max && 1ll * nblocks >= 2ll * bpc * 2 * sm_count()) bpc *= 2;
  const size_t smem = static_cast<size_t>(bpc) * (b == 16 ? CayleyBwdCfg<16>::SMEM_PER_BLOCK
                                                          : (b == 32 ? CayleyBwdCfg<32>::SMEM_PER_BLOCK
                                                                     : CayleyBwdCfg<64>::SMEM_PER_BLOCK));
  const int grid = static_cast<int>(std::min<long long>((nblocks + bpc - 1) / bpc, sm_count() * 3ll * (bpc_max / bpc)));
  if (b == 16) OFT_CUDA(cudaFuncSetAttribute(cayley_bwd_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  if (b == 32) OFT_CUDA(cudaFuncSetAttribute(cayley_bwd_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  if (b == 64) OFT_CUDA(cudaFuncSetAttribute(cayley_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  ProfScope ps(OFT_K_CAYLEY, st);
  if (b == 16) OFT_CUDA(launch_pdl(cayley_bwd_kernel<16>, grid, bpc * nt, smem, st, R, G, nparts, nblocks, dQ, map, n_map, per));
  if (b == 32) OFT_CUDA(launch_pdl(cayley_bwd_kernel<32>, grid, bpc * nt, smem, st, R, G, nparts, nblocks, dQ, map, n_map, per));
  if (b == 64) OFT_CUDA(launch_pdl(cayley_bwd_kernel<64>, grid, bpc * nt, smem, st, R, G, nparts, nblocks, dQ, map, n_map, per));
  OFT_LAUNCHED("cayley_bwd_kernel");
  return OFT_OK;
}

template <typename KernelT>
int set_smem(KernelT kernel, size_t bytes) {
  OFT_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)));
  return OFT_OK;
}

// X'_p = X R_p on the tensor cores (all P sub-projections in one pass).
int launch_rotate_fwd(const uint16_t* X, int M, int K, int P, int b, const float* R, uint16_t* Xr, cudaStream_t st,
                      bool transpose = false, int* zero_ptr = nullptr, int zero_n = 0) {
  rtc::FwdParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.transpose = transpose ? 1 : 0;
  prm.zero_ptr = zero_ptr;
  prm.zero_n = zero_ptr != nullptr ? zero_n : 0;
  if (int rc = make_map_bf16(&prm.tmX, X, K, M, K, rtc::TM)) return rc;
  if (int rc = make_map_bf16_3d_store(&prm.tmY, Xr, K, M, P)) return rc;
  prm.R = R;
  prm.Xr = Xr;
  prm.M = M;
  prm.K = K;
  prm.P = P;
  prm.b = b;
  prm.nb = K / b;
  prm.groups = (K + 63) / 64;
  prm.tiles_m = (M + rtc::TM - 1) / rtc::TM;
  {
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
      if (int rc = set_smem(rtc::rot_fwd_tc_kernel, rtc::kFwdSmem)) return rc;
      if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
  }
  const int grid = std::min(sm_count(), prm.groups * prm.tiles_m);
  ProfScope ps(OFT_K_ROTATE, st);
  OFT_CUDA(launch_pdl(rtc::rot_fwd_tc_kernel, grid, rtc::FWD_THREADS, rtc::kFwdSmem, st, prm));
  OFT_LAUNCHED("rot_fwd_tc_kernel");
  return OFT_OK;
}

// dX = sum_p dX'_p R_p^T on the tensor cores (tf32).
int launch_rotate_bwd(const float* dXr, int M, int K, int P, int b, const float* R, uint16_t* dX, cudaStream_t st) {
  rtc::BwdParams prm;
  memset(&prm, 0, sizeof(prm));
  if (int rc = make_map_f32_3d(&prm.tmD, dXr, K, M, P)) return rc;
  prm.R = R;
  prm.dX = dX;
  prm.M = M;
  prm.K = K;
  prm.P = P;
  prm.b = b;
  prm.nb = K / b;
  prm.groups = (K + 63) / 64;
  prm.tiles_m = (M + rtc::TM - 1) / rtc::TM;
  if (int rc = set_smem(rtc::rot_bwd_tc_kernel, rtc::kBwdSmem)) return rc;
  const int grid = std::min(sm_count(), prm.groups * prm.tiles_m);
  ProfScope ps(OFT_K_ROTATE, st);
  OFT_CUDA(launch_pdl(rtc::rot_bwd_tc_kernel, grid, rtc::NUM_THREADS, rtc::kBwdSmem, st, prm));
  OFT_LAUNCHED("rot_bwd_tc_kernel");
  return OFT_OK;
}

// Token chunking of the dR reduction (deterministic in the shape, fixed for a 148-SM
// part so the workspace size does not depend on the device): units are (128-column
// group, chunk of token tiles), spread over 148 CTAs in contiguous ranges.  The chunk
// length minimises the busiest CTA's work, ceil(units / 148) x (tiles per chunk + 1),
// the one counting a unit's accumulator drain and partial-sum writes; ties go to
// longer chunks (fewer partial sums).  The MXFP4 training step (56 groups, 128 token
// tiles) takes 5 chunks of 26 tiles: 52 tiles on the busiest CTA, against 64 with one
// chunk per SM's worth of groups.
struct GradChunks {
  int chunks, tiles_per_chunk;
};
GradChunks grad_chunks(int M, int K) {
  const int groups = (K + 127) / 128, tiles_m = (M + 127) / 128;
  int best_tpc = tiles_m;
  long long best = 1ll << 60;
  for (int tpc = tiles_m; tpc >= 1; --tpc) {
    const int chunks = (tiles_m + tpc - 1) / tpc;
    if ((chunks - 1) * tpc >= tiles_m) continue;  // the same chunking as a longer tpc
    const long long units = 1ll * groups * chunks;
    const long long cost = (units + 147) / 148 * (tpc + 1);
    if (cost < best) {
      best = cost;
      best_tpc = tpc;
    }
  }
  return GradChunks{(tiles_m + best_tpc - 1) / best_tpc, best_tpc};
}

int launch_grad(const uint16_t* X, const float* dXr, int M, int K, int P, int b, float* Gp, cudaStream_t st) {
  rtc::GradParams prm;
  memset(&prm, 0, sizeof(prm));
  if (int rc = make_map_f32_3d(&prm.tmD, dXr, K, M, P, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B)) return rc;
  if (int rc = make_map_bf16(&prm.tmX, X, K, M, K, rtc::TM)) return rc;
  const GradChunks gc = grad_chunks(M, K);
  prm.X = X;
  prm.Gp = Gp;
  prm.M = M;
  prm.K = K;
  prm.P = P;
  prm.b = b;
  prm.nb = K / b;
  prm.groups = (K + 127) / 128;
  prm.chunks = gc.chunks;
  prm.tiles_per_chunk = gc.tiles_per_chunk;
  prm.tiles_m = (M + rtc::TM - 1) / rtc::TM;
  if (int rc = set_smem(rtc::grad_tc_kernel, rtc::kGradSmem)) return rc;
  const int grid = std::min(sm_count(), prm.groups * prm.chunks);
  ProfScope ps(OFT_K_GRAD, st);
  OFT_CUDA(launch_pdl(rtc::grad_tc_kernel, grid, rtc::GR_THREADS, rtc::kGradSmem, st, prm));
  OFT_LAUNCHED("grad_tc_kernel");
  return OFT_OK;
}

// Longest-first static schedule for a plain grouped GEMM whose groups differ in depth (the
// dX' product of sub-projections of different widths): tiles in decreasing depth go to
// the CTA with the least work so far (ties to the lowest index), and each CTA runs its
// tiles in that order.  Round-robin would leave the CTAs that draw an extra deep tile
// with up to a quarter more work than the mean.  The last schedule built on this thread
// is kept, since a training loop repeats the same shapes.
bool build_gemm_schedule(gemm::Params& prm, int grid, int tile_rows) {
  if (prm.use_moe || grid <= 0 || grid > gemm::MAX_SCHED_CTAS) return false;
  std::vector<int> key{grid, tile_rows};
  std::vector<int> depth;  // k-steps per tile, in the order the kernel numbers the tiles
  int kmin = 1 << 30, kmax = 0;
  for (int gi = 0; gi < prm.num_groups; ++gi) {
    const gemm::Group& g = prm.groups[gi];
    if (g.m <= 0 || g.n <= 0) continue;
    const int tiles = ((g.m + tile_rows - 1) / tile_rows) * ((g.n + gemm::BN - 1) / gemm::BN);
    const int nk = (g.k + gemm::BK - 1) / gemm::BK;
    kmin = std::min(kmin, nk);
    kmax = std::max(kmax, nk);
    depth.insert(depth.end(), tiles, nk);
    key.insert(key.end(), {g.m, g.n, g.k});
  }
  if (depth.empty() || kmin == kmax || depth.size() > static_cast<size_t>(gemm::MAX_SCHED_TILES)) return false;
  static thread_local std::vector<int> last_key;
  static thread_local std::vector<uint16_t> last_off, last_tab;
  if (key != last_key) {
    std::vector<int> order(depth.size());
    for (size_t i = 0; i < order.size(); ++i) order[i] = static_cast<int>(i);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return depth[a] > depth[b]; });
    using Slot = std::pair<long long, int>;  // (work so far, CTA)
    std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
    for (int c = 0; c < grid; ++c) heap.push({0, c});
    std::vector<std::vector<uint16_t>> per(grid);
    for (int t : order) {
      Slot s = heap.top();
      heap.pop();
      per[s.second].push_back(static_cast<uint16_t>(t));
      heap.push({s.first + depth[t], s.second});
    }
    last_off.assign(grid + 1, 0);
    last_tab.clear();
    for (int c = 0; c < grid; ++c) {
      last_tab.insert(last_tab.end(), per[c].begin(), per[c].end());
      last_off[c + 1] = static_cast<uint16_t>(last_tab.size());
    }
    last_key = key;
  }
  std::copy(last_off.begin(), last_off.end(), prm.sched_off);
  std::copy(last_tab.begin(), last_tab.end(), prm.sched);
  prm.sched_ctas = grid;
  return true;
}

int launch_gemm(gemm::Params prm, int total_tiles_hint, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    OFT_CUDA(cudaFuncSetAttribute(gemm::gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(gemm::kSmemBytes)));
    attr_set[dev] = true;
  }
  int grid = sm_count();
  if (total_tiles_hint > 0 && total_tiles_hint < grid) grid = total_tiles_hint;
  prm.sched_ctas = 0;
  build_gemm_schedule(prm, grid, gemm::BM);
  ProfScope ps(OFT_K_GEMM, st);
  OFT_CUDA(launch_pdl(gemm::gemm_bf16_kernel, grid, gemm::NUM_THREADS, gemm::kSmemBytes, st, prm));
  OFT_LAUNCHED("gemm_bf16_kernel");
  return OFT_OK;
}

// Work units of the fused-dequant GEMM for one group: weight-row tiles (128 rows for the
// one-CTA kernel, 256 for the 2-SM pair) x token-tile pairs (2 x 192 tokens; 2 x 160 for the pair).
int dq_tiles(int rows, int tokens, int unit_rows = gdq::WM) {
  const int tn = unit_rows == gdq2::UROWS ? gdq2::TN : gdq::TN;
  return ((rows + unit_rows - 1) / unit_rows) * (((tokens + tn - 1) / tn + gdq::TP - 1) / gdq::TP);
}

// 0: choose by size; 1: always the one-CTA kernel; 2: always the 2-SM pair kernel.
int g_gemm_mode = 0;

template <int FMT, bool BWD, bool SCHED>
int launch_gemm_dq_k(const gdq::KParams<SCHED>& kp, int grid, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    OFT_CUDA(cudaFuncSetAttribute(gdq::gemm_dq_kernel<FMT, BWD, SCHED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(gdq::kSmemBytes)));
    attr_set[dev] = true;
  }
  ProfScope ps(OFT_K_GEMM, st);
  OFT_CUDA(launch_pdl(gdq::gemm_dq_kernel<FMT, BWD, SCHED>, grid, gdq::NUM_THREADS, gdq::kSmemBytes, st, kp));
  OFT_LAUNCHED("gemm_dq_kernel");
  return OFT_OK;
}

// Longest-first assignment of the launch's units to `grid` CTAs, each unit to the
// least-loaded CTA (ties: lowest index); a CTA runs its units in ascending order.
// Units are numbered as the kernel numbers them (groups in order, a group's units
// token-pair-major).  Returns false when the launch does not need or fit one.
bool build_schedule(const gdq::Params& prm, int grid, gdq::Sched& s, int unit_rows = gdq::WM) {
  struct Cls {
    int first, count, len;
  };
  std::vector<Cls> cls;
  int u0 = 0;
  bool mixed = false;
  for (int g = 0; g < prm.num_groups; ++g) {
    const gdq::Group& G = prm.groups[g];
    if (G.rows <= 0 || G.tokens <= 0) continue;
    const int n = dq_tiles(G.rows, G.tokens, unit_rows), len = (G.kred + gdq::BK - 1) / gdq::BK;
    if (!cls.empty() && cls.back().len != len) mixed = true;
    cls.push_back({u0, n, len});
    u0 += n;
  }
  if (!mixed || u0 > gdq::kMaxSchedUnits || grid > gdq::kMaxSchedCtas) return false;
  std::stable_sort(cls.begin(), cls.end(), [](const Cls& a, const Cls& b) { return a.len > b.len; });
  using Load = std::pair<long long, int>;  // (k-steps, cta)
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int b = 0; b < grid; ++b) heap.push({0ll, b});
  std::vector<std::vector<int>> per(grid);
  for (const Cls& c : cls)
    for (int k = 0; k < c.count; ++k) {
      Load l = heap.top();
      heap.pop();
      per[l.second].push_back(c.first + k);
      l.first += c.len;
      heap.push(l);
    }
  // keep round-robin (better L2 locality: all CTAs sweep the units together) unless
  // the balanced schedule shortens the longest CTA by more than 5 %
  long long lpt_max = 0;
  while (!heap.empty()) {
    lpt_max = std::max(lpt_max, heap.top().first);
    heap.pop();
  }
  std::vector<int> len_of(u0);
  for (const Cls& c : cls)
    for (int k = 0; k < c.count; ++k) len_of[c.first + k] = c.len;
  long long rr_max = 0;
  for (int b = 0; b < grid; ++b) {
    long long l = 0;
    for (int u = b; u < u0; u += grid) l += len_of[u];
    rr_max = std::max(rr_max, l);
  }
  if (lpt_max * 100 > rr_max * 95) return false;
  int pos = 0;
  for (int b = 0; b < grid; ++b) {
    s.off[b] = static_cast<uint16_t>(pos);
    std::sort(per[b].begin(), per[b].end());
    for (int u : per[b]) s.list[pos++] = static_cast<uint16_t>(u);
  }
  s.off[grid] = static_cast<uint16_t>(pos);
  return true;
}

template <int FMT, bool BWD>
int launch_gemm_dq_t(const gdq::Params& prm, int tiles, cudaStream_t st) {
  const int grid = std::max(1, std::min(sm_count(), tiles));
  if (BWD) {
    static thread_local gdq::KParams<true> kps;  // 25 KB: kept off the stack
    if (build_schedule(prm, grid, kps.s)) {
      kps.p = prm;
      return launch_gemm_dq_k<FMT, BWD, true>(kps, grid, st);
    }
  }
  gdq::KParams<false> kp;
  kp.p = prm;
  return launch_gemm_dq_k<FMT, BWD, false>(kp, grid, st);
}

template <int FMT, bool BWD, bool SCHED>
int launch_gemm_dq2_k(const gdq::KParams<SCHED>& kp, int clusters, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    OFT_CUDA(cudaFuncSetAttribute(gdq2::gemm_dq2_kernel<FMT, BWD, SCHED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(gdq2::kSmemBytes)));
    attr_set[dev] = true;
  }
  ProfScope ps(OFT_K_GEMM, st);
  OFT_CUDA(launch_pdl(gdq2::gemm_dq2_kernel<FMT, BWD, SCHED>, 2 * clusters, gdq2::NUM_THREADS, gdq2::kSmemBytes, st, kp));
  OFT_LAUNCHED("gemm_dq2_kernel");
  return OFT_OK;
}

// Number of 2-CTA clusters of the pair kernel that fit on the device at once (cached).
int pair_clusters_resident() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  cudaFuncSetAttribute(gdq2::gemm_dq2_kernel<gdq::kInt4, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(gdq2::kSmemBytes));
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(2 * sm_count());
  cfg.blockDim = dim3(gdq2::NUM_THREADS);
  cfg.dynamicSmemBytes = gdq2::kSmemBytes;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  if (cudaOccupancyMaxActiveClusters(&n, gdq2::gemm_dq2_kernel<gdq::kInt4, false, false>, &cfg) != cudaSuccess || n <= 0)
    n = sm_count() / 2;
  cudaGetLastError();
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

template <int FMT, bool BWD>
int launch_gemm_dq2_t(const gdq::Params& prm, int units, cudaStream_t st) {
  const int clusters = std::max(1, std::min(pair_clusters_resident(), units));
  if (BWD) {
    static thread_local gdq::KParams<true> kps;
    if (build_schedule(prm, clusters, kps.s, gdq2::UROWS)) {
      kps.p = prm;
      return launch_gemm_dq2_k<FMT, BWD, true>(kps, clusters, st);
    }
  }
  gdq::KParams<false> kp;
  kp.p = prm;
  return launch_gemm_dq2_k<FMT, BWD, false>(kp, clusters, st);
}

// The plain GEMM on 2-SM pairs: one persistent cluster per resident pair (the same
// one-CTA-per-SM footprint as the fused pair kernel), schedule in units of pair tiles.
int launch_gemm_pair(gemm::Params prm, int pair_tiles, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    OFT_CUDA(cudaFuncSetAttribute(gemm::gemm_bf16_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(gemm::kPairSmemBytes)));
    attr_set[dev] = true;
  }
  const int clusters = std::max(1, std::min(pair_clusters_resident(), pair_tiles));
  prm.sched_ctas = 0;
  build_gemm_schedule(prm, clusters, gemm::PM);
  ProfScope ps(OFT_K_GEMM, st);
  OFT_CUDA(launch_pdl(gemm::gemm_bf16_pair_kernel, 2 * clusters, gemm::NUM_THREADS, gemm::kPairSmemBytes, st, prm));
  OFT_LAUNCHED("gemm_bf16_pair_kernel");
  return OFT_OK;
}

// The dense path's plain GEMM: the pair kernel, or the one-CTA kernel in gemm mode 4.
// B tensor maps must have boxes of plain_b_rows() rows.
bool plain_pair() { return g_gemm_mode != 4; }
uint32_t plain_b_rows() { return plain_pair() ? 128u : static_cast<uint32_t>(gemm::BN); }
int launch_plain_gemm(const gemm::Params& prm, cudaStream_t st) {
  const int bm = plain_pair() ? gemm::PM : gemm::BM;
  int tiles = 0;
  for (int g = 0; g < prm.num_groups; ++g) {
    const gemm::Group& G = prm.groups[g];
    if (G.m > 0 && G.n > 0) tiles += ((G.m + bm - 1) / bm) * ((G.n + gemm::BN - 1) / gemm::BN);
  }
  return plain_pair() ? launch_gemm_pair(prm, tiles, st) : launch_gemm(prm, tiles, st);
}

// Pair kernel for launches of at least two one-CTA waves (unless forced).
bool use_pair(int tiles_one_cta) {
  if (g_gemm_mode == 1) return false;
  if (g_gemm_mode == 2) return true;
  return tiles_one_cta >= 2 * sm_count();
}

int launch_gemm_dq2(int fmt, bool bwd, const gdq::Params& prm, int units, cudaStream_t st) {
  if (fmt == OFT_W_INT4) return bwd ? launch_gemm_dq2_t<gdq::kInt4, true>(prm, units, st)
                                    : launch_gemm_dq2_t<gdq::kInt4, false>(prm, units, st);
  if (fmt == OFT_W_FP8) return bwd ? launch_gemm_dq2_t<gdq::kFp8, true>(prm, units, st)
                                   : launch_gemm_dq2_t<gdq::kFp8, false>(prm, units, st);
  return bwd ? launch_gemm_dq2_t<gdq::kMxfp4, true>(prm, units, st) : launch_gemm_dq2_t<gdq::kMxfp4, false>(prm, units, st);
}

int launch_gemm_dq(int fmt, bool bwd, const gdq::Params& prm, int tiles, cudaStream_t st) {
  if (fmt == OFT_W_INT4) return bwd ? launch_gemm_dq_t<gdq::kInt4, true>(prm, tiles, st)
                                    : launch_gemm_dq_t<gdq::kInt4, false>(prm, tiles, st);
  if (fmt == OFT_W_FP8) return bwd ? launch_gemm_dq_t<gdq::kFp8, true>(prm, tiles, st)
                                   : launch_gemm_dq_t<gdq::kFp8, false>(prm, tiles, st);
  return bwd ? launch_gemm_dq_t<gdq::kMxfp4, true>(prm, tiles, st) : launch_gemm_dq_t<gdq::kMxfp4, false>(prm, tiles, st);
}



// Large token counts take the weight through a bf16 copy and a plain tcgen05 GEMM
// (gemm.cuh); the dequant pass is cheap next to the product there, and the plain
// kernel runs closer to the tensor peak than the fused-decode kernels, which stay
// for small token counts where streaming the low-precision codes matters.
constexpr int kPlainMinTokens = 2048;
bool use_plain(int M) {
  if (g_gemm_mode == 3 || g_gemm_mode == 4) return true;
  if (g_gemm_mode == 1 || g_gemm_mode == 2) return false;
  return M >= kPlainMinTokens;
}

// The small-M path (few tokens against the whole weight, gsm::gemm_sm_kernel): forwards
// of 1 to 128 tokens in gemm mode 0.  Its e8m0 scale rows must be 16-byte strided.
constexpr int kSmallMaxTokens = gsm::MAX_TOKENS;
bool use_small(int M, int fmt, int N) {
  if (g_gemm_mode != 0) return false;
  if (M < 1 || M > kSmallMaxTokens) return false;
  return fmt != OFT_W_MXFP4 || N % 16 == 0;
}

// Split-K plan of the small-M kernel: 128-row weight tiles x `splits` reduction ranges,
// with the split count that minimises waves / splits over the SMs (ties to fewer splits).
struct SmallPlan {
  int tiles, splits, nkb, MN;
  size_t part_bytes, cnt_bytes;
};
SmallPlan small_plan(int M, int K, int fmt, const oft_split* S) {
  SmallPlan pl{};
  pl.MN = (M + 15) / 16 * 16;
  const int kbe = fmt == OFT_W_FP8 ? 128 : 256;
  pl.nkb = (K + kbe - 1) / kbe;
  for (int p = 0; p < S->n; ++p) pl.tiles += (S->sizes[p] + gsm::WM - 1) / gsm::WM;
  const int sms = sm_count();
  double best = 1e30;
  pl.splits = 1;
  for (int sp = 1; sp <= std::min(gsm::MAX_SPLITS, pl.nkb); ++sp) {
    const double waves = static_cast<double>((1ll * pl.tiles * sp + sms - 1) / sms) / sp;
    if (waves < best - 1e-9) {
      best = waves;
      pl.splits = sp;
    }
  }
  pl.cnt_bytes = pl.splits > 1 ? round_up(4ull * pl.tiles, 256) : 0;
  pl.part_bytes = pl.splits > 1 ? 4ull * pl.tiles * pl.splits * pl.MN * gsm::WM : 0;
  return pl;
}

struct FwdLayout {
  size_t xr, wdq, cnt, part, total;
};
// plain: the bf16 weight copy follows X'; small_extra: the small-M kernel's split-K
// counters and partial tiles follow X' instead
FwdLayout fwd_layout(int M, int K, int N, int P, bool plain, size_t cnt_bytes = 0, size_t part_bytes = 0) {
  FwdLayout L{};
  L.xr = 0;
  L.wdq = round_up(L.xr + 2ull * P * M * K, 256);
  L.cnt = L.wdq;
  L.part = round_up(L.cnt + cnt_bytes, 256);
  L.total = plain ? round_up(L.wdq + 2ull * N * K, 256) : round_up(L.part + part_bytes, 256);
  return L;
}
// The layout oft_linear_fwd uses when the plain (bf16 weight copy) path is not taken.
FwdLayout fwd_layout_fused(int M, const oft_weight* W, const oft_split* S) {
  if (use_small(M, W->fmt, W->d_out)) {
    const SmallPlan pl = small_plan(M, W->d_in, W->fmt, S);
    return fwd_layout(M, W->d_in, W->d_out, S->n, false, pl.cnt_bytes, pl.part_bytes);
  }
  return fwd_layout(M, W->d_in, W->d_out, S->n, false);
}


struct BwdLayout {
  size_t dxr, codes_t, gpart, factors, total;
  int nparts;
};
// Bytes of the backward's packed code blocks: per sub-projection, ceil(K/128) row
// tiles x ceil(N_p/64) k-steps of 128 x 64 codes.
size_t packed_bwd_code_bytes(int fmt, int K, const oft_split* S) {
  size_t blocks = 0;
  for (int p = 0; p < S->n; ++p) blocks += 1ull * ((K + 127) / 128) * ((S->sizes[p] + 63) / 64);
  return blocks * (fmt == OFT_W_FP8 ? 8192ull : 4096ull);
}

BwdLayout bwd_layout(int M, int K, int N, const oft_split* S, int b, int fmt, bool plain) {
  BwdLayout L{};
  const int P = S->n;
  L.nparts = grad_chunks(M, K).chunks;
  L.dxr = 0;
  L.codes_t = round_up(L.dxr + 4ull * P * M * K, 256);  // dX' kept in fp32
  // packed code blocks for the fused-decode kernels, or deq(W) as bf16 [K][N] for the plain GEMM
  L.gpart = round_up(L.codes_t + (plain ? 2ull * K * N : packed_bwd_code_bytes(fmt, K, S)), 256);
  L.factors = round_up(L.gpart + 4ull * P * (K / b) * L.nparts * b * b, 256);
  // MXFP4: one bf16 factor per e8m0 scale
  const size_t sbytes = fmt == OFT_W_MXFP4 ? 2ull * (K / 32) * N : 0ull;
  L.total = round_up(L.factors + sbytes, 256);
  return L;
}

// Tensor maps and launch of the small-M kernel (one CTA per SM, persistent over the
// tiles x splits units).
template <int FMT>
int launch_gemm_small_t(const gsm::Params& prm, int grid, size_t smem, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    OFT_CUDA(cudaFuncSetAttribute(gsm::gemm_sm_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(227 * 1024)));
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  ProfScope ps(OFT_K_GEMM, st);
  OFT_CUDA(launch_pdl(gsm::gemm_sm_kernel<FMT>, grid, gsm::NUM_THREADS, smem, st, prm));
  OFT_LAUNCHED("gemm_sm_kernel");
  return OFT_OK;
}

// The launch parameters of the last few small-M calls on this host thread, keyed by
// everything they are built from: a decode loop calls the same layers again and again,
// and encoding three tensor maps per call would dominate these short kernels' launch.
struct SmallKey {
  const void *codes, *scales, *xr, *y, *part, *counters;
  int dev, M, K, N, fmt, group, splits, sizes[4], n;
  bool operator==(const SmallKey& o) const { return memcmp(this, &o, sizeof(*this)) == 0; }
};
struct SmallEntry {
  SmallKey key;
  gsm::Params prm;
  int grid;
  size_t smem;
  bool valid = false;
};

int launch_gemm_small(const oft_weight* W, const oft_split* S, int M, const uint16_t* Xr, uint16_t* Y,
                      const SmallPlan& pl, int* counters, float* part, cudaStream_t st) {
  const int K = W->d_in, N = W->d_out, P = S->n;
  SmallKey key;
  memset(&key, 0, sizeof(key));
  key.codes = W->codes;
  key.scales = W->scales;
  key.xr = Xr;
  key.y = Y;
  key.part = part;
  key.counters = counters;
  cudaGetDevice(&key.dev);
  key.M = M;
  key.K = K;
  key.N = N;
  key.fmt = W->fmt;
  key.group = W->group;
  key.splits = pl.splits;
  key.n = P;
  for (int i = 0; i < P; ++i) key.sizes[i] = S->sizes[i];
  constexpr int kCache = 8;
  static thread_local std::unique_ptr<SmallEntry[]> cache(new SmallEntry[kCache]);
  static thread_local int next_slot = 0;
  for (int i = 0; i < kCache; ++i) {
    const SmallEntry& e = cache[i];
    if (e.valid && e.key == key) {
      if (W->fmt == OFT_W_INT4) return launch_gemm_small_t<gsm::kInt4>(e.prm, e.grid, e.smem, st);
      if (W->fmt == OFT_W_FP8) return launch_gemm_small_t<gsm::kFp8>(e.prm, e.grid, e.smem, st);
      return launch_gemm_small_t<gsm::kMxfp4>(e.prm, e.grid, e.smem, st);
    }
  }
  SmallEntry& ent = cache[next_slot];
  next_slot = (next_slot + 1) % kCache;
  ent.valid = false;
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(OFT_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  gsm::Params* prm = &ent.prm;
  memset(prm, 0, sizeof(*prm));
  {
    // codes: [N][row bytes] uint8, 128 x 128-byte boxes with the 128-byte swizzle
    const uint64_t row_bytes = W->fmt == OFT_W_FP8 ? 1ull * K : 1ull * K / 2;
    cuuint64_t dims[2] = {row_bytes, static_cast<cuuint64_t>(N)};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {128, gsm::WM};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&prm->tmC, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(W->codes), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(OFT_ERR_CUDA, "cuTensorMapEncodeTiled (codes) failed (%d)", int(r));
  }
  if (W->fmt == OFT_W_INT4) {
    if (int rc = make_map_plain_2d(&prm->tmS, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W->scales, N, K / W->group, 2ull * N,
                                   gsm::WM, 256 / W->group))
      return rc;
  } else if (W->fmt == OFT_W_MXFP4) {
    // e8m0 rows: the box starts at the 16-byte boundary at or below the tile's first column
    if (int rc = make_map_plain_2d(&prm->tmS, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->scales, N, K / 32, 1ull * N, 144, 8))
      return rc;
  }
  if (int rc = make_map_bf16(&prm->tmX, Xr, K, 1ull * P * M, K, pl.MN)) return rc;
  prm->fp8_scales = W->fmt == OFT_W_FP8 ? static_cast<const float*>(W->scales) : nullptr;
  prm->Y = Y;
  prm->part = part;
  prm->counters = counters;
  prm->M = M;
  prm->MN = pl.MN;
  prm->K = K;
  prm->N = N;
  prm->group = W->fmt == OFT_W_INT4 ? W->group : 32;
  prm->splits = pl.splits;
  prm->nkb = pl.nkb;
  prm->total_tiles = pl.tiles;
  prm->units = pl.tiles * pl.splits;
  const size_t base = gsm::smem_bytes(pl.MN, 0);
  prm->sx = static_cast<int>(std::min<size_t>(gsm::MAX_SX, (227ull * 1024 - base) / gsm::x_stage_bytes(pl.MN)));
  prm->num_groups = P;
  int off = 0, tile0 = 0;
  for (int p = 0; p < P; ++p) {
    gsm::Group& g = prm->groups[p];
    g.rows = S->sizes[p];
    g.w_row0 = off;
    g.b_row0 = p * M;
    g.tiles = (S->sizes[p] + gsm::WM - 1) / gsm::WM;
    g.tile0 = tile0;
    tile0 += g.tiles;
    off += S->sizes[p];
  }
  const size_t smem = gsm::smem_bytes(pl.MN, prm->sx);
  const int grid = std::min(prm->units, sm_count());
  ent.key = key;
  ent.grid = grid;
  ent.smem = smem;
  ent.valid = true;
  if (W->fmt == OFT_W_INT4) return launch_gemm_small_t<gsm::kInt4>(*prm, grid, smem, st);
  if (W->fmt == OFT_W_FP8) return launch_gemm_small_t<gsm::kFp8>(*prm, grid, smem, st);
  return launch_gemm_small_t<gsm::kMxfp4>(*prm, grid, smem, st);
}

}  // namespace

extern "C" {

const char* oft_version(void) { return "oft-b200 0.1 (sm_100a, tcgen05)"; }

const char* oft_last_error(void) { return g_last_error.c_str(); }

int oft_set_gemm_mode(int mode) {
  if (mode < 0 || mode > 4) return fail(OFT_ERR_INVALID_ARG, "gemm mode must be 0..4");
  g_gemm_mode = mode;
  return OFT_OK;
}

int oft_gemm_schedule(int n_groups, const int* m, const int* n, const int* k, int tile_rows, int grid, int* used,
                      int* off, int* tiles) {
  if (!m || !n || !k || !used || !off || !tiles) return fail(OFT_ERR_INVALID_ARG, "NULL pointer");
  if (n_groups < 1 || n_groups > gemm::MAX_GROUPS) return fail(OFT_ERR_INVALID_ARG, "n_groups must be 1..32");
  if (tile_rows != gemm::BM && tile_rows != gemm::PM) return fail(OFT_ERR_INVALID_ARG, "tile_rows must be 128 or 256");
  if (grid < 1) return fail(OFT_ERR_INVALID_ARG, "grid < 1");
  gemm::Params* prm = new gemm::Params;
  memset(prm, 0, sizeof(*prm));
  prm->num_groups = n_groups;
  for (int g = 0; g < n_groups; ++g) {
    prm->groups[g].m = m[g];
    prm->groups[g].n = n[g];
    prm->groups[g].k = k[g];
  }
  *used = build_gemm_schedule(*prm, grid, tile_rows) ? 1 : 0;
  if (*used) {
    for (int c = 0; c <= grid; ++c) off[c] = prm->sched_off[c];
    for (int i = 0; i < off[grid]; ++i) tiles[i] = prm->sched[i];
  }
  delete prm;
  return OFT_OK;
}

int oft_check_device(void* stream) {
  OFT_CUDA(cudaStreamSynchronize(as_stream(stream)));
  unsigned int word = 0, zero = 0;
  OFT_CUDA(cudaMemcpyFromSymbol(&word, g_dev_err, sizeof(word)));
  if (word != 0) {
    OFT_CUDA(cudaMemcpyToSymbol(g_dev_err, &zero, sizeof(zero)));
    return fail(OFT_ERR_TIMEOUT, "a bounded device wait ran out (error bits 0x%x)", word);
  }
  return OFT_OK;
}

int oft_build_rotation(const uint16_t* Q, int n_blocks, int b, float* R, void* stream) {
  if (n_blocks < 0) return fail(OFT_ERR_INVALID_ARG, "n_blocks < 0");
  if (n_blocks == 0) return OFT_OK;
  if (Q == nullptr || R == nullptr) return fail(OFT_ERR_INVALID_ARG, "Q/R NULL");
  if (!aligned16(Q) || !aligned16(R)) return fail(OFT_ERR_INVALID_ARG, "Q/R must be 16-byte aligned");
  if (int rc = check_b(b, b)) return rc;
  return launch_cayley(Q, n_blocks, b, R, nullptr, nullptr, 1, as_stream(stream));
}

int oft_cayley_backward(const float* R, const float* G, int n_blocks, int b, float* dQ, void* stream) {
  if (n_blocks < 0) return fail(OFT_ERR_INVALID_ARG, "n_blocks < 0");
  if (n_blocks == 0) return OFT_OK;
  if (!R || !G || !dQ) return fail(OFT_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(R) || !aligned16(G) || !aligned16(dQ)) return fail(OFT_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (int rc = check_b(b, b)) return rc;
  return launch_cayley_bwd(R, G, 1, n_blocks, b, dQ, as_stream(stream));
}

int oft_dequant_weight(const oft_weight* W, uint16_t* out, int transpose, void* stream) {
  if (int rc = check_weight(W, false)) return rc;
  if (out == nullptr || !aligned16(out)) return fail(OFT_ERR_INVALID_ARG, "out NULL or misaligned");
  return launch_dequant(view_of(W), out, transpose != 0, as_stream(stream));
}

int oft_rotate(const uint16_t* X, int M, int K, int P, int b, const float* R, uint16_t* Xr, void* stream) {
  if (M < 0 || K <= 0 || P < 1) return fail(OFT_ERR_INVALID_ARG, "bad sizes");
  if (P > 4) return fail(OFT_ERR_UNSUPPORTED, "1..4 sub-projections supported (got %d)", P);
  if (M == 0) return OFT_OK;
  if (!X || !R || !Xr || !aligned16(X) || !aligned16(R) || !aligned16(Xr))
    return fail(OFT_ERR_INVALID_ARG, "NULL or misaligned pointer");
  if (int rc = check_b(b, K)) return rc;
  if (K % 32 != 0) return fail(OFT_ERR_UNSUPPORTED, "K must be a multiple of 32");
  return launch_rotate_fwd(X, M, K, P, b, R, Xr, as_stream(stream));
}

size_t oft_linear_fwd_weight_side_workspace(const oft_weight* W) {
  if (W == nullptr || W->d_in <= 0 || W->d_out <= 0) return 0;
  return round_up(2ull * W->d_out * W->d_in, 256) + round_up(2ull * W->d_out * W->d_in, 256);
}

// Weight-side forward: V_p^T = deq(W_p)^T R_p^T (rows of split p), then Y = X V in one
// plain tcgen05 GEMM over all N columns.
int oft_linear_fwd_weight_side(const uint16_t* X, int M, const oft_weight* W, const oft_split* S, int b,
                               const float* R, uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_weight(W, false)) return rc;
  if (int rc = check_split(S, W->d_out)) return rc;
  const int K = W->d_in, N = W->d_out, P = S->n, nb = K / (b > 0 ? b : 1);
  if (int rc = check_b(b, K)) return rc;
  if (K % 32 != 0) return fail(OFT_ERR_UNSUPPORTED, "K must be a multiple of 32");
  if (M < 0) return fail(OFT_ERR_INVALID_ARG, "M < 0");
  if (M == 0) return OFT_OK;
  if (!X || !R || !Y || !ws) return fail(OFT_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(X) || !aligned16(R) || !aligned16(Y) || !aligned16(ws))
    return fail(OFT_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t need = oft_linear_fwd_weight_side_workspace(W);
  if (ws_bytes < need) return fail(OFT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  cudaStream_t st = as_stream(stream);
  uint16_t* Wd = static_cast<uint16_t*>(ws);
  uint16_t* V = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + round_up(2ull * N * K, 256));
  if (int rc = launch_dequant(view_of(W), Wd, false, st)) return rc;
  int off = 0;
  for (int p = 0; p < P; ++p) {
    if (int rc = launch_rotate_fwd(Wd + 1ull * off * K, S->sizes[p], K, 1, b, R + 1ull * p * nb * b * b,
                                   V + 1ull * off * K, st, true))
      return rc;
    off += S->sizes[p];
  }
  gemm::Params prm;
  memset(&prm, 0, sizeof(prm));
  if (int rc = make_map_bf16(&prm.tmA[0], X, K, M, K, gemm::BM)) return rc;
  if (int rc = make_map_bf16(&prm.tmB[0], V, K, N, K, plain_b_rows())) return rc;
  prm.C = Y;
  prm.ldc = N;
  prm.c_f32 = 0;
  prm.num_groups = 1;
  gemm::Group& g = prm.groups[0];
  g.m = M;
  g.n = N;
  g.k = K;
  return launch_plain_gemm(prm, st);
}

size_t oft_linear_fwd_workspace(int M, const oft_weight* W, const oft_split* S, int b) {
  if (W == nullptr || S == nullptr || M <= 0 || S->n < 1 || S->n > 4) return 0;
  (void)b;
  return use_plain(M) ? fwd_layout(M, W->d_in, W->d_out, S->n, true).total : fwd_layout_fused(M, W, S).total;
}

int oft_linear_fwd(const uint16_t* X, int M, const oft_weight* W, const oft_split* S, int b, const float* R,
                   uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_weight(W, false)) return rc;
  if (int rc = check_split(S, W->d_out)) return rc;
  const int K = W->d_in, N = W->d_out, P = S->n;
  if (int rc = check_b(b, K)) return rc;
  if (M < 0) return fail(OFT_ERR_INVALID_ARG, "M < 0");
  if (M == 0) return OFT_OK;
  if (!X || !R || !Y || !ws) return fail(OFT_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(X) || !aligned16(R) || !aligned16(Y) || !aligned16(ws))
    return fail(OFT_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  // the plain path when the token count calls for it and the workspace holds the bf16 weight
  const bool plain = use_plain(M) && ws_bytes >= fwd_layout(M, K, N, P, true).total;
  const bool small = !plain && use_small(M, W->fmt, N);
  const FwdLayout L = plain ? fwd_layout(M, K, N, P, true) : fwd_layout_fused(M, W, S);
  if (ws_bytes < L.total) return fail(OFT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint16_t* Xr = reinterpret_cast<uint16_t*>(wsb + L.xr);

  if (small) {
    // few tokens: the weight stream bounds the product (gsm::gemm_sm_kernel); the
    // rotation kernel also clears the split-K counters of the tiles
    const SmallPlan pl = small_plan(M, K, W->fmt, S);
    int* counters = reinterpret_cast<int*>(wsb + L.cnt);
    if (int rc = launch_rotate_fwd(X, M, K, P, b, R, Xr, st, false, pl.splits > 1 ? counters : nullptr, pl.tiles))
      return rc;
    return launch_gemm_small(W, S, M, Xr, Y, pl, counters, reinterpret_cast<float*>(wsb + L.part), st);
  }

  SidePipe* sp = nullptr;
  std::unique_lock<std::mutex> sp_lock;
  if (plain) {
    // deq(W) -> bf16 [N][K] on the side stream, alongside the rotation on this one: the two
    // read only inputs and write disjoint workspace regions, and the small dequant CTAs fit
    // next to the rotation's on the same SMs
    if (int rc = side_pipe(&sp, &sp_lock)) return rc;
    OFT_CUDA(cudaEventRecord(sp->start, st));
    OFT_CUDA(cudaStreamWaitEvent(sp->side, sp->start, 0));
    if (int rc = launch_dequant(view_of(W), reinterpret_cast<uint16_t*>(wsb + L.wdq), false, sp->side)) return rc;
    OFT_CUDA(cudaEventRecord(sp->dq_done[0], sp->side));
  }
  if (int rc = launch_rotate_fwd(X, M, K, P, b, R, Xr, st)) return rc;

  if (plain) {
    // Y[:, cols of p] = X'_p deq(W_p)^T-rows: one plain grouped GEMM over bf16 deq(W) [N][K]
    uint16_t* Wdq = reinterpret_cast<uint16_t*>(wsb + L.wdq);
    OFT_CUDA(cudaStreamWaitEvent(st, sp->dq_done[0], 0));
    gemm::Params prm;
    memset(&prm, 0, sizeof(prm));
    if (int rc = make_map_bf16(&prm.tmA[0], Xr, K, 1ull * P * M, K, gemm::BM)) return rc;
    if (int rc = make_map_bf16(&prm.tmB[0], Wdq, K, N, K, plain_b_rows())) return rc;
    prm.C = Y;
    prm.ldc = N;
    prm.c_f32 = 0;
    prm.num_groups = P;
    int off = 0;
    for (int p = 0; p < P; ++p) {
      gemm::Group& g = prm.groups[p];
      g.m = M;
      g.n = S->sizes[p];
      g.k = K;
      g.a_row0 = p * M;
      g.b_row0 = off;
      g.c_col0 = off;
      off += S->sizes[p];
    }
    return launch_plain_gemm(prm, st);
  }

  // Y[:, cols of p] = X'_p deq(W_p): dequant fused into the GEMM's weight operand
  int tiles1 = 0, units2 = 0;
  for (int p = 0; p < P; ++p) {
    tiles1 += dq_tiles(S->sizes[p], M);
    units2 += dq_tiles(S->sizes[p], M, gdq2::UROWS);
  }
  const bool pair = use_pair(tiles1);
  gdq::Params prm;
  memset(&prm, 0, sizeof(prm));
  if (int rc = make_map_bf16(&prm.tmB[0], Xr, K, 1ull * P * M, K, pair ? gdq2::TNC : gdq::TN)) return rc;
  for (int i = 1; i < gdq::MAX_GROUPS; ++i) prm.tmB[i] = prm.tmB[0];
  prm.codes = static_cast<const uint8_t*>(W->codes);
  prm.code_row_bytes = W->fmt == OFT_W_FP8 ? K : K / 2;
  prm.scales = W->scales;
  prm.N = N;
  prm.K = K;
  prm.group = W->fmt == OFT_W_INT4 ? W->group : 32;
  prm.num_groups = P;
  int off = 0;
  for (int p = 0; p < P; ++p) {
    gdq::Group& g = prm.groups[p];
    g.rows = S->sizes[p];
    g.tokens = M;
    g.kred = K;
    g.b_map = 0;
    g.b_row0 = p * M;
    g.w_row0 = off;
    g.w_k0 = 0;
    g.y_map = p;
    // Y[:, off : off + N_p] as its own tensor, so stores clip at the sub-projection's edge
    if (int rc = make_map_plain_2d(&prm.tmY[p], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y + off, S->sizes[p], M, 2ull * N,
                                   32, 32))
      return rc;
    off += S->sizes[p];
  }
  return pair ? launch_gemm_dq2(W->fmt, false, prm, units2, st) : launch_gemm_dq(W->fmt, false, prm, tiles1, st);
}

size_t oft_linear_bwd_workspace(int M, const oft_weight* W, const oft_split* S, int b) {
  if (W == nullptr || S == nullptr || M <= 0 || b <= 0) return 0;
  return bwd_layout(M, W->d_in, W->d_out, S, b, W->fmt, use_plain(M)).total;
}

int oft_linear_bwd(const uint16_t* dY, const uint16_t* X, int M, const oft_weight* W, const oft_split* S, int b,
                   const float* R, uint16_t* dX, float* dQ, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_weight(W, false)) return rc;
  if (int rc = check_split(S, W->d_out)) return rc;
  const int K = W->d_in, N = W->d_out, P = S->n, nb = K / (b > 0 ? b : 1);
  if (int rc = check_b(b, K)) return rc;
  if (M < 0) return fail(OFT_ERR_INVALID_ARG, "M < 0");
  if (!dQ || !R) return fail(OFT_ERR_INVALID_ARG, "NULL pointer");
  cudaStream_t st = as_stream(stream);
  if (M == 0) {  // no tokens: dX is empty and dQ is zero
    OFT_CUDA(cudaMemsetAsync(dQ, 0, sizeof(float) * P * nb * (b * (b - 1) / 2), st));
    return OFT_OK;
  }
  if (!dY || !X || !dX || !ws) return fail(OFT_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(dY) || !aligned16(X) || !aligned16(R) || !aligned16(dX) || !aligned16(dQ) || !aligned16(ws))
    return fail(OFT_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const bool plain = use_plain(M) && ws_bytes >= bwd_layout(M, K, N, S, b, W->fmt, true).total;
  const BwdLayout L = bwd_layout(M, K, N, S, b, W->fmt, plain);
  if (ws_bytes < L.total) return fail(OFT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* dXr = reinterpret_cast<float*>(wsb + L.dxr);
  uint8_t* codes_t = wsb + L.codes_t;
  float* Gp = reinterpret_cast<float*>(wsb + L.gpart);

  if (plain) {
    // dX'_p = dY_p deq(W_p): one plain grouped GEMM against bf16 deq(W) laid out [K][N]
    uint16_t* WdqT = reinterpret_cast<uint16_t*>(codes_t);
    if (int rc = launch_dequant(view_of(W), WdqT, true, st)) return rc;
    gemm::Params prm;
    memset(&prm, 0, sizeof(prm));
    int off = 0;
    for (int p = 0; p < P; ++p) {
      const int Np = S->sizes[p];
      if (int rc = make_map_bf16(&prm.tmA[p], dY + off, Np, M, N, gemm::BM)) return rc;
      if (int rc = make_map_bf16(&prm.tmB[p], WdqT + off, Np, K, N, plain_b_rows())) return rc;
      gemm::Group& g = prm.groups[p];
      g.m = M;
      g.n = K;
      g.k = Np;
      g.a_map = p;
      g.b_map = p;
      g.c_row0 = p * M;
      off += Np;
    }
    prm.C = dXr;
    prm.ldc = K;
    prm.c_f32 = 1;
    prm.num_groups = P;
    if (int rc = launch_plain_gemm(prm, st)) return rc;
    if (int rc = launch_rotate_bwd(dXr, M, K, P, b, R, dX, st)) return rc;
    if (int rc = launch_grad(X, dXr, M, K, P, b, Gp, st)) return rc;
    if (int rc = launch_cayley_bwd(R, Gp, L.nparts, P * nb, b, dQ, st)) return rc;
    return OFT_OK;
  }

  // codes re-laid out per (sub-projection, 128 input features, 64 channels) block for
  // the dequant producers: one row per input feature, coalesced across a warp
  long long code_off[gdq::MAX_GROUPS] = {0};
  {
    PackBwdParams pp;
    memset(&pp, 0, sizeof(pp));
    pp.num_groups = P;
    int blk = 0, n0 = 0;
    long long off = 0;
    const long long blk_bytes = W->fmt == OFT_W_FP8 ? 8192 : 4096;
    for (int p = 0; p < P; ++p) {
      pp.blk0[p] = blk;
      pp.n0[p] = n0;
      pp.np[p] = S->sizes[p];
      pp.nk[p] = (S->sizes[p] + 63) / 64;
      pp.off[p] = off;
      code_off[p] = off;
      const int nblk = ((K + 127) / 128) * pp.nk[p];
      blk += nblk;
      off += nblk * blk_bytes;
      n0 += S->sizes[p];
    }
    pp.blk0[P] = blk;
    ProfScope ps(OFT_K_DEQUANT, st);
    if (W->fmt == OFT_W_FP8)
      OFT_CUDA(launch_pdl(pack_codes_bwd_kernel<false>, blk, 256, 0, st, static_cast<const uint8_t*>(W->codes), N, K, pp, codes_t));
    else
      OFT_CUDA(launch_pdl(pack_codes_bwd_kernel<true>, blk, 256, 0, st, static_cast<const uint8_t*>(W->codes), N, K, pp, codes_t));
    OFT_LAUNCHED("pack_codes_bwd_kernel");
  }

  // dX'_p = dY_p deq(W_p)^T, dequant fused into the GEMM's weight operand, fp32 out
  gdq::Params prm;
  memset(&prm, 0, sizeof(prm));
  const int G = W->fmt == OFT_W_INT4 ? W->group : 32;
  if (W->fmt == OFT_W_INT4) {
    if (int rc = make_map_plain_2d(&prm.tmS, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W->scales, N, K / G, 2ull * N, 64,
                                   gdq::WM / G))
      return rc;
  } else if (W->fmt == OFT_W_MXFP4) {
    uint16_t* fac = reinterpret_cast<uint16_t*>(wsb + L.factors);
    const long long n = 1ll * (K / 32) * N;
    {
      ProfScope ps(OFT_K_DEQUANT, st);
      OFT_CUDA(launch_pdl(e8m0_factor_kernel, static_cast<unsigned>((n + 255) / 256), 256, 0, st,
                          static_cast<const uint8_t*>(W->scales), n, fac));
      OFT_LAUNCHED("e8m0_factor_kernel");
    }
    if (int rc = make_map_plain_2d(&prm.tmS, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, fac, N, K / 32, 2ull * N, 64,
                                   gdq::WM / 32))
      return rc;
  } else {
    // fp32 channel scales, one row
    if (int rc = make_map_plain_2d(&prm.tmS, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, W->scales, N, 1, 4ull * N, 64, 1))
      return rc;
  }
  const int tiles1 = P * dq_tiles(K, M), units2 = P * dq_tiles(K, M, gdq2::UROWS);
  const bool pair = use_pair(tiles1);
  int off = 0;
  for (int p = 0; p < P; ++p) {
    const int Np = S->sizes[p];
    if (int rc = make_map_bf16(&prm.tmB[p], dY + off, Np, M, N, pair ? gdq2::TNC : gdq::TN)) return rc;
    gdq::Group& g = prm.groups[p];
    g.rows = K;
    g.tokens = M;
    g.kred = Np;
    g.b_map = p;
    g.b_row0 = 0;
    g.w_row0 = 0;
    g.w_k0 = off;
    g.y_map = p;
    g.code_off = code_off[p];
    if (int rc = make_map_plain_2d(&prm.tmY[p], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, dXr + 1ull * p * M * K, K, M,
                                   4ull * K, 32, 32))
      return rc;
    off += Np;
  }
  for (int p = P; p < gdq::MAX_GROUPS; ++p) prm.tmB[p] = prm.tmB[0];
  prm.codes = codes_t;
  prm.code_row_bytes = 0;
  prm.scales = W->scales;
  prm.N = N;
  prm.K = K;
  prm.group = G;
  prm.num_groups = P;
  if (int rc = pair ? launch_gemm_dq2(W->fmt, true, prm, units2, st) : launch_gemm_dq(W->fmt, true, prm, tiles1, st))
    return rc;

  if (int rc = launch_rotate_bwd(dXr, M, K, P, b, R, dX, st)) return rc;
  if (int rc = launch_grad(X, dXr, M, K, P, b, Gp, st)) return rc;

  if (int rc = launch_cayley_bwd(R, Gp, L.nparts, P * nb, b, dQ, st)) return rc;
  return OFT_OK;
}

// ---------------------------------------------------------------------------
// MoE
// ---------------------------------------------------------------------------
namespace {
struct MoeLayout {
  size_t rex, xg, buf, ytk, inv, pexp, groups, meta, total;
};
// fused: no chunk buffers; a device-built group list instead
MoeLayout moe_layout(int T, int E, int top_k, int chunk, int K, int N, int b, bool fused = false) {
  MoeLayout L{};
  const size_t TK = 1ull * T * top_k;
  L.rex = 0;
  L.xg = round_up(L.rex + 4ull * E * 2 * (K / b) * b * b, 256);
  L.buf = round_up(L.xg + 2ull * 2 * TK * K, 256);
  L.ytk = round_up(L.buf + (fused ? 0ull : 2ull * 2 * chunk * N * K), 256);  // two chunk buffers (double-buffered)
  L.inv = round_up(L.ytk + 4ull * TK * N, 256);  // per-slot expert outputs kept in fp32
  L.pexp = round_up(L.inv + 4ull * TK, 256);
  L.groups = round_up(L.pexp + 4ull * TK, 256);
  L.meta = round_up(L.groups + (fused ? sizeof(gdq::Group) * 2ull * E : 0ull), 256);
  L.total = round_up(L.meta + (fused ? 16ull : 0ull), 256);
  return L;
}

int moe_oft_fwd_impl(bool fused, const uint16_t* X, int T, const float* logits, int E, int top_k, int chunk,
                     const oft_weight* W, int b, const uint16_t* Q, uint16_t* Y, int32_t* topk_idx, float* topk_w,
                     int32_t* offsets, int32_t* bucket, int32_t* chunk_table, int32_t* n_active, void* ws,
                     size_t ws_bytes, void* stream, bool combine = true);
}  // namespace

size_t moe_chunked_oft_workspace(int T, int E, int top_k, int chunk, const oft_weight* W, int b) {
  if (W == nullptr || T <= 0 || E <= 0 || top_k <= 0 || chunk <= 0 || b <= 0) return 0;
  return moe_layout(T, E, top_k, chunk, W->d_in, W->d_out, b).total;
}

int moe_chunked_oft_fwd(const uint16_t* X, int T, const float* logits, int E, int top_k, int chunk,
                        const oft_weight* W, int b, const uint16_t* Q, uint16_t* Y, int32_t* topk_idx, float* topk_w,
                        int32_t* offsets, int32_t* bucket, int32_t* chunk_table, int32_t* n_active, void* ws,
                        size_t ws_bytes, void* stream) {
  return moe_oft_fwd_impl(false, X, T, logits, E, top_k, chunk, W, b, Q, Y, topk_idx, topk_w, offsets, bucket,
                          chunk_table, n_active, ws, ws_bytes, stream);
}

size_t moe_fused_oft_workspace(int T, int E, int top_k, int chunk, const oft_weight* W, int b) {
  if (W == nullptr || T <= 0 || E <= 0 || top_k <= 0 || chunk <= 0 || b <= 0) return 0;
  return moe_layout(T, E, top_k, chunk, W->d_in, W->d_out, b, true).total;
}

int moe_fused_oft_fwd(const uint16_t* X, int T, const float* logits, int E, int top_k, int chunk,
                      const oft_weight* W, int b, const uint16_t* Q, uint16_t* Y, int32_t* topk_idx, float* topk_w,
                      int32_t* offsets, int32_t* bucket, int32_t* chunk_table, int32_t* n_active, void* ws,
                      size_t ws_bytes, void* stream) {
  return moe_oft_fwd_impl(true, X, T, logits, E, top_k, chunk, W, b, Q, Y, topk_idx, topk_w, offsets, bucket,
                          chunk_table, n_active, ws, ws_bytes, stream);
}

}  // extern "C"

namespace {
// combine = false stops before the weighted combine and leaves the per-slot outputs
// Ytk (fp32, bucket order), inv_pos and pos_expert in the workspace (full expert layer).
int moe_oft_fwd_impl(bool fused, const uint16_t* X, int T, const float* logits, int E, int top_k, int chunk,
                     const oft_weight* W, int b, const uint16_t* Q, uint16_t* Y, int32_t* topk_idx, float* topk_w,
                     int32_t* offsets, int32_t* bucket, int32_t* chunk_table, int32_t* n_active, void* ws,
                     size_t ws_bytes, void* stream, bool combine) {
  if (int rc = check_weight(W, true)) return rc;
  if (W->fmt != OFT_W_INT4) return fail(OFT_ERR_UNSUPPORTED, "the MoE expert bank must be INT4");
  const int K = W->d_in, N = W->d_out;
  if (int rc = check_b(b, K)) return rc;
  if (T <= 0) return fail(OFT_ERR_INVALID_ARG, "T must be positive");
  if (E < 1 || E > kMaxExperts || W->n_experts != E)
    return fail(OFT_ERR_UNSUPPORTED, "E must be 1..%d and match the bank's n_experts", kMaxExperts);
  if (top_k < 1 || top_k > kMaxTopK || top_k > E) return fail(OFT_ERR_UNSUPPORTED, "top_k must be 1..%d", kMaxTopK);
  if (chunk < 1 || chunk > gemm::MAX_GROUPS / 2) return fail(OFT_ERR_UNSUPPORTED, "chunk must be 1..%d", gemm::MAX_GROUPS / 2);
  if (N % 16 != 0) return fail(OFT_ERR_UNSUPPORTED, "expert d_out (gate+up) must be a multiple of 16");
  if (1ll * T * top_k * 2 > (1ll << 31) - 1) return fail(OFT_ERR_UNSUPPORTED, "too many routed rows");
  const void* ptrs[] = {X, logits, Q, combine ? static_cast<const void*>(Y) : ws, topk_idx, topk_w, offsets, bucket,
                        chunk_table, n_active, ws};
  for (const void* q : ptrs)
    if (q == nullptr || !aligned16(q)) return fail(OFT_ERR_INVALID_ARG, "NULL or misaligned pointer");
  const int n_proj = N / 2, TK = T * top_k, nb = K / b;
  const int n_chunks_max = (E + chunk - 1) / chunk;
  const MoeLayout L = moe_layout(T, E, top_k, chunk, K, N, b, fused);
  if (ws_bytes < L.total) return fail(OFT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* Rex = reinterpret_cast<float*>(wsb + L.rex);
  uint16_t* Xg = reinterpret_cast<uint16_t*>(wsb + L.xg);
  uint16_t* buf = reinterpret_cast<uint16_t*>(wsb + L.buf);
  float* Ytk = reinterpret_cast<float*>(wsb + L.ytk);
  int* inv = reinterpret_cast<int*>(wsb + L.inv);
  int* pexp = reinterpret_cast<int*>(wsb + L.pexp);

  // 1. top-k + gating
  {
    ProfScope ps(OFT_K_ROUTE, st);
    moe_topk_kernel<<<(T * 32 + 255) / 256, 256, 0, st>>>(logits, T, E, top_k, topk_idx, topk_w);
    OFT_LAUNCHED("moe_topk_kernel");
  }
  // 2. buckets, active experts, chunk table
  const size_t rsmem = sizeof(int) * (32 * E + 2 * E + 1);
  OFT_CUDA(cudaFuncSetAttribute(moe_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(rsmem)));
  {
    ProfScope ps(OFT_K_ROUTE, st);
    moe_route_kernel<<<1, 1024, rsmem, st>>>(topk_idx, TK, E, chunk, n_chunks_max, offsets, bucket, inv, pexp,
                                            chunk_table, n_active);
    OFT_LAUNCHED("moe_route_kernel");
  }
  // 3. rotations of the active experts (gate and up)
  // (as bf16 hi / lo parts of each block's transpose: the gather's MMA operand)
  const long long r_elems = 1ll * E * 2 * nb * b * b;
  if (int rc = launch_cayley(Q, E * 2 * nb, b, Rex, chunk_table, n_active, 2 * nb, st, r_elems)) return rc;
  const uint16_t* Rhi = reinterpret_cast<const uint16_t*>(Rex);
  const uint16_t* Rlo = Rhi + r_elems;
  // 4. rotated gather in bucket order: Xg[proj][pos] = X[t] R_{e,proj}
  //    on the tensor cores, units (active expert, 64-column group, 128-position tile)
  {
    const int rgrid = sm_count() * 4;  // four 128-thread CTAs per SM, persistent
    ProfScope ps(OFT_K_ROTATE, st);
    if (b == 16) {
      if (int rc = set_smem(moe_rot_tc_kernel<16>, kMoeRotSmem)) return rc;
      moe_rot_tc_kernel<16><<<rgrid, kMoeRotThreads, kMoeRotSmem, st>>>(X, K, top_k, bucket, offsets, chunk_table,
                                                                         n_active, Rhi, Rlo, TK, Xg);
    }
    if (b == 32) {
      if (int rc = set_smem(moe_rot_tc_kernel<32>, kMoeRotSmem)) return rc;
      moe_rot_tc_kernel<32><<<rgrid, kMoeRotThreads, kMoeRotSmem, st>>>(X, K, top_k, bucket, offsets, chunk_table,
                                                                         n_active, Rhi, Rlo, TK, Xg);
    }
    if (b == 64) {
      if (int rc = set_smem(moe_rot_tc_kernel<64>, kMoeRotSmem)) return rc;
      moe_rot_tc_kernel<64><<<rgrid, kMoeRotThreads, kMoeRotSmem, st>>>(X, K, top_k, bucket, offsets, chunk_table,
                                                                         n_active, Rhi, Rlo, TK, Xg);
    }
    OFT_LAUNCHED("moe_rot_tc_kernel");
  }
  if (fused) {
    // 5'. one grouped fused-dequant GEMM over every (active expert, projection): the INT4
    //     codes are decoded into the tensor-core operand; per-slot fp32 outputs to Ytk
    gdq::Group* groups = reinterpret_cast<gdq::Group*>(wsb + L.groups);
    int* meta = reinterpret_cast<int*>(wsb + L.meta);
    const long long code_stride = 1ll * N * K / 2, scale_stride = 2ll * (K / W->group) * N;
    {
      ProfScope ps(OFT_K_ROUTE, st);
      moe_groups_kernel<<<1, 32, 0, st>>>(chunk_table, n_active, offsets, TK, n_proj, K, code_stride, scale_stride,
                                          groups, meta);
      OFT_LAUNCHED("moe_groups_kernel");
    }
    gdq::KParams<false> kp;
    memset(&kp, 0, sizeof(kp));
    gdq::Params& gp = kp.p;
    if (int rc = make_map_bf16(&gp.tmB[0], Xg, K, 2ull * TK, K, gdq::TN)) return rc;
    gp.codes = static_cast<const uint8_t*>(W->codes);
    gp.code_row_bytes = K / 2;
    gp.scales = W->scales;
    gp.N = N;
    gp.K = K;
    gp.group = W->group;
    gp.num_groups = 0;
    gp.moe_groups = groups;
    gp.moe_meta = meta;
    gp.moe_out = Ytk;
    gp.moe_ldo = N;
    {
      static bool attr_set[64] = {false};
      int dev = 0;
      cudaGetDevice(&dev);
      if (dev < 64 && !attr_set[dev]) {
        OFT_CUDA(cudaFuncSetAttribute(gdq::gemm_dq_kernel<gdq::kInt4, false, false, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(gdq::kSmemBytes)));
        attr_set[dev] = true;
      }
      ProfScope ps(OFT_K_GEMM, st);
      gdq::gemm_dq_kernel<gdq::kInt4, false, false, true><<<sm_count(), gdq::NUM_THREADS, gdq::kSmemBytes, st>>>(kp);
      OFT_LAUNCHED("gemm_dq_kernel (MoE)");
    }
  } else {
  // 5. chunks: transient dequant of the chunk's experts, then one grouped GEMM
  gemm::Params prm;
  memset(&prm, 0, sizeof(prm));
  if (int rc = make_map_bf16(&prm.tmA[0], Xg, K, 2ull * TK, K, gemm::BM)) return rc;
  for (int i = 1; i < gemm::MAX_MAPS; ++i) prm.tmA[i] = prm.tmA[0];  // B maps: per chunk buffer, below
  prm.C = Ytk;
  prm.c_f32 = 1;
  prm.ldc = N;
  prm.use_moe = 1;
  prm.moe.chunk_table = chunk_table;
  prm.moe.offsets = offsets;
  prm.moe.chunk = chunk;
  prm.moe.TK = TK;
  prm.moe.n_proj = n_proj;
  prm.moe.K = K;
  WeightView bank = view_of(W);
  const size_t dq_smem = sizeof(uint16_t) * kChunkRows * chunk_scale_ld(K / W->group);
  if (dq_smem > 227 * 1024) return fail(OFT_ERR_UNSUPPORTED, "d_in / group too large for the chunk dequant");
  OFT_CUDA(cudaFuncSetAttribute(moe_chunk_dequant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(dq_smem)));
  // Chunk c is dequantised into buffer c % 2 on the side stream while the grouped
  // GEMM of chunk c - 1 runs on the caller's stream; the dequant of chunk c waits
  // for the GEMM of chunk c - 2 (the last reader of its buffer).
  SidePipe* sp = nullptr;
  std::unique_lock<std::mutex> sp_lock;
  if (int rc = side_pipe(&sp, &sp_lock)) return rc;
  OFT_CUDA(cudaEventRecord(sp->start, st));
  OFT_CUDA(cudaStreamWaitEvent(sp->side, sp->start, 0));
  const size_t buf_elems = 1ull * chunk * N * K;
  for (int c = 0; c < n_chunks_max; ++c) {
    const int h = c & 1;
    uint16_t* bufc = buf + h * buf_elems;
    if (c >= 2) OFT_CUDA(cudaStreamWaitEvent(sp->side, sp->gemm_done[h], 0));
    {
      ProfScope ps(OFT_K_DEQUANT, sp->side);
      moe_chunk_dequant_kernel<<<dim3((N + kChunkRows - 1) / kChunkRows, chunk), 256, dq_smem, sp->side>>>(
          bank, chunk_table, c, chunk, bufc);
      OFT_LAUNCHED("moe_chunk_dequant_kernel");
    }
    OFT_CUDA(cudaEventRecord(sp->dq_done[h], sp->side));
    OFT_CUDA(cudaStreamWaitEvent(st, sp->dq_done[h], 0));
    prm.moe.chunk_idx = c;
    if (int rc = make_map_bf16(&prm.tmB[0], bufc, K, 1ull * chunk * N, K, gemm::BN)) return rc;
    for (int i = 1; i < gemm::MAX_MAPS; ++i) prm.tmB[i] = prm.tmB[0];
    if (int rc = launch_gemm(prm, 0, st)) return rc;
    OFT_CUDA(cudaEventRecord(sp->gemm_done[h], st));
  }
  }
  if (!combine) return OFT_OK;
  // 6. weighted combine in slot order
  const long long cunits = 1ll * T * (N / 8);
  const int cgrid = static_cast<int>(std::min<long long>((cunits + 255) / 256, 148ll * 16));
  ProfScope ps(OFT_K_ROUTE, st);
  moe_combine_kernel<<<cgrid, 256, 0, st>>>(Ytk, topk_w, inv, T, N, top_k, Y);
  OFT_LAUNCHED("moe_combine_kernel");
  return OFT_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// MoE full expert layer (gate/up, SwiGLU, down projection)
// ---------------------------------------------------------------------------
namespace {
struct MoeLayerLayout {
  MoeLayout fwd;
  size_t idx, w, offsets, bucket, table, nact, rd, hg, z, total;
};
MoeLayerLayout moe_layer_layout(int T, int E, int top_k, int chunk, int K, int N, int b) {
  MoeLayerLayout L{};
  L.fwd = moe_layout(T, E, top_k, chunk, K, N, b);
  const size_t TK = 1ull * T * top_k, n = N / 2, nbd = n / b;
  const size_t n_chunks_max = (E + chunk - 1) / chunk;
  L.idx = L.fwd.total;
  L.w = round_up(L.idx + 4 * TK, 256);
  L.offsets = round_up(L.w + 4 * TK, 256);
  L.bucket = round_up(L.offsets + 4ull * (E + 1), 256);
  L.table = round_up(L.bucket + 4 * TK, 256);
  L.nact = round_up(L.table + 4 * n_chunks_max * chunk, 256);
  L.rd = round_up(L.nact + 16, 256);
  L.hg = round_up(L.rd + 4ull * E * nbd * b * b, 256);
  L.z = round_up(L.hg + 2 * TK * n, 256);
  L.total = round_up(L.z + 4 * TK * K, 256);
  return L;
}

int check_down_bank(const oft_weight* Wgu, const oft_weight* Wd, int b) {
  if (int rc = check_weight(Wd, true)) return rc;
  if (Wd->fmt != OFT_W_INT4) return fail(OFT_ERR_UNSUPPORTED, "the down-projection bank must be INT4");
  if (Wd->n_experts != Wgu->n_experts) return fail(OFT_ERR_INVALID_ARG, "gate/up and down banks differ in n_experts");
  if (Wd->d_in != Wgu->d_out / 2 || Wd->d_out != Wgu->d_in)
    return fail(OFT_ERR_INVALID_ARG, "down bank must map n_proj = %d to d_in = %d", Wgu->d_out / 2, Wgu->d_in);
  if (int rc = check_b(b, Wd->d_in)) return rc;
  return OFT_OK;
}

template <int B>
int launch_swiglu_rot(const float* Ytk, const int* pexp, int TK, int n, const float* Rd, uint16_t* Hg, cudaStream_t st) {
  const long long units = 1ll * ((TK + SwigluCfg<B>::PT - 1) / SwigluCfg<B>::PT) * (n / B);
  const int grid = static_cast<int>(std::min<long long>(units, 148ll * 8));
  moe_swiglu_rot_kernel<B><<<std::max(grid, 1), 256, 0, st>>>(Ytk, pexp, TK, n, Rd, Hg);
  OFT_LAUNCHED("moe_swiglu_rot_kernel");
  return OFT_OK;
}
}  // namespace

extern "C" {

size_t moe_chunked_oft_layer_workspace(int T, int E, int top_k, int chunk, const oft_weight* W_gu,
                                       const oft_weight* W_down, int b) {
  if (W_gu == nullptr || W_down == nullptr || T <= 0 || E <= 0 || top_k <= 0 || chunk <= 0 || b <= 0) return 0;
  return moe_layer_layout(T, E, top_k, chunk, W_gu->d_in, W_gu->d_out, b).total;
}

int moe_chunked_oft_layer_fwd(const uint16_t* X, int T, const float* logits, int E, int top_k, int chunk,
                              const oft_weight* W_gu, const oft_weight* W_down, int b, const uint16_t* Q_gu,
                              const uint16_t* Q_down, uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_weight(W_gu, true)) return rc;
  if (int rc = check_down_bank(W_gu, W_down, b)) return rc;
  const int K = W_gu->d_in, N = W_gu->d_out, n = N / 2, nbd = n / (b > 0 ? b : 1);
  if (T <= 0 || E <= 0 || top_k <= 0 || chunk <= 0) return fail(OFT_ERR_INVALID_ARG, "bad sizes");
  const void* ptrs[] = {X, logits, Q_gu, Q_down, Y, ws};
  for (const void* q : ptrs)
    if (q == nullptr || !aligned16(q)) return fail(OFT_ERR_INVALID_ARG, "NULL or misaligned pointer");
  const MoeLayerLayout L = moe_layer_layout(T, E, top_k, chunk, K, N, b);
  if (ws_bytes < L.total) return fail(OFT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  int* idx = reinterpret_cast<int*>(wsb + L.idx);
  float* wts = reinterpret_cast<float*>(wsb + L.w);
  int* offsets = reinterpret_cast<int*>(wsb + L.offsets);
  int* bucket = reinterpret_cast<int*>(wsb + L.bucket);
  int* table = reinterpret_cast<int*>(wsb + L.table);
  int* n_active = reinterpret_cast<int*>(wsb + L.nact);
  float* Rd = reinterpret_cast<float*>(wsb + L.rd);
  uint16_t* Hg = reinterpret_cast<uint16_t*>(wsb + L.hg);
  float* Z = reinterpret_cast<float*>(wsb + L.z);
  float* Ytk = reinterpret_cast<float*>(wsb + L.fwd.ytk);
  const int* inv = reinterpret_cast<const int*>(wsb + L.fwd.inv);
  const int* pexp = reinterpret_cast<const int*>(wsb + L.fwd.pexp);
  uint16_t* buf = reinterpret_cast<uint16_t*>(wsb + L.fwd.buf);
  const int TK = T * top_k, n_chunks_max = (E + chunk - 1) / chunk;

  // 1. routing, gate/up rotations, rotated gather, chunked gate/up GEMMs -> Ytk (fp32, bucket order)
  if (int rc = moe_oft_fwd_impl(false, X, T, logits, E, top_k, chunk, W_gu, b, Q_gu, nullptr, idx, wts, offsets,
                                bucket, table, n_active, ws, L.fwd.total, stream, false))
    return rc;
  // 2. down adapters of the active experts
  if (int rc = launch_cayley(Q_down, E * nbd, b, Rd, table, n_active, nbd, st)) return rc;
  // 3. h = silu(g) * u, rotated by R_e,down, bf16 in bucket order
  {
    ProfScope ps(OFT_K_ROTATE, st);
    int rc = OFT_OK;
    if (b == 16) rc = launch_swiglu_rot<16>(Ytk, pexp, TK, n, Rd, Hg, st);
    if (b == 32) rc = launch_swiglu_rot<32>(Ytk, pexp, TK, n, Rd, Hg, st);
    if (b == 64) rc = launch_swiglu_rot<64>(Ytk, pexp, TK, n, Rd, Hg, st);
    if (rc) return rc;
  }
  // 4. chunks of down projections: transient dequant (side stream, double-buffered, in the
  //    gate/up chunk buffers, which every gate/up GEMM has finished reading), one grouped GEMM each
  gemm::Params prm;
  memset(&prm, 0, sizeof(prm));
  if (int rc = make_map_bf16(&prm.tmA[0], Hg, n, 1ull * TK, n, gemm::BM)) return rc;
  for (int i = 1; i < gemm::MAX_MAPS; ++i) prm.tmA[i] = prm.tmA[0];
  prm.C = Z;
  prm.c_f32 = 1;
  prm.ldc = K;
  prm.use_moe = 1;
  prm.moe.chunk_table = table;
  prm.moe.offsets = offsets;
  prm.moe.chunk = chunk;
  prm.moe.TK = TK;
  prm.moe.n_proj = n;
  prm.moe.K = K;
  prm.moe.mode = gemm::kMoeDown;
  const WeightView dbank = view_of(W_down);  // N = K rows, K = n columns per expert
  const size_t dq_smem = sizeof(uint16_t) * kChunkRows * chunk_scale_ld(n / W_down->group);
  if (dq_smem > 227 * 1024) return fail(OFT_ERR_UNSUPPORTED, "n_proj / group too large for the chunk dequant");
  OFT_CUDA(cudaFuncSetAttribute(moe_chunk_dequant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(dq_smem)));
  SidePipe* sp = nullptr;
  std::unique_lock<std::mutex> sp_lock;
  if (int rc = side_pipe(&sp, &sp_lock)) return rc;
  OFT_CUDA(cudaEventRecord(sp->start, st));
  OFT_CUDA(cudaStreamWaitEvent(sp->side, sp->start, 0));
  const size_t buf_elems = 1ull * chunk * K * n;
  for (int c = 0; c < n_chunks_max; ++c) {
    const int h = c & 1;
    uint16_t* bufc = buf + h * buf_elems;
    if (c >= 2) OFT_CUDA(cudaStreamWaitEvent(sp->side, sp->gemm_done[h], 0));
    {
      ProfScope ps(OFT_K_DEQUANT, sp->side);
      moe_chunk_dequant_kernel<<<dim3((K + kChunkRows - 1) / kChunkRows, chunk), 256, dq_smem, sp->side>>>(
          dbank, table, c, chunk, bufc);
      OFT_LAUNCHED("moe_chunk_dequant_kernel");
    }
    OFT_CUDA(cudaEventRecord(sp->dq_done[h], sp->side));
    OFT_CUDA(cudaStreamWaitEvent(st, sp->dq_done[h], 0));
    prm.moe.chunk_idx = c;
    if (int rc = make_map_bf16(&prm.tmB[0], bufc, n, 1ull * chunk * K, n, gemm::BN)) return rc;
    for (int i = 1; i < gemm::MAX_MAPS; ++i) prm.tmB[i] = prm.tmB[0];
    if (int rc = launch_gemm(prm, 0, st)) return rc;
    OFT_CUDA(cudaEventRecord(sp->gemm_done[h], st));
  }
  // 5. Y[t] = sum_k w_tk Z[pos(t, k)] in slot order
  const long long cunits = 1ll * T * (K / 8);
  const int cgrid = static_cast<int>(std::min<long long>((cunits + 255) / 256, 148ll * 16));
  ProfScope ps(OFT_K_ROUTE, st);
  moe_combine_kernel<<<cgrid, 256, 0, st>>>(Z, wts, inv, T, K, top_k, Y);
  OFT_LAUNCHED("moe_combine_kernel");
  return OFT_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// MoE backward
// ---------------------------------------------------------------------------
namespace {
struct MoeBwdLayout {
  size_t idx, w, offsets, bucket, table, meta, order, inv, pexp, rex, dyg, buf, d, u, dw, row_t, row_w, total;
};
MoeBwdLayout moe_bwd_layout(int T, int E, int top_k, int chunk, int K, int N, int b) {
  MoeBwdLayout L{};
  const size_t TK = 1ull * T * top_k, n = N / 2, nb = K / b;
  const size_t n_chunks_max = (E + chunk - 1) / chunk;
  L.idx = 0;
  L.w = round_up(L.idx + 4 * TK, 256);
  L.offsets = round_up(L.w + 4 * TK, 256);
  L.bucket = round_up(L.offsets + 4ull * (E + 1), 256);
  L.table = round_up(L.bucket + 4 * TK, 256);
  L.meta = round_up(L.table + 4 * n_chunks_max * chunk, 256);  // n_active
  L.order = round_up(L.meta + 16, 256);
  L.inv = round_up(L.order + 4ull * E, 256);
  L.pexp = round_up(L.inv + 4 * TK, 256);
  L.rex = round_up(L.pexp + 4 * TK, 256);
  L.dyg = round_up(L.rex + 4ull * E * 2 * nb * b * b, 256);
  L.buf = round_up(L.dyg + 2 * 2 * TK * n, 256);
  // two transposed chunk buffers; after the last chunk's GEMM the same bytes hold the
  // active experts' adapter gradients G [E][2][nb][b][b]
  L.d = round_up(L.buf + std::max(2ull * 2 * chunk * N * K, 4ull * E * 2 * nb * b * b), 256);
  L.u = round_up(L.d + 4 * 2 * TK * K, 256);
  L.dw = round_up(L.u + 4 * TK * K, 256);
  L.row_t = round_up(L.dw + 4 * TK, 256);
  L.row_w = round_up(L.row_t + 4 * TK, 256);
  L.total = round_up(L.row_w + 4 * TK, 256);
  return L;
}

// Step 4 of the MoE backward on the tensor cores: U = sum_p D_p R^T per routed row, each
// active expert's adapter gradient G (into `G`, [E][2][nb][b][b]), then its Cayley backward.
int launch_moe_bwd_tc(const float* D, const uint16_t* X, int K, int TK, int E, int b, const int* row_t,
                      const float* row_w, const int* offsets, const int* order, const int* n_active, const float* R,
                      float* U, float* G, float* dQ, cudaStream_t st) {
  const int nb = K / b;
  {
    rtc::MoeRotbParams prm;
    memset(&prm, 0, sizeof(prm));
    if (int rc = make_map_f32_3d(&prm.tmD, D, K, TK, 2)) return rc;
    prm.R = R;
    prm.offsets = offsets;
    prm.order = order;
    prm.n_active = n_active;
    prm.U = U;
    prm.K = K;
    prm.TK = TK;
    prm.nb = nb;
    prm.groups = (K + 63) / 64;
    const int grid = static_cast<int>(std::min<long long>(sm_count(), 1ll * E * prm.groups));
    auto go = [&](auto kernel) -> int {
      if (int rc = set_smem(kernel, rtc::kMoeRotbSmem)) return rc;
      ProfScope ps(OFT_K_ROTATE, st);
      OFT_CUDA(launch_pdl(kernel, grid, rtc::NUM_THREADS, rtc::kMoeRotbSmem, st, prm));
      return OFT_OK;
    };
    int rc = OFT_OK;
    if (b == 16) rc = go(rtc::moe_rotb_tc_kernel<16>);
    if (b == 32) rc = go(rtc::moe_rotb_tc_kernel<32>);
    if (b == 64) rc = go(rtc::moe_rotb_tc_kernel<64>);
    if (rc) return rc;
    OFT_LAUNCHED("moe_rotb_tc_kernel");
  }
  {
    rtc::MoeGradParams prm;
    memset(&prm, 0, sizeof(prm));
    if (int rc = make_map_f32_3d(&prm.tmD, D, K, TK, 2, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B, rtc::MG_TP)) return rc;
    prm.X = X;
    prm.row_t = row_t;
    prm.row_w = row_w;
    prm.offsets = offsets;
    prm.order = order;
    prm.n_active = n_active;
    prm.G = G;
    prm.K = K;
    prm.TK = TK;
    prm.b = b;
    prm.nb = nb;
    prm.groups = (K + 127) / 128;
    if (int rc = set_smem(rtc::moe_grad_tc_kernel, rtc::kMoeGradSmem)) return rc;
    const int grid = static_cast<int>(std::min<long long>(sm_count(), 1ll * E * prm.groups));
    ProfScope ps(OFT_K_GRAD, st);
    OFT_CUDA(launch_pdl(rtc::moe_grad_tc_kernel, grid, rtc::NUM_THREADS, rtc::kMoeGradSmem, st, prm));
    OFT_LAUNCHED("moe_grad_tc_kernel");
  }
  return launch_cayley_bwd(R, G, 1, E * 2 * nb, b, dQ, st, order, n_active, 2 * nb);
}
}  // namespace

extern "C" {

size_t moe_chunked_oft_bwd_workspace(int T, int E, int top_k, int chunk, const oft_weight* W, int b) {
  if (W == nullptr || T <= 0 || E <= 0 || top_k <= 0 || chunk <= 0 || b <= 0) return 0;
  return moe_bwd_layout(T, E, top_k, chunk, W->d_in, W->d_out, b).total;
}

int moe_chunked_oft_bwd(const uint16_t* dY, const uint16_t* X, int T, const float* logits, int E, int top_k,
                        int chunk, const oft_weight* W, int b, const uint16_t* Q, uint16_t* dX, float* dQ,
                        float* dlogits, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_weight(W, true)) return rc;
  if (W->fmt != OFT_W_INT4) return fail(OFT_ERR_UNSUPPORTED, "the MoE expert bank must be INT4");
  const int K = W->d_in, N = W->d_out;
  if (int rc = check_b(b, K)) return rc;
  if (T <= 0) return fail(OFT_ERR_INVALID_ARG, "T must be positive");
  if (E < 1 || E > kMaxExperts || W->n_experts != E)
    return fail(OFT_ERR_UNSUPPORTED, "E must be 1..%d and match the bank's n_experts", kMaxExperts);
  if (top_k < 1 || top_k > kMaxTopK || top_k > E) return fail(OFT_ERR_UNSUPPORTED, "top_k must be 1..%d", kMaxTopK);
  if (chunk < 1 || chunk > gemm::MAX_GROUPS / 2) return fail(OFT_ERR_UNSUPPORTED, "chunk must be 1..%d", gemm::MAX_GROUPS / 2);
  if (N % 16 != 0) return fail(OFT_ERR_UNSUPPORTED, "expert d_out (gate+up) must be a multiple of 16");
  if (1ll * T * top_k * 2 > (1ll << 31) - 1 || 1ll * E * 2 * K > (1ll << 31) - 1)
    return fail(OFT_ERR_UNSUPPORTED, "too many routed rows");
  const void* ptrs[] = {dY, X, logits, Q, dX, dQ, ws};
  for (const void* q : ptrs)
    if (q == nullptr || !aligned16(q)) return fail(OFT_ERR_INVALID_ARG, "NULL or misaligned pointer");
  if (dlogits != nullptr && !aligned16(dlogits)) return fail(OFT_ERR_INVALID_ARG, "misaligned dlogits");
  const int n_proj = N / 2, TK = T * top_k, nb = K / b;
  const int n_chunks_max = (E + chunk - 1) / chunk;
  const MoeBwdLayout L = moe_bwd_layout(T, E, top_k, chunk, K, N, b);
  if (ws_bytes < L.total) return fail(OFT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  int* idx = reinterpret_cast<int*>(wsb + L.idx);
  float* wts = reinterpret_cast<float*>(wsb + L.w);
  int* offsets = reinterpret_cast<int*>(wsb + L.offsets);
  int* bucket = reinterpret_cast<int*>(wsb + L.bucket);
  int* table = reinterpret_cast<int*>(wsb + L.table);
  int* n_active = reinterpret_cast<int*>(wsb + L.meta);
  int* order = reinterpret_cast<int*>(wsb + L.order);
  int* inv = reinterpret_cast<int*>(wsb + L.inv);
  int* pexp = reinterpret_cast<int*>(wsb + L.pexp);
  float* Rex = reinterpret_cast<float*>(wsb + L.rex);
  uint16_t* dYg = reinterpret_cast<uint16_t*>(wsb + L.dyg);
  uint16_t* buf = reinterpret_cast<uint16_t*>(wsb + L.buf);
  float* D = reinterpret_cast<float*>(wsb + L.d);
  float* U = reinterpret_cast<float*>(wsb + L.u);
  float* dw = reinterpret_cast<float*>(wsb + L.dw);
  int* row_t = reinterpret_cast<int*>(wsb + L.row_t);
  float* row_w = reinterpret_cast<float*>(wsb + L.row_w);

  // 1. routing, as in the forward
  {
    ProfScope ps(OFT_K_ROUTE, st);
    moe_topk_kernel<<<(T * 32 + 255) / 256, 256, 0, st>>>(logits, T, E, top_k, idx, wts);
    OFT_LAUNCHED("moe_topk_kernel");
  }
  const size_t rsmem = sizeof(int) * (32 * E + 2 * E + 1);
  OFT_CUDA(cudaFuncSetAttribute(moe_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(rsmem)));
  {
    ProfScope ps(OFT_K_ROUTE, st);
    moe_route_kernel<<<1, 1024, rsmem, st>>>(idx, TK, E, chunk, n_chunks_max, offsets, bucket, inv, pexp, table,
                                            n_active);
    OFT_LAUNCHED("moe_route_kernel");
    moe_order_kernel<<<1, 1024, 0, st>>>(offsets, table, n_active, order);
    OFT_LAUNCHED("moe_order_kernel");
    const long long gunits = 1ll * TK * (N / 8);
    moe_gather_dy_kernel<<<static_cast<int>(std::min<long long>((gunits + 255) / 256, 148ll * 16)), 256, 0, st>>>(
        dY, bucket, wts, TK, top_k, n_proj, dYg, row_t, row_w);
    OFT_LAUNCHED("moe_gather_dy_kernel");
  }
  // 2. rotations of the active experts; the inactive experts' dQ is zero
  if (int rc = launch_cayley(Q, E * 2 * nb, b, Rex, table, n_active, 2 * nb, st)) return rc;
  OFT_CUDA(cudaMemsetAsync(dQ, 0, sizeof(float) * E * 2 * nb * (b * (b - 1) / 2), st));
  // 3. chunks: transposed dequant of the chunk's experts (side stream, double-buffered),
  //    then one grouped GEMM D[p][pos][:] = dYg[p][pos][:] W_e,p^T
  gemm::Params prm;
  memset(&prm, 0, sizeof(prm));
  if (int rc = make_map_bf16(&prm.tmA[0], dYg, n_proj, 2ull * TK, n_proj, gemm::BM)) return rc;
  for (int i = 1; i < gemm::MAX_MAPS; ++i) prm.tmA[i] = prm.tmA[0];
  prm.C = D;
  prm.c_f32 = 1;
  prm.ldc = K;
  prm.use_moe = 1;
  prm.moe.chunk_table = table;
  prm.moe.offsets = offsets;
  prm.moe.chunk = chunk;
  prm.moe.TK = TK;
  prm.moe.n_proj = n_proj;
  prm.moe.K = K;
  prm.moe.mode = gemm::kMoeBwd;
  const WeightView bank = view_of(W);
  SidePipe* sp = nullptr;
  std::unique_lock<std::mutex> sp_lock;
  if (int rc = side_pipe(&sp, &sp_lock)) return rc;
  OFT_CUDA(cudaEventRecord(sp->start, st));
  OFT_CUDA(cudaStreamWaitEvent(sp->side, sp->start, 0));
  const size_t buf_elems = 1ull * chunk * N * K;
  for (int c = 0; c < n_chunks_max; ++c) {
    const int h = c & 1;
    uint16_t* bufc = buf + h * buf_elems;
    if (c >= 2) OFT_CUDA(cudaStreamWaitEvent(sp->side, sp->gemm_done[h], 0));
    {
      ProfScope ps(OFT_K_DEQUANT, sp->side);
      moe_chunk_dequant_t_kernel<<<dqt_grid(K, N, chunk), 256, 0,
                                   sp->side>>>(bank, table, c, chunk,
                                                                                                  n_proj, bufc);
      OFT_LAUNCHED("moe_chunk_dequant_t_kernel");
    }
    OFT_CUDA(cudaEventRecord(sp->dq_done[h], sp->side));
    OFT_CUDA(cudaStreamWaitEvent(st, sp->dq_done[h], 0));
    prm.moe.chunk_idx = c;
    if (int rc = make_map_bf16(&prm.tmB[0], bufc, n_proj, 2ull * chunk * K, n_proj, gemm::BN)) return rc;
    for (int i = 1; i < gemm::MAX_MAPS; ++i) prm.tmB[i] = prm.tmB[0];
    if (int rc = launch_gemm(prm, 0, st)) return rc;
    OFT_CUDA(cudaEventRecord(sp->gemm_done[h], st));
  }
  // 4. per (active expert, column group): rows rotated back, the expert's adapter
  //    gradient (into the chunk buffers, free after the last GEMM), and the Cayley
  //    backward of the active experts' blocks
  if (int rc = launch_moe_bwd_tc(D, X, K, TK, E, b, row_t, row_w, offsets, order, n_active, Rex, U,
                                 reinterpret_cast<float*>(buf), dQ, st))
    return rc;
  // 5. dX[t] = sum_k w_tk U[pos(t, k)] in slot order with dw_tk = <U[pos(t, k)], X[t]>; logit gradients
  {
    ProfScope ps(OFT_K_ROUTE, st);
    const int cgrid = static_cast<int>(std::min<long long>((T + 7) / 8, 148ll * 16));
    moe_combine_bwd_kernel<<<cgrid, 256, 0, st>>>(U, wts, inv, X, T, K, top_k, dX, dw);
    OFT_LAUNCHED("moe_combine_bwd_kernel");
    if (dlogits != nullptr) {
      moe_dlogits_kernel<<<(T * 32 + 255) / 256, 256, 0, st>>>(dw, idx, wts, T, E, top_k, dlogits);
      OFT_LAUNCHED("moe_dlogits_kernel");
    }
  }
  return OFT_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// test hook: one chunk of the MoE transient dequant, as the MoE calls run it
// ---------------------------------------------------------------------------
extern "C" int oft_moe_chunk_dequant(const oft_weight* bank, const int32_t* chunk_table, int chunk_idx, int chunk,
                                     int transpose, uint16_t* out, void* stream) {
  if (int rc = check_weight(bank, true)) return rc;
  if (bank->fmt != OFT_W_INT4) return fail(OFT_ERR_UNSUPPORTED, "the MoE expert bank must be INT4");
  if (chunk < 1 || chunk > gemm::MAX_GROUPS / 2) return fail(OFT_ERR_UNSUPPORTED, "chunk must be 1..%d", gemm::MAX_GROUPS / 2);
  if (chunk_idx < 0) return fail(OFT_ERR_INVALID_ARG, "chunk_idx < 0");
  if (!chunk_table || !out || !aligned16(chunk_table) || !aligned16(out))
    return fail(OFT_ERR_INVALID_ARG, "NULL or misaligned pointer");
  const int K = bank->d_in, N = bank->d_out;
  const WeightView v = view_of(bank);
  cudaStream_t st = as_stream(stream);
  ProfScope ps(OFT_K_DEQUANT, st);
  if (!transpose) {
    const size_t dq_smem = sizeof(uint16_t) * kChunkRows * chunk_scale_ld(K / bank->group);
    if (dq_smem > 227 * 1024) return fail(OFT_ERR_UNSUPPORTED, "d_in / group too large for the chunk dequant");
    OFT_CUDA(cudaFuncSetAttribute(moe_chunk_dequant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(dq_smem)));
    moe_chunk_dequant_kernel<<<dim3((N + kChunkRows - 1) / kChunkRows, chunk), 256, dq_smem, st>>>(v, chunk_table,
                                                                                                  chunk_idx, chunk, out);
    OFT_LAUNCHED("moe_chunk_dequant_kernel");
  } else {
    if (N % 16 != 0) return fail(OFT_ERR_UNSUPPORTED, "the transposed chunk needs d_out (gate+up) % 16 == 0");
    moe_chunk_dequant_t_kernel<<<dqt_grid(K, N, chunk), 256, 0, st>>>(
        v, chunk_table, chunk_idx, chunk, N / 2, out);
    OFT_LAUNCHED("moe_chunk_dequant_t_kernel");
  }
  return OFT_OK;
}

// ---------------------------------------------------------------------------
// bounded-wait self test
// ---------------------------------------------------------------------------
namespace {
__global__ void debug_bounded_wait_kernel(unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, kErrWaitDebug, timeout_ns);  // nothing ever arrives
  __syncthreads();
}
}  // namespace

extern "C" int oft_debug_bounded_wait(int timeout_us, void* stream) {
  if (timeout_us <= 0 || timeout_us > 2000000) return fail(OFT_ERR_INVALID_ARG, "timeout_us must be 1..2000000");
  debug_bounded_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(1000ull * timeout_us);
  OFT_LAUNCHED("debug_bounded_wait_kernel");
  return OFT_OK;
}

extern "C" int oft_profile_begin(int max_launches) {
  if (max_launches < 1 || max_launches > (1 << 20)) return fail(OFT_ERR_INVALID_ARG, "max_launches must be 1..2^20");
  if (g_prof.cap < max_launches) {
    for (int i = 0; i < 2 * g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
    delete[] g_prof.ev;
    delete[] g_prof.kind;
    g_prof.ev = new cudaEvent_t[2 * max_launches];
    g_prof.kind = new int[max_launches];
    g_prof.cap = 0;
    for (int i = 0; i < 2 * max_launches; ++i) OFT_CUDA(cudaEventCreate(&g_prof.ev[i]));
    g_prof.cap = max_launches;
  }
  g_prof.n = 0;
  g_prof.dropped = 0;
  for (int k = 0; k < OFT_K_NUM; ++k) g_prof.counts[k] = 0;
  g_prof.on = true;
  return OFT_OK;
}

extern "C" int oft_profile_end(double* ms_by_kind, int* launches_by_kind, int n_kinds, int* dropped) {
  if (!g_prof.on) return fail(OFT_ERR_INVALID_ARG, "profiling was not started");
  g_prof.on = false;
  if (n_kinds < 0 || n_kinds > OFT_K_NUM) return fail(OFT_ERR_INVALID_ARG, "n_kinds must be 0..%d", OFT_K_NUM);
  double ms[OFT_K_NUM] = {0};
  for (int i = 0; i < g_prof.n; ++i) {
    OFT_CUDA(cudaEventSynchronize(g_prof.ev[2 * i + 1]));
    float t = 0.f;
    OFT_CUDA(cudaEventElapsedTime(&t, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]));
    ms[g_prof.kind[i]] += t;
  }
  for (int k = 0; k < n_kinds; ++k) {
    if (ms_by_kind) ms_by_kind[k] = ms[k];
    if (launches_by_kind) launches_by_kind[k] = g_prof.counts[k];
  }
  if (dropped) *dropped = g_prof.dropped;
  return OFT_OK;
}

// ---------------------------------------------------------------------------
// forward without a caller workspace: the scratch is a fixed device array
// ---------------------------------------------------------------------------
namespace {
// Scratch of oft_linear_fwd_noalloc.  A __device__ symbol: in host code its
// name is only a host-side stand-in, so the kernels get the device address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[OFT_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

// Once per device, with that device current: look up the array's device address.
int noalloc_scratch(void** out) {
  int dev = 0;
  OFT_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(OFT_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    OFT_CUDA(cudaGetSymbolAddress(&ptr, g_noalloc_scratch));
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return OFT_OK;
}
}  // namespace

extern "C" int oft_linear_fwd_noalloc(const uint16_t* X, int M, const oft_weight* W, const oft_split* S, int b,
                                      const float* R, uint16_t* Y, void* stream) {
  if (int rc = check_weight(W, false)) return rc;
  if (int rc = check_split(S, W->d_out)) return rc;
  if (int rc = check_b(b, W->d_in)) return rc;
  if (M < 0) return fail(OFT_ERR_INVALID_ARG, "M < 0");
  if (M == 0) return OFT_OK;
  // oft_linear_fwd takes the bf16-weight path only when its workspace also holds the
  // weight copy, and the fused-decode path otherwise; the smaller (fused) layout is
  // what must fit
  const size_t need = fwd_layout_fused(M, W, S).total;
  if (need > OFT_NOALLOC_SCRATCH_BYTES)
    return fail(OFT_ERR_WORKSPACE,
                "oft_linear_fwd_noalloc: this shape needs %zu bytes of scratch, more than the fixed %u-byte "
                "array; use oft_linear_fwd with a caller workspace",
                need, (unsigned)OFT_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if (int rc = noalloc_scratch(&scratch)) return rc;
  return oft_linear_fwd(X, M, W, S, b, R, Y, scratch, OFT_NOALLOC_SCRATCH_BYTES, stream);
}
