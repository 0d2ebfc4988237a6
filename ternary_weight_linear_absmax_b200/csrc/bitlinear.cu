// C-ABI entry points of libbitlinear: argument checks, workspace layout,
// kernel selection and launches. See include/bitlinear.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "bitlinear.h"
#include "bl_device.cuh"
#include "gemv_kernel.cuh"
#include "gemv_lut_kernel.cuh"
#include "gemv_r3_kernel.cuh"
#include "quant_kernels.cuh"
#include "skinny_kernel.cuh"
#include "ste_kernels.cuh"
#include "tc_gemm_kernel.cuh"

namespace bl {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kAbsmeanMaxBlocks = 1024;
constexpr size_t kAlign = 256;

inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define BL_TRY(expr)                 \
  do {                               \
    bl_status _s = (expr);           \
    if (_s != BL_OK) return _s;      \
  } while (0)

#define BL_CUDA(expr)                          \
  do {                                         \
    cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) return BL_ERR_CUDA; \
  } while (0)

// --------------------------------------------------------------------------
// Per-device state: architecture check and the number of SMs.
struct DeviceInfo {
  int checked = 0;
  int ok = 0;
  int sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

bl_status current_device(int* dev_out, int* sms_out) {
  int dev = 0;
  BL_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return BL_ERR_UNSUPPORTED;
  DeviceInfo& d = g_dev[dev];
  if (!d.checked) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!d.checked) {
      int major = 0, minor = 0, sms = 0;
      BL_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
      BL_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
      BL_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
      d.ok = (major == 10 && minor == 0);
      d.sms = sms;
      d.checked = 1;
    }
  }
  if (!d.ok) return BL_ERR_UNSUPPORTED;
  *dev_out = dev;
  if (sms_out) *sms_out = d.sms;
  return BL_OK;
}

// Opt a kernel into large dynamic shared memory, once per (kernel, device).
template <typename F>
bl_status ensure_smem(F* kernel, int dev, size_t bytes) {
  struct Entry {
    const void* fn;
    int dev;
    size_t bytes;
  };
  static Entry cache[512];
  static int n = 0;
  std::lock_guard<std::mutex> lk(g_mu);
  for (int i = 0; i < n; ++i)
    if (cache[i].fn == (const void*)kernel && cache[i].dev == dev && cache[i].bytes >= bytes)
      return BL_OK;
  BL_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
  // Every SM keeps its whole shared memory: with a smaller L1/shared split,
  // chosen per kernel, an SM that runs one kind of CTA may lack the room for
  // the next kernel's CTA in a chain of dependent launches, which then
  // doubles up on another SM (measured: 1-token FFN blocks 13.7 -> 10.5 us).
  BL_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared));
  if (n < 512) cache[n++] = Entry{(const void*)kernel, dev, bytes};
  return BL_OK;
}

// --------------------------------------------------------------------------
// Tensor maps (TMA descriptors) through the driver entry point, so the
// library does not link libcuda directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static int tried = 0;
  if (!tried) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!tried) {
      void* p = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
              cudaSuccess &&
          q == cudaDriverEntryPointSuccess)
        fn = reinterpret_cast<EncodeTiledFn>(p);
      tried = 1;
    }
  }
  return fn;
}

// 2-D uint8 tensor [rows, cols] (cols contiguous), box {box_cols, box_rows}.
bl_status make_map_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return BL_ERR_CUDA;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BL_OK : BL_ERR_CUDA;
}

// --------------------------------------------------------------------------
// Argument checks.
// K (and the FFN hidden size) ≤ BL_MAX_K = 2^22: every INT32 sum stays exact
// (127·K < 2^31), including the decode GEMV's per-thread sums scaled by up to
// 64 (each thread covers at most K/512 of a row's weights there).
bl_status check_k(int64_t K) {
  if (K <= 0 || K % 64 != 0) return BL_ERR_SHAPE;
  if (K > (int64_t)BL_MAX_K) return BL_ERR_SHAPE;
  return BL_OK;
}
bl_status check_rows(int64_t R) {
  if (R < 0 || R > ((int64_t)1 << 31) - 1) return BL_ERR_SHAPE;
  return BL_OK;
}
bl_status check_eps(float eps) {
  if (!(eps > 0.0f) || !std::isfinite(eps)) return BL_ERR_INVALID_ARG;
  return BL_OK;
}
bl_status check_ptr(const void* p) {
  if (p == nullptr) return BL_ERR_INVALID_ARG;
  if (!aligned16(p)) return BL_ERR_ALIGN;
  return BL_OK;
}
bl_status check_dtype(int d) {
  if (d != BL_F32 && d != BL_BF16) return BL_ERR_DTYPE;
  return BL_OK;
}

// --------------------------------------------------------------------------
// The fused GEMV (decode) path. Two CTAs per SM: 228 KiB of shared memory per
// SM, 1 KiB reserved per CTA.
constexpr size_t kGemvSmemCap = 112 * 1024;

// Up to bl_gemv_max_tokens() tokens a call takes the fused GEMV when a CTA's
// shared memory holds at least one weight row and the M int8 token rows
// (K up to 37,376 at 1 token, 18,624 at 4). Longer rows go through the
// activation quantiser and the warp-level kernel, whose stage ring streams any
// K; the workspaces are sized accordingly.
inline bool gemv_path(int64_t M, int64_t K) {
  return M <= kGemvMaxTokens && gemv_smem_bytes(K, 1, (int)M) <= kGemvSmemCap;
}

// --------------------------------------------------------------------------
// Workspace layouts (offsets are multiples of 256 bytes).
struct ActWs {
  size_t aq, gamma, rowsum, total;
};
ActWs act_ws(int64_t M, int64_t K) {
  ActWs w;
  w.aq = 0;
  w.gamma = align_up((size_t)M * K);
  w.rowsum = w.gamma + align_up((size_t)M * 4);
  w.total = w.rowsum + align_up((size_t)M * 4);
  return w;
}

struct FfnWs {
  ActWs x;        // quantised X (M > GEMV limit)
  size_t acc_up;  // int32 [M, H]
  size_t gamma_x; // [M] (GEMV path)
  size_t rmax;    // fp32 [M, up-projection CTAs ≤ H] per-CTA ReLU² maxima (GEMV path)
  size_t rq;      // int8 [M, H]
  size_t gamma_r, rs_r, total;
};
// The FFN block takes its GEMV form when both projections fit the GEMV.
inline bool ffn_gemv_path(int64_t M, int64_t K, int64_t H) {
  return gemv_path(M, K) && gemv_path(M, H);
}

FfnWs ffn_ws(int64_t M, int64_t K, int64_t H) {
  FfnWs w{};
  if (ffn_gemv_path(M, K, H)) {
    w.acc_up = 0;
    w.gamma_x = align_up((size_t)M * H * 4);
    w.rmax = w.gamma_x + align_up((size_t)M * 4);
    w.total = w.rmax + align_up((size_t)M * H * 4);
    return w;
  }
  w.x = act_ws(M, K);
  w.acc_up = w.x.total;
  w.rq = w.acc_up + align_up((size_t)M * H * 4);
  w.gamma_r = w.rq + align_up((size_t)M * H);
  w.rs_r = w.gamma_r + align_up((size_t)M * 4);
  w.total = w.rs_r + align_up((size_t)M * 4);
  return w;
}

// A kernel launched with programmatic dependent launch (it must wait for the
// previous grid before it reads what that grid may write).
template <typename... KArgs, typename... Args>
bl_status launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  BL_CUDA(cudaLaunchKernelEx(&cfg, k, static_cast<KArgs>(args)...));
  return BL_OK;
}

// --------------------------------------------------------------------------
// GEMV launches.
template <int MT, typename TA, int SRC, int OUT>
bl_status launch_gemv_t(const CUtensorMap& tw, const GemvParams& p, int grid, size_t smem,
                        bool pdl, int dev, cudaStream_t st) {
  auto* k = gemv_ternary_kernel<MT, TA, SRC, OUT>;
  BL_TRY(ensure_smem(k, dev, smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  BL_CUDA(cudaLaunchKernelEx(&cfg, k, tw, p));
  return BL_OK;
}

template <typename TA, int SRC, int OUT>
bl_status launch_gemv_mt(const CUtensorMap& tw, const GemvParams& p, int grid, size_t smem,
                         bool pdl, int dev, cudaStream_t st) {
  // Token counts 1 and 2 get their own instantiations (fewer registers);
  // 3 and 4 share MT = 4 with runtime guards.
  if (p.M == 1) return launch_gemv_t<1, TA, SRC, OUT>(tw, p, grid, smem, pdl, dev, st);
  if (p.M == 2) return launch_gemv_t<2, TA, SRC, OUT>(tw, p, grid, smem, pdl, dev, st);
  return launch_gemv_t<4, TA, SRC, OUT>(tw, p, grid, smem, pdl, dev, st);
}

// Choose rows per CTA: one wave over the SMs when shared memory allows,
// at most kGemvMaxRows rows.
// Grid of the one-CTA-per-row-slab kernels, rows split evenly: every SM
// gets the same number of CTAs of a launch (one when a slab of at most
// r_cap rows per SM covers N, else a multiple of the SM count). A launch
// with one CTA fewer than SMs leaves an SM free, which in a chain of
// programmatic dependent launches then takes two CTAs of the next launch
// and finishes it late. Returns the rows of the largest slab.
int even_grid(int64_t N, int64_t r_cap, int sms, int* grid) {
  const int64_t g0 = (N + r_cap - 1) / r_cap;
  int64_t g = g0 <= sms ? sms : (g0 + sms - 1) / sms * sms;
  if (g > N) g = N;
  if (g < 1) g = 1;
  *grid = (int)g;
  return (int)((N + g - 1) / g);
}

bl_status gemv_plan(int64_t N, int64_t K, int M, int sms, int* rows, int* grid, size_t* smem) {
  int64_t r = (N + sms - 1) / sms;
  if (r < 1) r = 1;
  if (r > kGemvMaxRows) r = kGemvMaxRows;
  while (r > 1 && gemv_smem_bytes(K, (int)r, M) > kGemvSmemCap) r = (r + 1) / 2;
  if (gemv_smem_bytes(K, (int)r, M) > kGemvSmemCap) return BL_ERR_SHAPE;
  *rows = even_grid(N, r, sms, grid);
  *smem = gemv_smem_bytes(K, *rows, M);
  return BL_OK;
}

// src: kSrcFloat (a_dtype says f32/bf16), kSrcFfnRequant, kSrcInt8.
// Taps in p (if any) report CTA p.tap_cta; a value past the last CTA (or
// negative) means the last CTA.
bl_status run_gemv(int src, int out, bl_dtype a_dtype, GemvParams p, bool pdl, int dev, int sms,
                   cudaStream_t st, int* grid_out = nullptr) {
  int rows, grid;
  size_t smem;
  BL_TRY(gemv_plan(p.N, p.K, p.M, sms, &rows, &grid, &smem));
  if (grid_out != nullptr) *grid_out = grid;
  if (p.tap_cta < 0 || p.tap_cta >= grid) p.tap_cta = grid - 1;
  p.rows_per_cta = rows;
  p.rows_pad = gemv_rows_pad(rows);
  CUtensorMap tw;
  BL_TRY(make_map_u8(&tw, p.W, (uint64_t)p.N, (uint64_t)(p.K / 4), 128, (uint32_t)p.rows_pad,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  if (src == kSrcFloat) {
    if (a_dtype == BL_BF16) {
      return out == kOutDequant
                 ? launch_gemv_mt<__nv_bfloat16, kSrcFloat, kOutDequant>(tw, p, grid, smem, pdl, dev, st)
                 : launch_gemv_mt<__nv_bfloat16, kSrcFloat, kOutRawI32>(tw, p, grid, smem, pdl, dev, st);
    }
    return out == kOutDequant
               ? launch_gemv_mt<float, kSrcFloat, kOutDequant>(tw, p, grid, smem, pdl, dev, st)
               : launch_gemv_mt<float, kSrcFloat, kOutRawI32>(tw, p, grid, smem, pdl, dev, st);
  }
  if (src == kSrcFfnRequant)
    return out == kOutDequant
               ? launch_gemv_mt<float, kSrcFfnRequant, kOutDequant>(tw, p, grid, smem, pdl, dev, st)
               : launch_gemv_mt<float, kSrcFfnRequant, kOutRawI32>(tw, p, grid, smem, pdl, dev, st);
  return out == kOutDequant
             ? launch_gemv_mt<float, kSrcInt8, kOutDequant>(tw, p, grid, smem, pdl, dev, st)
             : launch_gemv_mt<float, kSrcInt8, kOutRawI32>(tw, p, grid, smem, pdl, dev, st);
}

// --------------------------------------------------------------------------
// Tensor-core launches.
template <int BN, bool DUAL, int OUT>
bl_status launch_tc_t(const CUtensorMap& ta, const CUtensorMap& tw, const CUtensorMap& ty,
                      const TcParams& p, int splits, int dev, cudaStream_t st) {
  auto* k = tc_ternary_gemm_kernel<TcConfig<BN, DUAL>, OUT>;
  constexpr size_t smem = TcConfig<BN, DUAL>::kSmemBytes;
  BL_TRY(ensure_smem(k, dev, smem));
  // Always with programmatic dependent launch: the kernel waits for the
  // previous grid before it touches global memory.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((p.N + 127) / 128), (unsigned)((p.M + BN - 1) / BN), (unsigned)splits);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  BL_CUDA(cudaLaunchKernelEx(&cfg, k, ta, tw, ty, p));
  return BL_OK;
}

// Token tile of a launch: width 128, 192 or 256 (the tensor-core path only
// sees M > 32), one or two CTAs per SM.
struct TcTile {
  int bn;
  bool dual;
};

template <int OUT>
bl_status launch_tc_bn(TcTile t, const CUtensorMap& ta, const CUtensorMap& tw,
                       const CUtensorMap& ty, const TcParams& p, int splits, int dev,
                       cudaStream_t st) {
  if (t.bn == 128)
    return t.dual ? launch_tc_t<128, true, OUT>(ta, tw, ty, p, splits, dev, st)
                  : launch_tc_t<128, false, OUT>(ta, tw, ty, p, splits, dev, st);
  if (t.bn == 192)
    return t.dual ? launch_tc_t<192, true, OUT>(ta, tw, ty, p, splits, dev, st)
                  : launch_tc_t<192, false, OUT>(ta, tw, ty, p, splits, dev, st);
  return launch_tc_t<256, false, OUT>(ta, tw, ty, p, splits, dev, st);
}

// Token tile of K-split launches (and of the partial buffer's row padding).
int tc_split_bn(int64_t M) { return M <= 128 ? 128 : 256; }

// ---------------------------------------------------------------------------
// K ranges for tensor-core launches whose tiles fill at most half of the SMs
// (each range at least 8 K blocks, at most 4 ranges). The ranges write raw
// INT32 partials to an optional workspace part; splitk_reduce_kernel sums
// them (exact) and applies the epilogue.
constexpr int kSplitWsSms = 148;  // B200: the SM count workspaces are sized for

int tc_splits(int64_t M, int64_t N, int64_t K, int sms) {
  const int64_t tiles = ((N + 127) / 128) * ((M + tc_split_bn(M) - 1) / tc_split_bn(M));
  const int64_t KB = (K + kTcBK - 1) / kTcBK;
  if (tiles * 2 > sms) return 1;
  int64_t sp = sms / tiles;
  if (sp > 4) sp = 4;
  const int64_t most = KB / 8;
  if (sp > most) sp = most;
  return sp < 1 ? 1 : (int)sp;
}

// Rows per split in the partial buffer: M rounded up to the token tile.
int64_t tc_split_rows(int64_t M) {
  const int bn = tc_split_bn(M);
  return (M + bn - 1) / bn * bn;
}

size_t tc_split_ws_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= kSkPreferTokens) return 0;
  const int sp = tc_splits(M, N, K, kSplitWsSms);
  return sp > 1 ? align_up((size_t)sp * tc_split_rows(M) * N * 4) : 0;
}

// Token tile of an unsplit launch: the one with the fewest tile-time units,
// rounds of tiles over the SMs × (64 + tile width). A 128 × 256 tile costs
// about the MMAs of its 256 tokens plus a fixed part (expanding the weight
// tile, set-up, epilogue) worth ≈64 tokens; 512 tokens × 11008 rows make 172
// tiles of 256 (two rounds on 148 SMs) but 258 of 192 (also two, each 20 %
// cheaper).
TcTile tc_pick_tile(int64_t M, int64_t N, int sms) {
  if (M <= 128) return TcTile{128, false};
  const int64_t rt = (N + 127) / 128;
  int best = 256;
  int64_t best_cost = -1;
  for (int bn : {256, 192, 128}) {
    const int64_t rounds = (rt * ((M + bn - 1) / bn) + sms - 1) / sms;
    const int64_t cost = rounds * (64 + bn);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  // Two CTAs per SM with 192-token tiles when those fit in one co-resident
  // wave and the best single-CTA tile needs two or more rounds: one CTA's
  // epilogue and set-up then overlap the other's MMAs (512 tokens × 11008
  // rows: 258 tiles; FFN block 65.7 -> 60.8 us). The prefill shape (352
  // tiles of 192) stays on 256-token single tiles (32.4 us vs 37.4 dual).
  const int64_t t192 = rt * ((M + 191) / 192);
  const int64_t tbest = rt * ((M + best - 1) / best);
  if (t192 <= 2 * (int64_t)sms && tbest > sms) return TcTile{192, true};
  return TcTile{best, false};
}

// K ranges a launch gets: the split its tile count asks for, capped by the
// one workspaces are sized for, and 1 without room for the partials.
int tc_launch_splits(int64_t M, int64_t N, int64_t K, int sms, const void* split_ws,
                     size_t split_ws_bytes) {
  int sp = tc_splits(M, N, K, sms);
  const int sp_ws = tc_splits(M, N, K, kSplitWsSms);
  if (sp > sp_ws) sp = sp_ws;
  if (sp > 1 && (split_ws == nullptr || split_ws_bytes < tc_split_ws_bytes(M, N, K))) sp = 1;
  return sp;
}

// acc/Y[M,N] = epilogue(A_q[M,K] · W_q[N,K]ᵀ − rowsum).
bl_status run_tc(const int8_t* Aq, const uint8_t* Wp, int64_t M, int64_t K, int64_t N,
                 const float* gamma, const float* gammaA, const int32_t* rowsum, void* Y,
                 int out, int relu2, int y_bf16, void* split_ws, size_t split_ws_bytes, int dev,
                 int sms, cudaStream_t st, bool w_early = false) {
  if (M > 0x7FFFFFFF || N > 0x7FFFFFFF) return BL_ERR_SHAPE;
  const int KBall = (int)((K + kTcBK - 1) / kTcBK);
  int sp = tc_launch_splits(M, N, K, sms, split_ws, split_ws_bytes);
  const TcTile tile = sp > 1 ? TcTile{tc_split_bn(M), false} : tc_pick_tile(M, N, sms);
  const int bn = tile.bn;
  const int kbs = sp > 1 ? ((KBall + sp - 1) / sp + 3) / 4 * 4 : KBall;
  if (sp > 1) sp = (KBall + kbs - 1) / kbs;  // no empty ranges
  void* Yk = sp > 1 ? split_ws : Y;        // where the kernel writes
  const int outk = sp > 1 ? kTcRawI32 : out;
  CUtensorMap ta, tw;
  BL_TRY(make_map_u8(&ta, Aq, (uint64_t)M, (uint64_t)K, kTcBK, (uint32_t)bn,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  BL_TRY(make_map_u8(&tw, Wp, (uint64_t)N, (uint64_t)(K / 4), 128, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  // Output tensor map for the staged tensor-store epilogue (rows of N
  // elements must be a multiple of 16 bytes); split partials are [sp·M, N].
  const int esz = (outk == kTcRawI32 || !y_bf16) ? 4 : 2;
  CUtensorMap ty;
  std::memset(&ty, 0, sizeof(ty));
  int tma_store = 0;
  if (((uint64_t)N * esz) % 16 == 0) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return BL_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)N, sp > 1 ? (cuuint64_t)(tc_split_rows(M) * sp) : (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)N * esz};
    cuuint32_t box[2] = {128, (cuuint32_t)(bn < 32 ? bn : 32)};  // stored 32 tokens at a time
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&ty, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT32,
                     2, Yk, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return BL_ERR_CUDA;
    tma_store = 1;
  }
  TcParams p;
  p.tma_store = tma_store;
  p.gamma = gamma;
  p.gammaA = gammaA;
  p.rowsum = rowsum;
  p.Y = Yk;
  p.M = M;
  p.N = N;
  p.K = K;
  p.relu2 = relu2;
  p.y_bf16 = y_bf16;
  p.kb_per_split = kbs;
  p.split_rows = sp > 1 ? tc_split_rows(M) : 0;
  p.w_early = w_early ? 1 : 0;
  BL_TRY(outk == kTcDequant ? launch_tc_bn<kTcDequant>(tile, ta, tw, ty, p, sp, dev, st)
                            : launch_tc_bn<kTcRawI32>(tile, ta, tw, ty, p, sp, dev, st));
  if (sp == 1) return BL_OK;
  BL_TRY(ensure_smem(splitk_reduce_kernel, dev, 0));
  // With programmatic dependent launch: the reduce waits for the partials
  // (the kernel's first step) and its launch overlaps the contraction's tail.
  BL_TRY(launch_pdl(splitk_reduce_kernel, dim3((unsigned)((N + 1023) / 1024), (unsigned)M), dim3(256),
                    st, reinterpret_cast<const int32_t*>(Yk), sp, tc_split_rows(M) * N, M, N,
                    out == kTcRawI32 ? 1 : 0, gamma, gammaA, relu2, Y, y_bf16,
                    (N % 4 == 0 && (reinterpret_cast<uintptr_t>(Y) & 15) == 0) ? 1 : 0));
  return BL_OK;
}

// --------------------------------------------------------------------------
// Skinny launches (5 ≤ M ≤ 64 tokens, mma.sync over all SMs).
template <int MTT, int NTW, int KPS>
bl_status launch_skinny_t(const CUtensorMap& tw, const CUtensorMap& ta, const SkinnyParams& p,
                          int grid, size_t smem, bool pdl, int dev, cudaStream_t st) {
  auto* k = skinny_ternary_kernel<MTT, NTW, KPS>;
  BL_TRY(ensure_smem(k, dev, smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kSkThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  BL_CUDA(cudaLaunchKernelEx(&cfg, k, tw, ta, p));
  return BL_OK;
}

// Instantiated warp splits (NTW n-tiles per warp, KPS 32-K steps per warp
// and stage). With 16 warps, KPS n-tile groups cover KPS·NTW n-tiles.
struct SkinnySplit {
  int ntw, kps;
};
constexpr SkinnySplit kSkSplits[] = {{1, 2}, {2, 2}, {3, 2}, {5, 2}, {2, 4}, {3, 4}, {4, 4}};

template <int MTT>
bl_status launch_skinny_split(SkinnySplit sp, const CUtensorMap& tw, const CUtensorMap& ta,
                              const SkinnyParams& p, int grid, size_t smem, bool pdl, int dev,
                              cudaStream_t st) {
  if (sp.kps == 2) {
    switch (sp.ntw) {
      case 1: return launch_skinny_t<MTT, 1, 2>(tw, ta, p, grid, smem, pdl, dev, st);
      case 2: return launch_skinny_t<MTT, 2, 2>(tw, ta, p, grid, smem, pdl, dev, st);
      case 3: return launch_skinny_t<MTT, 3, 2>(tw, ta, p, grid, smem, pdl, dev, st);
      default:
        if constexpr (MTT <= 2) return launch_skinny_t<MTT, 5, 2>(tw, ta, p, grid, smem, pdl, dev, st);
        return BL_ERR_SHAPE;
    }
  }
  switch (sp.ntw) {
    case 2: return launch_skinny_t<MTT, 2, 4>(tw, ta, p, grid, smem, pdl, dev, st);
    case 3: return launch_skinny_t<MTT, 3, 4>(tw, ta, p, grid, smem, pdl, dev, st);
    default: return launch_skinny_t<MTT, 4, 4>(tw, ta, p, grid, smem, pdl, dev, st);
  }
}

inline int skinny_mtt(int64_t M) { return M <= 16 ? 1 : (M <= 32 ? 2 : 4); }

// Rows per CTA: one wave over the SMs (8..128 rows). The warp split
// minimises a cycle estimate per CTA: per stage the larger of the mma.sync
// time (≈2.2 SM cycles per m16n8k32, measured with the step loop unrolled)
// and the shared-memory time (a 512-byte ldmatrix per token fragment, 64
// bytes per weight fragment, 128 bytes per cycle), plus writing and reading
// the K-lanes' partial sums once. The ring is as deep as shared memory
// allows.
bl_status skinny_plan(int64_t M, int64_t N, int64_t K, int sms, SkinnyParams* p,
                      SkinnySplit* split, int* grid, size_t* smem) {
  const int mtt = skinny_mtt(M);
  int64_t r = (N + sms - 1) / sms;
  if (r < 8) r = 8;
  if (r > kSkMaxRowsPad) r = kSkMaxRowsPad;
  if ((N & 1) == 0 && (r & 1) != 0) ++r;  // even rows per CTA: paired output stores
  const int nt = (int)((r + 7) / 8);
  const int rp = nt * 8;
  const int nchunk = skinny_chunks(K);
  SkinnySplit best = {0, 0};
  double best_cost = 1e30;
  for (const SkinnySplit& sp : kSkSplits) {
    if (sp.ntw * sp.kps < nt) continue;      // n-tiles not covered
    if (sp.ntw * mtt > 16) continue;         // accumulator registers
    if (mtt == 4 && sp.ntw > 4) continue;    // not instantiated
    const double t_mma = (double)kSkWarps * sp.kps * sp.ntw * mtt * 2.2;
    const double t_smem = (double)kSkWarps * sp.kps * (4.0 * mtt + sp.ntw / 2.0);
    const double cost = nchunk * (t_mma > t_smem ? t_mma : t_smem) +
                        2.0 * (double)skinny_red_bytes(sp.ntw, mtt) / 128.0;
    if (cost < best_cost) {
      best_cost = cost;
      best = sp;
    }
  }
  if (best.ntw == 0) return BL_ERR_SHAPE;
  int stages = nchunk;
  while (stages > 1 && skinny_smem_bytes(rp, mtt, stages, best.ntw) > kSkSmemCap) --stages;
  if (skinny_smem_bytes(rp, mtt, stages, best.ntw) > kSkSmemCap) return BL_ERR_SHAPE;
  if (stages < 2 && nchunk > 1) return BL_ERR_SHAPE;
  p->rows_per_cta = (int)r;
  p->rows_pad = rp;
  p->stages = stages;
  *split = best;
  *grid = (int)((N + r - 1) / r);
  *smem = skinny_smem_bytes(rp, mtt, stages, best.ntw);
  return BL_OK;
}

// acc/Y[M,N] = epilogue(A_q[M,K] · W_q[N,K]ᵀ − rowsum) for 5 ≤ M ≤ 64.
// pdl: the preceding kernel on the stream does not write W_packed or gamma.
bl_status run_skinny(const int8_t* Aq, const uint8_t* Wp, int64_t M, int64_t K, int64_t N,
                     const float* gamma, const float* gammaA, const int32_t* rowsum, void* Y,
                     int raw, int relu2, int y_bf16, bool pdl, int dev, int sms,
                     cudaStream_t st) {
  SkinnyParams p = {};
  SkinnySplit split;
  int grid;
  size_t smem;
  BL_TRY(skinny_plan(M, N, K, sms, &p, &split, &grid, &smem));
  const int mtt = skinny_mtt(M);
  CUtensorMap tw, ta;
  BL_TRY(make_map_u8(&tw, Wp, (uint64_t)N, (uint64_t)(K / 4), 128, (uint32_t)p.rows_pad,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  BL_TRY(make_map_u8(&ta, Aq, (uint64_t)M, (uint64_t)K, 128, (uint32_t)(16 * mtt),
                     CU_TENSOR_MAP_SWIZZLE_128B));
  p.gamma = gamma;
  p.gammaA = gammaA;
  p.rowsum = rowsum;
  p.Y = Y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.relu2 = relu2;
  p.y_bf16 = y_bf16;
  p.raw = raw;
  if (mtt == 1) return launch_skinny_split<1>(split, tw, ta, p, grid, smem, pdl, dev, st);
  if (mtt == 2) return launch_skinny_split<2>(split, tw, ta, p, grid, smem, pdl, dev, st);
  return launch_skinny_split<4>(split, tw, ta, p, grid, smem, pdl, dev, st);
}

// Contraction of pre-quantised tokens: the skinny kernel up to 32 tokens,
// tensor-core tiles above 64. From 33 to 64 tokens the skinny kernel needs
// four 16-token m-tiles and costs what 64 tokens cost, while a 128-token tile
// costs about the same for any M ≤ 128, so the tiles take the call when they
// (times their K ranges) fill at least half of the SMs; otherwise the
// skinny kernel's spread over every SM wins. Measured in chains at 48-64
// tokens: 4096 -> 11008 (86 tiles) 15.2 us on tiles against 16.1 skinny;
// 11008 -> 4096 (32 tiles × 4 K ranges) 16.3-17.3 against 17.8-17.9; a
// 5504 -> 4096 shard without split workspace (32 tiles) ran slower on tiles.
// split_ws: optional scratch (tc_split_ws_bytes) that lets under-filled
// tensor-core launches split K.
bool contract_on_tiles(int64_t M, int64_t N, int64_t K, int sms, const void* split_ws,
                       size_t split_ws_bytes) {
  if (M > kSkMaxTokens) return true;
  return M > kSkPreferTokens &&
         2 * ((N + 127) / 128) * tc_launch_splits(M, N, K, sms, split_ws, split_ws_bytes) >= sms;
}

bl_status run_contract(const int8_t* Aq, const uint8_t* Wp, int64_t M, int64_t K, int64_t N,
                       const float* gamma, const float* gammaA, const int32_t* rowsum, void* Y,
                       int out, int relu2, int y_bf16, bool pdl, int dev, int sms,
                       cudaStream_t st, void* split_ws = nullptr, size_t split_ws_bytes = 0) {
  if (!contract_on_tiles(M, N, K, sms, split_ws, split_ws_bytes))
    return run_skinny(Aq, Wp, M, K, N, gamma, gammaA, rowsum, Y, out == kTcRawI32 ? 1 : 0, relu2,
                      y_bf16, pdl, dev, sms, st);
  return run_tc(Aq, Wp, M, K, N, gamma, gammaA, rowsum, Y, out, relu2, y_bf16, split_ws,
                split_ws_bytes, dev, sms, st, pdl);
}

// pdl: launch with programmatic dependent launch (the kernel waits for the
// previous grid before it touches global memory), so in a chain it is
// resident and ready when its predecessor completes.
bl_status run_quant_acts(const void* A, bl_dtype dt, int64_t M, int64_t K, float eps, int8_t* Aq,
                         float* gA, int32_t* rs, cudaStream_t st, bool pdl = false) {
  if (M == 0) return BL_OK;
  int dev;
  BL_CUDA(cudaGetDevice(&dev));
  BL_TRY(dt == BL_BF16 ? ensure_smem(quant_acts_kernel<__nv_bfloat16>, dev, 0)
                       : ensure_smem(quant_acts_kernel<float>, dev, 0));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)M);
  cfg.blockDim = dim3(kQuantThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (dt == BL_BF16)
    BL_CUDA(cudaLaunchKernelEx(&cfg, quant_acts_kernel<__nv_bfloat16>,
                               reinterpret_cast<const __nv_bfloat16*>(A), K, eps, Aq, gA, rs));
  else
    BL_CUDA(cudaLaunchKernelEx(&cfg, quant_acts_kernel<float>, reinterpret_cast<const float*>(A), K,
                               eps, Aq, gA, rs));
  return BL_OK;
}

// --------------------------------------------------------------------------
// Radix-3 decode GEMV launch.
template <int MT, typename TA>
bl_status launch_r3_t(const CUtensorMap& tw, const GemvR3Params& p, int grid, size_t smem, bool pdl,
                      int dev, cudaStream_t st) {
  auto* k = gemv_r3_kernel<MT, TA>;
  BL_TRY(ensure_smem(k, dev, smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  BL_CUDA(cudaLaunchKernelEx(&cfg, k, tw, p));
  return BL_OK;
}

bl_status run_r3(bl_dtype a_dtype, GemvR3Params p, bool pdl, int dev, int sms, cudaStream_t st) {
  // Two CTAs per SM when the token coefficients leave room, else one.
  const size_t cap = gemv_r3_smem_bytes(p.rb, 8, p.M) <= kGemvSmemCap ? kGemvSmemCap : kSkSmemCap;
  int64_t r = (p.N + sms - 1) / sms;
  if (r < 1) r = 1;
  if (r > kGemvMaxRows) r = kGemvMaxRows;
  while (r > 1 && gemv_r3_smem_bytes(p.rb, (int)r, p.M) > cap) r = (r + 1) / 2;
  if (gemv_r3_smem_bytes(p.rb, (int)r, p.M) > cap) return BL_ERR_SHAPE;
  int grid;
  p.rows_per_cta = even_grid(p.N, r, sms, &grid);
  p.rows_pad = gemv_rows_pad(p.rows_per_cta);
  const size_t smem = gemv_r3_smem_bytes(p.rb, p.rows_per_cta, p.M);
  CUtensorMap tw;
  BL_TRY(make_map_u8(&tw, p.W, (uint64_t)p.N, (uint64_t)p.rb, 128, (uint32_t)p.rows_pad,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  const bool bf = a_dtype == BL_BF16;
  if (p.M == 1)
    return bf ? launch_r3_t<1, __nv_bfloat16>(tw, p, grid, smem, pdl, dev, st)
              : launch_r3_t<1, float>(tw, p, grid, smem, pdl, dev, st);
  if (p.M == 2)
    return bf ? launch_r3_t<2, __nv_bfloat16>(tw, p, grid, smem, pdl, dev, st)
              : launch_r3_t<2, float>(tw, p, grid, smem, pdl, dev, st);
  return bf ? launch_r3_t<4, __nv_bfloat16>(tw, p, grid, smem, pdl, dev, st)
            : launch_r3_t<4, float>(tw, p, grid, smem, pdl, dev, st);
}

// --------------------------------------------------------------------------
// Lookup-table decode GEMV launch (one token).
template <typename TA>
bl_status launch_lut_t(const CUtensorMap& tw, const GemvLutParams& p, int grid, size_t smem,
                       bool pdl, int dev, cudaStream_t st) {
  auto* k = gemv_lut_kernel<TA>;
  BL_TRY(ensure_smem(k, dev, smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  BL_CUDA(cudaLaunchKernelEx(&cfg, k, tw, p));
  return BL_OK;
}

// --------------------------------------------------------------------------
// STE backward: bf16 GEMM launches and layouts.

// 2-D bf16 tensor [rows, cols] with row stride ld elements (ld·2 a multiple
// of 16 bytes), 64 × box_rows boxes, 128-byte swizzle.
bl_status make_map_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                        uint64_t ld, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return BL_ERR_CUDA;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)kGmBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BL_OK : BL_ERR_CUDA;
}

template <int BN, bool MASK, bool DUAL, int MAJ>
bl_status launch_gemm_t(const CUtensorMap& ta, const CUtensorMap& tb, const GmParams& p, int dev,
                        cudaStream_t st) {
  auto* k = bf16_gemm_kernel<BN, MASK, DUAL, MAJ>;
  constexpr size_t smem = GmConfig<BN, DUAL>::kSmem;
  BL_TRY(ensure_smem(k, dev, smem));
  const dim3 grid((unsigned)((p.rows + kGmBM - 1) / kGmBM), (unsigned)((p.cols + BN - 1) / BN));
  k<<<grid, kGmThreads, smem, st>>>(ta, tb, p);
  BL_CUDA(cudaGetLastError());
  return BL_OK;
}

template <int MAJ, bool MASK>
bl_status launch_gemm_form(const CUtensorMap& ta, const CUtensorMap& tb, const GmParams& p,
                           bool wide, bool dual, int dev, cudaStream_t st) {
  if (dual) return launch_gemm_t<256, MASK, true, MAJ>(ta, tb, p, dev, st);
  if (wide) return launch_gemm_t<256, MASK, false, MAJ>(ta, tb, p, dev, st);
  return launch_gemm_t<128, MASK, false, MAJ>(ta, tb, p, dev, st);
}

// C[rows, cols] (fp32) = epilogue(A · Bᵀ) over kdim, A and B bf16 with row
// strides lda, ldb elements. The two forms the STE backward uses:
//   maj = kMajBMN, no mask: A [rows, kdim], B stored [kdim, cols] (dA);
//   maj = kMajAMN | kMajBMN, mask: A stored [kdim, rows], B [kdim, cols] (dW).
bl_status run_bf16_gemm(const void* A, int64_t lda, const void* B, int64_t ldb, GmParams p,
                        int maj, int dev, cudaStream_t st) {
  if (p.rows > (int64_t)65535 * kGmBM) return BL_ERR_SHAPE;
  const bool mask = p.mask_w != nullptr;
  if (maj != (mask ? (kMajAMN | kMajBMN) : kMajBMN)) return BL_ERR_UNSUPPORTED;
  const bool wide = p.cols >= 256;
  CUtensorMap ta, tb;
  if (maj & kMajAMN)
    BL_TRY(make_map_bf16(&ta, A, (uint64_t)p.kdim, (uint64_t)p.rows, (uint64_t)lda, kGmBK));
  else
    BL_TRY(make_map_bf16(&ta, A, (uint64_t)p.rows, (uint64_t)p.kdim, (uint64_t)lda, kGmBM));
  BL_TRY(make_map_bf16(&tb, B, (uint64_t)p.kdim, (uint64_t)p.cols, (uint64_t)ldb, kGmBK));
  // More tiles than SMs: two CTAs per SM (two stages each), so one CTA's
  // epilogue overlaps the other's MMAs (2048 x 4096 x 4096: dA 69.4 -> 67.9 us,
  // dW 98.6 -> 96.7 us; 128-wide tiles two per SM were slower).
  int dev_sms = 0;
  BL_CUDA(cudaDeviceGetAttribute(&dev_sms, cudaDevAttrMultiProcessorCount, dev));
  const int64_t tiles = ((p.rows + kGmBM - 1) / kGmBM) * ((p.cols + 255) / 256);
  const bool dual = wide && tiles > dev_sms;
  return mask ? launch_gemm_form<kMajAMN | kMajBMN, true>(ta, tb, p, wide, dual, dev, st)
              : launch_gemm_form<kMajBMN, false>(ta, tb, p, wide, dual, dev, st);
}

inline int64_t round8(int64_t x) { return (x + 7) / 8 * 8; }

// Taps: argument checks and device-to-device copies of workspace pieces.
bl_status check_taps(const bl_taps* t, bool ffn) {
  if (t == nullptr) return BL_OK;
  if (t->reserved != 0) return BL_ERR_INVALID_ARG;
  if (!ffn && (t->acc_up || t->req_q || t->req_gamma || t->req_rowsum)) return BL_ERR_INVALID_ARG;
  const void* ptrs[] = {t->act_q, t->act_gamma, t->act_rowsum, t->acc_up,
                        t->req_q, t->req_gamma, t->req_rowsum};
  for (const void* q : ptrs)
    if (q != nullptr && !aligned16(q)) return BL_ERR_ALIGN;
  return BL_OK;
}

bl_status tap_copy(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (dst == nullptr || bytes == 0) return BL_OK;
  BL_CUDA(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st));
  return BL_OK;
}

// Points the GEMV prologue taps of p at (q, gamma, rowsum) when all are set.
void gemv_taps(GemvParams& p, int8_t* q, float* gamma, int32_t* rowsum, int cta) {
  if (q != nullptr && gamma != nullptr && rowsum != nullptr) {
    p.tap_q = q;
    p.tap_gamma = gamma;
    p.tap_rowsum = rowsum;
    p.tap_cta = cta;
  }
}

}  // namespace
}  // namespace bl

using namespace bl;

// ==========================================================================
// Public C ABI
// ==========================================================================
extern "C" {

const char* bl_status_string(bl_status s) {
  switch (s) {
    case BL_OK: return "BL_OK";
    case BL_ERR_INVALID_ARG: return "BL_ERR_INVALID_ARG: null pointer, bad eps, flag or value";
    case BL_ERR_SHAPE: return "BL_ERR_SHAPE: size negative, too large, or K/H not a positive multiple of 64";
    case BL_ERR_ALIGN: return "BL_ERR_ALIGN: pointer not 16-byte aligned";
    case BL_ERR_DTYPE: return "BL_ERR_DTYPE: dtype not supported for this argument";
    case BL_ERR_CUDA: return "BL_ERR_CUDA: CUDA call or kernel launch failed";
    case BL_ERR_TIMEOUT: return "BL_ERR_TIMEOUT: a device-side bounded wait gave up";
    case BL_ERR_UNSUPPORTED: return "BL_ERR_UNSUPPORTED: device is not sm_100 (B200)";
    case BL_ERR_WORKSPACE: return "BL_ERR_WORKSPACE: workspace missing or too small";
  }
  return "BL_ERR_UNKNOWN";
}

int bl_version(void) { return 100; }

int bl_gemv_max_tokens(void) { return kGemvMaxTokens; }

int bl_contraction_path(int64_t M, int64_t N, int64_t K, int sms, size_t split_ws_bytes) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 64 != 0 || sms <= 0) return -1;
  if (gemv_path(M, K)) return 0;
  // Any non-null pointer stands for a workspace part of split_ws_bytes.
  const void* ws = split_ws_bytes > 0 ? reinterpret_cast<const void*>(&split_ws_bytes) : nullptr;
  if (!contract_on_tiles(M, N, K, sms, ws, split_ws_bytes)) return 1;
  return tc_launch_splits(M, N, K, sms, ws, split_ws_bytes) > 1 ? 3 : 2;
}

size_t bl_quant_weights_workspace_bytes(int64_t N, int64_t K) {
  (void)N;
  (void)K;
  return (size_t)kAbsmeanMaxBlocks * sizeof(double);
}

bl_status bl_quant_weights(const void* W, bl_dtype w_dtype, int64_t N, int64_t K, float eps,
                           uint8_t* W_packed, float* gamma, void* workspace, size_t ws_bytes,
                           bl_stream_t stream) {
  BL_TRY(check_dtype(w_dtype));
  BL_TRY(check_k(K));
  BL_TRY(check_rows(N));
  BL_TRY(check_eps(eps));
  if (N == 0) return BL_OK;
  BL_TRY(check_ptr(W));
  BL_TRY(check_ptr(W_packed));
  if (gamma == nullptr) return BL_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(gamma) & 3u) != 0) return BL_ERR_ALIGN;
  if (workspace == nullptr || ws_bytes < bl_quant_weights_workspace_bytes(N, K))
    return BL_ERR_WORKSPACE;
  BL_TRY(check_ptr(workspace));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t count = N * K;
  const int vec = w_dtype == BL_BF16 ? 8 : 4;
  const int64_t nvec = count / vec;
  int64_t blocks = (nvec + kQuantThreads - 1) / kQuantThreads;
  if (blocks > kAbsmeanMaxBlocks) blocks = kAbsmeanMaxBlocks;
  if (blocks > 8 * (int64_t)sms) blocks = 8 * (int64_t)sms;
  double* partials = reinterpret_cast<double*>(workspace);
  const int64_t nwords = count / 16;
  int64_t pblocks = (nwords + kQuantThreads - 1) / kQuantThreads;
  if (pblocks > 16 * (int64_t)sms) pblocks = 16 * (int64_t)sms;
  if (w_dtype == BL_BF16) {
    auto* Wt = reinterpret_cast<const __nv_bfloat16*>(W);
    absmean_partial_kernel<__nv_bfloat16><<<(unsigned)blocks, kQuantThreads, 0, st>>>(Wt, count, partials);
    BL_CUDA(cudaGetLastError());
    ternary_pack_kernel<__nv_bfloat16><<<(unsigned)pblocks, kQuantThreads, 0, st>>>(
        Wt, nwords, (double)count, eps, partials, (int)blocks,
        reinterpret_cast<uint32_t*>(W_packed), gamma);
  } else {
    auto* Wt = reinterpret_cast<const float*>(W);
    absmean_partial_kernel<float><<<(unsigned)blocks, kQuantThreads, 0, st>>>(Wt, count, partials);
    BL_CUDA(cudaGetLastError());
    ternary_pack_kernel<float><<<(unsigned)pblocks, kQuantThreads, 0, st>>>(
        Wt, nwords, (double)count, eps, partials, (int)blocks,
        reinterpret_cast<uint32_t*>(W_packed), gamma);
  }
  BL_CUDA(cudaGetLastError());
  return BL_OK;
}

bl_status bl_quant_acts(const void* A, bl_dtype a_dtype, int64_t M, int64_t K, float eps,
                        int8_t* A_q, float* gamma_A, int32_t* rowsum, bl_stream_t stream) {
  BL_TRY(check_dtype(a_dtype));
  BL_TRY(check_k(K));
  BL_TRY(check_rows(M));
  BL_TRY(check_eps(eps));
  if (M == 0) return BL_OK;
  BL_TRY(check_ptr(A));
  BL_TRY(check_ptr(A_q));
  BL_TRY(check_ptr(gamma_A));
  if (rowsum != nullptr) BL_TRY(check_ptr(rowsum));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  return run_quant_acts(A, a_dtype, M, K, eps, A_q, gamma_A, rowsum,
                        reinterpret_cast<cudaStream_t>(stream));
}

size_t bl_zero_gemm_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  if (gemv_path(M, K)) return 0;
  return align_up((size_t)M * 4) + tc_split_ws_bytes(M, N, K);
}

bl_status bl_zero_gemm(const int8_t* A_q, int64_t M, int64_t K, const uint8_t* W_packed,
                       int64_t N, int32_t* acc, void* workspace, size_t ws_bytes,
                       bl_stream_t stream) {
  BL_TRY(check_k(K));
  BL_TRY(check_rows(M));
  BL_TRY(check_rows(N));
  if (M == 0 || N == 0) return BL_OK;
  BL_TRY(check_ptr(A_q));
  BL_TRY(check_ptr(W_packed));
  BL_TRY(check_ptr(acc));
  // Required: the row sums; the rest of bl_zero_gemm_workspace_bytes (K
  // ranges of under-filled tensor-core launches) is used when present.
  const size_t need = gemv_path(M, K) ? 0 : align_up((size_t)M * 4);
  if (need > 0) {
    if (workspace == nullptr || ws_bytes < need) return BL_ERR_WORKSPACE;
    BL_TRY(check_ptr(workspace));
  }
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (gemv_path(M, K)) {
    GemvParams p = {};
    p.A = A_q;
    p.W = W_packed;
    p.Y = acc;
    p.N = N;
    p.K = K;
    p.M = (int)M;
    p.eps = 1.0f;
    return run_gemv(kSrcInt8, kOutRawI32, BL_F32, p, false, dev, sms, st);
  }
  int32_t* rs = reinterpret_cast<int32_t*>(workspace);
  rowsum_i8_kernel<<<(unsigned)M, kQuantThreads, 0, st>>>(A_q, K, rs);
  BL_CUDA(cudaGetLastError());
  return run_contract(A_q, W_packed, M, K, N, nullptr, nullptr, rs, acc, kTcRawI32, 0, 0, true,
                      dev, sms, st, reinterpret_cast<uint8_t*>(workspace) + align_up((size_t)M * 4),
                      ws_bytes - align_up((size_t)M * 4));
}

size_t bl_linear_q_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  if (gemv_path(M, K)) return 0;
  return align_up((size_t)M * 4) + tc_split_ws_bytes(M, N, K);
}

bl_status bl_linear_q(const int8_t* A_q, const float* gamma_A, const int32_t* rowsum, int64_t M,
                      int64_t K, const uint8_t* W_packed, const float* gamma, int64_t N, int relu2,
                      void* Y, bl_dtype y_dtype, void* workspace, size_t ws_bytes,
                      bl_stream_t stream) {
  return bl_linear_q_ex(A_q, gamma_A, rowsum, M, K, W_packed, gamma, N, relu2, Y, y_dtype,
                        workspace, ws_bytes, 0u, stream);
}

bl_status bl_linear_q_ex(const int8_t* A_q, const float* gamma_A, const int32_t* rowsum,
                         int64_t M, int64_t K, const uint8_t* W_packed, const float* gamma,
                         int64_t N, int relu2, void* Y, bl_dtype y_dtype, void* workspace,
                         size_t ws_bytes, unsigned flags, bl_stream_t stream) {
  if ((flags & ~(unsigned)BL_FLAG_PDL) != 0) return BL_ERR_INVALID_ARG;
  const bool pdl = (flags & BL_FLAG_PDL) != 0;
  BL_TRY(check_dtype(y_dtype));
  BL_TRY(check_k(K));
  BL_TRY(check_rows(M));
  BL_TRY(check_rows(N));
  if (M == 0 || N == 0) return BL_OK;
  BL_TRY(check_ptr(A_q));
  BL_TRY(check_ptr(gamma_A));
  if (rowsum != nullptr) BL_TRY(check_ptr(rowsum));
  BL_TRY(check_ptr(W_packed));
  if (gamma == nullptr) return BL_ERR_INVALID_ARG;
  BL_TRY(check_ptr(Y));
  // The row sums' part is needed only without rowsum; the rest (K ranges of
  // under-filled tensor-core launches) is used when present.
  const size_t need = (rowsum || gemv_path(M, K)) ? 0 : align_up((size_t)M * 4);
  if (need > 0 && (workspace == nullptr || ws_bytes < need)) return BL_ERR_WORKSPACE;
  if (workspace != nullptr) BL_TRY(check_ptr(workspace));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (gemv_path(M, K)) {
    GemvParams p = {};
    p.A = A_q;
    p.a_scale = gamma_A;
    p.a_rowsum = rowsum;
    p.W = W_packed;
    p.gamma = gamma;
    p.Y = Y;
    p.N = N;
    p.K = K;
    p.M = (int)M;
    p.eps = 1.0f;
    p.relu2 = relu2 ? 1 : 0;
    p.y_bf16 = y_dtype == BL_BF16;
    return run_gemv(kSrcInt8, kOutDequant, BL_F32, p, pdl, dev, sms, st);
  }
  const int32_t* rs = rowsum;
  if (rs == nullptr) {
    int32_t* w = reinterpret_cast<int32_t*>(workspace);
    rowsum_i8_kernel<<<(unsigned)M, kQuantThreads, 0, st>>>(A_q, K, w);
    BL_CUDA(cudaGetLastError());
    rs = w;
  }
  // After this call's row-sum kernel the weights may stream early; without
  // it the preceding kernel is the caller's: early only with BL_FLAG_PDL.
  const size_t rs_part = align_up((size_t)M * 4);
  void* split_ws = (workspace != nullptr && ws_bytes > rs_part)
                       ? reinterpret_cast<uint8_t*>(workspace) + rs_part : nullptr;
  return run_contract(A_q, W_packed, M, K, N, gamma, gamma_A, rs, Y, kTcDequant, relu2 ? 1 : 0,
                      y_dtype == BL_BF16, pdl || rowsum == nullptr, dev, sms, st, split_ws,
                      split_ws ? ws_bytes - rs_part : 0);
}

size_t bl_linear_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  if (gemv_path(M, K)) return 0;
  return act_ws(M, K).total + tc_split_ws_bytes(M, N, K);
}

static bl_status linear_impl(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                             const uint8_t* W_packed, const float* gamma, int64_t N, float eps,
                             int relu2, void* Y, bl_dtype y_dtype, void* workspace,
                             size_t ws_bytes, unsigned flags, const bl_taps* taps,
                             cudaStream_t st) {
  BL_TRY(check_dtype(a_dtype));
  BL_TRY(check_dtype(y_dtype));
  BL_TRY(check_k(K));
  BL_TRY(check_rows(M));
  BL_TRY(check_rows(N));
  BL_TRY(check_eps(eps));
  BL_TRY(check_taps(taps, false));
  if ((flags & ~(unsigned)BL_FLAG_PDL) != 0) return BL_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return BL_OK;
  BL_TRY(check_ptr(A));
  BL_TRY(check_ptr(W_packed));
  if (gamma == nullptr) return BL_ERR_INVALID_ARG;
  BL_TRY(check_ptr(Y));
  // Required: the quantised tokens; the rest of bl_linear_workspace_bytes (K
  // ranges of under-filled tensor-core launches) is used when present.
  const size_t need = gemv_path(M, K) ? 0 : act_ws(M, K).total;
  if (need > 0) {
    if (workspace == nullptr || ws_bytes < need) return BL_ERR_WORKSPACE;
    BL_TRY(check_ptr(workspace));
  }
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  if (gemv_path(M, K)) {
    GemvParams p = {};
    p.A = A;
    p.W = W_packed;
    p.gamma = gamma;
    p.Y = Y;
    p.N = N;
    p.K = K;
    p.M = (int)M;
    p.eps = eps;
    p.relu2 = relu2 ? 1 : 0;
    p.y_bf16 = y_dtype == BL_BF16;
    if (taps) gemv_taps(p, taps->act_q, taps->act_gamma, taps->act_rowsum, taps->cta);
    return run_gemv(kSrcFloat, kOutDequant, a_dtype, p, (flags & BL_FLAG_PDL) != 0, dev, sms, st);
  }
  const ActWs w = act_ws(M, K);
  uint8_t* base = reinterpret_cast<uint8_t*>(workspace);
  int8_t* Aq = reinterpret_cast<int8_t*>(base + w.aq);
  float* gA = reinterpret_cast<float*>(base + w.gamma);
  int32_t* rs = reinterpret_cast<int32_t*>(base + w.rowsum);
  BL_TRY(run_quant_acts(A, a_dtype, M, K, eps, Aq, gA, rs, st, (flags & BL_FLAG_PDL) != 0));
  BL_TRY(run_contract(Aq, W_packed, M, K, N, gamma, gA, rs, Y, kTcDequant, relu2 ? 1 : 0,
                      y_dtype == BL_BF16, true, dev, sms, st, base + w.total, ws_bytes - w.total));
  if (taps) {
    BL_TRY(tap_copy(taps->act_q, Aq, (size_t)M * K, st));
    BL_TRY(tap_copy(taps->act_gamma, gA, (size_t)M * 4, st));
    BL_TRY(tap_copy(taps->act_rowsum, rs, (size_t)M * 4, st));
  }
  return BL_OK;
}

bl_status bl_linear_ex(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                       const uint8_t* W_packed, const float* gamma, int64_t N, float eps,
                       int relu2, void* Y, bl_dtype y_dtype, void* workspace, size_t ws_bytes,
                       unsigned flags, bl_stream_t stream) {
  return linear_impl(A, a_dtype, M, K, W_packed, gamma, N, eps, relu2, Y, y_dtype, workspace,
                     ws_bytes, flags, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

bl_status bl_linear_taps(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                         const uint8_t* W_packed, const float* gamma, int64_t N, float eps,
                         int relu2, void* Y, bl_dtype y_dtype, void* workspace, size_t ws_bytes,
                         unsigned flags, const bl_taps* taps, bl_stream_t stream) {
  return linear_impl(A, a_dtype, M, K, W_packed, gamma, N, eps, relu2, Y, y_dtype, workspace,
                     ws_bytes, flags, taps, reinterpret_cast<cudaStream_t>(stream));
}

bl_status bl_linear(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                    const uint8_t* W_packed, const float* gamma, int64_t N, float eps, int relu2,
                    void* Y, bl_dtype y_dtype, void* workspace, size_t ws_bytes,
                    bl_stream_t stream) {
  return bl_linear_ex(A, a_dtype, M, K, W_packed, gamma, N, eps, relu2, Y, y_dtype, workspace,
                      ws_bytes, 0u, stream);
}

size_t bl_ffn_workspace_bytes(int64_t M, int64_t K, int64_t H) {
  const size_t up = tc_split_ws_bytes(M, H, K), down = tc_split_ws_bytes(M, K, H);
  return ffn_ws(M, K, H).total + (up > down ? up : down);
}

static bl_status ffn_impl(const void* X, bl_dtype x_dtype, int64_t M, int64_t K, int64_t H,
                          const uint8_t* W_up, const float* gamma_up, const uint8_t* W_down,
                          const float* gamma_down, float eps, void* Y, bl_dtype y_dtype,
                          void* workspace, size_t ws_bytes, const bl_taps* taps, unsigned flags,
                          cudaStream_t st) {
  if ((flags & ~(unsigned)BL_FLAG_PDL) != 0) return BL_ERR_INVALID_ARG;
  const bool pdl = (flags & BL_FLAG_PDL) != 0;
  BL_TRY(check_dtype(x_dtype));
  BL_TRY(check_dtype(y_dtype));
  BL_TRY(check_k(K));
  BL_TRY(check_k(H));
  BL_TRY(check_rows(M));
  BL_TRY(check_eps(eps));
  BL_TRY(check_taps(taps, true));
  if (M == 0) return BL_OK;
  BL_TRY(check_ptr(X));
  BL_TRY(check_ptr(W_up));
  BL_TRY(check_ptr(W_down));
  if (gamma_up == nullptr || gamma_down == nullptr) return BL_ERR_INVALID_ARG;
  BL_TRY(check_ptr(Y));
  const FfnWs w = ffn_ws(M, K, H);
  if (workspace == nullptr || ws_bytes < w.total) return BL_ERR_WORKSPACE;
  BL_TRY(check_ptr(workspace));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  uint8_t* base = reinterpret_cast<uint8_t*>(workspace);
  int32_t* acc_up = reinterpret_cast<int32_t*>(base + w.acc_up);
  if (ffn_gemv_path(M, K, H)) {
    float* gX = reinterpret_cast<float*>(base + w.gamma_x);
    GemvParams up = {};
    up.A = X;
    up.W = W_up;
    up.gamma = gamma_up;
    up.Y = acc_up;
    up.gamma_out = gX;
    up.rmax_out = reinterpret_cast<float*>(base + w.rmax);
    up.N = H;
    up.K = K;
    up.M = (int)M;
    up.eps = eps;
    if (taps) gemv_taps(up, taps->act_q, taps->act_gamma, taps->act_rowsum, taps->cta);
    int up_grid = 0;
    BL_TRY(run_gemv(kSrcFloat, kOutRawI32, x_dtype, up, pdl, dev, sms, st, &up_grid));
    GemvParams dn = {};
    dn.A = acc_up;
    dn.a_scale = gX;
    dn.a_gamma_up = gamma_up;
    dn.rmax_in = up.rmax_out;  // γ_r from the up-projection's per-CTA maxima
    dn.rmax_n = up_grid;
    dn.W = W_down;
    dn.gamma = gamma_down;
    dn.Y = Y;
    dn.N = K;
    dn.K = H;
    dn.M = (int)M;
    dn.eps = eps;
    dn.y_bf16 = y_dtype == BL_BF16;
    if (taps) gemv_taps(dn, taps->req_q, taps->req_gamma, taps->req_rowsum, taps->cta);
    // The kernel before this one is the up-projection above, which does not
    // write W_down: the down-projection may stream its weights early (PDL).
    BL_TRY(run_gemv(kSrcFfnRequant, kOutDequant, BL_F32, dn, true, dev, sms, st));
    if (taps) BL_TRY(tap_copy(taps->acc_up, acc_up, (size_t)M * H * 4, st));
    return BL_OK;
  }
  int8_t* Xq = reinterpret_cast<int8_t*>(base + w.x.aq);
  float* gX = reinterpret_cast<float*>(base + w.x.gamma);
  int32_t* rsX = reinterpret_cast<int32_t*>(base + w.x.rowsum);
  int8_t* Rq = reinterpret_cast<int8_t*>(base + w.rq);
  float* gR = reinterpret_cast<float*>(base + w.gamma_r);
  int32_t* rsR = reinterpret_cast<int32_t*>(base + w.rs_r);
  BL_TRY(run_quant_acts(X, x_dtype, M, K, eps, Xq, gX, rsX, st, pdl));
  // Each contraction follows one of this call's own kernels, which write
  // neither W_up nor W_down: the weights may stream early (PDL).
  void* split_ws = base + w.total;
  const size_t split_bytes = ws_bytes - w.total;
  BL_TRY(run_contract(Xq, W_up, M, K, H, gamma_up, gX, rsX, acc_up, kTcRawI32, 0, 0, true, dev,
                      sms, st, split_ws, split_bytes));
  BL_TRY(ensure_smem(relu2_requant_kernel, dev, 0));
  BL_TRY(launch_pdl(relu2_requant_kernel, dim3((unsigned)M), dim3(kQuantThreads), st, acc_up, H, gX,
                    gamma_up, eps, Rq, gR, rsR));
  BL_TRY(run_contract(Rq, W_down, M, H, K, gamma_down, gR, rsR, Y, kTcDequant, 0,
                      y_dtype == BL_BF16, true, dev, sms, st, split_ws, split_bytes));
  if (taps) {
    BL_TRY(tap_copy(taps->act_q, Xq, (size_t)M * K, st));
    BL_TRY(tap_copy(taps->act_gamma, gX, (size_t)M * 4, st));
    BL_TRY(tap_copy(taps->act_rowsum, rsX, (size_t)M * 4, st));
    BL_TRY(tap_copy(taps->acc_up, acc_up, (size_t)M * H * 4, st));
    BL_TRY(tap_copy(taps->req_q, Rq, (size_t)M * H, st));
    BL_TRY(tap_copy(taps->req_gamma, gR, (size_t)M * 4, st));
    BL_TRY(tap_copy(taps->req_rowsum, rsR, (size_t)M * 4, st));
  }
  return BL_OK;
}

bl_status bl_ffn_relu2(const void* X, bl_dtype x_dtype, int64_t M, int64_t K, int64_t H,
                       const uint8_t* W_up, const float* gamma_up, const uint8_t* W_down,
                       const float* gamma_down, float eps, void* Y, bl_dtype y_dtype,
                       void* workspace, size_t ws_bytes, bl_stream_t stream) {
  return ffn_impl(X, x_dtype, M, K, H, W_up, gamma_up, W_down, gamma_down, eps, Y, y_dtype,
                  workspace, ws_bytes, nullptr, 0u, reinterpret_cast<cudaStream_t>(stream));
}

bl_status bl_ffn_relu2_ex(const void* X, bl_dtype x_dtype, int64_t M, int64_t K, int64_t H,
                          const uint8_t* W_up, const float* gamma_up, const uint8_t* W_down,
                          const float* gamma_down, float eps, void* Y, bl_dtype y_dtype,
                          void* workspace, size_t ws_bytes, unsigned flags, bl_stream_t stream) {
  return ffn_impl(X, x_dtype, M, K, H, W_up, gamma_up, W_down, gamma_down, eps, Y, y_dtype,
                  workspace, ws_bytes, nullptr, flags, reinterpret_cast<cudaStream_t>(stream));
}

bl_status bl_ffn_relu2_taps(const void* X, bl_dtype x_dtype, int64_t M, int64_t K, int64_t H,
                            const uint8_t* W_up, const float* gamma_up, const uint8_t* W_down,
                            const float* gamma_down, float eps, void* Y, bl_dtype y_dtype,
                            void* workspace, size_t ws_bytes, const bl_taps* taps,
                            bl_stream_t stream) {
  return ffn_impl(X, x_dtype, M, K, H, W_up, gamma_up, W_down, gamma_down, eps, Y, y_dtype,
                  workspace, ws_bytes, taps, 0u, reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Tensor-parallel FFN steps (one rank's shard of the hidden dimension).

size_t bl_ffn_tp_up_workspace_bytes(int64_t M, int64_t K) {
  if (gemv_path(M, K)) return 0;
  return align_up((size_t)M * K) + align_up((size_t)M * 4);
}

bl_status bl_ffn_tp_up(const void* X, bl_dtype x_dtype, int64_t M, int64_t K, int64_t H_r,
                       const uint8_t* W_up_r, const float* gamma_up, float eps, int32_t* acc_up,
                       float* gamma_x, float* rmax, void* workspace, size_t ws_bytes,
                       bl_stream_t stream) {
  BL_TRY(check_dtype(x_dtype));
  BL_TRY(check_k(K));
  BL_TRY(check_k(H_r));
  BL_TRY(check_rows(M));
  BL_TRY(check_eps(eps));
  if (M == 0) return BL_OK;
  BL_TRY(check_ptr(X));
  BL_TRY(check_ptr(W_up_r));
  if (gamma_up == nullptr) return BL_ERR_INVALID_ARG;
  BL_TRY(check_ptr(acc_up));
  BL_TRY(check_ptr(gamma_x));
  BL_TRY(check_ptr(rmax));
  const size_t need = bl_ffn_tp_up_workspace_bytes(M, K);
  if (need > 0) {
    if (workspace == nullptr || ws_bytes < need) return BL_ERR_WORKSPACE;
    BL_TRY(check_ptr(workspace));
  }
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (gemv_path(M, K)) {
    GemvParams up = {};
    up.A = X;
    up.W = W_up_r;
    up.gamma = gamma_up;
    up.Y = acc_up;
    up.gamma_out = gamma_x;
    // The shard's largest r per token, raised by every CTA from its rows.
    up.rmax_out = rmax;
    up.rmax_atomic = 1;
    up.N = H_r;
    up.K = K;
    up.M = (int)M;
    up.eps = eps;
    BL_CUDA(cudaMemsetAsync(rmax, 0, (size_t)M * 4, st));
    return run_gemv(kSrcFloat, kOutRawI32, x_dtype, up, false, dev, sms, st);
  } else {
    uint8_t* base = reinterpret_cast<uint8_t*>(workspace);
    int8_t* Xq = reinterpret_cast<int8_t*>(base);
    int32_t* rs = reinterpret_cast<int32_t*>(base + align_up((size_t)M * K));
    BL_TRY(run_quant_acts(X, x_dtype, M, K, eps, Xq, gamma_x, rs, st));
    BL_TRY(run_contract(Xq, W_up_r, M, K, H_r, gamma_up, gamma_x, rs, acc_up, kTcRawI32, 0, 0,
                        true, dev, sms, st));
  }
  relu2_rowmax_kernel<<<(unsigned)M, kQuantThreads, 0, st>>>(acc_up, H_r, gamma_x, gamma_up, rmax);
  BL_CUDA(cudaGetLastError());
  return BL_OK;
}

size_t bl_ffn_tp_down_workspace_bytes(int64_t M, int64_t H_r) {
  return align_up((size_t)M * H_r) + align_up((size_t)M * 4);
}

bl_status bl_ffn_tp_down(const int32_t* acc_up, const float* gamma_x, const float* gamma_up,
                         const float* gamma_r, int64_t M, int64_t H_r, const uint8_t* W_down_r,
                         int64_t K_out, float eps, int32_t* acc_down, void* workspace,
                         size_t ws_bytes, bl_stream_t stream) {
  BL_TRY(check_k(H_r));
  BL_TRY(check_rows(M));
  BL_TRY(check_rows(K_out));
  BL_TRY(check_eps(eps));
  if (M == 0 || K_out == 0) return BL_OK;
  BL_TRY(check_ptr(acc_up));
  BL_TRY(check_ptr(gamma_x));
  BL_TRY(check_ptr(gamma_r));
  if (gamma_up == nullptr) return BL_ERR_INVALID_ARG;
  BL_TRY(check_ptr(W_down_r));
  BL_TRY(check_ptr(acc_down));
  const size_t need = bl_ffn_tp_down_workspace_bytes(M, H_r);
  if (workspace == nullptr || ws_bytes < need) return BL_ERR_WORKSPACE;
  BL_TRY(check_ptr(workspace));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (gemv_path(M, H_r)) {
    // One launch: the GEMV's prologue requantises the shard with γ_r.
    GemvParams p = {};
    p.A = acc_up;
    p.a_scale = gamma_x;
    p.a_gamma_up = gamma_up;
    p.rmax_in = gamma_r;
    p.rmax_n = 1;
    p.W = W_down_r;
    p.Y = acc_down;
    p.N = K_out;
    p.K = H_r;
    p.M = (int)M;
    p.eps = eps;
    return run_gemv(kSrcFfnRequant, kOutRawI32, BL_F32, p, false, dev, sms, st);
  }
  uint8_t* base = reinterpret_cast<uint8_t*>(workspace);
  int8_t* Rq = reinterpret_cast<int8_t*>(base);
  int32_t* rs = reinterpret_cast<int32_t*>(base + align_up((size_t)M * H_r));
  relu2_requant_given_kernel<<<(unsigned)M, kQuantThreads, 0, st>>>(acc_up, H_r, gamma_x, gamma_up,
                                                                    gamma_r, eps, Rq, rs);
  BL_CUDA(cudaGetLastError());
  return run_contract(Rq, W_down_r, M, H_r, K_out, nullptr, nullptr, rs, acc_down, kTcRawI32, 0, 0,
                      true, dev, sms, st);
}

bl_status bl_dequant_i32(const int32_t* acc, const float* gamma_A, const float* gamma, int64_t M,
                         int64_t N, int relu2, void* Y, bl_dtype y_dtype, bl_stream_t stream) {
  BL_TRY(check_dtype(y_dtype));
  BL_TRY(check_rows(M));
  BL_TRY(check_rows(N));
  if (M == 0 || N == 0) return BL_OK;
  BL_TRY(check_ptr(acc));
  BL_TRY(check_ptr(gamma_A));
  if (gamma == nullptr) return BL_ERR_INVALID_ARG;
  BL_TRY(check_ptr(Y));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  const int64_t total = M * N;
  int64_t blocks = (total + kQuantThreads - 1) / kQuantThreads;
  if (blocks > 16 * (int64_t)sms) blocks = 16 * (int64_t)sms;
  dequant_i32_kernel<<<(unsigned)blocks, kQuantThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      acc, gamma_A, gamma, M, N, relu2 ? 1 : 0, Y, y_dtype == BL_BF16);
  BL_CUDA(cudaGetLastError());
  return BL_OK;
}

// ---------------------------------------------------------------------------
// Radix-3 storage and its decode GEMV.

int64_t bl_radix3_row_bytes(int64_t K) { return K > 0 ? radix3_row_bytes(K) : 0; }

bl_status bl_pack_radix3(const uint8_t* W_packed, int64_t N, int64_t K, uint8_t* W_r3,
                         bl_stream_t stream) {
  BL_TRY(check_k(K));
  BL_TRY(check_rows(N));
  if (N == 0) return BL_OK;
  BL_TRY(check_ptr(W_packed));
  BL_TRY(check_ptr(W_r3));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  const int64_t total = N * radix3_row_bytes(K);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 16 * (int64_t)sms) blocks = 16 * (int64_t)sms;
  radix3_pack_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      W_packed, N, K, radix3_row_bytes(K), W_r3);
  BL_CUDA(cudaGetLastError());
  return BL_OK;
}

bl_status bl_linear_radix3(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                           const uint8_t* W_r3, const float* gamma, int64_t N, float eps,
                           int relu2, void* Y, bl_dtype y_dtype, unsigned flags,
                           bl_stream_t stream) {
  BL_TRY(check_dtype(a_dtype));
  BL_TRY(check_dtype(y_dtype));
  BL_TRY(check_k(K));
  BL_TRY(check_rows(M));
  BL_TRY(check_rows(N));
  BL_TRY(check_eps(eps));
  if ((flags & ~(unsigned)(BL_FLAG_PDL | BL_FLAG_RAW_I32)) != 0) return BL_ERR_INVALID_ARG;
  if (M > kGemvMaxTokens) return BL_ERR_SHAPE;
  if (M == 0 || N == 0) return BL_OK;
  BL_TRY(check_ptr(A));
  BL_TRY(check_ptr(W_r3));
  if (gamma == nullptr) return BL_ERR_INVALID_ARG;
  BL_TRY(check_ptr(Y));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  GemvR3Params p = {};
  p.A = A;
  p.W = W_r3;
  p.gamma = gamma;
  p.Y = Y;
  p.N = N;
  p.K = K;
  p.rb = radix3_row_bytes(K);
  p.M = (int)M;
  p.eps = eps;
  p.relu2 = relu2 ? 1 : 0;
  p.y_bf16 = y_dtype == BL_BF16;
  p.raw = (flags & BL_FLAG_RAW_I32) != 0;
  return run_r3(a_dtype, p, (flags & BL_FLAG_PDL) != 0, dev, sms,
                reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Lookup-table weights and their decode GEMV (one token).

bl_status bl_pack_lut_index(const uint8_t* W_packed, int64_t N, int64_t K, uint8_t* W_idx,
                            bl_stream_t stream) {
  BL_TRY(check_k(K));
  BL_TRY(check_rows(N));
  if (N == 0) return BL_OK;
  BL_TRY(check_ptr(W_packed));
  BL_TRY(check_ptr(W_idx));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  const int64_t total = N * (K / 4);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 16 * (int64_t)sms) blocks = 16 * (int64_t)sms;
  lut_index_pack_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      W_packed, total, W_idx);
  BL_CUDA(cudaGetLastError());
  return BL_OK;
}

bl_status bl_linear_lut(const void* A, bl_dtype a_dtype, int64_t M, int64_t K, const uint8_t* W_idx,
                        const float* gamma, int64_t N, float eps, void* Y, bl_dtype y_dtype,
                        unsigned flags, bl_stream_t stream) {
  BL_TRY(check_dtype(a_dtype));
  BL_TRY(check_dtype(y_dtype));
  BL_TRY(check_k(K));
  BL_TRY(check_rows(M));
  BL_TRY(check_rows(N));
  BL_TRY(check_eps(eps));
  if ((flags & ~(unsigned)(BL_FLAG_PDL | BL_FLAG_RAW_I32)) != 0) return BL_ERR_INVALID_ARG;
  if (M > 1) return BL_ERR_SHAPE;
  if (M == 0 || N == 0) return BL_OK;
  BL_TRY(check_ptr(A));
  BL_TRY(check_ptr(W_idx));
  if (gamma == nullptr) return BL_ERR_INVALID_ARG;
  BL_TRY(check_ptr(Y));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  int64_t r = (N + sms - 1) / sms;
  if (r < 1) r = 1;
  if (r > kGemvMaxRows) r = kGemvMaxRows;
  while (r > 1 && gemv_lut_smem_bytes(K, (int)r) > kGemvSmemCap) r = (r + 1) / 2;
  if (gemv_lut_smem_bytes(K, (int)r) > kSkSmemCap) return BL_ERR_SHAPE;  // tables of very long rows do not fit
  int grid;
  r = even_grid(N, r, sms, &grid);
  const size_t smem = gemv_lut_smem_bytes(K, (int)r);
  GemvLutParams p = {};
  p.A = A;
  p.W = W_idx;
  p.gamma = gamma;
  p.Y = Y;
  p.N = N;
  p.K = K;
  p.rows_per_cta = (int)r;
  p.rows_pad = gemv_rows_pad((int)r);
  p.eps = eps;
  p.y_bf16 = y_dtype == BL_BF16;
  p.raw = (flags & BL_FLAG_RAW_I32) != 0;
  CUtensorMap tw;
  BL_TRY(make_map_u8(&tw, W_idx, (uint64_t)N, (uint64_t)(K / 4), 128, (uint32_t)p.rows_pad,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool pdl = (flags & BL_FLAG_PDL) != 0;
  return a_dtype == BL_BF16 ? launch_lut_t<__nv_bfloat16>(tw, p, grid, smem, pdl, dev, st)
                            : launch_lut_t<float>(tw, p, grid, smem, pdl, dev, st);
}

// ---------------------------------------------------------------------------
// STE backward.

size_t bl_ste_grad_input_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  // W_q [N, K] bf16 (room for K·N8), plus a bf16 copy of dY [M, N] when it is fp32
  return align_up((size_t)K * round8(N) * 2) + align_up((size_t)M * N * 2);
}

bl_status bl_ste_grad_input(const void* dY, bl_dtype dy_dtype, int64_t M, int64_t N,
                            const uint8_t* W_packed, const float* gamma, int64_t K, float* dA,
                            void* workspace, size_t ws_bytes, bl_stream_t stream) {
  BL_TRY(check_dtype(dy_dtype));
  BL_TRY(check_k(K));
  BL_TRY(check_rows(M));
  BL_TRY(check_rows(N));
  if (N % 8 != 0) return BL_ERR_SHAPE;
  if (M == 0) return BL_OK;
  if (N == 0) return BL_ERR_SHAPE;
  BL_TRY(check_ptr(dY));
  BL_TRY(check_ptr(W_packed));
  if (gamma == nullptr) return BL_ERR_INVALID_ARG;
  BL_TRY(check_ptr(dA));
  if (workspace == nullptr || ws_bytes < bl_ste_grad_input_workspace_bytes(M, N, K))
    return BL_ERR_WORKSPACE;
  BL_TRY(check_ptr(workspace));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = reinterpret_cast<uint8_t*>(workspace);
  // W_q in its own layout [N, K]: the GEMM reads it as an MN-major operand
  // (the contraction index N is its row index).
  __nv_bfloat16* wq = reinterpret_cast<__nv_bfloat16*>(base);
  const int64_t Np = round8(N);
  {
    const int64_t words = N * (K / 16);
    int64_t blocks = (words + 255) / 256;
    if (blocks > 16 * (int64_t)sms) blocks = 16 * (int64_t)sms;
    expand_wq_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const uint32_t*>(W_packed),
                                                       words, wq);
    BL_CUDA(cudaGetLastError());
  }
  const void* a = dY;
  if (dy_dtype == BL_F32) {  // one bf16 rounding of dY
    __nv_bfloat16* dyb = reinterpret_cast<__nv_bfloat16*>(base + align_up((size_t)K * Np * 2));
    const int64_t n = M * N;
    int64_t blocks = (n / 4 + 255) / 256;
    if (blocks > 16 * (int64_t)sms) blocks = 16 * (int64_t)sms;
    convert_bf16_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const float*>(dY), n, dyb);
    BL_CUDA(cudaGetLastError());
    a = dyb;
  }
  GmParams p = {};
  p.rows = M;
  p.cols = K;
  p.kdim = N;
  p.C = dA;
  p.scale = gamma;
  return run_bf16_gemm(a, N, wq, K, p, kMajBMN, dev, st);
}

size_t bl_ste_grad_weight_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  const size_t Mp = (size_t)round8(M);
  return align_up((size_t)N * Mp * 2) + align_up((size_t)K * Mp * 2);
}

bl_status bl_ste_grad_weight(const void* dY, bl_dtype dy_dtype, int64_t M, int64_t N,
                             const int8_t* A_q, const float* gamma_A, int64_t K, const void* W,
                             bl_dtype w_dtype, const float* gamma, float eps, float* dW,
                             void* workspace, size_t ws_bytes, bl_stream_t stream) {
  BL_TRY(check_dtype(dy_dtype));
  BL_TRY(check_dtype(w_dtype));
  BL_TRY(check_k(K));
  BL_TRY(check_rows(M));
  BL_TRY(check_rows(N));
  BL_TRY(check_eps(eps));
  if (N % 8 != 0) return BL_ERR_SHAPE;
  if (N == 0) return BL_OK;
  BL_TRY(check_ptr(dW));
  if (M == 0) {
    int dev, sms;
    BL_TRY(current_device(&dev, &sms));
    BL_CUDA(cudaMemsetAsync(dW, 0, (size_t)N * K * 4, reinterpret_cast<cudaStream_t>(stream)));
    return BL_OK;
  }
  BL_TRY(check_ptr(dY));
  BL_TRY(check_ptr(A_q));
  BL_TRY(check_ptr(gamma_A));
  BL_TRY(check_ptr(W));
  if (gamma == nullptr) return BL_ERR_INVALID_ARG;
  if (workspace == nullptr || ws_bytes < bl_ste_grad_weight_workspace_bytes(M, N, K))
    return BL_ERR_WORKSPACE;
  BL_TRY(check_ptr(workspace));
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t Mp = round8(M);
  uint8_t* base = reinterpret_cast<uint8_t*>(workspace);
  // The GEMM reads dY [M, N] and Â [M, K] in their own layouts, as MN-major
  // operands (the contraction index M is the row index of both): dY as given
  // when bf16, else a bf16 copy; Â scaled into bf16. Rows past M read as
  // zeros.
  const __nv_bfloat16* dyb = reinterpret_cast<const __nv_bfloat16*>(dY);
  if (dy_dtype != BL_BF16) {
    __nv_bfloat16* dyc = reinterpret_cast<__nv_bfloat16*>(base);
    int64_t blocks = (M * N / 4 + 255) / 256;
    if (blocks > 16 * (int64_t)sms) blocks = 16 * (int64_t)sms;
    convert_bf16_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const float*>(dY), M * N,
                                                          dyc);
    BL_CUDA(cudaGetLastError());
    dyb = dyc;
  }
  __nv_bfloat16* ahb = reinterpret_cast<__nv_bfloat16*>(base + align_up((size_t)N * Mp * 2));
  int64_t sblocks = (M * (K / 8) + 255) / 256;
  if (sblocks > 16 * (int64_t)sms) sblocks = 16 * (int64_t)sms;
  scale_rows_bf16_kernel<<<(unsigned)sblocks, 256, 0, st>>>(A_q, gamma_A, M, K, ahb);
  BL_CUDA(cudaGetLastError());
  GmParams p = {};
  p.rows = N;
  p.cols = K;
  p.kdim = M;
  p.C = dW;
  p.mask_w = W;
  p.mask_bf16 = w_dtype == BL_BF16;
  p.mask_gamma = gamma;
  p.eps = eps;
  return run_bf16_gemm(dyb, N, ahb, K, p, kMajAMN | kMajBMN, dev, st);
}

bl_status bl_check_device_error(bl_stream_t stream) {
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return BL_ERR_CUDA;
  unsigned flags = 0;
  BL_CUDA(cudaMemcpyFromSymbol(&flags, g_error_flags, sizeof(flags)));
  if (flags != 0) {
    const unsigned zero = 0;
    BL_CUDA(cudaMemcpyToSymbol(g_error_flags, &zero, sizeof(zero)));
    return BL_ERR_TIMEOUT;
  }
  return BL_OK;
}

}  // extern "C"

// ==========================================================================
// bl_linear_noalloc: bl_linear for callers that cannot allocate device
// memory. Its scratch (the quantised tokens, their scales and row sums) lives
// in the fixed array below instead of a caller-provided workspace.
// ==========================================================================
namespace {
constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;  // 4 MiB per device
}  // namespace

// Held by every GPU that loads this library, until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
struct NoAllocSlot {
  void* ptr = nullptr;
  CUcontext ctx = nullptr;  // context current when ptr was looked up
};
NoAllocSlot g_noalloc[bl::kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The current driver context, through the driver entry point (the library
// does not link libcuda directly). Null if it cannot be queried.
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static int tried = 0;
  if (!tried) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
    tried = 1;
  }
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of the scratch array for the current device. In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with the device current and cached; a call that finds another context
// current (the device was reset since) looks it up again.
bl_status noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(bl::g_mu);
  const CUcontext ctx = current_context();
  NoAllocSlot& slot = g_noalloc[dev];
  if (slot.ptr == nullptr || slot.ctx != ctx) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return BL_ERR_CUDA;
    slot.ptr = ptr;
    slot.ctx = ctx;
  }
  *out = slot.ptr;
  return BL_OK;
}
}  // namespace

extern "C" bl_status bl_linear_noalloc(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                                       const uint8_t* W_packed, const float* gamma, int64_t N,
                                       float eps, int relu2, void* Y, bl_dtype y_dtype,
                                       bl_stream_t stream) {
  BL_TRY(check_dtype(a_dtype));
  BL_TRY(check_dtype(y_dtype));
  BL_TRY(check_k(K));
  BL_TRY(check_rows(M));
  BL_TRY(check_rows(N));
  BL_TRY(check_eps(eps));
  if (M == 0 || N == 0) return BL_OK;
  BL_TRY(check_ptr(A));
  BL_TRY(check_ptr(W_packed));
  if (gamma == nullptr) return BL_ERR_INVALID_ARG;
  BL_TRY(check_ptr(Y));
  // Scratch this call needs; refuse what the fixed array cannot hold.
  const size_t need = gemv_path(M, K) ? 0 : act_ws(M, K).total;
  if (need > kNoAllocScratchBytes) return BL_ERR_WORKSPACE;
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (need == 0) {  // a few tokens: the fused GEMV needs no scratch at all
    GemvParams p = {};
    p.A = A;
    p.W = W_packed;
    p.gamma = gamma;
    p.Y = Y;
    p.N = N;
    p.K = K;
    p.M = (int)M;
    p.eps = eps;
    p.relu2 = relu2 ? 1 : 0;
    p.y_bf16 = y_dtype == BL_BF16;
    return run_gemv(kSrcFloat, kOutDequant, a_dtype, p, false, dev, sms, st);
  }
  void* scratch = nullptr;
  BL_TRY(noalloc_scratch(dev, &scratch));
  // Every scratch byte read below is first written by this call's quantiser,
  // so nothing has to start at zero.
  const ActWs w = act_ws(M, K);
  uint8_t* base = reinterpret_cast<uint8_t*>(scratch);
  int8_t* Aq = reinterpret_cast<int8_t*>(base + w.aq);
  float* gA = reinterpret_cast<float*>(base + w.gamma);
  int32_t* rs = reinterpret_cast<int32_t*>(base + w.rowsum);
  BL_TRY(run_quant_acts(A, a_dtype, M, K, eps, Aq, gA, rs, st));
  return run_contract(Aq, W_packed, M, K, N, gamma, gA, rs, Y, kTcDequant, relu2 ? 1 : 0,
                      y_dtype == BL_BF16, true, dev, sms, st);
}

namespace bl {
namespace {
// Measurement aid: the decode GEMV's launch (grid, 512 threads, dynamic
// shared memory, programmatic dependent launch) with no work, so a chain of
// it shows the launch-to-launch floor of a dependent chain.
__global__ void __launch_bounds__(kGemvThreads, 2) pdl_floor_kernel() {
  extern __shared__ uint8_t smem_unused[];
  (void)smem_unused;
  pdl_launch_dependents();
  pdl_wait_prior_grid();
}

__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    // Nothing ever arrives on `bar`: the bounded wait must give up.
    if (!mbar_wait_for(&bar, 0, limit_ns)) raise_error(kErrTimeout);
  }
}
}  // namespace
}  // namespace bl

extern "C" bl_status bl_probe_pdl_floor(int64_t M, int64_t K, int64_t N, bl_stream_t stream) {
  BL_TRY(check_k(K));
  BL_TRY(check_rows(N));
  if (M < 1 || M > kGemvMaxTokens || N == 0) return BL_ERR_SHAPE;
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  int rows, grid;
  size_t smem;
  BL_TRY(bl::gemv_plan(N, K, (int)M, sms, &rows, &grid, &smem));
  BL_TRY(bl::ensure_smem(bl::pdl_floor_kernel, dev, smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(bl::kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  BL_CUDA(cudaLaunchKernelEx(&cfg, bl::pdl_floor_kernel));
  return BL_OK;
}

extern "C" bl_status bl_selftest_wait_timeout(int64_t limit_ns, bl_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000) return BL_ERR_INVALID_ARG;
  int dev, sms;
  BL_TRY(current_device(&dev, &sms));
  bl::wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)limit_ns);
  BL_CUDA(cudaGetLastError());
  return BL_OK;
}
