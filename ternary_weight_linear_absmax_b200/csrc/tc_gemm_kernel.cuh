// Ternary × INT8 contraction on the 5th-generation tensor cores (tcgen05,
// kind::i8) for more than a handful of tokens (prefill, small batches, FFN).
//
// "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section
// "Como funciona a camada BitLinear ... (Zero-GEMM)?": acc = A_q·W_qᵀ in
// INT32, then Y = acc·(γ_A·γ)/127. The pages' add/subtract/skip is exact
// integer arithmetic; an INT8 MMA with operands in {0,1,2} × [-127,127]
// computes the same integers exactly.
//
// Orientation ("swap AB"): the MMA's M side is 128 weight rows (so small
// token counts still fill the 128-row instruction), its N side is BN tokens.
//  * warp 0   : TMA producer. Per 128-wide K block it loads the BN×128 int8
//               token tile (128-byte swizzle) and the 128×32-byte packed
//               weight tile into one shared-memory stage.
//  * warp 1   : allocates TMEM, issues tcgen05.mma (one elected thread) and
//               commits completion to the stage barriers.
//  * warps 2-5: expansion, then epilogue. Each thread owns one weight row
//               (one TMEM lane): it turns 32 packed bytes (128 codes) into
//               32 words of int8 codes {0,1,2} — two ALU ops per 4 weights —
//               and stores them with tcgen05.st straight into TMEM, where
//               the MMA reads its A operand. Nothing expanded goes through
//               shared memory.
//  * The accumulator D[weight row, token] lives in TMEM (int32). The
//    epilogue reads it with tcgen05.ld, subtracts the token's Σ A_q (codes
//    are w+1), scales by (γ_A·γ)/127 (optionally ReLU²) and stores.
// Every barrier wait is bounded; a wait that gives up raises the device
// error flag and the CTA drains and exits.
#pragma once

#include "bl_device.cuh"

namespace bl {

constexpr int kTcThreads = 192;
constexpr int kTcBK = 128;  // int8 K elements per stage (one 128-byte swizzle row)

enum TcOut : int { kTcDequant = 0, kTcRawI32 = 1 };

struct TcParams {
  const float* gamma;     // γ of W (1 value)
  const float* gammaA;    // [M] token scales
  const int32_t* rowsum;  // [M] Σ_k A_q[m,k]
  void* Y;                // [M, N] float/bf16 (dequant) or int32 (raw)
  int64_t M, N, K;
  int relu2;
  int y_bf16;
};

template <int BN>
struct TcConfig {
  static constexpr int kBStage = BN * kTcBK;     // bytes of token tile per stage
  static constexpr int kWStage = 128 * 32;       // bytes of packed weights per stage
  static constexpr int kSStages = BN >= 256 ? 4 : (BN >= 128 ? 6 : 8);
  static constexpr int kTStages = 4;             // TMEM A stages (32 columns each)
  static constexpr int kDCols = BN < 32 ? 32 : BN;
  static constexpr int kACol = kDCols;
  static constexpr int kColsNeeded = kDCols + kTStages * 32;
  static constexpr int kTmemCols = kColsNeeded <= 32 ? 32 : kColsNeeded <= 64 ? 64
                                   : kColsNeeded <= 128 ? 128 : kColsNeeded <= 256 ? 256 : 512;
  static constexpr int kRingBytes = kSStages * (kBStage + kWStage);
  static constexpr int kBarBytes = (2 * kSStages + 2 * kTStages + 1) * 8;
  static constexpr int kParamBytes = BN * 8;
  // 1 KiB slack for aligning the dynamic buffer to 1024 bytes. At least
  // 116 KiB are requested so that only one CTA is resident per SM: every CTA
  // then gets its TMEM columns without waiting on another CTA's allocation.
  static constexpr int kSmemUsed = 1024 + kRingBytes + kBarBytes + kParamBytes + 64;
  static constexpr int kSmemBytes = kSmemUsed > 116 * 1024 ? kSmemUsed : 116 * 1024;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long limit = g_wait_limit_ns;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit) {
      raise_error(kErrTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}

template <int BN, int OUT>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_ternary_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,
                       const __grid_constant__ CUtensorMap tm_w, const TcParams p) {
  using C = TcConfig<BN>;
  constexpr int SS = C::kSStages, TS = C::kTStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* s_b = smem;                              // SS × BN×128 (1024-aligned stages)
  uint8_t* s_w = smem + SS * C::kBStage;            // SS × 128×32
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kRingBytes);
  uint64_t* full = bars;                            // [SS] TMA landed
  uint64_t* empty = bars + SS;                      // [SS] MMA done with stage
  uint64_t* afull = bars + 2 * SS;                  // [TS] A operand in TMEM ready
  uint64_t* aempty = bars + 2 * SS + TS;            // [TS] MMA done with A stage
  uint64_t* done = bars + 2 * SS + 2 * TS;          // accumulator complete
  float* s_sc = reinterpret_cast<float*>(smem + C::kRingBytes + C::kBarBytes);
  int* s_rs = reinterpret_cast<int*>(s_sc + BN);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_rs + BN);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = (int64_t)blockIdx.x * 128;
  const int64_t m0 = (int64_t)blockIdx.y * BN;
  const int KB = (int)((p.K + kTcBK - 1) / kTcBK);

  // Per-token epilogue parameters.
  {
    // γ and γ_A are absent for raw INT32 output.
    const float g = p.gamma != nullptr ? *p.gamma : 0.0f;
    for (int j = tid; j < BN; j += kTcThreads) {
      const int64_t m = m0 + j;
      s_sc[j] = (m < p.M && p.gammaA != nullptr) ? __fdiv_rn(__fmul_rn(p.gammaA[m], g), 127.0f)
                                                  : 0.0f;
      s_rs[j] = m < p.M ? p.rowsum[m] : 0;
    }
  }
  if (tid == 0) {
    for (int s = 0; s < SS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int t = 0; t < TS; ++t) {
      mbar_init(&afull[t], 128);
      mbar_init(&aempty[t], 1);
    }
    mbar_init(done, 1);
    *s_abort = 0;
    fence_barrier_init();
    prefetch_tensormap(&tm_act);
    prefetch_tensormap(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int kb = 0;
      for (; kb < KB; ++kb) {
        const int s = kb % SS;
        if (kb >= SS && !wait_or_abort(&empty[s], ((kb / SS) + 1) & 1, s_abort)) break;
        mbar_arrive_expect_tx(&full[s], C::kBStage + C::kWStage);
        tma_load_2d(s_b + s * C::kBStage, &tm_act, kb * kTcBK, (int32_t)m0, &full[s]);
        tma_load_2d(s_w + s * C::kWStage, &tm_w, kb * (kTcBK / 4), (int32_t)n0, &full[s]);
      }
      if (*s_abort) {
        // Drain copies that may still be in flight (bounded) before exit.
        for (int d = max(0, kb - SS); d < kb; ++d)
          mbar_wait_for(&full[d % SS], (d / SS) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(128, BN);
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % SS, t = kb % TS;
        if (!wait_or_abort(&full[s], (kb / SS) & 1, s_abort)) break;
        if (!wait_or_abort(&afull[t], (kb / TS) & 1, s_abort)) break;
        tc_fence_after();
        const uint32_t b_addr = smem_u32(s_b + s * C::kBStage);
#pragma unroll
        for (int kk = 0; kk < kTcBK / 32; ++kk) {
          const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 32);
          mma_i8_ts(tmem, tmem + C::kACol + t * 32 + kk * 8, bdesc, idesc,
                    (kb > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        mma_commit(&aempty[t]);
      }
      mma_commit(done);  // also on abort: tracks every MMA issued
    }
  } else {
    // ---------------- expansion (warps 2..5) ----------------
    const int q = warp & 3;         // TMEM lane quarter this warp may access
    const int row = 32 * q + lane;  // weight row within the tile
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % SS, t = kb % TS;
      // tcgen05.st is warp-collective: the whole warp continues or stops.
      bool ok = wait_or_abort(&full[s], (kb / SS) & 1, s_abort);
      if (ok && kb >= TS) ok = wait_or_abort(&aempty[t], ((kb / TS) + 1) & 1, s_abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint4* src = reinterpret_cast<const uint4*>(s_w + s * C::kWStage + row * 32);
      const uint4 u0 = src[0], u1 = src[1];
      const uint32_t x[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      uint32_t v[32];
#pragma unroll
      for (int g = 0; g < 8; ++g) expand_word(x[g], v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
      tmem_st_32x32b_x32(tmem + lane_addr + C::kACol + t * 32, v);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&afull[t]);
    }
    // ---------------- epilogue ----------------
    bool ok = wait_or_abort(done, 0, s_abort);
    ok = __all_sync(0xffffffffu, ok && !*s_abort);  // tcgen05.ld is warp-collective
    if (ok) {
      tc_fence_after();
      const int64_t n = n0 + row;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t d[16];
        tmem_ld_32x32b_x16(tmem + lane_addr + c0, d);
        tmem_wait_ld();
        if (n < p.N) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int64_t m = m0 + c0 + j;
            if (m < p.M) {
              const int v = (int)d[j] - s_rs[c0 + j];
              const int64_t o = m * p.N + n;
              if constexpr (OUT == kTcRawI32) {
                reinterpret_cast<int32_t*>(p.Y)[o] = v;
              } else {
                float y = __fmul_rn((float)v, s_sc[c0 + j]);
                if (p.relu2) {
                  y = fmaxf(y, 0.0f);
                  y = __fmul_rn(y, y);
                }
                if (p.y_bf16)
                  reinterpret_cast<__nv_bfloat16*>(p.Y)[o] = __float2bfloat16_rn(y);
                else
                  reinterpret_cast<float*>(p.Y)[o] = y;
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // MMAs must be finished before TMEM is released (bounded on abort paths;
    // on the normal path the epilogue already observed `done`).
    if (*s_abort) mbar_wait_for(done, 0, 100000000ull);
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace bl
