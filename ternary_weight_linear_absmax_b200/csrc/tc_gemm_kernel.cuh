// Ternary × INT8 contraction on the 5th-generation tensor cores (tcgen05,
// kind::i8) for more than 64 tokens (prefill, the FFN at larger batches).
//
// "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section
// "Como funciona a camada BitLinear ... (Zero-GEMM)?": acc = A_q·W_qᵀ in
// INT32, then Y = acc·(γ_A·γ)/127. The pages' add/subtract/skip is exact
// integer arithmetic; an INT8 MMA with operands in {0,1,2} × [-127,127]
// computes the same integers exactly.
//
// Orientation ("swap AB"): the MMA's M side is 128 weight rows, its N side
// is BN tokens.
//  * warp 0   : TMA producer. Per 128-wide K block it loads the BN×128 int8
//               token tile (128-byte swizzle); every four K blocks, a
//               128×128-byte packed weight tile. After the main loop it
//               writes the staged output tile with tensor stores.
//  * warp 1   : allocates TMEM, issues tcgen05.mma (one elected thread) and
//               commits completion to the stage barriers.
//  * warps 2-9: expansion, then epilogue. Two warps share each TMEM lane
//               quarter; a thread owns one weight row (one TMEM lane) and
//               half of each K block: it turns 16 packed bytes (64 codes)
//               into 16 words of int8 codes {0,1,2} — two ALU ops per 4
//               weights — and stores them with tcgen05.st straight into
//               TMEM, where the MMA reads its A operand. Nothing expanded
//               goes through shared memory.
//  * The accumulator D[weight row, token] lives in TMEM (int32). The
//    epilogue reads it with tcgen05.ld, subtracts the token's Σ A_q (codes
//    are w+1), scales by (γ_A·γ)/127 (optionally ReLU²) and stores.
// Every barrier wait is bounded; a wait that gives up raises the device
// error flag and the CTA drains and exits.
#pragma once

#include "bl_device.cuh"

namespace bl {

// Warps: 0 TMA producer, 1 MMA issuer, 2..9 expansion + epilogue (two per
// TMEM lane quarter).
constexpr int kTcThreads = 320;
constexpr int kTcMathThreads = 256;
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
  int tma_store;  // 1: the epilogue stages the tile in shared memory and the producer warp
                  //    writes it with tensor stores of 32 tokens through tm_y (needs
                  //    N·element bytes % 16 == 0)
};

template <int BN>
struct TcConfig {
  // Token ring: one 128-byte-wide K block (BN rows, 128-byte swizzle) per stage.
  static constexpr int kBStage = BN * kTcBK;
  // Deep enough that the producer can run ahead over every weight stage
  // (4 K blocks per weight stage): small token tiles are cheap to stage.
  static constexpr int kSStages = BN >= 256 ? 4 : (BN >= 128 ? 6 : (BN >= 64 ? 12 : (BN >= 32 ? 16 : 24)));
  // Weight ring: 128 rows × 128 packed bytes (4 K blocks) per stage, 128-byte
  // swizzle. Wide rows keep the number of TMA requests per byte low, which is
  // what bounds the stream when few tokens share each weight byte.
  static constexpr int kWStage = 128 * 128;
  static constexpr int kWStages = BN >= 256 ? 2 : (BN >= 128 ? 3 : (BN >= 64 ? 4 : 6));
  static constexpr int kTStages = 4;  // TMEM A stages (32 columns = one K block each)
  // Independent accumulators: consecutive MMAs into one accumulator are
  // serialised by its read-modify-write, which dominates for small N. The
  // four MMAs of a stage rotate over kAcc accumulators, summed in the
  // epilogue (exact integer addition).
  static constexpr int kAcc = BN <= 64 ? 4 : (BN <= 128 ? 2 : 1);
  static constexpr int kDCols = BN < 32 ? 32 : BN;  // columns per accumulator
  static constexpr int kACol = kAcc * kDCols;
  static constexpr int kColsNeeded = kACol + kTStages * 32;
  static constexpr int kTmemCols = kColsNeeded <= 32 ? 32 : kColsNeeded <= 64 ? 64
                                   : kColsNeeded <= 128 ? 128 : kColsNeeded <= 256 ? 256 : 512;
  static constexpr int kRingBytes = kSStages * kBStage + kWStages * kWStage;
  // The staged output tile is stored in chunks of 32 tokens, each with its
  // own barrier, so the stores overlap the rest of the epilogue.
  static constexpr int kStoreChunks = (BN + 31) / 32;
  // Rounded to 16 bytes: the epilogue parameters after the barriers are read
  // with 16-byte vector loads.
  static constexpr int kBarBytes =
      ((2 * kSStages + 2 * kWStages + 2 * kTStages + 2 + kStoreChunks) * 8 + 15) / 16 * 16;
  static constexpr int kParamBytes = BN * 8;
  // 1 KiB slack for aligning the dynamic buffer to 1024 bytes. At least
  // 116 KiB are requested so that only one CTA is resident per SM: every CTA
  // then gets its TMEM columns without waiting on another CTA's allocation.
  static constexpr int kSmemUsed = 1024 + kRingBytes + kBarBytes + kParamBytes + 64;
  static constexpr int kSmemBytes = kSmemUsed > 116 * 1024 ? kSmemUsed : 116 * 1024;
  // The output staging tile reuses the ring.
  static_assert(BN * 128 * 4 <= kRingBytes, "staging tile must fit in the ring");
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

// Epilogue body for one chunk of CW accumulator columns (tokens) of this
// thread's row: undo the code offset, scale (and ReLU²), convert, and write
// either into the staged [BN x 128] tile or straight to global memory. The
// flags are template parameters so the unrolled body has no branches and the
// CW columns form independent instruction chains.
template <int CW, int OUT, bool RELU, bool BF16, bool STAGE>
__device__ __forceinline__ void tc_epilogue_chunk(const uint32_t (&d)[CW], int c0, int row,
                                                  const float* s_sc, const int* s_rs,
                                                  uint8_t* stage, const TcParams& p, int64_t m0,
                                                  int64_t n) {
  // Read all per-token scalars first: the stores below go to shared memory
  // too, and without this split they would order every following load.
  // c0 is a multiple of 16: 16-byte vector loads (warp-wide broadcasts).
  float sc[CW];
  int rs[CW];
#pragma unroll
  for (int j = 0; j < CW; j += 4) {
    const float4 f = *reinterpret_cast<const float4*>(s_sc + c0 + j);
    const int4 r = *reinterpret_cast<const int4*>(s_rs + c0 + j);
    sc[j] = f.x;
    sc[j + 1] = f.y;
    sc[j + 2] = f.z;
    sc[j + 3] = f.w;
    rs[j] = r.x;
    rs[j + 1] = r.y;
    rs[j + 2] = r.z;
    rs[j + 3] = r.w;
  }
  uint32_t bits[CW];
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    const int v = (int)d[j] - rs[j];
    if constexpr (OUT == kTcRawI32) {
      bits[j] = (uint32_t)v;
    } else {
      float y = __fmul_rn((float)v, sc[j]);
      if constexpr (RELU) {
        y = fmaxf(y, 0.0f);
        y = __fmul_rn(y, y);
      }
      if constexpr (BF16)
        bits[j] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y));
      else
        bits[j] = __float_as_uint(y);
    }
  }
  constexpr bool kHalf = (OUT != kTcRawI32) && BF16;
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    const int jj = c0 + j;
    if constexpr (STAGE) {
      if constexpr (kHalf)
        reinterpret_cast<uint16_t*>(stage)[jj * 128 + row] = (uint16_t)bits[j];
      else
        reinterpret_cast<uint32_t*>(stage)[jj * 128 + row] = bits[j];
    } else {
      const int64_t m = m0 + jj;
      if (m < p.M && n < p.N) {
        const int64_t o = m * p.N + n;
        if constexpr (kHalf)
          reinterpret_cast<uint16_t*>(p.Y)[o] = (uint16_t)bits[j];
        else
          reinterpret_cast<uint32_t*>(p.Y)[o] = bits[j];
      }
    }
  }
}

// Whole-tile epilogue for one thread's TMEM lane: loads CW columns at a time
// (summing the kAcc accumulators), with the next chunk's load issued before
// the current chunk is processed.
template <int BN, int OUT, bool RELU, bool BF16, bool STAGE>
__device__ __forceinline__ void tc_epilogue(uint32_t t_lane, int row, int half, const float* s_sc,
                                            const int* s_rs, uint8_t* stage, const TcParams& p,
                                            int64_t m0, int64_t n, uint64_t* staged) {
  using C = TcConfig<BN>;
  // 16-column chunks, alternating between the two warps of a lane quarter.
  constexpr int CW = 16;
  const int c_begin = half * CW;
  if (c_begin >= BN) return;
  auto load = [&](int c0, uint32_t (&d)[CW]) {
    tmem_ld_32x32b_x16(t_lane + c0, d);
    if constexpr (C::kAcc > 1) {
      tmem_wait_ld();
#pragma unroll
      for (int a = 1; a < C::kAcc; ++a) {
        uint32_t e[CW];
        tmem_ld_32x32b_x16(t_lane + a * C::kDCols + c0, e);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < CW; ++j) d[j] = (uint32_t)((int)d[j] + (int)e[j]);
      }
    }
  };
  uint32_t cur[CW], nxt[CW];
  load(c_begin, cur);
  tmem_wait_ld();
#pragma unroll 1
  for (int c0 = c_begin; c0 < BN; c0 += 2 * CW) {
    const bool more = c0 + 2 * CW < BN;
    if (more) load(c0 + 2 * CW, nxt);  // in flight while this chunk is processed
    tc_epilogue_chunk<CW, OUT, RELU, BF16, STAGE>(cur, c0, row, s_sc, s_rs, stage, p, m0, n);
    if constexpr (STAGE) {
      // This thread's part of tokens [32·(c0/32), +32) is staged: make it
      // visible to the tensor store and report it.
      fence_proxy_async_smem();
      mbar_arrive(&staged[c0 >> 5]);
    }
    if (more) {
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < CW; ++j) cur[j] = nxt[j];
    }
  }
}

template <int BN, int OUT>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_ternary_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,
                       const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_y, const TcParams p) {
  using C = TcConfig<BN>;
  constexpr int SS = C::kSStages, WS = C::kWStages, TS = C::kTStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* s_b = smem;                              // SS × BN×128 (1024-aligned stages)
  uint8_t* s_w = smem + SS * C::kBStage;            // WS × 128×128 (1024-aligned stages)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kRingBytes);
  uint64_t* full = bars;                            // [SS] token tile landed
  uint64_t* empty = bars + SS;                      // [SS] MMA done with token stage
  uint64_t* wfull = bars + 2 * SS;                  // [WS] weight tile landed
  uint64_t* wempty = bars + 2 * SS + WS;            // [WS] expansion done with weight stage
  uint64_t* afull = bars + 2 * SS + 2 * WS;         // [TS] A operand in TMEM ready
  uint64_t* aempty = afull + TS;                    // [TS] MMA done with A stage
  uint64_t* done = aempty + TS;                     // accumulator complete
  uint64_t* pready = done + 1;                      // epilogue parameters in shared memory
  uint64_t* staged = done + 2;                      // [kStoreChunks] 32 output tokens staged
  float* s_sc = reinterpret_cast<float*>(smem + C::kRingBytes + C::kBarBytes);
  int* s_rs = reinterpret_cast<int*>(s_sc + BN);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_rs + BN);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = (int64_t)blockIdx.x * 128;
  const int64_t m0 = (int64_t)blockIdx.y * BN;
  const int KB = (int)((p.K + kTcBK - 1) / kTcBK);

  if (tid == 0) {
    for (int s = 0; s < SS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int v = 0; v < WS; ++v) {
      mbar_init(&wfull[v], 1);
      mbar_init(&wempty[v], kTcMathThreads);
    }
    for (int t = 0; t < TS; ++t) {
      mbar_init(&afull[t], kTcMathThreads);
      mbar_init(&aempty[t], 1);
    }
    mbar_init(done, 1);
    mbar_init(pready, kTcMathThreads);
    for (int i = 0; i < C::kStoreChunks; ++i) mbar_init(&staged[i], kTcMathThreads);
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
  // Launched with programmatic dependent launch: the set-up above overlaps
  // the previous kernel's tail; global memory is touched only after it has
  // completed. The next kernel may start its own set-up from here on.
  pdl_launch_dependents();
  pdl_wait_prior_grid();

  if (warp == 0) {
    // ---------------- TMA producer (whole warp, one elected lane issues) ---
    int kb = 0, wissued = 0;
    for (; kb < KB; ++kb) {
      if ((kb & 3) == 0) {  // a new weight stage covers K blocks kb .. kb+3
        const int ws = kb >> 2, v = ws % WS;
        bool ok = ws < WS || wait_or_abort(&wempty[v], ((ws / WS) + 1) & 1, s_abort);
        if (!__all_sync(0xffffffffu, ok)) break;
        tma_load_1x2d_warp(&wfull[v], C::kWStage, s_w + v * C::kWStage, &tm_w, ws * 128,
                           (int32_t)n0);
        ++wissued;
      }
      const int s = kb % SS;
      bool ok = kb < SS || wait_or_abort(&empty[s], ((kb / SS) + 1) & 1, s_abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      tma_load_1x2d_warp(&full[s], C::kBStage, s_b + s * C::kBStage, &tm_act, kb * kTcBK,
                         (int32_t)m0);
      // Warm L2 with the token tile this stage will hold next time round.
      if (kb + SS < KB) tma_prefetch_2d_warp(&tm_act, (kb + SS) * kTcBK, (int32_t)m0);
    }
    if (*s_abort && lane == 0) {
      // Drain copies that may still be in flight (bounded) before exit.
      for (int d = max(0, kb - SS); d < kb; ++d)
        mbar_wait_for(&full[d % SS], (d / SS) & 1, 100000000ull);
      for (int d = max(0, wissued - WS); d < wissued; ++d)
        mbar_wait_for(&wfull[d % WS], (d / WS) & 1, 100000000ull);
    }
    // Output: store each 32-token chunk of the staged tile as soon as the
    // math warps have written it (the tile reuses the ring, whose loads have
    // all landed once the math warps observed `done`).
    if (p.tma_store && lane == 0 && !*s_abort) {
      const int esz = (OUT == kTcRawI32 || !p.y_bf16) ? 4 : 2;
      int issued = 0;
      for (int i = 0; i < C::kStoreChunks && m0 + 32 * i < p.M; ++i) {  // chunks past M: nothing
        if (!mbar_wait(&staged[i], 0) || *s_abort) break;
        tma_store_2d(&tm_y, (int32_t)n0, (int32_t)(m0 + 32 * i), smem + (size_t)i * 32 * 128 * esz);
        bulk_commit_group();
        ++issued;
      }
      if (issued) bulk_wait_group_read0();  // shared source read before the CTA may exit
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (whole warp, one elected lane issues) -----
    constexpr uint32_t idesc = idesc_i8(128, BN);
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    const uint32_t b_base = __shfl_sync(0xffffffffu, smem_u32(s_b), 0);
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % SS, t = kb % TS;
      bool ok = wait_or_abort(&full[s], (kb / SS) & 1, s_abort);
      if (ok) ok = wait_or_abort(&afull[t], (kb / TS) & 1, s_abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint64_t bdesc = smem_desc_sw128(b_base + s * C::kBStage);
      const uint32_t a_col = tm + C::kACol + t * 32;
#pragma unroll
      for (int kk = 0; kk < kTcBK / 32; ++kk) {
        const int acc = kk % C::kAcc;
        // +2 in the descriptor's address field = +32 bytes along K
        mma_i8_ts_warp(tm + acc * C::kDCols, a_col + kk * 8, bdesc + (uint64_t)(kk * 2), idesc,
                       (kb > 0 || kk >= C::kAcc) ? 1u : 0u);
      }
      mma_commit_warp(&empty[s]);
      mma_commit_warp(&aempty[t]);
    }
    mma_commit_warp(done);  // also on abort: tracks every MMA issued
  } else {
    // ---------------- expansion (warps 2..9) ----------------
    const int q = warp & 3;         // TMEM lane quarter this warp may access
    const int hw = (warp - 2) >> 2; // which half of each K block (and of the epilogue columns)
    const int row = 32 * q + lane;  // weight row within the tile
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    const int mtid = tid - 64;      // 0 .. 255 among the math warps
    // Per-token epilogue parameters, loaded now and parked in registers; they
    // are written to shared memory after the main loop (only the epilogue
    // reads them), so their memory latency overlaps the main loop.
    constexpr int kPar = (BN + kTcMathThreads - 1) / kTcMathThreads;
    float par_sc[kPar];
    int par_rs[kPar];
    {
      const float g = p.gamma != nullptr ? __ldg(p.gamma) : 0.0f;  // absent for raw INT32 output
#pragma unroll
      for (int i = 0; i < kPar; ++i) {
        const int j = mtid + i * kTcMathThreads;
        const int64_t m = m0 + j;
        const bool in = j < BN && m < p.M;
        par_sc[i] = (in && p.gammaA != nullptr) ? __fdiv_rn(__fmul_rn(__ldg(p.gammaA + m), g), 127.0f) : 0.0f;
        par_rs[i] = in ? __ldg(p.rowsum + m) : 0;
      }
    }
    for (int kb = 0; kb < KB; ++kb) {
      const int t = kb % TS, ws = kb >> 2, v = ws % WS, sub = kb & 3;
      // tcgen05.st is warp-collective: the whole warp continues or stops.
      bool ok = wait_or_abort(&wfull[v], (ws / WS) & 1, s_abort);
      if (ok && kb >= TS) ok = wait_or_abort(&aempty[t], ((kb / TS) + 1) & 1, s_abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      // This K block is 16-byte chunks 2·sub and 2·sub+1 of the row's 128-byte
      // line (this warp takes chunk 2·sub + hw); the 128-byte swizzle stores
      // chunk j at slot j ^ (row mod 8).
      const uint8_t* line = s_w + v * C::kWStage + row * 128;
      const uint4 u = *reinterpret_cast<const uint4*>(line + (((2 * sub + hw) ^ (row & 7)) << 4));
      if (sub == 3 || kb == KB - 1) mbar_arrive(&wempty[v]);  // done reading this stage
      const uint32_t x[4] = {u.x, u.y, u.z, u.w};
      uint32_t vv[16];
#pragma unroll
      for (int g = 0; g < 4; ++g) expand_word(x[g], vv[4 * g], vv[4 * g + 1], vv[4 * g + 2], vv[4 * g + 3]);
      tmem_st_32x32b_x16(tmem + lane_addr + C::kACol + t * 32 + hw * 16, vv);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&afull[t]);
    }
#pragma unroll
    for (int i = 0; i < kPar; ++i) {
      const int j = mtid + i * kTcMathThreads;
      if (j < BN) {
        s_sc[j] = par_sc[i];
        s_rs[j] = par_rs[i];
      }
    }
    mbar_arrive(pready);  // parameters visible to all math warps
    // ---------------- epilogue ----------------
    bool ok = wait_or_abort(done, 0, s_abort);
    if (ok) ok = wait_or_abort(pready, 0, s_abort);
    ok = __all_sync(0xffffffffu, ok && !*s_abort);  // tcgen05.ld is warp-collective
    if (ok) {
      tc_fence_after();
      const int64_t n = n0 + row;
      // The staging tile reuses the ring: once `done` has been observed every
      // load has landed and every MMA has finished reading it.
      const uint32_t t_lane = tmem + lane_addr;
      if constexpr (OUT == kTcRawI32) {
        if (p.tma_store)
          tc_epilogue<BN, OUT, false, false, true>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, staged);
        else
          tc_epilogue<BN, OUT, false, false, false>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, staged);
      } else {
        const int sel = (p.tma_store ? 4 : 0) | (p.y_bf16 ? 2 : 0) | (p.relu2 ? 1 : 0);
        switch (sel) {
          case 0: tc_epilogue<BN, OUT, false, false, false>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, staged); break;
          case 1: tc_epilogue<BN, OUT, true, false, false>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, staged); break;
          case 2: tc_epilogue<BN, OUT, false, true, false>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, staged); break;
          case 3: tc_epilogue<BN, OUT, true, true, false>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, staged); break;
          case 4: tc_epilogue<BN, OUT, false, false, true>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, staged); break;
          case 5: tc_epilogue<BN, OUT, true, false, true>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, staged); break;
          case 6: tc_epilogue<BN, OUT, false, true, true>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, staged); break;
          default: tc_epilogue<BN, OUT, true, true, true>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, staged); break;
        }
      }
    }
    // Every epilogue thread arrives on every chunk barrier exactly once: the
    // epilogue arrives per chunk it staged; the rest (a skipped epilogue, or
    // the second half of a 16-token tile) arrive here, so the storing
    // thread's bounded waits can only time out on a failed CTA.
    if (p.tma_store) {
      const int first = (ok && hw * 16 < BN) ? (BN - hw * 16 + 31) / 32 : 0;
      for (int i = first; i < C::kStoreChunks; ++i) mbar_arrive(&staged[i]);
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

// ===========================================================================
// Persistent variant: one CTA per SM walks work items (a 128-weight × 256-token
// tile, or a K-range of one when the tiles alone would leave SMs idle).
//  * warp 0       : TMA producer (token tiles, packed weight tiles).
//  * warp 1       : TMEM owner (all 512 columns = two 256-column INT32
//                   accumulators) and MMA issuer; A and B both come from
//                   shared memory (128-byte swizzle, K-major).
//  * warps 2..9   : expansion — 2-bit codes → int8 codes {0,1,2} written into
//                   the swizzled A stage (two ALU ops per 4 weights).
//  * warps 10..13 : epilogue — one TMEM lane quarter each; drains accumulator
//                   i while the MMAs fill accumulator i+1, stores directly
//                   (lanes are consecutive output columns, so each warp store
//                   covers 64 or 128 contiguous bytes).
// K-split items write raw INT32 partials to a [splits, M, N] workspace; the
// last split to finish a tile (elected by an atomic counter — no CTA ever
// waits for another) sums the partials and runs the epilogue.
constexpr int kTc2Threads = 448;
constexpr int kTc2BN = 256;

struct Tc2 {
  static constexpr int kSS = 3;             // token stages (one 128-byte K block each)
  static constexpr int kWS = 2;             // packed weight stages (four K blocks each)
  static constexpr int kAS = 4;             // expanded A stages (one K block each)
  static constexpr int kBStage = kTc2BN * 128;
  static constexpr int kWStage = 128 * 128;
  static constexpr int kAStage = 128 * 128;
  static constexpr int kRing = kSS * kBStage + kWS * kWStage + kAS * kAStage;
  static constexpr int kBars = 2 * kSS + 2 * kWS + 2 * kAS + 5;  // + accfull[2], accempty[2], done
  static constexpr int kBarBytes = (kBars * 8 + 15) / 16 * 16;
  static constexpr int kParamBytes = 2 * kTc2BN * 8;  // [2][BN] scales, [2][BN] row sums
  static constexpr int kSmem = 1024 + kRing + kBarBytes + kParamBytes + 64;
};

struct Tc2Params {
  const float* gamma;     // γ of W (1 value); null for raw output
  const float* gammaA;    // [M]
  const int32_t* rowsum;  // [M]
  void* Y;                // [M, N] float/bf16 (dequant) or int32 (raw)
  int64_t M, N, K;
  int relu2, y_bf16;
  int tiles_n;            // ceil(N / 128)
  int tiles;              // tiles_n · ceil(M / 256)
  int splits;             // K ranges per tile (1: none)
  int kb_per_split;       // K blocks (128) per range, a multiple of 4
  int32_t* part;          // splits > 1: [splits, M, N] partial accumulators
  int32_t* counter;       // splits > 1: [tiles] arrival counters, zero at launch
};

__device__ __forceinline__ void mma_i8_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// One output element: undo the code offset, then dequantise (or keep raw).
template <int OUT>
__device__ __forceinline__ void tc2_store(const Tc2Params& p, int64_t m, int64_t n, int acc, int rs,
                                          float sc) {
  const int v = acc - rs;
  const int64_t o = m * p.N + n;
  if constexpr (OUT == kTcRawI32) {
    reinterpret_cast<int32_t*>(p.Y)[o] = v;
  } else {
    float y = __fmul_rn((float)v, sc);
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

template <int OUT>
__global__ void __launch_bounds__(kTc2Threads, 1)
tc_persistent_kernel(const __grid_constant__ CUtensorMap tm_act,
                     const __grid_constant__ CUtensorMap tm_w, const Tc2Params p) {
  constexpr int SS = Tc2::kSS, WS = Tc2::kWS, AS = Tc2::kAS, BN = kTc2BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* s_b = smem;
  uint8_t* s_w = s_b + SS * Tc2::kBStage;
  uint8_t* s_a = s_w + WS * Tc2::kWStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tc2::kRing);
  uint64_t* full = bars;
  uint64_t* empty = full + SS;
  uint64_t* wfull = empty + SS;
  uint64_t* wempty = wfull + WS;
  uint64_t* afull = wempty + WS;
  uint64_t* aempty = afull + AS;
  uint64_t* accfull = aempty + AS;
  uint64_t* accempty = accfull + 2;
  uint64_t* done = accempty + 2;
  float* s_sc = reinterpret_cast<float*>(smem + Tc2::kRing + Tc2::kBarBytes);  // [2][BN]
  int* s_rs = reinterpret_cast<int*>(s_sc + 2 * BN);                          // [2][BN]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_rs + 2 * BN);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  volatile int* s_last = s_abort + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = (int)((p.K + kTcBK - 1) / kTcBK);
  const int items = p.tiles * p.splits;

  if (tid == 0) {
    for (int s = 0; s < SS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int v = 0; v < WS; ++v) {
      mbar_init(&wfull[v], 1);
      mbar_init(&wempty[v], 256);
    }
    for (int a = 0; a < AS; ++a) {
      mbar_init(&afull[a], 256);
      mbar_init(&aempty[a], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 128);
    }
    mbar_init(done, 1);
    *s_abort = 0;
    fence_barrier_init();
    prefetch_tensormap(&tm_act);
    prefetch_tensormap(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  pdl_launch_dependents();
  pdl_wait_prior_grid();

  // Work item it → tile (weight tile fastest, so concurrent CTAs share token
  // tiles in L2) and its K-block range [kb0, kb1).
  auto item = [&](int it, int64_t& m0, int64_t& n0, int& kb0, int& kb1, int& tile, int& split) {
    tile = it / p.splits;
    split = it - tile * p.splits;
    n0 = (int64_t)(tile % p.tiles_n) * 128;
    m0 = (int64_t)(tile / p.tiles_n) * BN;
    kb0 = split * p.kb_per_split;
    kb1 = min(KB, kb0 + p.kb_per_split);
  };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    uint32_t tcnt = 0, wcnt = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
      int64_t m0, n0;
      int kb0, kb1, tile, split;
      item(it, m0, n0, kb0, kb1, tile, split);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (((kb - kb0) & 3) == 0) {  // a new packed stage covers K blocks kb .. kb+3
          const int v = (int)(wcnt % WS);
          ok = wcnt < (uint32_t)WS || wait_or_abort(&wempty[v], ((wcnt / WS) + 1) & 1, s_abort);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tma_load_1x2d_warp(&wfull[v], Tc2::kWStage, s_w + v * Tc2::kWStage, &tm_w, kb * 32,
                             (int32_t)n0);
          ++wcnt;
        }
        const int s = (int)(tcnt % SS);
        ok = tcnt < (uint32_t)SS || wait_or_abort(&empty[s], ((tcnt / SS) + 1) & 1, s_abort);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tma_load_1x2d_warp(&full[s], Tc2::kBStage, s_b + s * Tc2::kBStage, &tm_act, kb * kTcBK,
                           (int32_t)m0);
        ++tcnt;
      }
    }
    if (!ok && lane == 0) {  // drain copies that may be in flight (bounded)
      for (uint32_t d = tcnt > (uint32_t)SS ? tcnt - SS : 0; d < tcnt; ++d)
        mbar_wait_for(&full[d % SS], (d / SS) & 1, 100000000ull);
      for (uint32_t d = wcnt > (uint32_t)WS ? wcnt - WS : 0; d < wcnt; ++d)
        mbar_wait_for(&wfull[d % WS], (d / WS) & 1, 100000000ull);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idesc = idesc_i8(128, BN);
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    const uint32_t b_base = __shfl_sync(0xffffffffu, smem_u32(s_b), 0);
    const uint32_t a_base = __shfl_sync(0xffffffffu, smem_u32(s_a), 0);
    uint32_t tcnt = 0, acnt = 0;
    int itc = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x, ++itc) {
      int64_t m0, n0;
      int kb0, kb1, tile, split;
      item(it, m0, n0, kb0, kb1, tile, split);
      const int acc = itc & 1;
      ok = itc < 2 || wait_or_abort(&accempty[acc], ((itc >> 1) + 1) & 1, s_abort);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      for (int kb = kb0; kb < kb1; ++kb) {
        const int s = (int)(tcnt % SS), a = (int)(acnt % AS);
        ok = wait_or_abort(&full[s], (tcnt / SS) & 1, s_abort);
        if (ok) ok = wait_or_abort(&afull[a], (acnt / AS) & 1, s_abort);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        const uint64_t bd = smem_desc_sw128(b_base + s * Tc2::kBStage);
        const uint64_t ad = smem_desc_sw128(a_base + a * Tc2::kAStage);
#pragma unroll
        for (int kk = 0; kk < kTcBK / 32; ++kk)
          mma_i8_ss_warp(tm + acc * BN, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc,
                         (kb > kb0 || kk > 0) ? 1u : 0u);
        mma_commit_warp(&empty[s]);
        mma_commit_warp(&aempty[a]);
        ++tcnt;
        ++acnt;
      }
      if (ok) mma_commit_warp(&accfull[acc]);
    }
    mma_commit_warp(done);  // tracks every MMA issued
  } else if (warp < 10) {
    // ---------------- expansion (warps 2..9) ----------------
    const int ew = warp - 2;
    const int row = 32 * (ew & 3) + lane;  // weight row of the tile
    const int h = ew >> 2;                 // half of each K block: A chunks 4h .. 4h+3
    uint32_t wcnt = 0, acnt = 0;
    int v = 0;
    uint32_t wpar = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
      int64_t m0, n0;
      int kb0, kb1, tile, split;
      item(it, m0, n0, kb0, kb1, tile, split);
      for (int kb = kb0; kb < kb1; ++kb) {
        const int sub = (kb - kb0) & 3;
        if (sub == 0) {
          v = (int)(wcnt % WS);
          wpar = (wcnt / WS) & 1;
          ++wcnt;
        }
        const int a = (int)(acnt % AS);
        ok = wait_or_abort(&wfull[v], wpar, s_abort);
        if (ok && acnt >= (uint32_t)AS) ok = wait_or_abort(&aempty[a], ((acnt / AS) + 1) & 1, s_abort);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        // K block kb is 16-byte chunks 2·sub, 2·sub+1 of the row's 128-byte packed line.
        const uint4 u = *reinterpret_cast<const uint4*>(s_w + v * Tc2::kWStage + row * 128 +
                                                        (((2 * sub + h) ^ (row & 7)) << 4));
        if (sub == 3 || kb == kb1 - 1) mbar_arrive(&wempty[v]);
        uint8_t* dst = s_a + a * Tc2::kAStage + row * 128;
        const uint32_t x[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // packed word q → 16 codes = A chunk 4h + q
          uint32_t o0, o1, o2, o3;
          expand_word(x[q], o0, o1, o2, o3);
          *reinterpret_cast<uint4*>(dst + (((4 * h + q) ^ (row & 7)) << 4)) = make_uint4(o0, o1, o2, o3);
        }
        fence_proxy_async_smem();  // generic-proxy writes → visible to the MMA (async proxy)
        mbar_arrive(&afull[a]);
        ++acnt;
      }
    }
  } else {
    // ---------------- epilogue (warps 10..13) ----------------
    const int q = warp & 3;  // TMEM lane quarter
    const int row = 32 * q + lane;
    const int et = tid - 320;  // 0 .. 127
    const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
    const float g = p.gamma != nullptr ? __ldg(p.gamma) : 0.0f;
    bool dead = false;  // an aborted CTA still walks the same barriers
    int itc = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++itc) {
      int64_t m0, n0;
      int kb0, kb1, tile, split;
      item(it, m0, n0, kb0, kb1, tile, split);
      const int acc = itc & 1;
      float* sc = s_sc + acc * BN;
      int* rs = s_rs + acc * BN;
      for (int j = et; j < BN; j += 128) {
        const int64_t m = m0 + j;
        const bool in = m < p.M;
        sc[j] = (in && p.gammaA != nullptr) ? __fdiv_rn(__fmul_rn(__ldg(p.gammaA + m), g), 127.0f) : 0.0f;
        rs[j] = in ? __ldg(p.rowsum + m) : 0;
      }
      epilogue_bar();
      bool ok = !dead && wait_or_abort(&accfull[acc], (itc >> 1) & 1, s_abort);
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld is warp-collective
      dead = dead || !ok;
      const int64_t n = n0 + row;
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t d[16];
          tmem_ld_32x32b_x16(t_lane + acc * BN + c0, d);
          tmem_wait_ld();
          if (n < p.N) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int64_t m = m0 + c0 + j;
              if (m < p.M) {
                if (p.splits > 1)
                  p.part[((int64_t)split * p.M + m) * p.N + n] = (int32_t)d[j];
                else
                  tc2_store<OUT>(p, m, n, (int)d[j], rs[c0 + j], sc[c0 + j]);
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&accempty[acc]);
      }
      if (p.splits > 1) {
        // The last of the tile's K ranges to finish sums the partials.
        __threadfence();
        epilogue_bar();
        if (et == 0) *s_last = (!dead && atomicAdd(p.counter + tile, 1) == p.splits - 1) ? 1 : 0;
        epilogue_bar();
        if (*s_last && n < p.N) {
          __threadfence();
          for (int j = 0; j < BN; ++j) {
            const int64_t m = m0 + j;
            if (m >= p.M) break;
            int sum = 0;
            for (int sp = 0; sp < p.splits; ++sp) sum += __ldcg(p.part + ((int64_t)sp * p.M + m) * p.N + n);
            tc2_store<OUT>(p, m, n, sum, rs[j], sc[j]);
          }
        }
        if (*s_last && et == 0) p.counter[tile] = 0;  // ready for the next launch
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every MMA must be complete before TMEM is released (bounded)
    mbar_wait_for(done, 0, 1000000000ull);
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bl
