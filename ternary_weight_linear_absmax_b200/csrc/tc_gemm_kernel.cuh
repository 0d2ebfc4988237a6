// Ternary × INT8 contraction on the 5th-generation tensor cores (tcgen05,
// kind::i8) for more than 32 tokens (prefill, the FFN at larger batches).
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
  int kb_per_split;  // K blocks per blockIdx.z (a multiple of 4); all of K when unsplit.
                     // Split z writes raw INT32 partials to rows [z·Mp, z·Mp + M) of Y,
                     // Mp = M rounded up to the token tile, so a tile's rows past M
                     // (stored whole by the tensor stores) stay in z's own padding.
                     // Only split 0 subtracts the row sums.
  int64_t split_rows;  // Mp (0 when unsplit)
  int w_early;         // 1: the kernel before this one does not write the packed weights, so
                       //    the first weight stages are requested before the dependency wait
};

// DUAL: two CTAs per SM (BN 128 or 192). Each CTA then fits in half of the
// SM's shared memory and TMEM (256 columns: one accumulator, and 4 or 2 A
// stages), so one CTA's epilogue and set-up overlap the other's MMAs.
template <int BN_, bool DUAL_ = false>
struct TcConfig {
  static constexpr int BN = BN_;
  static constexpr bool kDual = DUAL_;
  static_assert(!DUAL_ || BN_ == 128 || BN_ == 192, "two CTAs per SM need BN 128 or 192");
  // Token ring: one 128-byte-wide K block (BN rows, 128-byte swizzle) per stage.
  static constexpr int kBStage = BN * kTcBK;
  // Deep enough to cover the L2 latency of the token tiles at the rate the
  // MMAs consume them (one 256-token tile, 32 KB, per ≈640 cycles): with four
  // stages the loads alone, without any MMA, bounded the prefill at 29 us.
  // Single configurations use what the 227 KB of shared memory allows.
  static constexpr int kSStages = DUAL_ ? (BN > 128 ? 3 : 4)
                                        : BN > 192 ? 5 : (BN > 128 ? 7 : (BN >= 128 ? 10 : (BN >= 64 ? 12 : (BN >= 32 ? 16 : 24))));
  // Weight ring: 128 rows × 128 packed bytes (4 K blocks) per stage, 128-byte
  // swizzle. Wide rows keep the number of TMA requests per byte low, which is
  // what bounds the stream when few tokens share each weight byte.
  static constexpr int kWStage = 128 * 128;
  static constexpr int kWStages = DUAL_ ? 2 : BN > 128 ? 2 : (BN >= 128 ? 3 : (BN >= 64 ? 4 : 6));
  // TMEM A stages (32 columns = one K block each).
  static constexpr int kTStages = DUAL_ && BN > 128 ? 2 : 4;
  // Independent accumulators: consecutive MMAs into one accumulator are
  // serialised by its read-modify-write, which dominates for small N. The
  // four MMAs of a stage rotate over kAcc accumulators, summed in the
  // epilogue (exact integer addition).
  static constexpr int kAcc = DUAL_ ? 1 : BN <= 64 ? 4 : (BN <= 128 ? 2 : 1);
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
  // 1 KiB slack for aligning the dynamic buffer to 1024 bytes. Single
  // configurations request at least 116 KiB so that only one CTA is resident
  // per SM: every CTA then gets its TMEM columns without waiting on another
  // CTA's allocation. Dual ones fit two per SM, 256 TMEM columns each.
  static constexpr int kSmemUsed = 1024 + kRingBytes + kBarBytes + kParamBytes + 64;
  static constexpr int kSmemBytes = DUAL_ ? kSmemUsed : (kSmemUsed > 116 * 1024 ? kSmemUsed : 116 * 1024);
  static_assert(!DUAL_ || (kTmemCols <= 256 && kSmemBytes <= 112 * 1024), "dual CTA too large");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory of one CTA");
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
                                                  int64_t n, int64_t zrow) {
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
        const int64_t o = (zrow + m) * p.N + n;
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
template <class C, int OUT, bool RELU, bool BF16, bool STAGE>
__device__ __forceinline__ void tc_epilogue(uint32_t t_lane, int row, int half, const float* s_sc,
                                            const int* s_rs, uint8_t* stage, const TcParams& p,
                                            int64_t m0, int64_t n, int64_t zrow, uint64_t* staged) {
  constexpr int BN = C::BN;
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
    tc_epilogue_chunk<CW, OUT, RELU, BF16, STAGE>(cur, c0, row, s_sc, s_rs, stage, p, m0, n, zrow);
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

template <class C, int OUT>
__global__ void __launch_bounds__(kTcThreads, C::kDual ? 2 : 1)
tc_ternary_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,
                       const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_y, const TcParams p) {
  constexpr int BN = C::BN;
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
  // This CTA's K blocks [kb_lo, kb_lo + KB); stage bookkeeping uses the local
  // index, TMA coordinates the global one.
  const int KBall = (int)((p.K + kTcBK - 1) / kTcBK);
  const int kb_lo = (int)blockIdx.z * p.kb_per_split;
  const int KB = min(KBall, kb_lo + p.kb_per_split) - kb_lo;
  const int64_t zrow = (int64_t)blockIdx.z * p.split_rows;  // output row offset of this split

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
  // completed, except the first weight stages when the caller says the
  // weights are not written by that kernel (w_early). The next kernel may
  // start its own set-up from here on.
  pdl_launch_dependents();
  // Weight stages requested before the dependency wait (w_early; warp 0).
  int w_pre = 0;
  if (warp == 0 && p.w_early) {
    w_pre = min((KB + 3) / 4, WS);
    for (int ws = 0; ws < w_pre; ++ws)
      tma_load_1x2d_warp(&wfull[ws], C::kWStage, s_w + ws * C::kWStage, &tm_w,
                         (kb_lo + 4 * ws) * 32, (int32_t)n0);
  }
  pdl_wait_prior_grid();

  if (warp == 0) {
    // ---------------- TMA producer (whole warp, one elected lane issues) ---
    int kb = 0, wissued = w_pre;
    for (; kb < KB; ++kb) {
      if ((kb & 3) == 0 && (kb >> 2) >= w_pre) {  // a new weight stage covers K blocks kb .. kb+3
        const int ws = kb >> 2, v = ws % WS;
        bool ok = ws < WS || wait_or_abort(&wempty[v], ((ws / WS) + 1) & 1, s_abort);
        if (!__all_sync(0xffffffffu, ok)) break;
        tma_load_1x2d_warp(&wfull[v], C::kWStage, s_w + v * C::kWStage, &tm_w, (kb_lo + kb) * 32,
                           (int32_t)n0);
        ++wissued;
      }
      const int s = kb % SS;
      bool ok = kb < SS || wait_or_abort(&empty[s], ((kb / SS) + 1) & 1, s_abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      tma_load_1x2d_warp(&full[s], C::kBStage, s_b + s * C::kBStage, &tm_act, (kb_lo + kb) * kTcBK,
                         (int32_t)m0);
      // Warm L2 with the token tile this stage will hold next time round.
      if (kb + SS < KB) tma_prefetch_2d_warp(&tm_act, (kb_lo + kb + SS) * kTcBK, (int32_t)m0);
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
        tma_store_2d(&tm_y, (int32_t)n0, (int32_t)(zrow + m0 + 32 * i), smem + (size_t)i * 32 * 128 * esz);
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
        par_rs[i] = (in && blockIdx.z == 0) ? __ldg(p.rowsum + m) : 0;  // subtracted once
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
          tc_epilogue<C, OUT, false, false, true>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, zrow, staged);
        else
          tc_epilogue<C, OUT, false, false, false>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, zrow, staged);
      } else {
        const int sel = (p.tma_store ? 4 : 0) | (p.y_bf16 ? 2 : 0) | (p.relu2 ? 1 : 0);
        switch (sel) {
          case 0: tc_epilogue<C, OUT, false, false, false>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, zrow, staged); break;
          case 1: tc_epilogue<C, OUT, true, false, false>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, zrow, staged); break;
          case 2: tc_epilogue<C, OUT, false, true, false>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, zrow, staged); break;
          case 3: tc_epilogue<C, OUT, true, true, false>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, zrow, staged); break;
          case 4: tc_epilogue<C, OUT, false, false, true>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, zrow, staged); break;
          case 5: tc_epilogue<C, OUT, true, false, true>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, zrow, staged); break;
          case 6: tc_epilogue<C, OUT, false, true, true>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, zrow, staged); break;
          default: tc_epilogue<C, OUT, true, true, true>(t_lane, row, hw, s_sc, s_rs, smem, p, m0, n, zrow, staged); break;
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

}  // namespace bl
