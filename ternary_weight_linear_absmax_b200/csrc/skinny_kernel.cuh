// Skinny contraction: 5 ≤ M ≤ 64 int8 tokens against a packed ternary
// matrix (small-batch decode, and the FFN block at small M).
//
// "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section
// "Como funciona a camada BitLinear ... (Zero-GEMM)?": acc = A_q·W_qᵀ in
// INT32 (add on +1, subtract on -1, skip on 0), then (γ_A·γ)/127.
//
// Why not tcgen05 here: one kind::i8 tcgen05.mma (M = 128, K = 32) takes
// ≈170-185 cycles whatever its N, so with N ≤ 64 tokens it runs far below
// the tensor peak, and 128-row weight tiles leave most SMs idle when there
// are only 4096 outputs. This kernel spreads every matrix over all SMs like
// the decode GEMV and does the multiply-adds with warp-level
// mma.sync.m16n8k32 (s8·s8 → s32) on register fragments:
//  * A = tokens, 16-token m-tiles, read with ldmatrix from 128-byte-swizzled
//    TMA boxes (conflict-free).
//  * B = weights, 8-row n-tiles. Each fragment register is expanded from
//    the packed words in place: (word >> 2t) & 0x03030303 holds the codes
//    c = w+1 ∈ {0,1,2} of 4 consecutive weights, in the order the fragment
//    wants them.
//  * Σ c·a − Σ a = Σ w·a: the token row sums are subtracted in the epilogue.
//  * The CTA's weight rows and the tokens stream through a ring of stages of
//    512 K each (one weight box of 128 packed bytes per row, four token
//    boxes), with a full and an empty barrier per stage. The weight boxes of
//    the first stages are requested before the programmatic-dependent-launch
//    wait, so they stream while the kernel that produces the tokens runs.
//    A TMA request costs its issuing thread tens of cycles, so the five
//    requests of a stage are spread over the lane 0s of different warps.
//  * Every CTA reads the same token lines. CTA b walks the K chunks starting
//    at chunk b mod (number of chunks), so at any moment the CTAs spread
//    their token requests over all chunks instead of all asking L2 for the
//    same lines (integer sums do not depend on the order).
//  * The 16 warps form NG n-tile groups × KS K-lanes (NG = KPS, KS = 16/KPS).
//    Warp (ng, ks) owns n-tiles [ng·NTW, ng·NTW+NTW) for all MTT m-tiles and
//    the KPS consecutive 32-K steps ks·KPS … ks·KPS+KPS-1 of each stage (a
//    pair of steps shares one 16-byte load of packed weights). KPS is a
//    compile-time constant so the step loop unrolls and fragment loads run
//    ahead of the mma.sync chain (a rolled loop measured ~2.7x slower). The
//    K-lanes'
//    partial sums are written in fragment order to shared memory
//    (conflict-free 16-byte stores) and summed by the epilogue, which
//    dequantises (or writes raw INT32) straight from fragment coordinates.
// All waits are bounded; on give-up the error flag is raised and the CTA
// leaves its outputs untouched.
#pragma once

#include "bl_device.cuh"

namespace bl {

constexpr int kSkThreads = 512;
constexpr int kSkWarps = kSkThreads / 32;
constexpr int kSkKC = 512;              // K values per stage (one weight box)
constexpr int kSkMaxTokens = 64;
// Above this many tokens the tensor-core tiles take a contraction when they
// fill at least half of the SMs.
constexpr int kSkPreferTokens = 32;
constexpr int kSkMaxRowsPad = 128;      // rows computed per CTA ≤ 128: ≤ 16 n-tiles
constexpr size_t kSkSmemCap = 226 * 1024;  // of the 227 KiB a CTA may opt into

struct SkinnyParams {
  const float* gamma;     // γ of W (1 value); unused for raw output
  const float* gammaA;    // [M]; unused for raw output
  const int32_t* rowsum;  // [M]  Σ_k A_q[m,k]
  void* Y;                // [M, N] float/bf16 (dequant) or int32 (raw)
  int64_t M, N, K;
  int rows_per_cta;       // R: rows owned (and stored) by a CTA
  int rows_pad;           // R_pad = 8·NT ≥ R: rows loaded and computed
  int stages;             // S: ring depth
  int relu2;
  int y_bf16;
  int raw;                // 1: raw INT32 output (acc = A_q·W_qᵀ)
};

__host__ __device__ inline int skinny_chunks(int64_t K) { return (int)((K + kSkKC - 1) / kSkKC); }
__host__ __device__ inline size_t skinny_stage_bytes(int rows_pad, int mtt) {
  return (size_t)rows_pad * 128 + 4 * (size_t)(16 * mtt) * 128;
}
// Fragment-order partial sums: 16 warps × NTW × MTT × 32 lanes × 16 bytes.
__host__ __device__ inline size_t skinny_red_bytes(int ntw, int mtt) {
  return (size_t)kSkWarps * ntw * mtt * 512;
}
// [ring S × (weight box, 4 token boxes), aliased by the partial sums after the
//  main loop][scale: 64 fp32][row sums: 64 int32][full S][empty S]
__host__ __device__ inline size_t skinny_smem_bytes(int rows_pad, int mtt, int stages, int ntw) {
  size_t ring = (size_t)stages * skinny_stage_bytes(rows_pad, mtt);
  const size_t red = skinny_red_bytes(ntw, mtt);
  if (red > ring) ring = red;
  return 1024 + ring + 2 * kSkMaxTokens * 4 + (size_t)stages * 16;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma_s8_16832(int (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Issuers of sequence c's five TMA requests (lane 0 of these warps): warp
// c mod 16 for the weight box, warp (4c + q + 8) mod 16 for token box q.
// Inverted: warp w issues token box q = w mod 4 of sequences c ≡ c0 (mod 4),
// c0 = (w/4 + 2) mod 4.
__device__ __forceinline__ int skinny_t_box(int warp) { return warp & 3; }
__device__ __forceinline__ int skinny_t_first(int warp) { return ((warp >> 2) + 2) & 3; }

// MTT: token m-tiles (16 tokens each; rows past M read as zero).
// NTW: n-tiles (8 weight rows each) per warp. KPS: 32-K steps per warp and
// stage (warps = KPS n-tile groups × 16/KPS K-lanes).
template <int MTT, int NTW, int KPS>
__global__ void __launch_bounds__(kSkThreads, 1)
skinny_ternary_kernel(const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_a, const SkinnyParams p) {
  constexpr int MB = 16 * MTT;  // token rows per box
  constexpr int NG = KPS, KS = kSkWarps / KPS;
  constexpr uint32_t kTokBox = MB * 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int RP = p.rows_pad, NT = RP / 8;
  const int S = p.stages;
  const uint32_t wbox = (uint32_t)RP * 128;
  const uint32_t stage_bytes = wbox + 4 * kTokBox;
  size_t ring = (size_t)S * stage_bytes;
  const size_t red_bytes = skinny_red_bytes(NTW, MTT);
  if (red_bytes > ring) ring = red_bytes;
  float* s_sc = reinterpret_cast<float*>(smem + ring);
  int* s_rs = reinterpret_cast<int*>(s_sc + kSkMaxTokens);
  uint64_t* full = reinterpret_cast<uint64_t*>(s_rs + kSkMaxTokens);
  uint64_t* empty = full + S;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;  // mma fragment coordinates
  const int64_t r0 = (int64_t)blockIdx.x * p.rows_per_cta;
  const int nchunk = skinny_chunks(p.K);
  const int rot = (int)(blockIdx.x % (unsigned)nchunk);
  const int M = (int)p.M;

  auto issue_w = [&](int c, int st) {  // weight box of sequence c into stage st
    const int cc = (c + rot) % nchunk;
    mbar_arrive_expect_tx(&full[st], wbox);
    tma_load_2d(smem + (size_t)st * stage_bytes, &tm_w, cc * 128, (int32_t)r0, &full[st]);
  };
  auto issue_t = [&](int c, int st, int q) {  // token box q of sequence c into stage st
    const int cc = (c + rot) % nchunk;
    mbar_arrive_expect_tx(&full[st], kTokBox);
    tma_load_2d(smem + (size_t)st * stage_bytes + wbox + q * kTokBox, &tm_a, cc * kSkKC + q * 128, 0,
                &full[st]);
  };

  // 1. Barriers (one arrival per request of a fill: the weight box and four
  //    token boxes), then the weight boxes of the first S stages: they do
  //    not depend on the previous kernel.
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 5);
      mbar_init(&empty[s], kSkWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (lane == 0) {
    if (warp == 1) prefetch_tensormap(&tm_a);
    for (int c = warp; c < S; c += kSkWarps) issue_w(c, c);
  }
  pdl_launch_dependents();
  // 2. Tokens, their scales and row sums come from the previous kernel.
  pdl_wait_prior_grid();
  const int tq = skinny_t_box(warp), tc0 = skinny_t_first(warp);
  if (lane == 0) {
    for (int c = tc0; c < S; c += 4) issue_t(c, c, tq);
  }
  if (tid < M) {
    s_rs[tid] = __ldg(p.rowsum + tid);
    s_sc[tid] = p.raw ? 0.0f : __fdiv_rn(__fmul_rn(__ldg(p.gammaA + tid), __ldg(p.gamma)), 127.0f);
  }

  const int ng = warp % NG, ks = warp / NG;
  int acc[NTW][MTT][4];
#pragma unroll
  for (int j = 0; j < NTW; ++j)
#pragma unroll
    for (int m = 0; m < MTT; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][m][e] = 0;
  // This warp's 32-K steps of a stage: kk = ks·KPS + i, i < KPS (KPS even),
  // so pairs (kk, kk+1) share one 16-byte chunk of packed weights.
  // Byte offsets inside a stage (the 128-byte swizzle puts 16-byte chunk x of
  // row r at x ^ (r % 8)):
  //  * tokens, ldmatrix: lane → (row lrow of the m-tile, 16-byte half lhi of
  //    the step): matrices 0..3 are (rows 0-7, K 0-15), (rows 8-15, K 0-15),
  //    (rows 0-7, K 16-31), (rows 8-15, K 16-31), i.e. registers a0..a3.
  //    Step kk is token box kk/4, chunks 2·(kk%4) and 2·(kk%4)+1.
  //  * weights: slot j reads row 8·min(ng·NTW+j, NT-1)+g (slots past the last
  //    n-tile repeat it and are dropped by the epilogue); step kk is packed
  //    bytes [8·kk, +8): chunk kk/2, half kk%2.
  const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int lhi = lane >> 4;
  uint32_t toff[KPS];
#pragma unroll
  for (int i = 0; i < KPS; ++i) {
    const int kk = ks * KPS + i;
    toff[i] = (uint32_t)((kk >> 2) * kTokBox + lrow * 128 + (((2 * (kk & 3) + lhi) ^ (lane & 7)) << 4));
  }
  uint32_t woff[NTW];
#pragma unroll
  for (int j = 0; j < NTW; ++j) woff[j] = (uint32_t)(min(ng * NTW + j, NT - 1) * 8 + g) * 128;
  uint32_t wsub[KPS / 2];
#pragma unroll
  for (int q = 0; q < KPS / 2; ++q) wsub[q] = (uint32_t)((((ks * KPS) / 2 + q) ^ g) << 4);

  bool ok = true;
  int s = 0, sp = 0;
  uint32_t par = 0, ppar = 0;
  for (int c = 0; c < nchunk; ++c) {
    // Refill the stage that sequence c-1 used (sp) with sequence c-1+S once
    // every warp has released it.
    if (lane == 0 && c >= 1 && c - 1 + S < nchunk) {
      const int cn = c - 1 + S;
      const bool wi = (cn & (kSkWarps - 1)) == warp, ti = ((cn - tc0) & 3) == 0;
      if ((wi || ti) && mbar_wait(&empty[sp], ppar)) {
        if (wi) issue_w(cn, sp);
        if (ti) issue_t(cn, sp, tq);
      }
    }
    ok = __all_sync(0xffffffffu, mbar_wait(&full[s], par));
    if (!ok) break;
    const uint8_t* wst = smem + (size_t)s * stage_bytes;
    const uint8_t* tk = wst + wbox;
#pragma unroll
    for (int q = 0; q < KPS / 2; ++q) {
      uint4 w[NTW];
#pragma unroll
      for (int j = 0; j < NTW; ++j) w[j] = *reinterpret_cast<const uint4*>(wst + woff[j] + wsub[q]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t a[MTT][4];
#pragma unroll
        for (int m = 0; m < MTT; ++m) ldmatrix_x4(a[m], tk + toff[2 * q + h] + m * 16 * 128);
#pragma unroll
        for (int j = 0; j < NTW; ++j) {
          // b0 = codes of k = 4t..4t+3, b1 = codes of k = 16+4t..16+4t+3
          const uint32_t b0 = ((h ? w[j].z : w[j].x) >> (2 * t)) & 0x03030303u;
          const uint32_t b1 = ((h ? w[j].w : w[j].y) >> (2 * t)) & 0x03030303u;
#pragma unroll
          for (int m = 0; m < MTT; ++m) mma_s8_16832(acc[j][m], a[m], b0, b1);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    sp = s;
    ppar = par;
    if (++s == S) {
      s = 0;
      par ^= 1u;
    }
  }
  // A warp that gave up raised the error flag; the whole CTA leaves.
  if (__syncthreads_or(!ok)) return;

  // 3. Partial sums in fragment order (the ring is free: every stage was
  //    waited for and consumed).
  int4* red = reinterpret_cast<int4*>(smem);
#pragma unroll
  for (int j = 0; j < NTW; ++j)
#pragma unroll
    for (int m = 0; m < MTT; ++m)
      red[(((ks * NG + ng) * NTW + j) * MTT + m) * 32 + lane] =
          make_int4(acc[j][m][0], acc[j][m][1], acc[j][m][2], acc[j][m][3]);
  __syncthreads();

  // 4. Epilogue: sum the K-lanes of one fragment slot (ng, j, m, lane),
  //    undo the code offset (Σ A_q), scale, store. Fragment c0, c1: token
  //    16m+g, weight rows 8·tile+2t, +1; c2, c3: token 16m+g+8.
  const int Rv = (int)min((int64_t)p.rows_per_cta, p.N - r0);  // rows stored by this CTA
  // Rows 8·tile+2t, +1 are adjacent outputs; with N and r0 even their offset
  // is even, so the pair is one aligned vector store.
  const bool pair_ok = ((p.N | r0) & 1) == 0;
  constexpr int kSlots = NG * NTW * MTT * 32;
  for (int sl = tid; sl < kSlots; sl += kSkThreads) {
    const int ln = sl & 31, m = (sl >> 5) % MTT, tile = (sl >> 5) / MTT;  // tile = ng·NTW + j
    if (tile >= NT) continue;
    int4 v = red[sl];
#pragma unroll
    for (int q = 1; q < KS; ++q) {
      const int4 u = red[q * kSlots + sl];
      v.x += u.x;
      v.y += u.y;
      v.z += u.z;
      v.w += u.w;
    }
    const int gg = ln >> 2, tt = ln & 3;
    const int row = tile * 8 + 2 * tt;  // even
    const int vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // token 16m+g, then 16m+g+8
      const int tok = 16 * m + gg + 8 * h;
      if (tok >= M || row >= Rv) continue;
      const int rs = s_rs[tok];
      const int a0 = vals[2 * h] - rs, a1 = vals[2 * h + 1] - rs;
      const bool two = row + 1 < Rv;
      const int64_t o = (int64_t)tok * p.N + r0 + row;
      if (p.raw) {
        int32_t* y = reinterpret_cast<int32_t*>(p.Y) + o;
        if (two && pair_ok) {
          *reinterpret_cast<int2*>(y) = make_int2(a0, a1);
        } else {
          y[0] = a0;
          if (two) y[1] = a1;
        }
      } else {
        const float sc = s_sc[tok];
        float y0 = __fmul_rn((float)a0, sc), y1 = __fmul_rn((float)a1, sc);
        if (p.relu2) {
          y0 = fmaxf(y0, 0.0f);
          y0 = __fmul_rn(y0, y0);
          y1 = fmaxf(y1, 0.0f);
          y1 = __fmul_rn(y1, y1);
        }
        if (p.y_bf16) {
          __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(p.Y) + o;
          if (two && pair_ok) {
            *reinterpret_cast<__nv_bfloat162*>(y) = __floats2bfloat162_rn(y0, y1);
          } else {
            y[0] = __float2bfloat16_rn(y0);
            if (two) y[1] = __float2bfloat16_rn(y1);
          }
        } else {
          float* y = reinterpret_cast<float*>(p.Y) + o;
          if (two && pair_ok) {
            *reinterpret_cast<float2*>(y) = make_float2(y0, y1);
          } else {
            y[0] = y0;
            if (two) y[1] = y1;
          }
        }
      }
    }
  }
}

}  // namespace bl
