// Decode GEMV: a few tokens (M ≤ 4) against a packed ternary matrix.
//
// "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", sections
// "Como funciona a camada BitLinear ... (Zero-GEMM)?" (INT32 add/subtract/skip
// contraction, then one scale (γ_A·γ)/127) and "Como o BitNet quebra o Memory
// Wall ..." (decode streams 0.25 byte per weight; the kernel is HBM-bound).
//
// Design (one launch per call, 512 threads per CTA, two CTAs per SM so the
// next call's CTA can already be resident):
//  * Each CTA owns a contiguous slab of R ≤ 128 weight rows. One thread
//    issues K/512 tensor copies (TMA, 128-byte swizzle) of R rows × 128
//    bytes each into shared memory before anything else. With programmatic
//    dependent launch this happens while the previous kernel on the stream
//    is still running, so in a decode chain the weight stream overlaps the
//    previous layer's work.
//  * The CTA then waits for the previous grid (griddepcontrol.wait) and runs
//    the token prologue in one pass over global memory: AbsMax quantisation
//    of the tokens, or the FFN ReLU² requantisation, or a copy of int8 tokens.
//  * Each thread owns two rows (r and r + ⌈R/2⌉) and a chunk group (every
//    CG-th 64-weight chunk of K), so the R·K/64 chunk tasks spread evenly over
//    the 512 threads and each token load serves two rows. The swizzle places
//    16-byte chunk j of row r at position j ^ (r mod 8) of its 128-byte line,
//    so consecutive lanes (consecutive rows, same chunk) load without bank
//    conflicts; token words are broadcast loads.
//  * Contraction with codes c = w+1 ∈ {0,1,2}: a packed word x holds, in byte
//    i, the codes of weights 4j+i at bits 2j. For each j, x & (3·0x01010101
//    << 2j) is a vector of four unsigned bytes c·4^j, so one LOP3 and one
//    dp4a (unsigned × signed) per 4 weights accumulate 4^j·Σ c·a into acc[j];
//    Σ c·a = acc[0] + acc[1]/4 + acc[2]/16 + acc[3]/64 exactly. Σ w·a is then
//    Σ c·a − Σ a, with Σ a (the token's row sum) taken once.
//  * Partial sums are combined in shared memory; the epilogue
//    applies (γ_A·γ)/127 (and ReLU²) or writes the raw INT32 result.
#pragma once

#include "bl_device.cuh"

namespace bl {

constexpr int kGemvThreads = 512;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvMaxTokens = 4;
constexpr int kGemvMaxRows = 128;
// 16-byte token vectors kept in registers per thread and token.
template <int MT>
__host__ __device__ constexpr int gemv_reg_vecs() { return MT == 1 ? 4 : (MT == 2 ? 2 : 1); }

enum GemvSrc : int { kSrcFloat = 0, kSrcFfnRequant = 1, kSrcInt8 = 2 };
enum GemvOut : int { kOutDequant = 0, kOutRawI32 = 1 };

struct GemvParams {
  const void* A;            // kSrcFloat: T[M,K]; kSrcFfnRequant: int32[M,K]; kSrcInt8: int8[M,K]
  const float* a_scale;     // kSrcFfnRequant: γ_X[M]; kSrcInt8: γ_A[M]
  const float* a_gamma_up;  // kSrcFfnRequant: γ_up (1 value)
  const int32_t* a_rowsum;  // kSrcInt8: Σ A_q per token, or nullptr
  const uint8_t* W;         // packed [N, K/4]
  const float* gamma;       // γ of W (1 value); may be null for raw output
  void* Y;                  // kOutDequant: float/bf16 [M,N]; kOutRawI32: int32 [M,N]
  float* gamma_out;         // optional: per-token γ_A (or γ_r) written by CTA 0
  // FFN hand-off (one-token blocks). kOutRawI32 with rmax_out: each CTA also
  // writes, per token m, the largest r = max(h,0)² over its rows, h =
  // fp32(acc · s_sc[m]) — the values the down-projection requantises — to
  // rmax_out[m·gridDim.x + blockIdx.x]. kSrcFfnRequant with rmax_in: γ_r of
  // token m is the largest of rmax_in[m·rmax_n .. m·rmax_n + rmax_n), so
  // the prologue reads the accumulators once (no separate max pass).
  // rmax_atomic: instead, every CTA raises rmax_out[m] (zeroed by the caller)
  // to its maximum with an atomic max on the float bits (r ≥ 0).
  float* rmax_out;
  const float* rmax_in;
  int rmax_n;
  int rmax_atomic;
  // Optional taps (all null = off): the int8 tokens [M,K], their per-token
  // scale γ and Σ of the int8 tokens, as the prologue of CTA tap_cta made them.
  int8_t* tap_q;
  float* tap_gamma;
  int32_t* tap_rowsum;
  int tap_cta;
  int64_t N;
  int64_t K;
  int rows_per_cta;
  int rows_pad;  // rows per CTA rounded up to 8 (rows of one swizzled box)
  int M;
  float eps;
  int relu2;
  int y_bf16;
};

// Shared memory holds the slab as K/512 boxes of rows_pad × 128 bytes.
__host__ __device__ inline int gemv_boxes(int64_t K) { return (int)((K / 4 + 127) / 128); }
__host__ __device__ inline int gemv_rows_pad(int rows) { return (rows + 7) & ~7; }

// Chunk groups per row: as many as the 512 threads allow, at most one per
// 64-weight chunk.
__host__ __device__ inline int gemv_chunk_groups(int rows, int64_t K) {
  int cg = kGemvThreads / (rows > 0 ? rows : 1);
  const int nchunks = (int)(K / 64);
  if (cg > nchunks) cg = nchunks;
  return cg < 1 ? 1 : cg;
}

// Shared memory: [0,1024) mbarrier + per-token scalars; then the weight
// boxes (1024-byte aligned, as the 128-byte swizzle requires); then the int8
// tokens; then the per-warp partial sums.
constexpr int kGemvHeader = 1024;

__host__ __device__ inline size_t gemv_smem_bytes(int64_t K, int rows, int M) {
  size_t s = kGemvHeader;
  s += (size_t)gemv_boxes(K) * gemv_rows_pad(rows) * 128;  // weights
  s += (size_t)M * K;                                      // int8 tokens
  s += (size_t)M * rows * sizeof(int);                     // per-row sums
  return s + 1024;                                         // base alignment slack
}

// d = Σ_i ua[i]·sb[i] + c over the four bytes; a unsigned, b signed.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Combine the per-warp entries of one token (16 values, 16-byte aligned).
__device__ __forceinline__ unsigned warp_slots_max(const unsigned (&v)[kGemvWarps]) {
  unsigned r = 0u;
#pragma unroll
  for (int i = 0; i < kGemvWarps; i += 4) {
    const uint4 q = *reinterpret_cast<const uint4*>(v + i);
    r = max(r, max(max(q.x, q.y), max(q.z, q.w)));
  }
  return r;
}
__device__ __forceinline__ int warp_slots_sum(const int (&v)[kGemvWarps]) {
  int r = 0;
#pragma unroll
  for (int i = 0; i < kGemvWarps; i += 4) {
    const int4 q = *reinterpret_cast<const int4*>(v + i);
    r += (q.x + q.y) + (q.z + q.w);
  }
  return r;
}

template <int MT, typename TA, int SRC, int OUT>
__global__ void __launch_bounds__(kGemvThreads, 2)
gemv_ternary_kernel(const __grid_constant__ CUtensorMap tm_w, const GemvParams p) {
  // The one-token FFN requantiser keeps a whole 11008-accumulator row in
  // registers (6 vectors per thread): one L2 round trip after the wait.
  constexpr int RV = (SRC == kSrcFfnRequant && MT == 1) ? 6 : gemv_reg_vecs<MT>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  // Per-warp partial results (no shared atomics): the max as float bits (all
  // values are ≥ 0) and Σ A_q; every reader combines the 16 entries itself.
  __shared__ __align__(16) unsigned s_wmax[MT][kGemvWarps];
  __shared__ __align__(16) int s_wsum[MT][kGemvWarps];
  __shared__ float s_sc[MT];      // per-token dequant scale (γ_A·γ)/127
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t K = p.K;
  // Rows [r0, r1) of an even split over the grid (at most rows_per_cta).
  const int64_t r0 = (int64_t)blockIdx.x * p.N / gridDim.x;
  const int R = (int)((int64_t)(blockIdx.x + 1) * p.N / gridDim.x - r0);
  const int M = p.M;

  uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem);
  uint8_t* s_w = smem + kGemvHeader;
  const int nbox = gemv_boxes(K);
  const int box_bytes = p.rows_pad * 128;
  int8_t* s_a = reinterpret_cast<int8_t*>(s_w + (size_t)nbox * box_bytes);
  int* s_part = reinterpret_cast<int*>(s_a + (size_t)M * K);

  // 1. Stream this CTA's weight rows into shared memory (independent of the
  //    previous kernel on the stream).
  if (tid == 0) {
    mbar_init(s_bar, 1);
    fence_barrier_init();
  }
  for (int i = tid; i < M * p.rows_per_cta; i += kGemvThreads) s_part[i] = 0;
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(s_bar, (uint32_t)nbox * (uint32_t)box_bytes);
    for (int b = 0; b < nbox; ++b)
      tma_load_2d(s_w + (size_t)b * box_bytes, &tm_w, b * 128, (int32_t)r0, s_bar);
  } else if (tid == 32) {
    // Warm L2 with the tokens (the reads themselves wait for the prior grid).
    const size_t tok_bytes = (size_t)M * K *
        (SRC == kSrcFloat ? sizeof(TA) : (SRC == kSrcFfnRequant ? 4 : 1));
    for (size_t o = 0; o < tok_bytes; o += 65536)
      prefetch_l2(reinterpret_cast<const uint8_t*>(p.A) + o,
                  (uint32_t)min((size_t)65536, tok_bytes - o));
  }
  // γ of W is as static as W itself (see BL_FLAG_PDL), so it is read before
  // the dependency wait.
  const float gamma_w = p.gamma != nullptr ? __ldg(p.gamma) : 0.0f;
  pdl_launch_dependents();

  // Contraction mapping (see step 5): thread t < RH·CG owns rows ra = t mod RH
  // and rb = ra + RH (RH = ⌈R/2⌉) and chunk group cg = t / RH, i.e. the
  // 64-weight chunks cg, cg + CG, ... of both rows.
  const int RH = (R + 1) >> 1;
  const int CG = gemv_chunk_groups(RH, K);
  const int nchunks = (int)(K / 64);
  const bool active = tid < RH * CG;
  const int ra = active ? tid % RH : 0;
  const int cg = active ? tid / RH : 0;
  const bool has_b = ra + RH < R;
  const int rb = has_b ? ra + RH : ra;
  const uint8_t* wa = s_w + (size_t)ra * 128;
  const uint8_t* wb = s_w + (size_t)rb * 128;
  const int swa = ra & 7, swb = rb & 7;
  auto wload = [&](const uint8_t* w, int sw, int c) {
    // chunk c: box c/8, 16-byte slot (c mod 8) XOR (row mod 8)
    return *reinterpret_cast<const uint4*>(w + (size_t)(c >> 3) * box_bytes + (((c & 7) ^ sw) << 4));
  };

  // 2. The weights do not depend on the previous kernel either: wait for
  //    them and move this thread's first kRegChunks chunks into registers
  //    before the dependency wait, so the contraction after it starts from
  //    registers.
  //    One thread waits (bounded) and the outcome is made CTA-uniform, so a
  //    give-up returns every thread together and no barrier is left waiting.
  __shared__ int s_wok;
  if (tid == 0) s_wok = mbar_wait(s_bar, 0) ? 1 : 0;
  __syncthreads();
  if (!s_wok) {
    // Gave up: the error flag is raised and this CTA's outputs stay
    // untouched. The CTA still waits for the previous grid, so that a kernel
    // launched after this one stays ordered after it, and gives its own
    // copies a last bounded chance to land before shared memory is released.
    if (warp == 0) pdl_wait_prior_grid();
    if (tid == 0) mbar_wait_for(s_bar, 0, 100000000ull);
    return;
  }
  mbar_wait(s_bar, 0);  // phase complete: acquires the copies for this thread
  constexpr int kRegChunks = MT <= 2 ? 2 : 0;
  uint4 rwa[kRegChunks > 0 ? kRegChunks : 1], rwb[kRegChunks > 0 ? kRegChunks : 1];
#pragma unroll
  for (int i = 0; i < kRegChunks; ++i) {
    const int c = cg + i * CG;
    if (active && c < nchunks) {
      rwa[i] = wload(wa, swa, c);
      rwb[i] = wload(wb, swb, c);
    }
  }

  // Tokens and outputs are ordered after the previous kernel: every thread
  // waits for the prior grid itself (no CTA barrier after the release; in a
  // 1000-call decode chain this measured 2 % faster than one waiting warp).
  pdl_wait_prior_grid();

  // 3. Token prologue → int8 tokens in shared memory, Σ A_q and the scales.
  //    Warp reductions use redux.sync; warps combine through shared atomics.
  if constexpr (SRC == kSrcFloat || SRC == kSrcFfnRequant) {
    constexpr int VEC = SRC == kSrcFloat ? 16 / (int)sizeof(TA) : 4;
    const int64_t nvec = K / VEC;
    float scu[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) scu[m] = 0.0f;
    if constexpr (SRC == kSrcFfnRequant) {
      const float gup = *p.a_gamma_up;
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < M) scu[m] = __fdiv_rn(__fmul_rn(p.a_scale[m], gup), 127.0f);
    }
    // The value each element is quantised from.
    auto value = [&](const uint4& u, int i, int m) -> float {
      if constexpr (SRC == kSrcFloat) {
        return to_f32<TA>(reinterpret_cast<const TA*>(&u)[i]);
      } else {
        // r = max(h,0)² with h = fp32(acc · fp32((γ_X·γ_up)/127))
        const float h =
            fmaxf(__fmul_rn((float)reinterpret_cast<const int*>(&u)[i], scu[m]), 0.0f);
        return __fmul_rn(h, h);
      }
    };
    auto row_ptr = [&](int m) {
      return reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(p.A) +
                                            (size_t)m * (size_t)nvec * 16);
    };
    // γ_r handed over by the up-projection: the accumulator loads below
    // only fill registers, and the max comes from the per-CTA maxima.
    const bool given = SRC == kSrcFfnRequant && p.rmax_in != nullptr;
    uint4 reg[MT][RV];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float mx = 0.0f;
      if (m < M) {
        const uint4* src = row_ptr(m);
#pragma unroll
        for (int r = 0; r < RV; ++r) {
          const int64_t v = tid + (int64_t)r * kGemvThreads;
          if (v < nvec) reg[m][r] = __ldg(src + v);
        }
        if (given) {
          for (int j = tid; j < p.rmax_n; j += kGemvThreads)
            mx = fmaxf(mx, __ldg(p.rmax_in + (int64_t)m * p.rmax_n + j));
        } else {
#pragma unroll
          for (int r = 0; r < RV; ++r) {
            const int64_t v = tid + (int64_t)r * kGemvThreads;
            if (v < nvec) {
#pragma unroll
              for (int i = 0; i < VEC; ++i) mx = fmaxf(mx, fabsf(value(reg[m][r], i, m)));
            }
          }
          for (int64_t v = tid + (int64_t)RV * kGemvThreads; v < nvec; v += kGemvThreads) {
            const uint4 u = __ldg(src + v);
#pragma unroll
            for (int i = 0; i < VEC; ++i) mx = fmaxf(mx, fabsf(value(u, i, m)));
          }
        }
      }
      const unsigned wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
      if (lane == 0) s_wmax[m][warp] = wmax;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      int tsum = 0;
      if (m < M) {
        const float g = __uint_as_float(warp_slots_max(s_wmax[m]));  // γ_A (or γ_r)
        const float s = __fdiv_rn(127.0f, __fadd_rn(g, p.eps));
        const uint4* src = row_ptr(m);
        auto emit = [&](const uint4& u, int64_t v) {
          uint32_t b[VEC], w[VEC / 4];
#pragma unroll
          for (int i = 0; i < VEC; ++i) b[i] = quant_i8_bits(value(u, i, m), s);
#pragma unroll
          for (int i = 0; i < VEC / 4; ++i) {
            w[i] = pack4_low_bytes(b[4 * i], b[4 * i + 1], b[4 * i + 2], b[4 * i + 3]);
            tsum = dp4a(w[i], 0x01010101u, tsum);  // Σ of the four int8 values
          }
          if constexpr (VEC == 8)
            *reinterpret_cast<uint2*>(s_a + m * K + v * VEC) = make_uint2(w[0], w[1]);
          else
            *reinterpret_cast<uint32_t*>(s_a + m * K + v * VEC) = w[0];
        };
#pragma unroll
        for (int r = 0; r < RV; ++r) {
          const int64_t v = tid + (int64_t)r * kGemvThreads;
          if (v < nvec) emit(reg[m][r], v);
        }
        for (int64_t v = tid + (int64_t)RV * kGemvThreads; v < nvec; v += kGemvThreads)
          emit(__ldg(src + v), v);
        // The last thread has no token vector when K/VEC < 512: it makes the
        // scale while the others quantise.
        if (tid == kGemvThreads - 1) {
          s_sc[m] = __fdiv_rn(__fmul_rn(g, gamma_w), 127.0f);  // (γ_A·γ)/127
          if (p.gamma_out != nullptr && blockIdx.x == 0) p.gamma_out[m] = g;
        }
      }
      const int wsum = __reduce_add_sync(0xffffffffu, tsum);
      if (lane == 0) s_wsum[m][warp] = wsum;
    }
  } else {  // kSrcInt8
    const int8_t* A = reinterpret_cast<const int8_t*>(p.A);
    const int64_t nvec = K / 16;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      int tsum = 0;
      if (m < M) {
        for (int64_t v = tid; v < nvec; v += kGemvThreads) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(A + m * K) + v);
          *reinterpret_cast<uint4*>(s_a + m * K + v * 16) = u;
          tsum = dp4a(u.x, 0x01010101u, tsum);
          tsum = dp4a(u.y, 0x01010101u, tsum);
          tsum = dp4a(u.z, 0x01010101u, tsum);
          tsum = dp4a(u.w, 0x01010101u, tsum);
        }
        if (tid == kGemvThreads - 1) {
          const float g = p.a_scale != nullptr ? p.a_scale[m] : 0.0f;
          s_sc[m] = __fdiv_rn(__fmul_rn(g, gamma_w), 127.0f);
        }
      }
      const int wsum = __reduce_add_sync(0xffffffffu, tsum);
      if (lane == 0) s_wsum[m][warp] = wsum;
    }
  }
  __syncthreads();

  // 4. Taps: CTA tap_cta reports its int8 tokens, scales and sums.
  if (p.tap_q != nullptr && (int)blockIdx.x == p.tap_cta) {
    const int64_t nv = (int64_t)M * K / 16;
    for (int64_t v = tid; v < nv; v += kGemvThreads)
      reinterpret_cast<uint4*>(p.tap_q)[v] = reinterpret_cast<const uint4*>(s_a)[v];
    if (tid < M) {
      if constexpr (SRC == kSrcInt8)
        p.tap_gamma[tid] = p.a_scale != nullptr ? p.a_scale[tid] : 0.0f;
      else
        p.tap_gamma[tid] = __uint_as_float(warp_slots_max(s_wmax[tid]));
      p.tap_rowsum[tid] = warp_slots_sum(s_wsum[tid]);
    }
  }

  // 5. Contraction (mapping above). The two rows share every token load
  //    and keep 8 independent accumulators per token. Consecutive lanes take
  //    consecutive rows at the same chunk: the swizzle keeps their weight
  //    loads conflict-free and the token loads are broadcasts.
  int acc[2][MT][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[h][m][j] = 0;
  auto contract = [&](const uint4& va, const uint4& vb, int c) {
    const uint32_t xa[4] = {va.x, va.y, va.z, va.w};
    const uint32_t xb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m < M) {
        const uint4* ap = reinterpret_cast<const uint4*>(s_a + m * K + c * 64);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 a = ap[q];  // token words 16c+4q .. 16c+4q+3
          acc[0][m][0] = dp4a_us(xa[q] & 0x03030303u, a.x, acc[0][m][0]);
          acc[1][m][0] = dp4a_us(xb[q] & 0x03030303u, a.x, acc[1][m][0]);
          acc[0][m][1] = dp4a_us(xa[q] & 0x0C0C0C0Cu, a.y, acc[0][m][1]);
          acc[1][m][1] = dp4a_us(xb[q] & 0x0C0C0C0Cu, a.y, acc[1][m][1]);
          acc[0][m][2] = dp4a_us(xa[q] & 0x30303030u, a.z, acc[0][m][2]);
          acc[1][m][2] = dp4a_us(xb[q] & 0x30303030u, a.z, acc[1][m][2]);
          acc[0][m][3] = dp4a_us(xa[q] & 0xC0C0C0C0u, a.w, acc[0][m][3]);
          acc[1][m][3] = dp4a_us(xb[q] & 0xC0C0C0C0u, a.w, acc[1][m][3]);
        }
      }
    }
  };
  if (active) {
#pragma unroll
    for (int i = 0; i < kRegChunks; ++i) {
      const int c = cg + i * CG;
      if (c < nchunks) contract(rwa[i], rwb[i], c);
    }
#pragma unroll 2
    for (int c = cg + kRegChunks * CG; c < nchunks; c += CG)
      contract(wload(wa, swa, c), wload(wb, swb, c), c);
    // Σ c·a over this thread's chunks (acc[j] is a multiple of 4^j, so the
    // arithmetic shifts are exact), accumulated per row in shared memory.
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m < M) {
        atomicAdd(&s_part[m * R + ra],
                  acc[0][m][0] + (acc[0][m][1] >> 2) + (acc[0][m][2] >> 4) + (acc[0][m][3] >> 6));
        if (has_b)
          atomicAdd(&s_part[m * R + rb],
                    acc[1][m][0] + (acc[1][m][1] >> 2) + (acc[1][m][2] >> 4) + (acc[1][m][3] >> 6));
      }
    }
  }
  __syncthreads();

  // 6. Epilogue: undo the code offset, scale.
  if constexpr (OUT == kOutRawI32) {
    if (p.rmax_out != nullptr) {
      // One warp stores this CTA's accumulators and reduces, per token, the
      // largest r = max(h,0)² (h = fp32(acc · s_sc[m])) for the hand-off.
      if (warp == 0) {
        float lm[MT], sc[MT];
        int ts[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          lm[m] = 0.0f;
          sc[m] = m < M ? s_sc[m] : 0.0f;
          ts[m] = m < M ? warp_slots_sum(s_wsum[m]) : 0;
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m < M) {
            for (int r = lane; r < R; r += 32) {
              const int v = s_part[m * R + r] - ts[m];
              reinterpret_cast<int32_t*>(p.Y)[(int64_t)m * p.N + r0 + r] = v;
              const float h = fmaxf(__fmul_rn((float)v, sc[m]), 0.0f);
              lm[m] = fmaxf(lm[m], __fmul_rn(h, h));
            }
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const unsigned w = __reduce_max_sync(0xffffffffu, __float_as_uint(lm[m]));
          if (lane == 0 && m < M) {
            if (p.rmax_atomic)
              atomicMax(reinterpret_cast<unsigned*>(p.rmax_out) + m, w);
            else
              p.rmax_out[(int64_t)m * gridDim.x + blockIdx.x] = __uint_as_float(w);
          }
        }
      }
      return;
    }
  }
  for (int e = tid; e < M * R; e += kGemvThreads) {
    const int m = e / R, r = e - m * R;
    const int v = s_part[m * R + r] - warp_slots_sum(s_wsum[m]);
    const int64_t o = (int64_t)m * p.N + r0 + r;
    if constexpr (OUT == kOutRawI32) {
      reinterpret_cast<int32_t*>(p.Y)[o] = v;
    } else {
      float y = __fmul_rn((float)v, s_sc[m]);
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

}  // namespace bl
