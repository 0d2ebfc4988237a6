// Decode GEMV: a few tokens (M ≤ 4) against a packed ternary matrix.
//
// "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", sections
// "Como funciona a camada BitLinear ... (Zero-GEMM)?" (INT32 add/subtract/skip
// contraction, then one scale (γ_A·γ)/127) and "Como o BitNet quebra o Memory
// Wall ..." (decode streams 0.25 byte per weight; the kernel is HBM-bound).
//
// Design (one launch per call):
//  * Each CTA owns a contiguous slab of R weight rows. Its first warp issues
//    one bulk copy (TMA, cp.async.bulk) per row into shared memory before
//    anything else — with programmatic dependent launch this happens while
//    the previous kernel on the stream is still running.
//  * The CTA then waits for the previous grid (griddepcontrol.wait) and
//    quantises the M tokens into shared memory (AbsMax prologue), or
//    requantises the FFN intermediate, or copies pre-quantised int8 tokens.
//  * Warps split K, lanes split rows: lane l of warp w handles rows l, l+32,
//    ... and 64-weight chunks w, w+8, .... Weight rows sit in shared memory
//    at a pitch chosen so a quarter-warp's 16-byte loads hit 8 distinct bank
//    groups; activations are read as broadcasts.
//  * Codes c = w+1 ∈ {0,1,2} are used directly as int8 operands of dp4a:
//    Σ c·a = Σ w·a + Σ a, so the token's Σ a is subtracted once per row.
//  * Partial sums of the 8 warps are combined in shared memory; the epilogue
//    applies (γ_A·γ)/127 (and ReLU²) or writes the raw INT32 result.
#pragma once

#include "bl_device.cuh"

namespace bl {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvMaxTokens = 4;

enum GemvSrc : int { kSrcFloat = 0, kSrcFfnRequant = 1, kSrcInt8 = 2 };
enum GemvOut : int { kOutDequant = 0, kOutRawI32 = 1 };

struct GemvParams {
  const void* A;            // kSrcFloat: T[M,K]; kSrcFfnRequant: int32[M,K]; kSrcInt8: int8[M,K]
  const float* a_scale;     // kSrcFfnRequant: γ_X[M]; kSrcInt8: γ_A[M]
  const float* a_gamma_up;  // kSrcFfnRequant: γ_up (1 value)
  const int32_t* a_rowsum;  // kSrcInt8: Σ A_q per token, or nullptr
  const uint8_t* W;         // packed [N, K/4]
  const float* gamma;       // γ of W (1 value)
  void* Y;                  // kOutDequant: float/bf16 [M,N]; kOutRawI32: int32 [M,N]
  float* gamma_out;         // optional: per-token γ_A written by CTA 0
  int64_t N;
  int64_t K;
  int rows_per_cta;
  int pitch;  // bytes between weight rows in shared memory
  int M;
  float eps;
  int relu2;
  int y_bf16;
};

__host__ __device__ inline int gemv_pitch(int64_t K) {
  // Row pitch in 32-bit words ≡ 4 (mod 8): 16-byte loads of 8 consecutive
  // lanes (8 consecutive rows) then cover all 32 banks exactly once.
  const int w = (int)(K / 16);
  return 4 * (w + ((4 - (w % 8)) + 8) % 8);
}

// Shared memory: [0,128) mbarrier + per-token scalars; then R weight rows at
// the padded pitch; then the int8 tokens; then the per-warp partial sums.
constexpr int kGemvHeader = 128;

__host__ __device__ inline size_t gemv_smem_bytes(int64_t K, int rows, int M) {
  size_t s = kGemvHeader;
  s += (size_t)rows * gemv_pitch(K);                  // weights
  s += (size_t)M * K;                                  // int8 activations
  s += (size_t)kGemvWarps * M * rows * sizeof(int);    // warp partials
  return (s + 127) & ~(size_t)127;
}

template <int MT, int RPL, typename TA, int SRC, int OUT>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_ternary_kernel(const GemvParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t K = p.K;
  const int kbytes = (int)(K / 4);
  const int64_t r0 = (int64_t)blockIdx.x * p.rows_per_cta;
  const int R = (int)min((int64_t)p.rows_per_cta, p.N - r0);
  const int M = p.M;

  uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem);
  float* s_sc = reinterpret_cast<float*>(smem + 16);   // [MT] dequant scale (γ_A·γ)/127
  int* s_sum = reinterpret_cast<int*>(smem + 32);      // [MT] Σ A_q
  float* s_tok = reinterpret_cast<float*>(smem + 48);  // [MT] token scale γ_A (or γ_r)
  uint8_t* s_w = smem + kGemvHeader;
  int8_t* s_a = reinterpret_cast<int8_t*>(s_w + (size_t)p.rows_per_cta * p.pitch);
  int* s_part = reinterpret_cast<int*>(s_a + (size_t)M * K);

  // 1. Stream this CTA's weight rows into shared memory (independent of the
  //    previous kernel on the stream).
  if (tid == 0) {
    mbar_init(s_bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(s_bar, (uint32_t)R * (uint32_t)kbytes);
    __syncwarp();
    for (int i = lane; i < R; i += 32)
      bulk_g2s(s_w + (size_t)i * p.pitch, p.W + (r0 + i) * kbytes, (uint32_t)kbytes, s_bar);
  }
  pdl_launch_dependents();
  // 2. Activations and outputs are ordered after the previous kernel.
  pdl_wait_prior_grid();

  // 3. Token prologue → int8 tokens in shared memory, Σ A_q, scales.
  if constexpr (SRC == kSrcFloat) {
    __shared__ float red[kGemvWarps][MT];
    const TA* A = reinterpret_cast<const TA*>(p.A);
    constexpr int VEC = 16 / sizeof(TA);
    const int64_t nvec = K / VEC;
    float mx[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) mx[m] = 0.0f;
    for (int64_t v = tid; v < nvec; v += kGemvThreads) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          uint4 u = __ldg(reinterpret_cast<const uint4*>(A + m * K) + v);
          const TA* e = reinterpret_cast<const TA*>(&u);
#pragma unroll
          for (int i = 0; i < VEC; ++i) mx[m] = fmaxf(mx[m], fabsf(to_f32<TA>(e[i])));
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float t = warp_max(mx[m]);
      if (lane == 0) red[warp][m] = t;
    }
    __syncthreads();
    if (tid < MT) {
      float t = 0.0f;
      for (int w = 0; w < kGemvWarps; ++w) t = fmaxf(t, red[w][tid]);
      s_tok[tid] = t;  // γ_A
      if (tid < M && p.gamma_out != nullptr && blockIdx.x == 0) p.gamma_out[tid] = t;
    }
    __syncthreads();
    int sum[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) sum[m] = 0;
    for (int64_t v = tid; v < nvec; v += kGemvThreads) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          const float s = __fdiv_rn(127.0f, __fadd_rn(s_tok[m], p.eps));
          uint4 u = __ldg(reinterpret_cast<const uint4*>(A + m * K) + v);
          const TA* e = reinterpret_cast<const TA*>(&u);
          int8_t q[VEC];
#pragma unroll
          for (int i = 0; i < VEC; ++i) {
            q[i] = quant_i8(to_f32<TA>(e[i]), s);
            sum[m] += q[i];
          }
          if constexpr (VEC == 8)
            *reinterpret_cast<uint2*>(s_a + m * K + v * VEC) = *reinterpret_cast<uint2*>(q);
          else
            *reinterpret_cast<uint32_t*>(s_a + m * K + v * VEC) = *reinterpret_cast<uint32_t*>(q);
        }
      }
    }
    __shared__ int redi[kGemvWarps][MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      int t = warp_sum_i(sum[m]);
      if (lane == 0) redi[warp][m] = t;
    }
    __syncthreads();
    if (tid < MT) {
      int t = 0;
      for (int w = 0; w < kGemvWarps; ++w) t += redi[w][tid];
      s_sum[tid] = t;
    }
  } else if constexpr (SRC == kSrcFfnRequant) {
    // h = fp32(acc·fp32((γ_X·γ_up)/127)); r = max(h,0)²; γ_r = max r;
    // q = Clip(Round(r·127/(γ_r+ε))).
    __shared__ float red[kGemvWarps][MT];
    const int32_t* A = reinterpret_cast<const int32_t*>(p.A);
    const float gup = *p.a_gamma_up;
    float scu[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m)
      scu[m] = m < M ? __fdiv_rn(__fmul_rn(p.a_scale[m], gup), 127.0f) : 0.0f;
    const int64_t nvec = K / 4;
    float mx[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) mx[m] = 0.0f;
    for (int64_t v = tid; v < nvec; v += kGemvThreads) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          int4 u = __ldg(reinterpret_cast<const int4*>(A + m * K) + v);
          const int e[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float h = fmaxf(__fmul_rn((float)e[i], scu[m]), 0.0f);
            mx[m] = fmaxf(mx[m], __fmul_rn(h, h));
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float t = warp_max(mx[m]);
      if (lane == 0) red[warp][m] = t;
    }
    __syncthreads();
    if (tid < MT) {
      float t = 0.0f;
      for (int w = 0; w < kGemvWarps; ++w) t = fmaxf(t, red[w][tid]);
      s_tok[tid] = t;  // γ_r
      if (tid < M && p.gamma_out != nullptr && blockIdx.x == 0) p.gamma_out[tid] = t;
    }
    __syncthreads();
    int sum[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) sum[m] = 0;
    for (int64_t v = tid; v < nvec; v += kGemvThreads) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          const float s = __fdiv_rn(127.0f, __fadd_rn(s_tok[m], p.eps));
          int4 u = __ldg(reinterpret_cast<const int4*>(A + m * K) + v);
          const int e[4] = {u.x, u.y, u.z, u.w};
          int8_t q[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float h = fmaxf(__fmul_rn((float)e[i], scu[m]), 0.0f);
            q[i] = quant_i8(__fmul_rn(h, h), s);
            sum[m] += q[i];
          }
          *reinterpret_cast<uint32_t*>(s_a + m * K + v * 4) = *reinterpret_cast<uint32_t*>(q);
        }
      }
    }
    __shared__ int redi[kGemvWarps][MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      int t = warp_sum_i(sum[m]);
      if (lane == 0) redi[warp][m] = t;
    }
    __syncthreads();
    if (tid < MT) {
      int t = 0;
      for (int w = 0; w < kGemvWarps; ++w) t += redi[w][tid];
      s_sum[tid] = t;
    }
  } else {  // kSrcInt8
    const int8_t* A = reinterpret_cast<const int8_t*>(p.A);
    const int64_t nvec = K / 16;
    int sum[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) sum[m] = 0;
    for (int64_t v = tid; v < nvec; v += kGemvThreads) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          uint4 u = __ldg(reinterpret_cast<const uint4*>(A + m * K) + v);
          *reinterpret_cast<uint4*>(s_a + m * K + v * 16) = u;
          sum[m] = dp4a(u.x, 0x01010101u, sum[m]);
          sum[m] = dp4a(u.y, 0x01010101u, sum[m]);
          sum[m] = dp4a(u.z, 0x01010101u, sum[m]);
          sum[m] = dp4a(u.w, 0x01010101u, sum[m]);
        }
      }
    }
    __shared__ int redi[kGemvWarps][MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      int t = warp_sum_i(sum[m]);
      if (lane == 0) redi[warp][m] = t;
    }
    __syncthreads();
    if (tid < MT) {
      int t = 0;
      for (int w = 0; w < kGemvWarps; ++w) t += redi[w][tid];
      s_sum[tid] = (p.a_rowsum != nullptr && tid < M) ? p.a_rowsum[tid] : t;
      s_tok[tid] = (tid < M && p.a_scale != nullptr) ? p.a_scale[tid] : 0.0f;
    }
  }
  if (tid < MT) {
    const float g = p.gamma != nullptr ? *p.gamma : 0.0f;  // absent for raw INT32 output
    s_sc[tid] = __fdiv_rn(__fmul_rn(s_tok[tid], g), 127.0f);  // (γ_A·γ)/127
  }
  __syncthreads();

  // 4. Weights must have landed.
  __shared__ int s_ok;
  if (tid == 0) s_ok = mbar_wait(s_bar, 0) ? 1 : 0;
  __syncthreads();
  // On give-up the error flag is raised and the outputs are left untouched.
  // The wait that gave up was the wait for this CTA's own copies.
  if (!s_ok) return;
  // Each thread observes the completed phase itself (acquire of the
  // bulk-copy writes); the phase is already complete, so this returns at once.
  mbar_wait(s_bar, 0);

  // 5. Contraction.
  int acc[RPL][MT];
#pragma unroll
  for (int t = 0; t < RPL; ++t)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[t][m] = 0;
  const int nchunks = (int)(K / 64);
  for (int c = warp; c < nchunks; c += kGemvWarps) {
    uint32_t a[MT][16];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m < M) {
        const uint4* src = reinterpret_cast<const uint4*>(s_a + m * K + c * 64);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 u = src[v];
          a[m][4 * v + 0] = u.x;
          a[m][4 * v + 1] = u.y;
          a[m][4 * v + 2] = u.z;
          a[m][4 * v + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int v = 0; v < 16; ++v) a[m][v] = 0u;
      }
    }
#pragma unroll
    for (int t = 0; t < RPL; ++t) {
      const int i = lane + 32 * t;
      if (i < R) {
        const uint4 wv = *reinterpret_cast<const uint4*>(s_w + (size_t)i * p.pitch + c * 16);
        const uint32_t x[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t e0, e1, e2, e3;
          expand_word(x[q], e0, e1, e2, e3);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            acc[t][m] = dp4a(e0, a[m][4 * q + 0], acc[t][m]);
            acc[t][m] = dp4a(e1, a[m][4 * q + 1], acc[t][m]);
            acc[t][m] = dp4a(e2, a[m][4 * q + 2], acc[t][m]);
            acc[t][m] = dp4a(e3, a[m][4 * q + 3], acc[t][m]);
          }
        }
      }
    }
  }
  const int RP = p.rows_per_cta;
#pragma unroll
  for (int t = 0; t < RPL; ++t) {
    const int i = lane + 32 * t;
    if (i < R) {
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < M) s_part[(warp * M + m) * RP + i] = acc[t][m];
    }
  }
  __syncthreads();

  // 6. Epilogue: combine the warps, undo the code offset, scale.
  for (int e = tid; e < M * R; e += kGemvThreads) {
    const int m = e / R, i = e - m * R;
    int d = 0;
#pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) d += s_part[(w * M + m) * RP + i];
    const int v = d - s_sum[m];
    const int64_t o = (int64_t)m * p.N + r0 + i;
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
