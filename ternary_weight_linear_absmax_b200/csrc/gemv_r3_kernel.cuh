// Decode GEMV on radix-3 weights: five ternary weights per byte.
//
// "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section "Como
// o ecossistema bitnet.cpp acelera inferência em CPUs e borda?": 3^5 = 243
// ≤ 256, so one byte holds five weights (1.60 bits per weight, 20 % fewer
// weight bytes than the 2-bit codes).
//
// Storage (the library's): a row is split into groups t of five weights,
// first most significant, b = Σ_i d_i·3^(4-i) with d = w + 1; the byte kept
// is q = ceil(256·b/243). Rows are padded with all-zero groups to a multiple
// of 16 bytes.
//
// Decoding without a table: with H_i = floor(3^i·q/256), the digits are
// d_i = H_{i+1} - 3·H_i, so for tokens a_0..a_4 of the group
//   Σ_i d_i·a_i = Σ_{i=1..4} H_i·(a_{i-1} - 3·a_i) + H_5·a_4 .
// The token coefficients β_i = a_{i-1} - 3·a_i (β_5 = a_4, |β| ≤ 508) are
// computed once per call in shared memory; the weights only need the H_i.
// For the four bytes of a 32-bit word, H_i of bytes 0, 2 and of bytes 1, 3
// come from two 16-bit-lane products (3^i·q < 2^16 for every i ≤ 5) and one
// byte permute gathers the four H_i bytes; dp2a (two int16 β × two uint8 H)
// accumulates. Σ w·a is then Σ d·a - Σ a.
//
// Layout and launch follow the 2-bit decode GEMV: 512 threads, two CTAs per
// SM, each CTA a slab of rows streamed by TMA (128-byte swizzle) before the
// programmatic-dependent-launch wait, then the token prologue.
#pragma once

#include "bl_device.cuh"
#include "gemv_kernel.cuh"
#include "gemv_prologue.cuh"

namespace bl {

struct GemvR3Params {
  const void* A;       // tokens [M, K] fp32/bf16
  const uint8_t* W;    // radix-3 [N, rb]
  const float* gamma;  // γ of W
  void* Y;             // [M, N] fp32/bf16, or int32 when raw
  int64_t N, K, rb;    // rb: bytes per row (multiple of 16)
  int rows_per_cta, rows_pad, M;
  float eps;
  int relu2, y_bf16, raw;
};

__host__ __device__ inline int64_t radix3_row_bytes(int64_t K) { return ((K + 4) / 5 + 15) / 16 * 16; }
__host__ __device__ inline int gemv_r3_boxes(int64_t rb) { return (int)((rb + 127) / 128); }

// [header 1024][weights nbox·rows_pad·128][int8 tokens M·5rb][β M·(rb/4)·40][row sums M·R·4]
__host__ __device__ inline size_t gemv_r3_smem_bytes(int64_t rb, int rows, int M) {
  size_t s = kGemvHeader;
  s += (size_t)gemv_r3_boxes(rb) * gemv_rows_pad(rows) * 128;
  s += (size_t)M * 5 * rb;
  s += (size_t)M * (rb / 4) * 40;
  s += (size_t)M * rows * sizeof(int);
  return s + 1024;
}

// d = c + β.lo·H.byte0 + β.hi·H.byte1 (lo) or ·H.byte2, ·H.byte3 (hi):
// two signed 16-bit × unsigned 8-bit products.
__device__ __forceinline__ int dp2a_lo_su(uint32_t beta, uint32_t h, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(beta), "r"(h), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi_su(uint32_t beta, uint32_t h, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(beta), "r"(h), "r"(c));
  return d;
}

// Radix-3 bytes from the 2-bit codes: one thread per output byte.
__global__ void __launch_bounds__(256)
radix3_pack_kernel(const uint8_t* __restrict__ W2, int64_t N, int64_t K, int64_t rb,
                   uint8_t* __restrict__ out) {
  const int64_t total = N * rb;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = e / rb, t = e - n * rb;
    const uint8_t* row = W2 + n * (K / 4);
    int b = 0;
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      const int64_t k = 5 * t + i;
      int d = 1;  // past K: weight 0
      if (k < K) {
        const uint32_t word = __ldg(reinterpret_cast<const uint32_t*>(row) + (k >> 4));
        d = (int)((word >> (8 * (k & 3) + 2 * ((k >> 2) & 3))) & 3u);
      }
      b = 3 * b + d;
    }
    out[e] = (uint8_t)((256 * b + 242) / 243);
  }
}

template <int MT, typename TA>
__global__ void __launch_bounds__(kGemvThreads, 2)
gemv_r3_kernel(const __grid_constant__ CUtensorMap tm_w, const GemvR3Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(16) unsigned s_wmax[MT][kGemvWarps];
  __shared__ __align__(16) int s_wsum[MT][kGemvWarps];
  __shared__ float s_sc[MT];
  __shared__ int s_wok;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t K = p.K, rb = p.rb, Kp = 5 * rb;
  // Rows [r0, r1) of an even split over the grid (at most rows_per_cta).
  const int64_t r0 = (int64_t)blockIdx.x * p.N / gridDim.x;
  const int R = (int)((int64_t)(blockIdx.x + 1) * p.N / gridDim.x - r0);
  const int M = p.M;
  const int nbox = gemv_r3_boxes(rb);
  const int box_bytes = p.rows_pad * 128;
  const int nwords = (int)(rb / 4);  // 32-bit words of a row (4 groups each)

  uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem);
  uint8_t* s_w = smem + kGemvHeader;
  int8_t* s_a = reinterpret_cast<int8_t*>(s_w + (size_t)nbox * box_bytes);
  uint2* s_beta = reinterpret_cast<uint2*>(s_a + (size_t)M * Kp);  // [M][nwords][5]
  int* s_part = reinterpret_cast<int*>(s_beta + (size_t)M * nwords * 5);

  // 1. Weight slab → shared memory, before the dependency wait.
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
    const size_t tok_bytes = (size_t)M * K * sizeof(TA);
    for (size_t o = 0; o < tok_bytes; o += 65536)
      prefetch_l2(reinterpret_cast<const uint8_t*>(p.A) + o, (uint32_t)min((size_t)65536, tok_bytes - o));
  }
  const float gamma_w = p.gamma != nullptr ? __ldg(p.gamma) : 0.0f;
  pdl_launch_dependents();
  if (tid == 0) s_wok = mbar_wait(s_bar, 0) ? 1 : 0;
  __syncthreads();
  if (!s_wok) {  // gave up (error flag raised): stay ordered, drain own copies, leave
    if (warp == 0) pdl_wait_prior_grid();
    if (tid == 0) mbar_wait_for(s_bar, 0, 100000000ull);
    return;
  }
  mbar_wait(s_bar, 0);
  if (warp == 0) pdl_wait_prior_grid();
  __syncthreads();

  // 2. AbsMax per token → int8 tokens (positions K .. 5·rb-1 are zero), Σ A_q.
  gemv_absmax_prologue<MT, TA>(reinterpret_cast<const TA*>(p.A), M, K, Kp, p.eps, gamma_w, s_a,
                               s_wmax, s_wsum, s_sc);

  // 3. Token coefficients: word u holds groups t = 4u + j (j = 0..3); for digit
  //    i = 1..5, β_i of the four groups as int16 pairs (j = 0, 1 | j = 2, 3).
  for (int e = tid; e < M * nwords; e += kGemvThreads) {
    const int m = e / nwords, u = e - m * nwords;
    const int8_t* a = s_a + m * Kp + 20 * (int64_t)u;  // tokens 20u .. 20u+19
    int beta[5][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int i = 1; i <= 4; ++i) beta[i - 1][j] = (int)a[5 * j + i - 1] - 3 * (int)a[5 * j + i];
      beta[4][j] = (int)a[5 * j + 4];
    }
    uint2* dst = s_beta + ((size_t)m * nwords + u) * 5;
#pragma unroll
    for (int i = 0; i < 5; ++i)
      dst[i] = make_uint2((uint32_t)(beta[i][0] & 0xFFFF) | ((uint32_t)beta[i][1] << 16),
                          (uint32_t)(beta[i][2] & 0xFFFF) | ((uint32_t)beta[i][3] << 16));
  }
  __syncthreads();

  // 4. Contraction: thread t < RH·CG owns rows ra = t mod RH, rb2 = ra + RH and
  //    the 16-byte chunks cg, cg + CG, ... (chunk = 4 words = 80 weights).
  const int RH = (R + 1) >> 1;
  const int nchunks = (int)(rb / 16);
  int CG = kGemvThreads / (RH > 0 ? RH : 1);
  if (CG > nchunks) CG = nchunks;
  if (CG < 1) CG = 1;
  const bool active = tid < RH * CG;
  const int ra = active ? tid % RH : 0, cg = active ? tid / RH : 0;
  const bool has_b = ra + RH < R;
  const int rbw = has_b ? ra + RH : ra;
  int acc[2][MT];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[h][m] = 0;
  if (active) {
    for (int c = cg; c < nchunks; c += CG) {
      uint4 wv[2];
      const int rows[2] = {ra, rbw};
#pragma unroll
      for (int h = 0; h < 2; ++h)
        wv[h] = *reinterpret_cast<const uint4*>(s_w + (size_t)(c >> 3) * box_bytes + rows[h] * 128 +
                                                (((c & 7) ^ (rows[h] & 7)) << 4));
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int u = 4 * c + q;
        uint32_t H[2][5];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t w = q == 0 ? wv[h].x : (q == 1 ? wv[h].y : (q == 2 ? wv[h].z : wv[h].w));
          const uint32_t E = __byte_perm(w, 0u, 0x4240), O = __byte_perm(w, 0u, 0x4341);
          uint32_t pe = E, po = O;
#pragma unroll
          for (int i = 0; i < 5; ++i) {
            pe *= 3u;
            po *= 3u;
            H[h][i] = __byte_perm(pe, po, 0x7351);  // H_{i+1} of bytes 0, 1, 2, 3
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m < M) {
            const uint2* bt = s_beta + ((size_t)m * nwords + u) * 5;
#pragma unroll
            for (int i = 0; i < 5; ++i) {
              const uint2 b = bt[i];
#pragma unroll
              for (int h = 0; h < 2; ++h)
                acc[h][m] = dp2a_hi_su(b.y, H[h][i], dp2a_lo_su(b.x, H[h][i], acc[h][m]));
            }
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m < M) {
        atomicAdd(&s_part[m * R + ra], acc[0][m]);
        if (has_b) atomicAdd(&s_part[m * R + rbw], acc[1][m]);
      }
    }
  }
  __syncthreads();

  // 5. Epilogue: Σ w·a = Σ d·a − Σ a; scale or raw.
  for (int e = tid; e < M * R; e += kGemvThreads) {
    const int m = e / R, r = e - m * R;
    const int v = s_part[m * R + r] - warp_slots_sum(s_wsum[m]);
    const int64_t o = (int64_t)m * p.N + r0 + r;
    if (p.raw) {
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
