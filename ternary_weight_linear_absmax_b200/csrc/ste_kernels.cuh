// Straight-through-estimator (STE) backward of BitLinear.
//
// "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section "Como
// funciona a camada BitLinear ... (Zero-GEMM)?", STE paragraph: in the
// backward pass the gradient of the quantisation is the identity inside the
// valid range. With the forward Y = Â·Ŵᵀ (Ŵ = γ·W_q, Â = (γ_A/127)·A_q):
//   dA = dY·Ŵ                         [M, K]   (contraction over N)
//   dW = 1[|W ÷ (γ+ε)| ≤ 1] ⊙ dYᵀ·Â   [N, K]   (contraction over M)
// Both are dense contractions, so both run as one tcgen05 kind::f16 GEMM
// (bf16 operands, fp32 accumulation in tensor memory) after small layout
// kernels that put the contraction dimension innermost:
//   dA:  A = dY [M, N] (as given, bf16), B = W_qᵀ [K, N] bf16 {-1, 0, +1}
//        expanded from the packed codes, scale γ in the epilogue;
//   dW:  A = dYᵀ [N, M] bf16, B = Âᵀ [K, M] bf16, mask in the epilogue.
// W_q is exact in bf16; dY (when fp32) and Â are rounded to bf16 once.
#pragma once

#include "bl_device.cuh"

namespace bl {

// ---------------------------------------------------------------------------
// GEMM C[r, c] = scale · Σ_k A[r, k]·B[c, k], A [rows, kdim], B [cols, kdim]
// bf16 with kdim contiguous. Tile 128 × BN, 64 bf16 (128 bytes) of K per
// stage. Warp 0 issues the TMA loads, warp 1 owns TMEM and issues the MMAs,
// warps 2..5 read the accumulator (one TMEM lane quarter each) and store.
constexpr int kGmThreads = 192;
constexpr int kGmBM = 128;
constexpr int kGmBK = 64;  // bf16 per stage row: one 128-byte swizzle row

template <int BN>
struct GmConfig {
  static constexpr int kStageA = kGmBM * 128;
  static constexpr int kStageB = BN * 128;
  static constexpr int kStages = BN >= 256 ? 4 : 6;
  static constexpr int kRing = kStages * (kStageA + kStageB);
  static constexpr int kSmem = 1024 + kRing + (2 * kStages + 2) * 8 + 16;
  static constexpr int kTmemCols = BN;
};

struct GmParams {
  int64_t rows, cols, kdim;
  float* C;               // [rows, cols] fp32, row-major
  const float* scale;     // optional device scalar multiplying C
  const void* mask_w;     // optional [rows, cols] fp32/bf16 latent weights for the STE mask
  int mask_bf16;
  const float* mask_gamma;  // γ of those weights (device)
  float eps;
};

// Instruction descriptor for kind::f16 with bf16 A and B, fp32 D, both
// K-major, M = m, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t m, uint32_t n) {
  return (1u << 4)           // D format: f32
         | (1u << 7)         // A: bf16
         | (1u << 10)        // B: bf16
         | ((n >> 3) << 17)  // N / 8
         | ((m >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void mma_bf16_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One elected lane arms `bar` for `tx` bytes and issues two 2-D tensor loads
// completing on it.
__device__ __forceinline__ void tma_load_2x2d_warp(uint64_t* bar, uint32_t tx, void* dst0,
                                                   const CUtensorMap* m0, void* dst1,
                                                   const CUtensorMap* m1, int32_t x, int32_t y0,
                                                   int32_t y1) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t"
      "@e cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%2], [%3, {%6, %7}], [%0];\n\t"
      "@e cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%4], [%5, {%6, %8}], [%0];\n\t}" ::"r"(smem_u32(bar)),
      "r"(tx), "r"(smem_u32(dst0)), "l"(reinterpret_cast<uint64_t>(m0)), "r"(smem_u32(dst1)),
      "l"(reinterpret_cast<uint64_t>(m1)), "r"(x), "r"(y0), "r"(y1)
      : "memory");
}

template <int BN, bool MASK>
__global__ void __launch_bounds__(kGmThreads, 1)
bf16_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const GmParams p) {
  using C = GmConfig<BN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* s_a = smem;                                 // S × 128 rows × 128 B
  uint8_t* s_b = smem + S * C::kStageA;                // S × BN rows × 128 B
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kRing);
  uint64_t* empty = full + S;
  uint64_t* done = empty + S;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(done + 2);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t r0 = (int64_t)blockIdx.x * kGmBM;
  const int64_t c0 = (int64_t)blockIdx.y * BN;
  const int KB = (int)((p.kdim + kGmBK - 1) / kGmBK);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *s_abort = 0;
    fence_barrier_init();
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
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
    // ---- TMA producer ----
    int kb = 0;
    for (; kb < KB; ++kb) {
      const int s = kb % S;
      bool ok = kb < S || mbar_wait(&empty[s], ((kb / S) + 1) & 1);
      if (!__all_sync(0xffffffffu, ok)) {
        *s_abort = 1;
        break;
      }
      tma_load_2x2d_warp(&full[s], C::kStageA + C::kStageB, s_a + s * C::kStageA, &tm_a,
                         s_b + s * C::kStageB, &tm_b, kb * kGmBK, (int32_t)r0, (int32_t)c0);
    }
    if (*s_abort && lane == 0) {  // drain copies in flight (bounded) before exit
      for (int d = max(0, kb - S); d < kb; ++d) mbar_wait_for(&full[d % S], (d / S) & 1, 100000000ull);
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    constexpr uint32_t idesc = idesc_bf16(kGmBM, BN);
    const uint32_t a_base = __shfl_sync(0xffffffffu, smem_u32(s_a), 0);
    const uint32_t b_base = __shfl_sync(0xffffffffu, smem_u32(s_b), 0);
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % S;
      bool ok = mbar_wait(&full[s], (kb / S) & 1);
      if (!__all_sync(0xffffffffu, ok && !*s_abort)) {  // warp-uniform: the MMAs are warp-collective
        *s_abort = 1;
        break;
      }
      tc_fence_after();
      const uint64_t ad = smem_desc_sw128(a_base + s * C::kStageA);
      const uint64_t bd = smem_desc_sw128(b_base + s * C::kStageB);
#pragma unroll
      for (int kk = 0; kk < kGmBK / 16; ++kk)  // 16 bf16 = 32 bytes per MMA: +2 in the address field
        mma_bf16_ss_warp(tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
      mma_commit_warp(&empty[s]);
    }
    mma_commit_warp(done);  // tracks every MMA issued, also on abort
  } else {
    // ---- epilogue: warps 2..5, TMEM lane quarter warp % 4 ----
    const int q = warp & 3;
    const int64_t r = r0 + 32 * q + lane;
    bool ok = mbar_wait(done, 0);
    ok = __all_sync(0xffffffffu, ok && !*s_abort);  // tcgen05.ld is warp-collective
    if (ok) {
      tc_fence_after();
      const float scale = p.scale != nullptr ? __ldg(p.scale) : 1.0f;
      double thr = 0.0;
      if constexpr (MASK) {
        const float g = __fadd_rn(__ldg(p.mask_gamma), p.eps);
        thr = (double)g * (1.0 + 0x1p-24);  // |fl32(W ÷ g)| ≤ 1  ⟺  |W| ≤ g·(1 + 2^-24)
      }
      const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
      for (int cc = 0; cc < BN; cc += 16) {
        uint32_t d[16];
        tmem_ld_32x32b_x16(t_lane + cc, d);
        tmem_wait_ld();
        const int64_t col = c0 + cc;
        if (r >= p.rows || col >= p.cols) continue;
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(__uint_as_float(d[j]), scale);
        if constexpr (MASK) {
          // This thread's 16 contiguous latent weights in 16-byte loads
          // (cols is a multiple of 64 and col of 16, so they are aligned).
          float w[16];
          const int64_t o = r * p.cols + col;
          if (p.mask_bf16) {
            const uint4* src = reinterpret_cast<const uint4*>(
                reinterpret_cast<const __nv_bfloat16*>(p.mask_w) + o);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint4 u = __ldg(src + h);
              const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
              for (int j = 0; j < 8; ++j) w[8 * h + j] = __bfloat162float(e[j]);
            }
          } else {
            const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.mask_w) + o);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float4 f = __ldg(src + h);
              w[4 * h] = f.x;
              w[4 * h + 1] = f.y;
              w[4 * h + 2] = f.z;
              w[4 * h + 3] = f.w;
            }
          }
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (fabs((double)w[j]) > thr) v[j] = 0.0f;
        }
        float* out = p.C + r * p.cols + col;
        if (col + 16 <= p.cols && (p.cols & 3) == 0) {
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<float4*>(out + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (col + j < p.cols) out[j] = v[j];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*s_abort) mbar_wait_for(done, 0, 100000000ull);  // MMAs finished before TMEM is freed
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Layout kernels (32 × 32 tiles through shared memory, 256 threads).

// W_qᵀ [K, Np] bf16 from the packed codes [N, K/4]: element (k, n) = c(n,k) - 1
// (columns n ≥ N are zero). Block tile: 32 rows n × 64 weights k. 128 threads
// each load one 32-bit word (16 codes) and expand it into the tile; then all
// 256 threads write 64 rows k × 32 columns n (64 contiguous bytes per row).
__global__ void __launch_bounds__(256)
expand_wqt_kernel(const uint8_t* __restrict__ W, int64_t N, int64_t K, int64_t Np,
                  __nv_bfloat16* __restrict__ out) {
  __shared__ __nv_bfloat16 tile[64][34];
  const int64_t n0 = (int64_t)blockIdx.x * 32, k0 = (int64_t)blockIdx.y * 64;
  const int tid = threadIdx.x;
  if (tid < 128) {
    const int i = tid >> 2, q = tid & 3;  // row n0+i, word q of the 64 weights
    const int64_t n = n0 + i;
    uint32_t word = 0x55555555u;          // codes 1 (w = 0) past N
    if (n < N) word = __ldg(reinterpret_cast<const uint32_t*>(W + n * (K / 4)) + (k0 >> 4) + q);
#pragma unroll
    for (int e = 0; e < 16; ++e) {  // weight 16q + 4j + i2 at bits 8·i2 + 2·j
      const int j = e >> 2, i2 = e & 3;
      const int c = (int)((word >> (8 * i2 + 2 * j)) & 3u);
      tile[16 * q + e][i] = __float2bfloat16_rn((float)(c - 1));
    }
  }
  __syncthreads();
  const int tx = tid & 31, ty = tid >> 5;
  for (int r = ty; r < 64; r += 8) {
    const int64_t k = k0 + r, n = n0 + tx;
    if (k < K && n < Np) out[k * Np + n] = tile[r][tx];
  }
}

// Transpose-convert an [R, Cc] fp32/bf16 matrix, with rows scaled by an
// optional per-row factor, into [Cc, Rp] bf16 (columns r ≥ R zero).
// Used for dYᵀ (factor none) and for Âᵀ from int8 A_q (see below).
template <typename T>
__global__ void __launch_bounds__(256)
transpose_bf16_kernel(const T* __restrict__ in, int64_t R, int64_t Cc, int64_t Rp,
                      __nv_bfloat16* __restrict__ out) {
  __shared__ float tile[32][33];
  const int64_t c0 = (int64_t)blockIdx.x * 32, rr0 = (int64_t)blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < 32; i += 8) {
    const int64_t r = rr0 + i, c = c0 + tx;
    tile[i][tx] = (r < R && c < Cc) ? to_f32<T>(in[r * Cc + c]) : 0.0f;
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int64_t c = c0 + i, r = rr0 + tx;
    if (c < Cc && r < Rp) out[c * Rp + r] = __float2bfloat16_rn(tile[tx][i]);
  }
}

// bf16 copy of an fp32 array (n a multiple of 4, 16-byte aligned).
__global__ void __launch_bounds__(256)
convert_bf16_kernel(const float* __restrict__ in, int64_t n, __nv_bfloat16* __restrict__ out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n / 4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(in) + i);
    __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(out + 4 * i);
    o[0] = __floats2bfloat162_rn(v.x, v.y);
    o[1] = __floats2bfloat162_rn(v.z, v.w);
  }
}

// Âᵀ [K, Mp] bf16: Â[m, k] = fp32(γ_A[m] ÷ 127) · A_q[m, k] (columns m ≥ M zero).
__global__ void __launch_bounds__(256)
ahat_t_kernel(const int8_t* __restrict__ Aq, const float* __restrict__ gammaA, int64_t M,
              int64_t K, int64_t Mp, __nv_bfloat16* __restrict__ out) {
  __shared__ float tile[32][33];
  const int64_t k0 = (int64_t)blockIdx.x * 32, m0 = (int64_t)blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < 32; i += 8) {
    const int64_t m = m0 + i, k = k0 + tx;
    float a = 0.0f;
    if (m < M && k < K) a = __fmul_rn(__fdiv_rn(__ldg(gammaA + m), 127.0f), (float)Aq[m * K + k]);
    tile[i][tx] = a;
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int64_t k = k0 + i, m = m0 + tx;
    if (k < K && m < Mp) out[k * Mp + m] = __float2bfloat16_rn(tile[tx][i]);
  }
}

}  // namespace bl
