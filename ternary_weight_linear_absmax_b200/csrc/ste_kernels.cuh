// Straight-through-estimator (STE) backward of BitLinear.
//
// "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section "Como
// funciona a camada BitLinear ... (Zero-GEMM)?", STE paragraph: in the
// backward pass the gradient of the quantisation is the identity inside the
// valid range. With the forward Y = Â·Ŵᵀ (Ŵ = γ·W_q, Â = (γ_A/127)·A_q):
//   dA = dY·Ŵ                         [M, K]   (contraction over N)
//   dW = 1[|W ÷ (γ+ε)| ≤ 1] ⊙ dYᵀ·Â   [N, K]   (contraction over M)
// Both are dense contractions, so both run as one tcgen05 kind::f16 GEMM
// (bf16 operands, fp32 accumulation in tensor memory):
//   dA:  A = dY [M, N] (as given, bf16; K-major), B = W_q [N, K] bf16
//        {-1, 0, +1} expanded from the packed codes in its own layout and
//        read as an MN-major operand; scale γ in the epilogue;
//   dW:  A = dY and B = Â [M, K] bf16 in their natural row-major layouts,
//        both read as MN-major operands (the contraction index M is the row
//        index of both); mask in the epilogue.
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

// DUAL: two CTAs per SM (each at most half of the shared memory, BN TMEM
// columns), so one CTA's epilogue overlaps the other's MMAs.
template <int BN, bool DUAL = false>
struct GmConfig {
  static constexpr int kStageA = kGmBM * 128;
  static constexpr int kStageB = BN * 128;
  static constexpr int kStages = DUAL ? (BN >= 256 ? 2 : 3) : (BN >= 256 ? 4 : 6);
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

// MN-major operand tile with the 128-byte swizzle, as a TMA box of 64
// elements × 64 rows writes it: each 128-byte row holds 64 consecutive MN
// elements of one K index, 8 K rows form a 1024-byte swizzle atom (stride
// byte offset), and 64-element MN chunks sit `lbo` bytes apart (leading byte
// offset). Same field encoding as smem_desc_sw128.
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(uint32_t saddr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}
// Operand majors of the GEMM (instruction descriptor bits 15 and 16).
constexpr int kMajAMN = 1, kMajBMN = 2;

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

// MAJ: kMajAMN — A is stored [kdim, rows] instead of [rows, kdim]; kMajBMN —
// B is stored [kdim, cols] instead of [cols, kdim] (row-major, the MN index
// innermost). An MN-major operand takes one 64 × 64 box per 64 rows (cols)
// of its tile and stage, a K-major one a single box of 64 K × its rows.
template <int BN, bool MASK, bool DUAL = false, int MAJ = 0>
__global__ void __launch_bounds__(kGmThreads, DUAL ? 2 : 1)
bf16_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const GmParams p) {
  using C = GmConfig<BN, DUAL>;
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
      if constexpr (MAJ != 0) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], C::kStageA + C::kStageB);
          uint8_t* da = s_a + s * C::kStageA;
          uint8_t* db = s_b + s * C::kStageB;
          if constexpr ((MAJ & kMajAMN) != 0) {
#pragma unroll
            for (int j = 0; j < kGmBM / 64; ++j)
              tma_load_2d(da + j * 8192, &tm_a, (int32_t)(r0 + 64 * j), kb * kGmBK, &full[s]);
          } else {
            tma_load_2d(da, &tm_a, kb * kGmBK, (int32_t)r0, &full[s]);
          }
          if constexpr ((MAJ & kMajBMN) != 0) {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d(db + j * 8192, &tm_b, (int32_t)(c0 + 64 * j), kb * kGmBK, &full[s]);
          } else {
            tma_load_2d(db, &tm_b, kb * kGmBK, (int32_t)c0, &full[s]);
          }
        }
        __syncwarp();
      } else {
        tma_load_2x2d_warp(&full[s], C::kStageA + C::kStageB, s_a + s * C::kStageA, &tm_a,
                           s_b + s * C::kStageB, &tm_b, kb * kGmBK, (int32_t)r0, (int32_t)c0);
      }
    }
    if (*s_abort && lane == 0) {  // drain copies in flight (bounded) before exit
      for (int d = max(0, kb - S); d < kb; ++d) mbar_wait_for(&full[d % S], (d / S) & 1, 100000000ull);
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    constexpr uint32_t idesc = idesc_bf16(kGmBM, BN) | ((MAJ & kMajAMN) ? (1u << 15) : 0u) |
                               ((MAJ & kMajBMN) ? (1u << 16) : 0u);
    // Per 16-K MMA: a K-major tile advances 32 bytes inside its swizzle rows
    // (+2 in the address field); an MN-major tile (64 K rows of 128 bytes per
    // 64-element chunk) advances 16 K rows, two swizzle atoms (+128).
    constexpr uint64_t a_step = (MAJ & kMajAMN) ? 128 : 2, b_step = (MAJ & kMajBMN) ? 128 : 2;
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
      const uint64_t ad = (MAJ & kMajAMN) ? smem_desc_sw128_mn(a_base + s * C::kStageA, 64 * 128)
                                          : smem_desc_sw128(a_base + s * C::kStageA);
      const uint64_t bd = (MAJ & kMajBMN) ? smem_desc_sw128_mn(b_base + s * C::kStageB, 64 * 128)
                                          : smem_desc_sw128(b_base + s * C::kStageB);
#pragma unroll
      for (int kk = 0; kk < kGmBK / 16; ++kk)
        mma_bf16_ss_warp(tmem, ad + kk * a_step, bd + kk * b_step, idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
      mma_commit_warp(&empty[s]);
    }
    mma_commit_warp(done);  // tracks every MMA issued, also on abort
  } else {
    // ---- epilogue: warps 2..5, TMEM lane quarter warp % 4 ----
    const int q = warp & 3;
    const int64_t r = r0 + 32 * q + lane;
    // STE mask of this thread's row, read while the MMAs run (the latent
    // weights are read once): bit c of mbits[c/32] keeps column c0 + c.
    // |fl32(W ÷ g)| ≤ 1 ⟺ |W| ≤ g·(1 + 2^-24) (exact in double); for an fp32
    // W that equals |W| ≤ the largest fp32 not above that bound.
    uint32_t mbits[MASK ? BN / 32 : 1];
    if constexpr (MASK) {
      const float g = __fadd_rn(__ldg(p.mask_gamma), p.eps);
      const float thr = __double2float_rd((double)g * (1.0 + 0x1p-24));
#pragma unroll
      for (int cw = 0; cw < BN / 32; ++cw) {
        uint32_t bits = 0u;
        const int64_t col = c0 + 32 * cw;
        if (r < p.rows && col < p.cols) {  // cols is a multiple of 64: whole groups of 32
          const int64_t o = r * p.cols + col;
          float w[32];
          if (p.mask_bf16) {
            const uint4* src = reinterpret_cast<const uint4*>(
                reinterpret_cast<const __nv_bfloat16*>(p.mask_w) + o);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const uint4 u = __ldg(src + h);
              const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
              for (int j = 0; j < 8; ++j) w[8 * h + j] = __bfloat162float(e[j]);
            }
          } else {
            const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.mask_w) + o);
#pragma unroll
            for (int h = 0; h < 8; ++h) {
              const float4 f = __ldg(src + h);
              w[4 * h] = f.x;
              w[4 * h + 1] = f.y;
              w[4 * h + 2] = f.z;
              w[4 * h + 3] = f.w;
            }
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) bits |= (fabsf(w[j]) <= thr ? 1u : 0u) << j;
        }
        mbits[cw] = bits;
      }
    }
    bool ok = mbar_wait(done, 0);
    ok = __all_sync(0xffffffffu, ok && !*s_abort);  // tcgen05.ld is warp-collective
    if (ok) {
      tc_fence_after();
      const float scale = p.scale != nullptr ? __ldg(p.scale) : 1.0f;
      const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
      // Chunk cc+16 is loaded (warp-collective) while chunk cc is processed.
      uint32_t d[2][16];
      tmem_ld_32x32b_x16(t_lane, d[0]);
#pragma unroll
      for (int cc = 0; cc < BN; cc += 16) {
        tmem_wait_ld();
        if (cc + 16 < BN) tmem_ld_32x32b_x16(t_lane + cc + 16, d[((cc >> 4) + 1) & 1]);
        const uint32_t(&dc)[16] = d[(cc >> 4) & 1];
        const int64_t col = c0 + cc;
        if (r >= p.rows || col >= p.cols) continue;
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(__uint_as_float(dc[j]), scale);
        if constexpr (MASK) {
          const uint32_t bits = mbits[cc >> 5] >> (cc & 31);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (!((bits >> j) & 1u)) v[j] = 0.0f;
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
// Layout kernels (256 threads).

// W_q [N, K] bf16 from the packed codes [N, K/4]: element (n, k) = c(n, k) - 1.
// Each thread expands one 32-bit word (16 codes; weight 16g + 4j + i of a row
// sits at bits 8i + 2j of its word g) into 16 consecutive bf16 of the same
// row: two 16-byte stores.
__global__ void __launch_bounds__(256)
expand_wq_kernel(const uint32_t* __restrict__ W, int64_t words, __nv_bfloat16* __restrict__ out) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < words;
       t += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t word = __ldg(W + t);
    uint32_t h[8];
#pragma unroll
    for (int e2 = 0; e2 < 8; ++e2) {  // weights 2·e2 and 2·e2 + 1 of the word
      uint32_t pair = 0;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int e = 2 * e2 + u, i = e & 3, jj = e >> 2;
        const int c = (int)((word >> (8 * i + 2 * jj)) & 3u);
        pair |= (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn((float)(c - 1))) << (16 * u);
      }
      h[e2] = pair;
    }
    uint4* o = reinterpret_cast<uint4*>(out + 16 * t);
    o[0] = make_uint4(h[0], h[1], h[2], h[3]);
    o[1] = make_uint4(h[4], h[5], h[6], h[7]);
  }
}

// Conversion helpers: two floats to a bf16 pair (round to nearest even), and
// eight consecutive elements of an int8 / bf16 / fp32 row to fp32.
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}

template <typename T>
__device__ __forceinline__ void load8_f32(const T* p, float (&v)[8]) {
  if constexpr (sizeof(T) == 1) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    const int8_t* b = reinterpret_cast<const int8_t*>(&u);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = (float)b[j];
  } else if constexpr (sizeof(T) == 2) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __bfloat162float(b[j]);
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// Â = bf16(fp32(rscale[r] ÷ 127) · A_q[r, c]) for an int8 [R, Cc] matrix (Cc a
// multiple of 8), in its own layout: one fp32 division per row, one fp32
// product and one rounding to bf16 per element; eight elements per thread
// and 16-byte stores.
__global__ void __launch_bounds__(256)
scale_rows_bf16_kernel(const int8_t* __restrict__ in, const float* __restrict__ rscale, int64_t R,
                       int64_t Cc, __nv_bfloat16* __restrict__ out) {
  const int64_t per_row = Cc / 8;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < R * per_row;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = t / per_row, c = (t - r * per_row) * 8;
    float v[8];
    load8_f32<int8_t>(in + r * Cc + c, v);
    const float sc = __fdiv_rn(__ldg(rscale + r), 127.0f);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(sc, v[j]);
    uint4 w;
    w.x = bf16x2_bits(v[0], v[1]);
    w.y = bf16x2_bits(v[2], v[3]);
    w.z = bf16x2_bits(v[4], v[5]);
    w.w = bf16x2_bits(v[6], v[7]);
    *reinterpret_cast<uint4*>(out + r * Cc + c) = w;
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

}  // namespace bl
