// AbsMax token prologue shared by the decode GEMV variants that read float
// tokens (radix-3 and lookup-table weights).
//
// "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section "Por
// que 1,58 bits por peso ...", activation paragraph: per token,
// γ_A = max|A|, A_q = Clip(Round(A·(127 ÷ (γ_A+ε))), -128, 127) in fp32,
// round half to even (the magic-add rounding of quant_i8_bits).
#pragma once

#include "bl_device.cuh"
#include "gemv_kernel.cuh"

namespace bl {

// All kGemvThreads threads call it. Writes the int8 tokens of token m to
// s_a[m·stride + k] (k < K; zeros for K ≤ k < stride, stride a multiple of 4),
// the per-warp Σ A_q slots s_wsum[m][·] and s_sc[m] = (γ_A·γ_w)/127. Returns
// after a CTA barrier, so everything written is visible.
template <int MT, typename TA>
__device__ __forceinline__ void gemv_absmax_prologue(const TA* __restrict__ A, int M, int64_t K,
                                                     int64_t stride, float eps, float gamma_w,
                                                     int8_t* s_a, unsigned (&s_wmax)[MT][kGemvWarps],
                                                     int (&s_wsum)[MT][kGemvWarps], float* s_sc) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int VEC = 16 / (int)sizeof(TA);
  const int64_t nvec = K / VEC;
  for (int m = 0; m < MT; ++m) {
    float mx = 0.0f;
    if (m < M) {
      const uint4* src = reinterpret_cast<const uint4*>(A + m * K);
      for (int64_t v = tid; v < nvec; v += kGemvThreads) {
        const uint4 u = __ldg(src + v);
#pragma unroll
        for (int i = 0; i < VEC; ++i) mx = fmaxf(mx, fabsf(to_f32<TA>(reinterpret_cast<const TA*>(&u)[i])));
      }
    }
    const unsigned wm = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
    if (lane == 0) s_wmax[m][warp] = wm;
  }
  __syncthreads();
  for (int m = 0; m < MT; ++m) {
    int tsum = 0;
    if (m < M) {
      const float g = __uint_as_float(warp_slots_max(s_wmax[m]));
      const float s = __fdiv_rn(127.0f, __fadd_rn(g, eps));
      const uint4* src = reinterpret_cast<const uint4*>(A + m * K);
      for (int64_t v = tid; v < nvec; v += kGemvThreads) {
        const uint4 u = __ldg(src + v);
#pragma unroll
        for (int i = 0; i < VEC / 4; ++i) {
          const TA* e = reinterpret_cast<const TA*>(&u) + 4 * i;
          const uint32_t w =
              pack4_low_bytes(quant_i8_bits(to_f32<TA>(e[0]), s), quant_i8_bits(to_f32<TA>(e[1]), s),
                              quant_i8_bits(to_f32<TA>(e[2]), s), quant_i8_bits(to_f32<TA>(e[3]), s));
          tsum = dp4a(w, 0x01010101u, tsum);
          *reinterpret_cast<uint32_t*>(s_a + m * stride + v * VEC + 4 * i) = w;
        }
      }
      for (int64_t v = K / 4 + tid; v < stride / 4; v += kGemvThreads)
        *reinterpret_cast<uint32_t*>(s_a + m * stride + 4 * v) = 0u;
      if (tid == kGemvThreads - 1) s_sc[m] = __fdiv_rn(__fmul_rn(g, gamma_w), 127.0f);
    }
    const int ws = __reduce_add_sync(0xffffffffu, tsum);
    if (lane == 0) s_wsum[m][warp] = ws;
  }
  __syncthreads();
}

}  // namespace bl
