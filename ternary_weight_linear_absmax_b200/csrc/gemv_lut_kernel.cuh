// Decode GEMV by table lookup (one token): the lookup-table contraction of
// "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section "Como
// o ecossistema bitnet.cpp acelera inferência em CPUs e borda?" (figure
// "Fluxo de Execução com Lookup Table (LUT-GEMM)"), run on the GPU.
//
// Weights: one index byte per group of four weights, idx = 27·d0 + 9·d1 +
// 3·d2 + d3 with d_i = w_i + 1 (first weight most significant: index 0 = all
// -1, 40 = all 0, 80 = all +1), stored [N, K/4] like the 2-bit codes (same
// 2 bits per weight).
// Tables: after the AbsMax prologue every CTA tabulates, for each block of 4
// int8 activations, the signed sums of the 41 patterns with index ≤ 40; the
// other 40 are their negatives (index 80 - idx flips every sign), so the
// table of a token takes K/4 · 41 int16.
// Contraction: per index byte one shared-memory read of T[min(idx, 80-idx)],
// negated when idx > 40, and one add; no multiplications and no row-sum
// correction (the table holds Σ w·a directly).
// This is the pages' CPU method transplanted for comparison; on this GPU the
// dp4a contraction of the 2-bit codes does the same work in fewer issue slots.
#pragma once

#include "bl_device.cuh"
#include "gemv_kernel.cuh"
#include "gemv_prologue.cuh"

namespace bl {

constexpr int kLutHalf = 41;  // entries kept per block: indices 0..40

struct GemvLutParams {
  const void* A;       // token [1, K] fp32/bf16
  const uint8_t* W;    // index bytes [N, K/4]
  const float* gamma;
  void* Y;             // [1, N] fp32/bf16 or int32 (raw)
  int64_t N, K;
  int rows_per_cta, rows_pad;
  float eps;
  int y_bf16, raw;
};

// [header][index slab gemv_boxes(K)·rows_pad·128][int8 token K][tables K/4·41·2][row sums R·4]
__host__ __device__ inline size_t gemv_lut_smem_bytes(int64_t K, int rows) {
  size_t s = kGemvHeader;
  s += (size_t)gemv_boxes(K) * gemv_rows_pad(rows) * 128;
  s += (size_t)K;
  s += ((size_t)(K / 4) * kLutHalf * 2 + 15) / 16 * 16;
  s += (size_t)rows * sizeof(int);
  return s + 1024;
}

// 2-bit codes → index bytes: byte g of a row = base-3 number of the codes of
// weights 4g .. 4g+3 (first most significant). One thread per byte.
__global__ void __launch_bounds__(256)
lut_index_pack_kernel(const uint8_t* __restrict__ W2, int64_t total, uint8_t* __restrict__ out) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    // index byte e covers weights 4e .. 4e+3: in the 2-bit layout those are
    // bit pair j = e mod 4 of each byte i of 32-bit word e/4 (rows have K/16
    // whole words, so global indices work)
    const uint32_t word = __ldg(reinterpret_cast<const uint32_t*>(W2) + (e >> 2));
    const int j = (int)(e & 3);
    uint32_t idx = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) idx = 3u * idx + ((word >> (8 * i + 2 * j)) & 3u);
    out[e] = (uint8_t)idx;
  }
}

template <typename TA>
__global__ void __launch_bounds__(kGemvThreads, 2)
gemv_lut_kernel(const __grid_constant__ CUtensorMap tm_w, const GemvLutParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(16) unsigned s_wmax[1][kGemvWarps];
  __shared__ __align__(16) int s_wsum[1][kGemvWarps];
  __shared__ float s_sc[1];
  __shared__ int s_wok;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t K = p.K, G = K / 4;
  // Rows [r0, r1) of an even split over the grid (at most rows_per_cta).
  const int64_t r0 = (int64_t)blockIdx.x * p.N / gridDim.x;
  const int R = (int)((int64_t)(blockIdx.x + 1) * p.N / gridDim.x - r0);
  const int nbox = gemv_boxes(K);
  const int box_bytes = p.rows_pad * 128;
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem);
  uint8_t* s_w = smem + kGemvHeader;
  int8_t* s_a = reinterpret_cast<int8_t*>(s_w + (size_t)nbox * box_bytes);
  int16_t* s_t = reinterpret_cast<int16_t*>(s_a + K);
  int* s_part = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(s_t) +
                                       ((size_t)G * kLutHalf * 2 + 15) / 16 * 16);

  if (tid == 0) {
    mbar_init(s_bar, 1);
    fence_barrier_init();
  }
  for (int i = tid; i < p.rows_per_cta; i += kGemvThreads) s_part[i] = 0;
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(s_bar, (uint32_t)nbox * (uint32_t)box_bytes);
    for (int b = 0; b < nbox; ++b)
      tma_load_2d(s_w + (size_t)b * box_bytes, &tm_w, b * 128, (int32_t)r0, s_bar);
  }
  const float gamma_w = p.gamma != nullptr ? __ldg(p.gamma) : 0.0f;
  pdl_launch_dependents();
  if (tid == 0) s_wok = mbar_wait(s_bar, 0) ? 1 : 0;
  __syncthreads();
  if (!s_wok) {
    if (warp == 0) pdl_wait_prior_grid();
    if (tid == 0) mbar_wait_for(s_bar, 0, 100000000ull);
    return;
  }
  mbar_wait(s_bar, 0);
  if (warp == 0) pdl_wait_prior_grid();
  __syncthreads();

  gemv_absmax_prologue<1, TA>(reinterpret_cast<const TA*>(p.A), 1, K, K, p.eps, gamma_w, s_a,
                              s_wmax, s_wsum, s_sc);

  // Tables: entries of the last j activations extended by -a, 0, +a.
  for (int64_t g = tid; g < G; g += kGemvThreads) {
    const int a0 = s_a[4 * g], a1 = s_a[4 * g + 1], a2 = s_a[4 * g + 2], a3 = s_a[4 * g + 3];
    int t123[27];
#pragma unroll
    for (int r = 0; r < 27; ++r) {
      const int d1 = r / 9, d2 = (r / 3) % 3, d3 = r % 3;
      t123[r] = (d1 - 1) * a1 + (d2 - 1) * a2 + (d3 - 1) * a3;
    }
    int16_t* t = s_t + g * kLutHalf;
#pragma unroll
    for (int idx = 0; idx < kLutHalf; ++idx)
      t[idx] = (int16_t)(idx < 27 ? t123[idx] - a0 : t123[idx - 27]);
  }
  __syncthreads();

  // Contraction: thread t < RH·CG owns rows ra = t mod RH and ra + RH and the
  // 16-byte chunks (16 groups) cg, cg + CG, ...
  const int RH = (R + 1) >> 1;
  const int nchunks = (int)(G / 16);
  int CG = kGemvThreads / (RH > 0 ? RH : 1);
  if (CG > nchunks) CG = nchunks;
  if (CG < 1) CG = 1;
  const bool active = tid < RH * CG;
  const int ra = active ? tid % RH : 0, cg = active ? tid / RH : 0;
  const bool has_b = ra + RH < R;
  const int rows[2] = {ra, has_b ? ra + RH : ra};
  int acc[2] = {0, 0};
  if (active) {
    for (int c = cg; c < nchunks; c += CG) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 v = *reinterpret_cast<const uint4*>(s_w + (size_t)(c >> 3) * box_bytes +
                                                        rows[h] * 128 + (((c & 7) ^ (rows[h] & 7)) << 4));
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int idx = (int)((wv[q] >> (8 * b)) & 0xFFu);
            const int64_t g = 16 * (int64_t)c + 4 * q + b;
            const int e = s_t[g * kLutHalf + min(idx, 80 - idx)];
            acc[h] += idx > 40 ? -e : e;
          }
        }
      }
    }
    atomicAdd(&s_part[ra], acc[0]);
    if (has_b) atomicAdd(&s_part[ra + RH], acc[1]);
  }
  __syncthreads();

  for (int r = tid; r < R; r += kGemvThreads) {
    const int v = s_part[r];
    const int64_t o = r0 + r;
    if (p.raw) {
      reinterpret_cast<int32_t*>(p.Y)[o] = v;
    } else {
      const float y = __fmul_rn((float)v, s_sc[0]);
      if (p.y_bf16)
        reinterpret_cast<__nv_bfloat16*>(p.Y)[o] = __float2bfloat16_rn(y);
      else
        reinterpret_cast<float*>(p.Y)[o] = y;
    }
  }
}

}  // namespace bl
