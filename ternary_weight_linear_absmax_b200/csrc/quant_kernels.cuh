// Quantiser kernels: AbsMean ternary weight quantisation + 2-bit packing,
// AbsMax per-token INT8 activation quantisation, and the FFN ReLU²
// requantisation. All are single-pass, HBM-bound streaming kernels.
//
// Formulas: "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM",
// section "Por que 1,58 bits por peso e qual a matemática da ternarização?"
// (γ = mean|W|, W_q = Round(Clip(W/(γ+ε), -1, 1)); γ_A = max|A| per token,
// A_q = Clip(Round(A·127/(γ_A+ε)), -128, 127)); ReLU² from the BitLinear
// utilities (ReLUSquared) of "Arquitetura Hibrida Multimodal para bitnet.cpp".
#pragma once

#include "bl_device.cuh"

namespace bl {

constexpr int kQuantThreads = 256;

// ---------------------------------------------------------------------------
// AbsMean, pass 1: per-block partial sums of |W| in double. Each thread
// reads 16-byte vectors (8 bf16 or 4 fp32) in a grid-stride loop.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
absmean_partial_kernel(const T* __restrict__ W, int64_t count, double* __restrict__ partials) {
  constexpr int VEC = 16 / sizeof(T);
  const int64_t nvec = count / VEC;
  const uint4* W4 = reinterpret_cast<const uint4*>(W);
  double s = 0.0;
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < nvec;
       v += (int64_t)gridDim.x * blockDim.x) {
    uint4 u = __ldg(W4 + v);
    const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
    for (int i = 0; i < VEC; ++i) s += fabs((double)to_f32<T>(e[i]));
  }
  // tail (count not a multiple of VEC cannot happen: K % 64 == 0)
  s = warp_sum_d(s);
  __shared__ double red[kQuantThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double t = threadIdx.x < kQuantThreads / 32 ? red[threadIdx.x] : 0.0;
    t = warp_sum_d(t);
    if (threadIdx.x == 0) partials[blockIdx.x] = t;
  }
}

// Deterministic block-wide sum of the partials (fixed order for a given
// partial count), result broadcast through shared memory.
__device__ __forceinline__ double sum_partials(const double* __restrict__ partials, int n) {
  __shared__ double red[kQuantThreads / 32];
  __shared__ double total;
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += partials[i];
  s = warp_sum_d(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double t = threadIdx.x < (int)(blockDim.x / 32) ? red[threadIdx.x] : 0.0;
    t = warp_sum_d(t);
    if (threadIdx.x == 0) total = t;
  }
  __syncthreads();
  return total;
}

// AbsMean, pass 2: γ from the partials, then ternary codes and packing.
// One thread produces one 32-bit packed word (16 consecutive weights).
//
// Code decision. The pages' rule is Round(Clip(x)) with x = fl32(W/g),
// g = fl32(γ+ε). Since fl32 is monotone and the quotients in
// (1/2, 1/2 + 2^-25] round to 1/2 (a tie that round-half-even sends to 0),
//   Round(Clip(fl32(W/g))) = +1  iff  W >  g·(1/2 + 2^-25),
//                            -1  iff  W < -g·(1/2 + 2^-25),   else 0,
// where the threshold g·(1/2 + 2^-25) is exact in double (24 + 25 bits).
// This reproduces the fp32 division bit for bit without dividing per weight.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
ternary_pack_kernel(const T* __restrict__ W, int64_t nwords, double count, float eps,
                    const double* __restrict__ partials, int npartials,
                    uint32_t* __restrict__ packed, float* __restrict__ gamma_out) {
  const double total = sum_partials(partials, npartials);
  const float gamma = (float)(total / count);  // mean in double, rounded once
  if (blockIdx.x == 0 && threadIdx.x == 0) *gamma_out = gamma;
  const float g = __fadd_rn(gamma, eps);
  const double thr = (double)g * (0.5 + 0x1p-25);
  constexpr int VEC = 16 / sizeof(T);
  constexpr int NV = 16 / VEC;  // 16-byte vectors per 16 weights
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < nwords;
       w += (int64_t)gridDim.x * blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(W + w * 16);
    T e[16];
#pragma unroll
    for (int v = 0; v < NV; ++v) *reinterpret_cast<uint4*>(&e[v * VEC]) = __ldg(src + v);
    uint32_t word = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const double x = (double)to_f32<T>(e[k]);
      const uint32_t c = x > thr ? 2u : (x < -thr ? 0u : 1u);
      const int j = k >> 2, i = k & 3;
      word |= c << (8 * i + 2 * j);
    }
    packed[w] = word;
  }
}

// ---------------------------------------------------------------------------
// AbsMax activation quantisation: one block per token row.
// Writes int8 A_q, γ_A and (optionally) the row sum of A_q. The first
// kQuantRegVecs 16-byte vectors of each thread stay in registers between the
// max pass and the quantise pass (all of a row up to 8192 bf16 / 4096 fp32
// values), so the row is read from memory once.
constexpr int kQuantRegVecs = 4;

template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
quant_acts_kernel(const T* __restrict__ A, int64_t K, float eps, int8_t* __restrict__ Aq,
                  float* __restrict__ gammaA, int32_t* __restrict__ rowsum) {
  // A kernel launched after this one with programmatic dependent launch may
  // start its own independent work now; it waits for this grid's results.
  // This grid itself, when launched early, reads and writes global memory
  // only after the previous kernel has completed.
  pdl_launch_dependents();
  pdl_wait_prior_grid();
  const int64_t m = blockIdx.x;
  const T* row = A + m * K;
  constexpr int VEC = 16 / sizeof(T);
  const int64_t nvec = K / VEC;
  const uint4* r4 = reinterpret_cast<const uint4*>(row);
  __shared__ float redf[kQuantThreads / 32];
  __shared__ int redi[kQuantThreads / 32];
  __shared__ float s_scale;

  uint4 reg[kQuantRegVecs];
  float mx = 0.0f;
#pragma unroll
  for (int r = 0; r < kQuantRegVecs; ++r) {
    const int64_t v = threadIdx.x + (int64_t)r * kQuantThreads;
    if (v < nvec) {
      reg[r] = __ldg(r4 + v);
      const T* e = reinterpret_cast<const T*>(&reg[r]);
#pragma unroll
      for (int i = 0; i < VEC; ++i) mx = fmaxf(mx, fabsf(to_f32<T>(e[i])));
    }
  }
  for (int64_t v = threadIdx.x + (int64_t)kQuantRegVecs * kQuantThreads; v < nvec;
       v += kQuantThreads) {
    const uint4 u = __ldg(r4 + v);
    const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
    for (int i = 0; i < VEC; ++i) mx = fmaxf(mx, fabsf(to_f32<T>(e[i])));
  }
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) redf[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < kQuantThreads / 32 ? redf[threadIdx.x] : 0.0f;
    t = warp_max(t);
    if (threadIdx.x == 0) {
      gammaA[m] = t;
      s_scale = __fdiv_rn(127.0f, __fadd_rn(t, eps));
    }
  }
  __syncthreads();
  const float s = s_scale;
  int sum = 0;
  auto emit = [&](const uint4& u, int64_t v) {
    const T* e = reinterpret_cast<const T*>(&u);
    uint32_t w[VEC / 4];
#pragma unroll
    for (int i = 0; i < VEC / 4; ++i) {
      w[i] = pack4_low_bytes(quant_i8_bits(to_f32<T>(e[4 * i]), s),
                             quant_i8_bits(to_f32<T>(e[4 * i + 1]), s),
                             quant_i8_bits(to_f32<T>(e[4 * i + 2]), s),
                             quant_i8_bits(to_f32<T>(e[4 * i + 3]), s));
      sum = dp4a(w[i], 0x01010101u, sum);  // Σ of the four int8 values
    }
    if constexpr (VEC == 8)
      *reinterpret_cast<uint2*>(Aq + m * K + v * VEC) = make_uint2(w[0], w[1]);
    else
      *reinterpret_cast<uint32_t*>(Aq + m * K + v * VEC) = w[0];
  };
#pragma unroll
  for (int r = 0; r < kQuantRegVecs; ++r) {
    const int64_t v = threadIdx.x + (int64_t)r * kQuantThreads;
    if (v < nvec) emit(reg[r], v);
  }
  for (int64_t v = threadIdx.x + (int64_t)kQuantRegVecs * kQuantThreads; v < nvec;
       v += kQuantThreads)
    emit(__ldg(r4 + v), v);
  if (rowsum != nullptr) {
    sum = warp_sum_i(sum);
    if ((threadIdx.x & 31) == 0) redi[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x < 32) {
      int t = threadIdx.x < kQuantThreads / 32 ? redi[threadIdx.x] : 0;
      t = warp_sum_i(t);
      if (threadIdx.x == 0) rowsum[m] = t;
    }
  }
}

// Row sums of an int8 matrix (one block per row), for callers that pass
// quantised activations without their sums.
__global__ void __launch_bounds__(kQuantThreads)
rowsum_i8_kernel(const int8_t* __restrict__ Aq, int64_t K, int32_t* __restrict__ rowsum) {
  pdl_launch_dependents();
  const int64_t m = blockIdx.x;
  const uint4* r4 = reinterpret_cast<const uint4*>(Aq + m * K);
  int sum = 0;
  for (int64_t v = threadIdx.x; v < K / 16; v += blockDim.x) {
    uint4 u = __ldg(r4 + v);
    sum = dp4a(u.x, 0x01010101u, sum);
    sum = dp4a(u.y, 0x01010101u, sum);
    sum = dp4a(u.z, 0x01010101u, sum);
    sum = dp4a(u.w, 0x01010101u, sum);
  }
  __shared__ int redi[kQuantThreads / 32];
  sum = warp_sum_i(sum);
  if ((threadIdx.x & 31) == 0) redi[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x < 32) {
    int t = threadIdx.x < kQuantThreads / 32 ? redi[threadIdx.x] : 0;
    t = warp_sum_i(t);
    if (threadIdx.x == 0) rowsum[m] = t;
  }
}

// ---------------------------------------------------------------------------
// FFN requantisation of the up-projection, one block per token:
//   h = fp32(acc · fp32((γ_X·γ_up)/127)),  r = max(h,0)²  (fp32),
//   γ_r = max_n r,  q = Clip(Round(r · 127/(γ_r+ε)), -128, 127),  Σq.
// ReLU² is monotone in acc and fp32 rounding is monotone, so γ_r is also
// the image of the largest accumulator; computing it from r keeps the
// kernel a literal restatement. The two passes are also launched apart for
// the tensor-parallel block, where γ_r is the maximum over every rank's
// shard of H.

__device__ __forceinline__ float relu2_of(int acc, float sc) {
  const float h = __fmul_rn((float)acc, sc);
  const float p = fmaxf(h, 0.0f);
  return __fmul_rn(p, p);
}

// Pass 1: block-wide max of r over one token's row (returned to all threads).
__device__ __forceinline__ float relu2_row_max(const int4* __restrict__ a4, int64_t H, float sc) {
  __shared__ float redf[kQuantThreads / 32];
  __shared__ float total;
  float mx = 0.0f;
  for (int64_t v = threadIdx.x; v < H / 4; v += blockDim.x) {
    const int4 u = __ldg(a4 + v);
    mx = fmaxf(fmaxf(mx, fmaxf(relu2_of(u.x, sc), relu2_of(u.y, sc))),
               fmaxf(relu2_of(u.z, sc), relu2_of(u.w, sc)));
  }
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) redf[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < kQuantThreads / 32 ? redf[threadIdx.x] : 0.0f;
    t = warp_max(t);
    if (threadIdx.x == 0) total = t;
  }
  __syncthreads();
  return total;
}

// Pass 2: quantise one token's row of r with γ_r, write q and Σq.
__device__ __forceinline__ void relu2_row_quant(const int4* __restrict__ a4, int64_t H, float sc,
                                                float gamma_r, float eps, int8_t* __restrict__ q_row,
                                                int32_t* __restrict__ rowsum) {
  __shared__ int redi[kQuantThreads / 32];
  const float s = __fdiv_rn(127.0f, __fadd_rn(gamma_r, eps));
  int sum = 0;
  for (int64_t v = threadIdx.x; v < H / 4; v += blockDim.x) {
    const int4 u = __ldg(a4 + v);
    const uint32_t w = pack4_low_bytes(quant_i8_bits(relu2_of(u.x, sc), s),
                                       quant_i8_bits(relu2_of(u.y, sc), s),
                                       quant_i8_bits(relu2_of(u.z, sc), s),
                                       quant_i8_bits(relu2_of(u.w, sc), s));
    sum = dp4a(w, 0x01010101u, sum);
    *reinterpret_cast<uint32_t*>(q_row + v * 4) = w;
  }
  sum = warp_sum_i(sum);
  if ((threadIdx.x & 31) == 0) redi[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x < 32) {
    int t = threadIdx.x < kQuantThreads / 32 ? redi[threadIdx.x] : 0;
    t = warp_sum_i(t);
    if (threadIdx.x == 0) *rowsum = t;
  }
}

// The single-device kernel keeps each thread's first kRequantRegVecs
// 16-byte vectors of accumulators in registers between the max and the
// quantise pass (rows up to 12288 accumulators), so the row is read from
// memory once, and all of a thread's loads are in flight together.
constexpr int kRequantRegVecs = 12;

__global__ void __launch_bounds__(kQuantThreads)
relu2_requant_kernel(const int32_t* __restrict__ acc, int64_t H, const float* __restrict__ gammaX,
                     const float* __restrict__ g_up, float eps, int8_t* __restrict__ Rq,
                     float* __restrict__ gammaR, int32_t* __restrict__ rowsum) {
  pdl_launch_dependents();
  pdl_wait_prior_grid();  // no-op unless launched with programmatic dependent launch
  const int64_t m = blockIdx.x;
  const int4* a4 = reinterpret_cast<const int4*>(acc + m * H);
  const int64_t nvec = H / 4;
  __shared__ float redf[kQuantThreads / 32];
  __shared__ int redi[kQuantThreads / 32];
  __shared__ float s_scale;
  const float sc = __fdiv_rn(__fmul_rn(gammaX[m], *g_up), 127.0f);
  int4 reg[kRequantRegVecs];
#pragma unroll
  for (int r = 0; r < kRequantRegVecs; ++r) {
    const int64_t v = threadIdx.x + (int64_t)r * kQuantThreads;
    if (v < nvec) reg[r] = __ldg(a4 + v);
  }
  float mx = 0.0f;
  auto vmax = [&](const int4& u) {
    mx = fmaxf(fmaxf(mx, fmaxf(relu2_of(u.x, sc), relu2_of(u.y, sc))),
               fmaxf(relu2_of(u.z, sc), relu2_of(u.w, sc)));
  };
#pragma unroll
  for (int r = 0; r < kRequantRegVecs; ++r)
    if (threadIdx.x + (int64_t)r * kQuantThreads < nvec) vmax(reg[r]);
  for (int64_t v = threadIdx.x + (int64_t)kRequantRegVecs * kQuantThreads; v < nvec;
       v += kQuantThreads)
    vmax(__ldg(a4 + v));
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) redf[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < kQuantThreads / 32 ? redf[threadIdx.x] : 0.0f;
    t = warp_max(t);
    if (threadIdx.x == 0) {
      gammaR[m] = t;
      s_scale = __fdiv_rn(127.0f, __fadd_rn(t, eps));
    }
  }
  __syncthreads();
  const float s = s_scale;
  int8_t* q_row = Rq + m * H;
  int sum = 0;
  auto emit = [&](const int4& u, int64_t v) {
    const uint32_t w = pack4_low_bytes(quant_i8_bits(relu2_of(u.x, sc), s),
                                       quant_i8_bits(relu2_of(u.y, sc), s),
                                       quant_i8_bits(relu2_of(u.z, sc), s),
                                       quant_i8_bits(relu2_of(u.w, sc), s));
    sum = dp4a(w, 0x01010101u, sum);
    *reinterpret_cast<uint32_t*>(q_row + v * 4) = w;
  };
#pragma unroll
  for (int r = 0; r < kRequantRegVecs; ++r) {
    const int64_t v = threadIdx.x + (int64_t)r * kQuantThreads;
    if (v < nvec) emit(reg[r], v);
  }
  for (int64_t v = threadIdx.x + (int64_t)kRequantRegVecs * kQuantThreads; v < nvec;
       v += kQuantThreads)
    emit(__ldg(a4 + v), v);
  sum = warp_sum_i(sum);
  if ((threadIdx.x & 31) == 0) redi[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x < 32) {
    int t = threadIdx.x < kQuantThreads / 32 ? redi[threadIdx.x] : 0;
    t = warp_sum_i(t);
    if (threadIdx.x == 0) rowsum[m] = t;
  }
}

// Tensor-parallel FFN, pass 1 on one rank's shard: rmax[m] = max_n r.
__global__ void __launch_bounds__(kQuantThreads)
relu2_rowmax_kernel(const int32_t* __restrict__ acc, int64_t H, const float* __restrict__ gammaX,
                    const float* __restrict__ g_up, float* __restrict__ rmax) {
  pdl_launch_dependents();
  const int64_t m = blockIdx.x;
  const float sc = __fdiv_rn(__fmul_rn(gammaX[m], *g_up), 127.0f);
  const float g = relu2_row_max(reinterpret_cast<const int4*>(acc + m * H), H, sc);
  if (threadIdx.x == 0) rmax[m] = g;
}

// Tensor-parallel FFN, pass 2 on one rank's shard with the all-ranks γ_r.
__global__ void __launch_bounds__(kQuantThreads)
relu2_requant_given_kernel(const int32_t* __restrict__ acc, int64_t H,
                           const float* __restrict__ gammaX, const float* __restrict__ g_up,
                           const float* __restrict__ gammaR, float eps, int8_t* __restrict__ Rq,
                           int32_t* __restrict__ rowsum) {
  pdl_launch_dependents();
  const int64_t m = blockIdx.x;
  const float sc = __fdiv_rn(__fmul_rn(gammaX[m], *g_up), 127.0f);
  relu2_row_quant(reinterpret_cast<const int4*>(acc + m * H), H, sc, gammaR[m], eps, Rq + m * H,
                  rowsum + m);
}

// Dequantisation of INT32 accumulators: y = acc · ((γ_A·γ)/127) in fp32
// (optionally ReLU²), the same arithmetic as the contraction epilogues.
// One thread per 4 outputs (N % 4 == 0 is not required; row tails handled).
__global__ void __launch_bounds__(kQuantThreads)
dequant_i32_kernel(const int32_t* __restrict__ acc, const float* __restrict__ gammaA,
                   const float* __restrict__ gamma, int64_t M, int64_t N, int relu2, void* Y,
                   int y_bf16) {
  const float g = __ldg(gamma);
  const int64_t total = M * N;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = i / N;
    const float sc = __fdiv_rn(__fmul_rn(__ldg(gammaA + m), g), 127.0f);
    float y = __fmul_rn((float)__ldg(acc + i), sc);
    if (relu2) {
      y = fmaxf(y, 0.0f);
      y = __fmul_rn(y, y);
    }
    if (y_bf16)
      reinterpret_cast<__nv_bfloat16*>(Y)[i] = __float2bfloat16_rn(y);
    else
      reinterpret_cast<float*>(Y)[i] = y;
  }
}

__device__ __forceinline__ float dequant_value(int v, float sc, int relu2) {
  float y = __fmul_rn((float)v, sc);
  if (relu2) {
    y = fmaxf(y, 0.0f);
    y = __fmul_rn(y, y);
  }
  return y;
}

// Sum of the INT32 partials of a K-split contraction (split z at
// part + z·stride, rows of N; split 0 already subtracted the row sums), then
// the epilogue: raw INT32, or y = v · ((γ_A·γ)/127) in fp32 (ReLU² optional)
// as fp32/bf16. One block per output row (blockIdx.y) and 1024 columns per
// block (blockIdx.x), four columns per thread: 16-byte loads and stores
// when vec (N a multiple of 4, part and Y 16-byte aligned), else scalar.
__global__ void __launch_bounds__(256)
splitk_reduce_kernel(const int32_t* __restrict__ part, int splits, int64_t stride, int64_t M,
                     int64_t N, int raw, const float* __restrict__ gamma,
                     const float* __restrict__ gammaA, int relu2, void* Y, int y_bf16,
                     int vec) {
  pdl_launch_dependents();
  pdl_wait_prior_grid();  // no-op unless launched with programmatic dependent launch
  const int64_t m = blockIdx.y;
  const float sc = raw ? 0.0f : __fdiv_rn(__fmul_rn(__ldg(gammaA + m), __ldg(gamma)), 127.0f);
  auto finish = [sc, relu2](int v) -> float { return dequant_value(v, sc, relu2); };
  const int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (c >= N) return;
  const int64_t o = m * N + c;
  if (vec) {
    int4 v = __ldg(reinterpret_cast<const int4*>(part + o));
    for (int z = 1; z < splits; ++z) {
      const int4 u = __ldg(reinterpret_cast<const int4*>(part + (int64_t)z * stride + o));
      v.x += u.x;
      v.y += u.y;
      v.z += u.z;
      v.w += u.w;
    }
    if (raw) {
      *reinterpret_cast<int4*>(reinterpret_cast<int32_t*>(Y) + o) = v;
    } else if (y_bf16) {
      __nv_bfloat162* yp = reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(Y) + o);
      yp[0] = __floats2bfloat162_rn(finish(v.x), finish(v.y));
      yp[1] = __floats2bfloat162_rn(finish(v.z), finish(v.w));
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(Y) + o) =
          make_float4(finish(v.x), finish(v.y), finish(v.z), finish(v.w));
    }
    return;
  }
  for (int64_t cc = c; cc < c + 4 && cc < N; ++cc) {
    int v = 0;
    for (int z = 0; z < splits; ++z) v += __ldg(part + (int64_t)z * stride + m * N + cc);
    if (raw)
      reinterpret_cast<int32_t*>(Y)[m * N + cc] = v;
    else if (y_bf16)
      reinterpret_cast<__nv_bfloat16*>(Y)[m * N + cc] = __float2bfloat16_rn(finish(v));
    else
      reinterpret_cast<float*>(Y)[m * N + cc] = finish(v);
  }
}

}  // namespace bl
