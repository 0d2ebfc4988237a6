// Plain CPU oracle for the BitNet b1.58 BitLinear forward pass.
//
// TEST INFRASTRUCTURE ONLY. This file is the independent reference that the
// CUDA path is checked against. Only the test-suite, the smoke check and the
// benchmark's CPU-baseline leg may load it; the product path never does. It
// shares no code, header, table or helper with the CUDA library.
//
// Sources (page titles and the section each function follows):
//   [BLOG] "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM"
//          (produtoramaxvision.com.br blog post)
//     §"qual a matemática da ternarização?"  AbsMean scale γ and the ternary
//          weight rule W_q = Round(Clip(W ÷ (γ+ε), -1, 1)); Ŵ = γ·W_q.
//     same section, activation paragraph: AbsMax γ_A = max|A_k| per token,
//          A_q = Clip(Round(A × 127 ÷ (γ_A+ε)), -128, 127).
//     §"Como funciona a camada BitLinear ... (Zero-GEMM)?": add on +1,
//          subtract on -1, skip on 0, INT32 accumulation; worked example;
//          the result A_q·W_qᵀ is scaled once by (γ_A × γ) ÷ 127.
//     §"Como o ecossistema bitnet.cpp acelera ...": 81-entry table of
//          pre-summed signs for a block of 4 activations (index 0 = all -1,
//          40 = all 0, 80 = all +1) — used here as an independent second
//          way to compute the integer contraction.
//   [REPO] "Arquitetura Hibrida Multimodal para bitnet.cpp", §utils/ —
//          bit_layers.py: BitLinear, quantise_weights_ternary,
//          quantise_activations_8bit, ReLUSquared ("ReLU² as in BitNet").
//
// Readings where the pages are silent (each is listed in the design notes):
//   * "Round" is round-half-to-even (nearbyint under FE_TONEAREST).
//   * γ is a per-tensor mean: |W| summed in double in row-major order,
//     divided by N·K in double, then rounded once to fp32.
//   * Every floating-point step that decides an integer (a ternary code, an
//     int8 activation, the FFN requantisation) is taken in fp32, the
//     precision the GPU kernels use, with the pages' literal operation order:
//     x = W ÷ (γ+ε);  s = 127 ÷ (γ_A+ε);  A·s;  h = acc·((γ_A·γ)÷127).
//   * Final float outputs are computed in double from the integer result and
//     the fp32 scales: y = acc × ((γ_A × γ) ÷ 127); optional ReLU² on y.
//   * FFN block: h = dequantised up-projection (fp32), r = max(h,0)² (fp32),
//     per-token AbsMax requantisation of r, then the down-projection.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fopenmp -shared -fPIC
// (no fast-math; x86-64 SSE arithmetic, no excess precision).

#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// ---------------------------------------------------------------------------
// Threads used by the parallel drivers (independent output rows only; no
// arithmetic is reordered by threading).
int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

// ---------------------------------------------------------------------------
// [BLOG] §"qual a matemática da ternarização?": γ = (1 ÷ (n×m)) × Σ|W_ij|.
// Sum of |W| in double, row-major order.
double orc_sum_abs(const float* W, int64_t count) {
  double s = 0.0;
  for (int64_t i = 0; i < count; ++i) s += std::fabs((double)W[i]);
  return s;
}

// γ rounded once to fp32.
float orc_absmean_gamma(const float* W, int64_t N, int64_t K) {
  double s = orc_sum_abs(W, N * K);
  return (float)(s / (double)(N * K));
}

// Round-half-to-even of an fp32 value (FE_TONEAREST is the default mode).
static float round_half_even(float x) {
  return std::nearbyint(x);
}

static float clipf(float x, float lo, float hi) {
  return x < lo ? lo : (x > hi ? hi : x);
}

// [BLOG] §"qual a matemática da ternarização?":
// W_q = Round(Clip(W ÷ (γ+ε), -1, 1)) ∈ {-1, 0, +1}, taken in fp32.
void orc_ternary_codes(const float* W, int64_t N, int64_t K, float gamma,
                       float eps, int8_t* Wq) {
  const float g = gamma + eps;  // fp32 add
  for (int64_t i = 0; i < N * K; ++i) {
    float x = W[i] / g;  // IEEE fp32 division
    float q = round_half_even(clipf(x, -1.0f, 1.0f));
    Wq[i] = (int8_t)q;  // -0.0 converts to 0
  }
}

// quantise_weights_ternary: γ then codes.
float orc_quant_weights(const float* W, int64_t N, int64_t K, float eps,
                        int8_t* Wq) {
  float gamma = orc_absmean_gamma(W, N, K);
  orc_ternary_codes(W, N, K, gamma, eps, Wq);
  return gamma;
}

// ---------------------------------------------------------------------------
// 2-bit storage of the ternary weights ([BLOG] §"Memory Wall": "pesos
// compactados em 2 bits", 0.25 byte per weight). The pages give no bit
// layout; this library's layout is:
//   * code c = w + 1 ∈ {0, 1, 2} (3 is never written), so code order follows
//     the table order of [BLOG] §bitnet.cpp (index 0 = all -1, 80 = all +1);
//   * each row of K weights is K/16 little-endian 32-bit words (K/4 bytes);
//   * within word g, weight k = 16·g + 4·j + i (i, j ∈ 0..3) occupies bits
//     8·i + 2·j and 8·i + 2·j + 1.
// Requires K % 16 == 0.
void orc_pack_ternary(const int8_t* Wq, int64_t N, int64_t K, uint8_t* packed) {
  const int64_t words = K / 16;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < words; ++g) {
      uint32_t word = 0;
      for (int j = 0; j < 4; ++j) {
        for (int i = 0; i < 4; ++i) {
          int64_t k = 16 * g + 4 * j + i;
          uint32_t c = (uint32_t)(Wq[n * K + k] + 1);
          word |= c << (8 * i + 2 * j);
        }
      }
      uint8_t* dst = packed + n * (K / 4) + 4 * g;
      dst[0] = (uint8_t)(word & 0xFF);
      dst[1] = (uint8_t)((word >> 8) & 0xFF);
      dst[2] = (uint8_t)((word >> 16) & 0xFF);
      dst[3] = (uint8_t)((word >> 24) & 0xFF);
    }
  }
}

// Inverse of orc_pack_ternary. Returns the number of invalid codes (3), which
// are decoded as 0.
int64_t orc_unpack_ternary(const uint8_t* packed, int64_t N, int64_t K,
                           int8_t* Wq) {
  const int64_t words = K / 16;
  int64_t bad = 0;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < words; ++g) {
      const uint8_t* src = packed + n * (K / 4) + 4 * g;
      uint32_t word = (uint32_t)src[0] | ((uint32_t)src[1] << 8) |
                      ((uint32_t)src[2] << 16) | ((uint32_t)src[3] << 24);
      for (int j = 0; j < 4; ++j) {
        for (int i = 0; i < 4; ++i) {
          int64_t k = 16 * g + 4 * j + i;
          uint32_t c = (word >> (8 * i + 2 * j)) & 3u;
          if (c == 3u) {
            ++bad;
            c = 1u;
          }
          Wq[n * K + k] = (int8_t)((int)c - 1);
        }
      }
    }
  }
  return bad;
}

// ---------------------------------------------------------------------------
// [BLOG] §"qual a matemática da ternarização?", activation paragraph
// (quantise_activations_8bit): per token m,
//   γ_A = max_k |A[m,k]|;  A_q = Clip(Round(A × (127 ÷ (γ_A+ε))), -128, 127).
void orc_quant_acts(const float* A, int64_t M, int64_t K, float eps, int8_t* Aq,
                    float* gammaA) {
  for (int64_t m = 0; m < M; ++m) {
    const float* row = A + m * K;
    float gmax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = std::fabs(row[k]);
      if (a > gmax) gmax = a;
    }
    gammaA[m] = gmax;
    const float s = 127.0f / (gmax + eps);  // fp32: 127 ÷ (γ_A+ε)
    for (int64_t k = 0; k < K; ++k) {
      float v = row[k] * s;  // fp32 product
      float q = clipf(round_half_even(v), -128.0f, 127.0f);
      Aq[m * K + k] = (int8_t)q;
    }
  }
}

// ---------------------------------------------------------------------------
// [BLOG] §Zero-GEMM: acc[m,n] = Σ_k over the ternary weight row, adding the
// activation on +1, subtracting it on -1 and skipping it on 0, in INT32.
// Output rows are independent, so they are spread over threads.
void orc_zero_gemm(const int8_t* Aq, const int8_t* Wq, int64_t M, int64_t N,
                   int64_t K, int32_t* acc) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      const int8_t* a = Aq + m * K;
      const int8_t* w = Wq + n * K;
      int32_t s = 0;
      for (int64_t k = 0; k < K; ++k) {
        if (w[k] == 1) {
          s += a[k];
        } else if (w[k] == -1) {
          s -= a[k];
        }  // w == 0: skip
      }
      acc[m * N + n] = s;
    }
  }
}

// [BLOG] §bitnet.cpp: for each block of 4 int8 activations, a table of the 81
// signed sums over all ternary weight patterns. Pattern index is base-3 with
// digit d = w + 1, first weight most significant, so index 0 is -a0-a1-a2-a3,
// 40 is 0 and 80 is +a0+a1+a2+a3. The contraction then adds one table entry
// per 4 weights. Independent of orc_zero_gemm; used to cross-check it.
// Requires K % 4 == 0.
void orc_lut_gemm(const int8_t* Aq, const int8_t* Wq, int64_t M, int64_t N,
                  int64_t K, int32_t* acc) {
  const int64_t blocks = K / 4;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    std::vector<int32_t> table((size_t)blocks * 81);
    for (int64_t b = 0; b < blocks; ++b) {
      const int8_t* a = Aq + m * K + 4 * b;
      for (int idx = 0; idx < 81; ++idx) {
        int d0 = idx / 27, d1 = (idx / 9) % 3, d2 = (idx / 3) % 3, d3 = idx % 3;
        table[(size_t)b * 81 + idx] = (d0 - 1) * a[0] + (d1 - 1) * a[1] +
                                      (d2 - 1) * a[2] + (d3 - 1) * a[3];
      }
    }
    for (int64_t n = 0; n < N; ++n) {
      const int8_t* w = Wq + n * K;
      int32_t s = 0;
      for (int64_t b = 0; b < blocks; ++b) {
        int idx = 27 * (w[4 * b] + 1) + 9 * (w[4 * b + 1] + 1) +
                  3 * (w[4 * b + 2] + 1) + (w[4 * b + 3] + 1);
        s += table[(size_t)b * 81 + idx];
      }
      acc[m * N + n] = s;
    }
  }
}

// ---------------------------------------------------------------------------
// [BLOG] §Zero-GEMM, last paragraph: one scalar multiply by (γ_A × γ) ÷ 127.
// Computed in double from the fp32 scales; optional ReLU² ([REPO]
// ReLUSquared) applied to the dequantised value.
void orc_dequant(const int32_t* acc, const float* gammaA, float gamma,
                 int64_t M, int64_t N, int relu2, double* Y) {
  for (int64_t m = 0; m < M; ++m) {
    const double sc = ((double)gammaA[m] * (double)gamma) / 127.0;
    for (int64_t n = 0; n < N; ++n) {
      double y = (double)acc[m * N + n] * sc;
      if (relu2) {
        double r = y > 0.0 ? y : 0.0;
        y = r * r;
      }
      Y[m * N + n] = y;
    }
  }
}

// The same scaling taken in fp32, in the pages' order: sc = (γ_A·γ)÷127,
// h = (float)acc · sc. This is the value the FFN requantisation is decided on.
void orc_dequant_f32(const int32_t* acc, const float* gammaA, float gamma,
                     int64_t M, int64_t N, float* H) {
  for (int64_t m = 0; m < M; ++m) {
    const float sc = (gammaA[m] * gamma) / 127.0f;
    for (int64_t n = 0; n < N; ++n) {
      H[m * N + n] = (float)acc[m * N + n] * sc;
    }
  }
}

// ---------------------------------------------------------------------------
// BitLinear forward (inference): AbsMax act quant, Zero-GEMM with the given
// ternary codes, dequant (+ optional ReLU²). Outputs the int8 activations,
// γ_A, the INT32 accumulators and the float result.
void orc_bitlinear(const float* A, int64_t M, int64_t K, const int8_t* Wq,
                   float gamma, int64_t N, float eps, int relu2, int8_t* Aq,
                   float* gammaA, int32_t* acc, double* Y) {
  orc_quant_acts(A, M, K, eps, Aq, gammaA);
  orc_zero_gemm(Aq, Wq, M, N, K, acc);
  orc_dequant(acc, gammaA, gamma, M, N, relu2, Y);
}

// FFN requantisation of the up-projection ([REPO] ReLUSquared, then the
// [BLOG] AbsMax rule applied per token to r): all in fp32.
//   h = acc·((γ_A·γ_up)÷127);  r = max(h,0)·max(h,0);
//   γ_r = max_n r;  q = Clip(Round(r × (127 ÷ (γ_r+ε))), -128, 127).
void orc_relu2_requant(const int32_t* acc_up, const float* gammaA, float g_up,
                       int64_t M, int64_t H, float eps, int8_t* Rq,
                       float* gammaR) {
  std::vector<float> h((size_t)H), r((size_t)H);
  for (int64_t m = 0; m < M; ++m) {
    orc_dequant_f32(acc_up + m * H, gammaA + m, g_up, 1, H, h.data());
    float gmax = 0.0f;
    for (int64_t n = 0; n < H; ++n) {
      float p = h[n] > 0.0f ? h[n] : 0.0f;
      r[n] = p * p;  // fp32 product
      if (r[n] > gmax) gmax = r[n];
    }
    gammaR[m] = gmax;
    const float s = 127.0f / (gmax + eps);
    for (int64_t n = 0; n < H; ++n) {
      float q = clipf(round_half_even(r[n] * s), -128.0f, 127.0f);
      Rq[m * H + n] = (int8_t)q;
    }
  }
}

// Ternary FFN block: up BitLinear (K→H), ReLU², per-token requant, down
// BitLinear (H→K_out). Intermediates are returned for staged checks.
void orc_ffn_relu2(const float* X, int64_t M, int64_t K, int64_t H,
                   const int8_t* Wup, float g_up, const int8_t* Wdown,
                   float g_down, int64_t Nout, float eps, int8_t* Xq,
                   float* gammaX, int32_t* acc_up, int8_t* Rq, float* gammaR,
                   int32_t* acc_down, double* Y) {
  orc_quant_acts(X, M, K, eps, Xq, gammaX);
  orc_zero_gemm(Xq, Wup, M, H, K, acc_up);
  orc_relu2_requant(acc_up, gammaX, g_up, M, H, eps, Rq, gammaR);
  orc_zero_gemm(Rq, Wdown, M, Nout, H, acc_down);
  orc_dequant(acc_down, gammaR, g_down, M, Nout, 0, Y);
}

// ---------------------------------------------------------------------------
// Radix-3 storage ([BLOG] §"Como o ecossistema bitnet.cpp acelera ...": five
// ternary weights in one byte, 3^5 = 243 ≤ 256, 1.60 bits per weight).
// This library's layout of it:
//   * a row of K weights is split into groups t of five consecutive weights
//     k = 5t .. 5t+4 (weights past K count as 0);
//   * the group's value is b = Σ_i d_i·3^(4-i) with d_i = w_{5t+i} + 1 (the
//     first weight most significant, the digit order of the lookup-table
//     figure), so b ∈ [0, 242];
//   * the byte stored is q = ceil(256·b ÷ 243), b scaled to a fraction of
//     256, which is what lets a decoder peel digits off with multiplies by 3;
//     b = floor(243·q ÷ 256) recovers the group value;
//   * a row takes ceil(K/5) bytes, padded with zero-valued groups (q of all
//     weights 0) to a multiple of 16 bytes: row_bytes = 16·ceil(ceil(K/5)/16).
int64_t orc_radix3_row_bytes(int64_t K) {
  const int64_t groups = (K + 4) / 5;
  return (groups + 15) / 16 * 16;
}

void orc_pack_radix3(const int8_t* Wq, int64_t N, int64_t K, uint8_t* out) {
  const int64_t rb = orc_radix3_row_bytes(K);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t t = 0; t < rb; ++t) {
      int b = 0;
      for (int i = 0; i < 5; ++i) {
        const int64_t k = 5 * t + i;
        const int d = (k < K) ? (int)Wq[n * K + k] + 1 : 1;
        b = 3 * b + d;
      }
      out[n * rb + t] = (uint8_t)((256 * b + 242) / 243);  // ceil(256·b / 243)
    }
  }
}

// Inverse of orc_pack_radix3 (weights past K are dropped). Returns the
// number of bytes that are not the image of a group value (never written
// by the packer); those decode as their floor group value.
int64_t orc_unpack_radix3(const uint8_t* in, int64_t N, int64_t K, int8_t* Wq) {
  const int64_t rb = orc_radix3_row_bytes(K);
  int64_t bad = 0;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t t = 0; t < rb; ++t) {
      const int q = in[n * rb + t];
      const int b = (243 * q) / 256;  // floor
      if ((256 * b + 242) / 243 != q) ++bad;
      int rest = b;
      for (int i = 0; i < 5; ++i) {
        int p = 1;
        for (int j = 0; j < 4 - i; ++j) p *= 3;
        const int d = rest / p;
        rest -= d * p;
        const int64_t k = 5 * t + i;
        if (k < K) Wq[n * K + k] = (int8_t)(d - 1);
      }
    }
  }
  return bad;
}

// ---------------------------------------------------------------------------
// [BLOG] §Zero-GEMM, paragraph after the worked example: training uses the
// Straight-Through Estimator; in the backward pass the gradient of the
// quantisation is taken as the identity (∂W_q ÷ ∂W = 1) for values inside
// the valid range. Reading (the page states no more): the forward is
// Y = Â·Ŵᵀ with Ŵ = γ·W_q and Â = (γ_A ÷ 127)·A_q; the backward passes the
// output gradient dY through both quantisers as if they were the identity,
// except that the weight gradient is zero where the Clip of W ÷ (γ+ε) to
// [-1, 1] was active. Sums in double.
//   dA[m,k] = Σ_n dY[m,n]·Ŵ[n,k] = γ·(Σ_{W_q=+1} dY[m,n] − Σ_{W_q=−1} dY[m,n])
//   dW[n,k] = 1[−1 ≤ W ÷ (γ+ε) ≤ 1] · Σ_m dY[m,n]·Â[m,k]
// The range test uses the same fp32 quotient the forward rounds.
void orc_ste_grad_input(const float* dY, int64_t M, int64_t N, const int8_t* Wq,
                        int64_t K, float gamma, double* dA) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t k = 0; k < K; ++k) {
      double s = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        const int8_t w = Wq[n * K + k];
        if (w == 1) {
          s += (double)dY[m * N + n];
        } else if (w == -1) {
          s -= (double)dY[m * N + n];
        }
      }
      dA[m * K + k] = (double)gamma * s;
    }
  }
}

// 1 where the forward's Clip(W ÷ (γ+ε), -1, 1) left the quotient unchanged.
void orc_ste_weight_mask(const float* W, int64_t N, int64_t K, float gamma,
                         float eps, uint8_t* mask) {
  const float g = gamma + eps;  // fp32 add, as in the forward
  for (int64_t i = 0; i < N * K; ++i) {
    const float x = W[i] / g;  // fp32 division, as in the forward
    mask[i] = (x >= -1.0f && x <= 1.0f) ? 1 : 0;
  }
}

void orc_ste_grad_weight(const float* dY, int64_t M, int64_t N, const int8_t* Aq,
                         const float* gammaA, int64_t K, const float* W,
                         float gamma, float eps, double* dW) {
  std::vector<uint8_t> mask((size_t)N * K);
  orc_ste_weight_mask(W, N, K, gamma, eps, mask.data());
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      double s = 0.0;
      if (mask[n * K + k]) {
        for (int64_t m = 0; m < M; ++m) {
          const double a_hat = (double)gammaA[m] / 127.0 * (double)Aq[m * K + k];
          s += (double)dY[m * N + n] * a_hat;
        }
      }
      dW[n * K + k] = s;
    }
  }
}

}  // extern "C"
