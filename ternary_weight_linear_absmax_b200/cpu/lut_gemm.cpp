// Host table-lookup BitLinear contraction (see include/bitlinear_lut_cpu.h).
//
// "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section
// "Como o ecossistema bitnet.cpp acelera inferência em CPUs e borda?": per
// token, one 81-entry table of signed sums for every block of 4 int8
// activations; each group of 4 ternary weights is an index into it, so the
// contraction adds one table entry per 4 weights.
//
// x86-64 design: the tables of one token are int16 (|entry| ≤ 4·127) and
// stay in L1/L2 (K/4 · 81 · 2 bytes: 104 KB at K = 2560). Weights are stored
// as one index byte per group, 16 rows interleaved per group, so one 16-byte
// load brings the indices of 16 rows for the same activation block; a
// gather (AVX-512: 16 lanes, AVX2: 8) reads their 16 table entries and one
// add accumulates them in INT32. The path is chosen at run time from the
// CPU's features; the scalar path is the same loop without SIMD.
#include "bitlinear_lut_cpu.h"

#include <immintrin.h>
#include <omp.h>

#include <cmath>
#include <cstring>
#include <vector>

namespace {

constexpr int kRowBlock = 16;
constexpr int kEntries = 81;
constexpr int kZeroIndex = 40;  // all four weights 0

inline int64_t row_blocks(int64_t N) { return (N + kRowBlock - 1) / kRowBlock; }

// Table of one 4-activation block, in the figure's order (d_i = w_i + 1,
// first weight most significant). Built by adding one activation at a time:
// the entries of the last j weights are extended by -a, 0 or +a.
void build_table(const int8_t* a, int16_t* t) {
  int16_t t3[3], t23[9], t123[27];
  for (int d3 = 0; d3 < 3; ++d3) t3[d3] = (int16_t)(d3 == 0 ? -a[3] : (d3 == 2 ? a[3] : 0));
  for (int d2 = 0; d2 < 3; ++d2)
    for (int r = 0; r < 3; ++r)
      t23[3 * d2 + r] = (int16_t)(t3[r] + (d2 == 0 ? -a[2] : (d2 == 2 ? a[2] : 0)));
  for (int d1 = 0; d1 < 3; ++d1)
    for (int r = 0; r < 9; ++r)
      t123[9 * d1 + r] = (int16_t)(t23[r] + (d1 == 0 ? -a[1] : (d1 == 2 ? a[1] : 0)));
  for (int d0 = 0; d0 < 3; ++d0)
    for (int r = 0; r < 27; ++r)
      t[27 * d0 + r] = (int16_t)(t123[r] + (d0 == 0 ? -a[0] : (d0 == 2 ? a[0] : 0)));
}

// One row block (16 rows) of one token: acc16[r] = Σ_g T[g][idx[g][r]].
void block_scalar(const int16_t* T, const uint8_t* idx, int64_t groups, int32_t* acc16) {
  int32_t s[kRowBlock] = {0};
  for (int64_t g = 0; g < groups; ++g) {
    const int16_t* tg = T + g * kEntries;
    const uint8_t* ig = idx + g * kRowBlock;
    for (int r = 0; r < kRowBlock; ++r) s[r] += tg[ig[r]];
  }
  std::memcpy(acc16, s, sizeof(s));
}

__attribute__((target("avx2"))) void block_avx2(const int16_t* T, const uint8_t* idx,
                                                 int64_t groups, int32_t* acc16) {
  __m256i s0 = _mm256_setzero_si256(), s1 = _mm256_setzero_si256();
  const int* base = reinterpret_cast<const int*>(T);
  for (int64_t g = 0; g < groups; ++g) {
    const __m128i ib = _mm_loadu_si128(reinterpret_cast<const __m128i*>(idx + g * kRowBlock));
    const __m256i off = _mm256_set1_epi32((int)(g * kEntries));
    const __m256i i0 = _mm256_add_epi32(_mm256_cvtepu8_epi32(ib), off);
    const __m256i i1 = _mm256_add_epi32(_mm256_cvtepu8_epi32(_mm_srli_si128(ib, 8)), off);
    // 4-byte reads at T + 2·index: the low half is the int16 entry.
    const __m256i v0 = _mm256_i32gather_epi32(base, i0, 2);
    const __m256i v1 = _mm256_i32gather_epi32(base, i1, 2);
    s0 = _mm256_add_epi32(s0, _mm256_srai_epi32(_mm256_slli_epi32(v0, 16), 16));
    s1 = _mm256_add_epi32(s1, _mm256_srai_epi32(_mm256_slli_epi32(v1, 16), 16));
  }
  _mm256_storeu_si256(reinterpret_cast<__m256i*>(acc16), s0);
  _mm256_storeu_si256(reinterpret_cast<__m256i*>(acc16 + 8), s1);
}

__attribute__((target("avx512f"))) void block_avx512(const int16_t* T, const uint8_t* idx,
                                                      int64_t groups, int32_t* acc16) {
  __m512i s = _mm512_setzero_si512();
  for (int64_t g = 0; g < groups; ++g) {
    const __m128i ib = _mm_loadu_si128(reinterpret_cast<const __m128i*>(idx + g * kRowBlock));
    const __m512i i = _mm512_add_epi32(_mm512_cvtepu8_epi32(ib), _mm512_set1_epi32((int)(g * kEntries)));
    const __m512i v = _mm512_i32gather_epi32(i, T, 2);
    s = _mm512_add_epi32(s, _mm512_srai_epi32(_mm512_slli_epi32(v, 16), 16));
  }
  _mm512_storeu_si512(acc16, s);
}

typedef void (*BlockFn)(const int16_t*, const uint8_t*, int64_t, int32_t*);

bool isa_supported(int isa) {
  __builtin_cpu_init();
  switch (isa) {
    case BLC_ISA_SCALAR: return true;
    case BLC_ISA_AVX2: return __builtin_cpu_supports("avx2");
    case BLC_ISA_AVX512: return __builtin_cpu_supports("avx512f");
  }
  return false;
}

BlockFn block_fn(int isa) {
  switch (isa) {
    case BLC_ISA_AVX512: return block_avx512;
    case BLC_ISA_AVX2: return block_avx2;
    default: return block_scalar;
  }
}

int resolve(int isa) {
  if (isa == BLC_ISA_AUTO) return blc_best_isa();
  return isa_supported(isa) ? isa : -1;
}

}  // namespace

extern "C" {

int blc_best_isa(void) {
  if (isa_supported(BLC_ISA_AVX512)) return BLC_ISA_AVX512;
  if (isa_supported(BLC_ISA_AVX2)) return BLC_ISA_AVX2;
  return BLC_ISA_SCALAR;
}

size_t blc_lut_index_bytes(int64_t N, int64_t K) {
  return (size_t)row_blocks(N) * kRowBlock * (size_t)(K / 4);
}

int64_t blc_lut_index_from_packed(const uint8_t* W_packed, int64_t N, int64_t K, uint8_t* idx) {
  const int64_t groups = K / 4, nb = row_blocks(N);
  int64_t bad = 0;
  for (int64_t b = 0; b < nb; ++b) {
    for (int r = 0; r < kRowBlock; ++r) {
      const int64_t n = b * kRowBlock + r;
      for (int64_t g = 0; g < groups; ++g) {
        uint8_t* dst = idx + (b * groups + g) * kRowBlock + r;
        if (n >= N) {
          *dst = kZeroIndex;
          continue;
        }
        // weights 4g..4g+3 = 16·w + 4·j + i for word w = g/4, j = g%4, i = 0..3
        const uint8_t* wp = W_packed + n * (K / 4) + 4 * (g >> 2);
        const uint32_t word = (uint32_t)wp[0] | ((uint32_t)wp[1] << 8) |
                              ((uint32_t)wp[2] << 16) | ((uint32_t)wp[3] << 24);
        const int j = (int)(g & 3);
        int index = 0;
        for (int i = 0; i < 4; ++i) {
          uint32_t c = (word >> (8 * i + 2 * j)) & 3u;
          if (c == 3u) {
            ++bad;
            c = 1u;
          }
          index = 3 * index + (int)c;
        }
        *dst = (uint8_t)index;
      }
    }
  }
  return bad;
}

void blc_lut_table(const int8_t a[4], int16_t table[81]) { build_table(a, table); }

int blc_lut_gemm(const int8_t* A_q, int64_t M, int64_t K, const uint8_t* idx, int64_t N,
                 int32_t* acc, int threads, int isa) {
  const int use = resolve(isa);
  if (use < 0) return -1;
  if (M <= 0 || N <= 0) return 0;
  const BlockFn fn = block_fn(use);
  const int64_t groups = K / 4, nb = row_blocks(N);
  // One token's tables, plus 2 bytes so the last 4-byte gather read stays inside.
  std::vector<int16_t> T((size_t)groups * kEntries + 2, 0);
  const int nt = threads > 0 ? threads : omp_get_max_threads();
  for (int64_t m = 0; m < M; ++m) {
    const int8_t* a = A_q + m * K;
    int32_t* out = acc + m * N;
#pragma omp parallel num_threads(nt)
    {
#pragma omp for schedule(static)
      for (int64_t g = 0; g < groups; ++g) build_table(a + 4 * g, T.data() + g * kEntries);
      // (implicit barrier: every table is built before any lookup)
#pragma omp for schedule(static)
      for (int64_t b = 0; b < nb; ++b) {
        int32_t s[kRowBlock];
        fn(T.data(), idx + b * groups * kRowBlock, groups, s);
        const int64_t n0 = b * kRowBlock;
        const int rows = (int)(N - n0 < kRowBlock ? N - n0 : kRowBlock);
        std::memcpy(out + n0, s, (size_t)rows * sizeof(int32_t));
      }
    }
  }
  return 0;
}

int blc_bitlinear_lut(const float* A, int64_t M, int64_t K, const uint8_t* idx, float gamma,
                      int64_t N, float eps, float* Y, int8_t* A_q, float* gamma_A, int threads,
                      int isa) {
  if (resolve(isa) < 0) return -1;
  if (M <= 0 || N <= 0) return 0;
  std::vector<int8_t> q((size_t)M * K);
  std::vector<float> gA((size_t)M);
  for (int64_t m = 0; m < M; ++m) {
    const float* row = A + m * K;
    float mx = 0.0f;
    for (int64_t k = 0; k < K; ++k) mx = std::fmax(mx, std::fabs(row[k]));
    const float s = 127.0f / (mx + eps);
    for (int64_t k = 0; k < K; ++k) {
      float v = std::nearbyint(row[k] * s);
      v = v < -128.0f ? -128.0f : (v > 127.0f ? 127.0f : v);
      q[(size_t)m * K + k] = (int8_t)v;
    }
    gA[m] = mx;
  }
  std::vector<int32_t> acc((size_t)M * N);
  const int rc = blc_lut_gemm(q.data(), M, K, idx, N, acc.data(), threads, isa);
  if (rc != 0) return rc;
  for (int64_t m = 0; m < M; ++m) {
    const float sc = (gA[m] * gamma) / 127.0f;
    for (int64_t n = 0; n < N; ++n) Y[m * N + n] = (float)acc[(size_t)m * N + n] * sc;
  }
  if (A_q) std::memcpy(A_q, q.data(), q.size());
  if (gamma_A) std::memcpy(gamma_A, gA.data(), gA.size() * sizeof(float));
  return 0;
}

}  // extern "C"
