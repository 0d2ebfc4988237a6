/*
 * bitlinear_lut_cpu.h — host (x86-64) table-lookup BitLinear contraction.
 *
 * The lookup-table method of "BitNet b1.58 — quantização ternária,
 * BitLinear, Zero-GEMM", section "Como o ecossistema bitnet.cpp acelera
 * inferência em CPUs e borda?" (figure "Fluxo de Execução com Lookup Table
 * (LUT-GEMM)"): for every block of 4 int8 activations the 3^4 = 81 possible
 * signed sums are tabulated once per token; a group of 4 ternary weights is
 * then one table index, so the contraction is one table read and one add per
 * 4 weights, with no multiplication. Table order follows the figure: index
 * 27·d0 + 9·d1 + 3·d2 + d3 with d_i = w_i + 1 (first weight most
 * significant), so index 0 holds -a0-a1-a2-a3, 40 holds 0 and 80 holds
 * +a0+a1+a2+a3.
 *
 * This library runs on the host CPU only: it is the second CPU baseline of
 * the benchmark and an independent cross-check of the integer contraction.
 * Every pointer is a HOST pointer owned by the caller; nothing is allocated
 * beyond per-call tables on the stack/heap of the calling threads, and
 * nothing is kept after a call returns. Results are exact (int16 table
 * entries, |entry| ≤ 508, INT32 sums).
 *
 * Index layout ("LUT-indexed weights"): rows are grouped in blocks of 16;
 * block b holds, for each of the K/4 weight groups g, the 16 index bytes of
 * rows 16b .. 16b+15 (rows past N hold index 40, all zero):
 *   idx[(b·(K/4) + g)·16 + r] = index of weights 4g..4g+3 of row 16b + r.
 * Size: ceil(N/16)·16·K/4 bytes (2 bits per weight, like the 2-bit format).
 */
#ifndef BITLINEAR_LUT_CPU_H_
#define BITLINEAR_LUT_CPU_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Instruction-set paths of blc_lut_gemm. */
enum { BLC_ISA_AUTO = 0, BLC_ISA_SCALAR = 1, BLC_ISA_AVX2 = 2, BLC_ISA_AVX512 = 3 };

/* The best path this CPU supports (BLC_ISA_SCALAR/AVX2/AVX512). */
int blc_best_isa(void);

/* Bytes of the LUT-indexed weight layout for an N×K matrix. */
size_t blc_lut_index_bytes(int64_t N, int64_t K);

/* Converts packed ternary weights in the 2-bit format of bitlinear.h
 * ([N, K/4] bytes; weight 16g+4j+i at bits 8i+2j of 32-bit word g) into the
 * LUT-indexed layout above. K must be a positive multiple of 16.
 * Returns the number of invalid codes (3) met, which are read as 0. */
int64_t blc_lut_index_from_packed(const uint8_t* W_packed, int64_t N, int64_t K,
                                  uint8_t* idx);

/* The 81-entry table of one block of 4 activations (figure's order). */
void blc_lut_table(const int8_t a[4], int16_t table[81]);

/* acc[m, n] = Σ_k A_q[m,k]·W_q[n,k] by table lookup. A_q [M, K] int8,
 * idx from blc_lut_index_from_packed, acc [M, N] int32. K % 4 == 0.
 * threads ≤ 0: all hardware threads. isa: BLC_ISA_* (AUTO = best).
 * Returns 0, or -1 if the requested isa is not supported by this CPU. */
int blc_lut_gemm(const int8_t* A_q, int64_t M, int64_t K, const uint8_t* idx,
                 int64_t N, int32_t* acc, int threads, int isa);

/* Whole BitLinear forward on the host: AbsMax per-token quantisation of A
 * (fp32: γ_A = max|A|, A_q = Clip(Round(A·(127/(γ_A+ε))), -128, 127), round
 * half to even), the table-lookup contraction, and Y = acc·((γ_A·γ)/127)
 * in fp32. A [M, K] fp32; Y [M, N] fp32; A_q / gamma_A may be NULL. */
int blc_bitlinear_lut(const float* A, int64_t M, int64_t K, const uint8_t* idx,
                      float gamma, int64_t N, float eps, float* Y, int8_t* A_q,
                      float* gamma_A, int threads, int isa);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_LUT_CPU_H_ */
