/*
 * tgemm_oracle.h -- plain CPU oracle for the ternary / 4-bit dequant-fused matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or call
 * this code: it exists so that tests/, the smoke check and the benchmark's CPU
 * baseline can compare the CUDA library against an independent, obviously-correct
 * restatement of what the source pages define.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * Sources (page title, section):
 *   [P2-LB]  "We're Teaching Your Browser to Paint: A 4B Image Model on WebGPU",
 *            section "The lucky break that wasn't luck" -- Q2_0: 128-weight blocks,
 *            one f16 scale d per block, 2-bit codes {0,1,2} packed LSB-first four per
 *            byte along the input axis, w = (q - 1) * d; the only rounding is the
 *            scale's f32 -> f16 conversion, which must round-trip exactly.
 *   [P2-GD]  same page, "The GPU driver, and the bug that looked like broken math" --
 *            quantized rows are independent byte runs (row slicing); a projection
 *            whose input is two activations concatenated per token is split along its
 *            input axis into two matmuls that are summed ("Slice weights, not
 *            activations").
 *   [P2-WL]  same page, "What's left" -- the 4-bit format dequantizes as
 *            (q - zero) * scale.
 *   [P3-FB]  "You Can Now Just Ask for an Image -- and Your Browser Draws It",
 *            section "The bug that hid in one flipped bit" -- two 4-bit codes per
 *            byte, the code of even index t sits in the low nibble:
 *            code = (byte >> ((t & 1) * 4)) & 0xF.
 *   [P5-1S]  "mindview-t2i-turbo" model card, section "One step" -- side branch
 *            y = W x + B (A x).
 *
 * Conventions (readings where the pages are silent; each is listed in the design notes):
 *   - packed Q2 weights: wq[N][K/4] bytes and d[N][K/128] f16 bit patterns, two planes;
 *   - packed Q4 weights: wq[N][K/2] bytes and sz[N][K/64][2] f16 bit patterns (s, z);
 *     the Q4 group is 64 weights along K; t is the index along K within the row;
 *   - activations x[M][K] and low-rank factors A[r][K], B[N][r] are bf16 bit patterns;
 *   - outputs y[M][N] in f64, accumulated in ascending k.
 */
#ifndef TGEMM_ORACLE_H
#define TGEMM_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status bits returned by the pack functions */
#define ORACLE_PACK_BAD_CODE  1u
#define ORACLE_PACK_INEXACT   2u
#define ORACLE_PACK_NONFINITE 4u
#define ORACLE_PACK_ZERO_MISMATCH  8u   /* gemlite import: zero != -scale */
#define ORACLE_PACK_GROUP_MISMATCH 16u  /* gemlite import: groups of one 128-block differ */

/* IEEE 754 binary16 and bfloat16, converted bit by bit (round to nearest, ties to even). */
float    oracle_f16_to_f32(uint16_t h);
uint16_t oracle_f32_to_f16_rne(float f);
float    oracle_bf16_to_f32(uint16_t b);
uint16_t oracle_f32_to_bf16_rne(float f);
uint16_t oracle_f64_to_bf16_rne(double v);
void     oracle_f64_to_bf16_array(const double* v, int64_t n, uint16_t* out);

/* Q2_0 [P2-LB] */
void     oracle_q2_unpack(const uint8_t* wq, int64_t N, int64_t K, uint8_t* codes);
uint32_t oracle_q2_pack(const uint8_t* codes, const float* scale, int64_t N, int64_t K,
                        uint8_t* wq, uint16_t* d);
void     oracle_q2_dequant(const uint8_t* wq, const uint16_t* d, int64_t N, int64_t K, float* w);

/* gemlite-int2 -> Q2_0 [P2-LB]: the pages give gemlite's codes ({0,1,2}, LSB-first, four
 * per byte along the input axis), its dequant ((q - zero) * scale with zeros == -scales,
 * i.e. (q - 1) * scale) and the conversion ("a transpose and regroup", scales f32 -> f16
 * with an exact roundtrip).  Layout reading: wq_g[K/4][N] bytes, byte (i, n) holding the
 * codes of k = 4i..4i+3 of output row n; scale and zero f32 [N][K/g], group j covering
 * k in [j g, (j + 1) g).  Q2_0 block b takes the scale of the groups covering
 * [128 b, 128 b + 128), which must all be equal.  g divides 128, or is a multiple of 128
 * dividing K.  Returns the Q2 pack status plus the two import bits above. */
uint32_t oracle_q2_from_gemlite(const uint8_t* wq_g, const float* scale, const float* zero,
                                int64_t N, int64_t K, int64_t g, uint8_t* wq, uint16_t* d);

/* 4-bit group format [P3-FB], [P2-WL] */
void     oracle_q4_unpack(const uint8_t* wq, int64_t N, int64_t K, uint8_t* codes);
uint32_t oracle_q4_pack(const uint8_t* codes, const float* s, const float* z, int64_t N,
                        int64_t K, uint8_t* wq, uint16_t* sz);
void     oracle_q4_dequant(const uint8_t* wq, const uint16_t* sz, int64_t N, int64_t K, float* w);

/* y[m][n] = sum_k w[n][k] * x[m][k] in f64 (the plain definition of the matmul). */
void oracle_gemm_f64(const uint16_t* x, const float* w, int64_t M, int64_t N, int64_t K,
                     double* y);
/* y[m][n] += sum_i B[n][i] * (sum_k A[i][k] * x[m][k]) in f64 [P5-1S]. */
void oracle_lora_add_f64(const uint16_t* x, const uint16_t* a, const uint16_t* b, int64_t r,
                         int64_t M, int64_t N, int64_t K, double* y);

/* Whole-matrix composites: dequantize, then multiply (and add the side branch). */
void oracle_q2_gemm(const uint16_t* x, const uint8_t* wq, const uint16_t* d, int64_t M,
                    int64_t N, int64_t K, double* y);
void oracle_q2_lora_gemm(const uint16_t* x, const uint8_t* wq, const uint16_t* d,
                         const uint16_t* a, const uint16_t* b, int64_t r, int64_t M,
                         int64_t N, int64_t K, double* y);
void oracle_q4_gemm(const uint16_t* x, const uint8_t* wq, const uint16_t* sz, int64_t M,
                    int64_t N, int64_t K, double* y);

/* A projection split along its input axis [P2-GD]: y = x1 W1^T + x2 W2^T, with
 * x1 [M][K1], W1 packed [N][K1/4] + [N][K1/128], x2 [M][K2], W2 packed likewise.  Two
 * independent f64 products, added element by element. */
void oracle_q2_dual_gemm(const uint16_t* x1, const uint8_t* wq1, const uint16_t* d1, int64_t K1,
                         const uint16_t* x2, const uint8_t* wq2, const uint16_t* d2, int64_t K2,
                         int64_t M, int64_t N, double* y);
void oracle_q2_dual_gemm_at(const uint16_t* x1, const uint8_t* wq1, const uint16_t* d1,
                            int64_t K1, const uint16_t* x2, const uint8_t* wq2,
                            const uint16_t* d2, int64_t K2, int64_t M, int64_t N,
                            const int64_t* mi, const int64_t* ni, int64_t count, double* out);

/* Sampled outputs, one at a time: out[i] = y[mi[i]][ni[i]].  a/b may be NULL (no branch). */
void oracle_q2_gemm_at(const uint16_t* x, const uint8_t* wq, const uint16_t* d,
                       const uint16_t* a, const uint16_t* b, int64_t r, int64_t M, int64_t N,
                       int64_t K, const int64_t* mi, const int64_t* ni, int64_t count,
                       double* out);
void oracle_q4_gemm_at(const uint16_t* x, const uint8_t* wq, const uint16_t* sz, int64_t M,
                       int64_t N, int64_t K, const int64_t* mi, const int64_t* ni,
                       int64_t count, double* out);

/* Number of OpenMP threads the oracle uses (1 when built without OpenMP). */
int oracle_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
