/*
 * tgemm_oracle.c -- plain CPU oracle (TEST INFRASTRUCTURE ONLY; see tgemm_oracle.h).
 *
 * Written to be read against the pages, not to be fast: byte-by-byte unpacking, f32
 * dequantization, an f64 triple loop in ascending k.  OpenMP only splits independent
 * output rows across threads; it does not change any sum.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fopenmp -fPIC -shared (see oracle/build.py).
 * -ffp-contract=off keeps (q - z) * s as two rounded f32 operations.
 *
 * ORACLE_PLANT_* macros exist only for the mutation tests, which rebuild this file with
 * one deliberate mistake and check that the pins catch it.  The normal build defines
 * none of them.
 */
#include "tgemm_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------------------
 * Scalar conversions.  IEEE 754 binary16: 1 sign, 5 exponent (bias 15), 10 fraction
 * bits.  bfloat16: the top 16 bits of binary32.  Rounding: to nearest, ties to even.
 * ---------------------------------------------------------------------------------- */

float oracle_f16_to_f32(uint16_t h) {
  unsigned sign = (h >> 15) & 1u;
  unsigned expo = (h >> 10) & 0x1Fu;
  unsigned frac = h & 0x3FFu;
  float v;
  if (expo == 0) {
    v = ldexpf((float)frac, -24); /* subnormal: frac * 2^-24 */
  } else if (expo == 31) {
    v = frac ? NAN : INFINITY;
  } else {
    v = ldexpf((float)(frac | 0x400u), (int)expo - 25); /* 1.frac * 2^(expo-15) */
  }
  return sign ? -v : v;
}

/* Shift a right by s bits, rounding to nearest, ties to even. */
static uint32_t shr_rne(uint32_t a, int s) {
  if (s <= 0) return a;
  if (s >= 32) return 0;
  uint32_t q = a >> s;
  uint32_t rem = a & ((1u << s) - 1u);
  uint32_t half = 1u << (s - 1);
#ifdef ORACLE_PLANT_F16_TRUNCATE
  (void)rem; (void)half;
  return q;
#else
  if (rem > half || (rem == half && (q & 1u))) q += 1u;
  return q;
#endif
}

uint16_t oracle_f32_to_f16_rne(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
  uint32_t ax = x & 0x7FFFFFFFu;
  if (ax > 0x7F800000u) return (uint16_t)(sign | 0x7E00u); /* NaN */
  if (ax == 0x7F800000u) return (uint16_t)(sign | 0x7C00u); /* inf */
  int e = (int)(ax >> 23) - 127;                             /* unbiased f32 exponent */
  uint32_t sig = (ax >> 23) ? ((ax & 0x7FFFFFu) | 0x800000u) : (ax & 0x7FFFFFu);
  if (!(ax >> 23)) e = -126; /* f32 subnormal */
  if (e >= -14) {
    /* normal f16 range (or overflow): keep 11 significant bits */
    uint32_t m = shr_rne(sig, 13);         /* 1.xxxxxxxxxx, may carry to 2.0 */
    int ee = e + 15;
    if (m >= 0x800u) { m >>= 1; ee += 1; } /* carry out of the significand */
    if (ee >= 31) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | ((uint32_t)ee << 10) | (m & 0x3FFu));
  }
  /* subnormal f16: value = sig * 2^(e-23); in units of 2^-24 that is sig * 2^(e+1) */
  int s = -(e + 1);
  uint32_t m = shr_rne(sig, s); /* may round up to 0x400 = smallest normal, still right */
  return (uint16_t)(sign | m);
}

float oracle_bf16_to_f32(uint16_t b) {
  uint32_t x = (uint32_t)b << 16;
  float f;
  memcpy(&f, &x, 4);
  return f;
}

uint16_t oracle_f32_to_bf16_rne(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  if ((x & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((x >> 16) | 0x40u); /* NaN */
  uint32_t upper = x >> 16;
  uint32_t lower = x & 0xFFFFu;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
  return (uint16_t)upper;
}

uint16_t oracle_f64_to_bf16_rne(double v) {
  if (isnan(v)) return 0x7FC0u;
  if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
  int sign = v < 0;
  double a = fabs(v);
  int e;
  frexp(a, &e); /* a = frac * 2^e, frac in [0.5, 1): leading bit has weight 2^(e-1) */
  int lead = e - 1;
  if (lead < -126) lead = -126; /* bf16 subnormals share f32's minimum exponent */
  /* 8 significant bits: units of 2^(lead-7); rint rounds to nearest, ties to even */
#ifdef ORACLE_PLANT_BF16_TRUNCATE
  double q = trunc(ldexp(a, 7 - lead));
#else
  double q = rint(ldexp(a, 7 - lead));
#endif
  double r = ldexp(q, lead - 7);
  if (r >= 0x1p128) return sign ? 0xFF80u : 0x7F80u;
  float rf = (float)r; /* exact: at most 8 significant bits inside f32's range */
  uint32_t bits;
  memcpy(&bits, &rf, 4);
  return (uint16_t)((bits >> 16) | (sign ? 0x8000u : 0u));
}

void oracle_f64_to_bf16_array(const double* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_f64_to_bf16_rne(v[i]);
}

/* ------------------------------------------------------------------------------------
 * Q2_0 [P2-LB]: four 2-bit codes per byte, LSB first along the input axis; one f16
 * scale per 128 weights; w = (q - 1) * d.
 * ---------------------------------------------------------------------------------- */

static unsigned q2_code_of(uint8_t byte, int j) {
#ifdef ORACLE_PLANT_Q2_MSB_FIRST
  return (unsigned)(byte >> (6 - 2 * j)) & 3u;
#else
  return (unsigned)(byte >> (2 * j)) & 3u; /* code j of the byte sits at bits 2j, 2j+1 */
#endif
}

void oracle_q2_unpack(const uint8_t* wq, int64_t N, int64_t K, uint8_t* codes) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      codes[n * K + k] = (uint8_t)q2_code_of(wq[n * (K / 4) + k / 4], (int)(k % 4));
}

static int is_finite_f32(float v) { return !isnan(v) && !isinf(v); }

uint32_t oracle_q2_pack(const uint8_t* codes, const float* scale, int64_t N, int64_t K,
                        uint8_t* wq, uint16_t* d) {
  uint32_t status = 0;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t i = 0; i < K / 4; ++i) {
      unsigned byte = 0;
      for (int j = 0; j < 4; ++j) {
        unsigned q = codes[n * K + 4 * i + j];
        if (q > 2u) status |= ORACLE_PACK_BAD_CODE;
#ifdef ORACLE_PLANT_Q2_MSB_FIRST
        byte |= (q & 3u) << (6 - 2 * j);
#else
        byte |= (q & 3u) << (2 * j);
#endif
      }
      wq[n * (K / 4) + i] = (uint8_t)byte;
    }
    for (int64_t b = 0; b < K / 128; ++b) {
      float v = scale[n * (K / 128) + b];
      uint16_t h = oracle_f32_to_f16_rne(v);
      if (!is_finite_f32(v)) status |= ORACLE_PACK_NONFINITE;
      else if (oracle_f16_to_f32(h) != v) status |= ORACLE_PACK_INEXACT;
      d[n * (K / 128) + b] = h;
    }
  }
  return status;
}

uint32_t oracle_q2_from_gemlite(const uint8_t* wq_g, const float* scale, const float* zero,
                                int64_t N, int64_t K, int64_t g, uint8_t* wq, uint16_t* d) {
  const int64_t ng = K / g, nb = K / 128;
  uint8_t* codes = (uint8_t*)malloc((size_t)(N * K));
  float* bs = (float*)malloc((size_t)(N * nb) * sizeof(float));
  uint32_t status = 0;
  /* the transpose: gemlite's byte (k / 4, n) -> codes[n][k] */
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
#ifdef ORACLE_PLANT_GEMLITE_NO_TRANSPOSE
      unsigned byte = wq_g[n * (K / 4) + k / 4];
#else
      unsigned byte = wq_g[(k / 4) * N + n];
#endif
      codes[n * K + k] = (uint8_t)((byte >> (2 * (k % 4))) & 3u);
    }
  /* zeros == -scales, every group */
#ifndef ORACLE_PLANT_GEMLITE_ZERO_UNCHECKED
  for (int64_t i = 0; i < N * ng; ++i)
    if (!(zero[i] == -scale[i])) status |= ORACLE_PACK_ZERO_MISMATCH;
#endif
  /* the regroup: block b of row n takes the scale of the groups covering it */
  for (int64_t n = 0; n < N; ++n)
    for (int64_t b = 0; b < nb; ++b) {
      const int64_t k0 = 128 * b, k1 = 128 * b + 128;
#ifdef ORACLE_PLANT_GEMLITE_GROUP_INDEX
      const int64_t j0 = b % ng;
#else
      const int64_t j0 = k0 / g;
#endif
      const float s = scale[n * ng + j0];
      for (int64_t j = k0 / g; j * g < k1; ++j)
        if (!(scale[n * ng + j] == s)) status |= ORACLE_PACK_GROUP_MISMATCH;
      bs[n * nb + b] = s;
    }
  status |= oracle_q2_pack(codes, bs, N, K, wq, d);
  free(codes);
  free(bs);
  return status;
}

void oracle_q2_dequant(const uint8_t* wq, const uint16_t* d, int64_t N, int64_t K, float* w) {
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      int q = (int)q2_code_of(wq[n * (K / 4) + k / 4], (int)(k % 4));
#ifdef ORACLE_PLANT_Q2_SCALE_BLOCK64
      float dd = oracle_f16_to_f32(d[n * (K / 128) + (k / 64) % (K / 128)]);
#else
      float dd = oracle_f16_to_f32(d[n * (K / 128) + k / 128]);
#endif
#if defined(ORACLE_PLANT_Q2_NO_OFFSET)
      w[n * K + k] = (float)q * dd;
#elif defined(ORACLE_PLANT_Q2_SIGN)
      w[n * K + k] = (float)(1 - q) * dd;
#else
      w[n * K + k] = (float)(q - 1) * dd;
#endif
    }
  }
}

/* ------------------------------------------------------------------------------------
 * 4-bit group format [P3-FB], [P2-WL]: code t of a row is (byte[t/2] >> ((t&1)*4)) & 0xF,
 * i.e. the even index in the low nibble; w = (q - z) * s, s and z per 64 weights.
 * ---------------------------------------------------------------------------------- */

static unsigned q4_code_of(uint8_t byte, int64_t t) {
#ifdef ORACLE_PLANT_Q4_NIBBLE_SWAP
  return (unsigned)(byte >> (((t & 1) ^ 1) * 4)) & 0xFu;
#else
  return (unsigned)(byte >> ((t & 1) * 4)) & 0xFu;
#endif
}

void oracle_q4_unpack(const uint8_t* wq, int64_t N, int64_t K, uint8_t* codes) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t t = 0; t < K; ++t)
      codes[n * K + t] = (uint8_t)q4_code_of(wq[n * (K / 2) + t / 2], t);
}

uint32_t oracle_q4_pack(const uint8_t* codes, const float* s, const float* z, int64_t N,
                        int64_t K, uint8_t* wq, uint16_t* sz) {
  uint32_t status = 0;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t i = 0; i < K / 2; ++i) {
      unsigned lo = codes[n * K + 2 * i], hi = codes[n * K + 2 * i + 1];
      if (lo > 15u || hi > 15u) status |= ORACLE_PACK_BAD_CODE;
#ifdef ORACLE_PLANT_Q4_NIBBLE_SWAP
      wq[n * (K / 2) + i] = (uint8_t)((hi & 0xFu) | ((lo & 0xFu) << 4));
#else
      wq[n * (K / 2) + i] = (uint8_t)((lo & 0xFu) | ((hi & 0xFu) << 4));
#endif
    }
    for (int64_t g = 0; g < K / 64; ++g) {
      float vs = s[n * (K / 64) + g], vz = z[n * (K / 64) + g];
      uint16_t hs = oracle_f32_to_f16_rne(vs), hz = oracle_f32_to_f16_rne(vz);
      if (!is_finite_f32(vs) || !is_finite_f32(vz)) status |= ORACLE_PACK_NONFINITE;
      else if (oracle_f16_to_f32(hs) != vs || oracle_f16_to_f32(hz) != vz)
        status |= ORACLE_PACK_INEXACT;
      sz[(n * (K / 64) + g) * 2 + 0] = hs;
      sz[(n * (K / 64) + g) * 2 + 1] = hz;
    }
  }
  return status;
}

void oracle_q4_dequant(const uint8_t* wq, const uint16_t* sz, int64_t N, int64_t K, float* w) {
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t t = 0; t < K; ++t) {
      float q = (float)q4_code_of(wq[n * (K / 2) + t / 2], t);
#ifdef ORACLE_PLANT_Q4_GROUP32
      int64_t g = (t / 32) % (K / 64); /* groups of 32 weights, kept inside the row */
#else
      int64_t g = t / 64;
#endif
      float sc = oracle_f16_to_f32(sz[(n * (K / 64) + g) * 2 + 0]);
      float ze = oracle_f16_to_f32(sz[(n * (K / 64) + g) * 2 + 1]);
#ifdef ORACLE_PLANT_Q4_ZERO_SIGN
      float diff = q + ze;
#else
      float diff = q - ze;
#endif
      w[n * K + t] = diff * sc;
    }
  }
}

/* ------------------------------------------------------------------------------------
 * The matmul: y = x . w^T, f64 accumulation in ascending k.
 * ---------------------------------------------------------------------------------- */

void oracle_gemm_f64(const uint16_t* x, const float* w, int64_t M, int64_t N, int64_t K,
                     double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
#ifdef ORACLE_PLANT_GEMM_TRANSPOSED
        /* reads w as if it were stored [K][N]; the mutation test uses N == K */
        double wv = (double)w[(N == K) ? (k * K + n) : (n * K + k)];
#else
        double wv = (double)w[n * K + k];
#endif
        acc += wv * (double)oracle_bf16_to_f32(x[m * K + k]);
      }
      y[m * N + n] = acc;
    }
  }
}

void oracle_lora_add_f64(const uint16_t* x, const uint16_t* a, const uint16_t* b, int64_t r,
                         int64_t M, int64_t N, int64_t K, double* y) {
#ifdef ORACLE_PLANT_LORA_DROPPED
  (void)x; (void)a; (void)b; (void)r; (void)M; (void)N; (void)K; (void)y;
#else
  /* u[m][i] = sum_k A[i][k] x[m][k], kept in f64 (never rounded) */
  double* u = (double*)malloc((size_t)(M * r) * sizeof(double));
  if (!u) return;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t i = 0; i < r; ++i) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k)
#ifdef ORACLE_PLANT_LORA_A_TRANSPOSED
        /* reads A as if it were stored [K][r]; the index stays inside the buffer */
        acc += (double)oracle_bf16_to_f32(a[k * r + i]) * (double)oracle_bf16_to_f32(x[m * K + k]);
#else
        acc += (double)oracle_bf16_to_f32(a[i * K + k]) * (double)oracle_bf16_to_f32(x[m * K + k]);
#endif
      u[m * r + i] = acc;
    }
  }
  /* y[m][n] += sum_i B[n][i] u[m][i] */
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0;
#ifdef ORACLE_PLANT_LORA_B_TRANSPOSED
      /* reads B as if it were stored [r][N]; the index stays inside the buffer */
      for (int64_t i = 0; i < r; ++i) acc += (double)oracle_bf16_to_f32(b[i * N + n]) * u[m * r + i];
#else
      for (int64_t i = 0; i < r; ++i) acc += (double)oracle_bf16_to_f32(b[n * r + i]) * u[m * r + i];
#endif
      y[m * N + n] += acc;
    }
  }
  free(u);
#endif
}

/* ------------------------------------------------------------------------------------
 * Composites.
 * ---------------------------------------------------------------------------------- */

void oracle_q2_gemm(const uint16_t* x, const uint8_t* wq, const uint16_t* d, int64_t M,
                    int64_t N, int64_t K, double* y) {
  float* w = (float*)malloc((size_t)(N * K) * sizeof(float));
  if (!w) return;
  oracle_q2_dequant(wq, d, N, K, w);
  oracle_gemm_f64(x, w, M, N, K, y);
  free(w);
}

void oracle_q2_lora_gemm(const uint16_t* x, const uint8_t* wq, const uint16_t* d,
                         const uint16_t* a, const uint16_t* b, int64_t r, int64_t M,
                         int64_t N, int64_t K, double* y) {
  oracle_q2_gemm(x, wq, d, M, N, K, y);
  oracle_lora_add_f64(x, a, b, r, M, N, K, y);
}

void oracle_q4_gemm(const uint16_t* x, const uint8_t* wq, const uint16_t* sz, int64_t M,
                    int64_t N, int64_t K, double* y) {
  float* w = (float*)malloc((size_t)(N * K) * sizeof(float));
  if (!w) return;
  oracle_q4_dequant(wq, sz, N, K, w);
  oracle_gemm_f64(x, w, M, N, K, y);
  free(w);
}

/* y = x1 W1^T + x2 W2^T [P2-GD]: the two products of a projection split along its input
 * axis, each computed on its own, then summed. */
void oracle_q2_dual_gemm(const uint16_t* x1, const uint8_t* wq1, const uint16_t* d1, int64_t K1,
                         const uint16_t* x2, const uint8_t* wq2, const uint16_t* d2, int64_t K2,
                         int64_t M, int64_t N, double* y) {
  double* y2 = (double*)malloc((size_t)(M * N) * sizeof(double));
  if (!y2) return;
  oracle_q2_gemm(x1, wq1, d1, M, N, K1, y);
  oracle_q2_gemm(x2, wq2, d2, M, N, K2, y2);
#ifndef ORACLE_PLANT_DUAL_SECOND_DROPPED
  for (int64_t i = 0; i < M * N; ++i) y[i] += y2[i];
#endif
  free(y2);
}

/* ------------------------------------------------------------------------------------
 * Sampled outputs: each requested y[m][n] computed on its own from the packed row n
 * (row slicing [P2-GD]: row n is the byte run wq[n*K/4 ...], scales d[n*K/128 ...]).
 * ---------------------------------------------------------------------------------- */

void oracle_q2_gemm_at(const uint16_t* x, const uint8_t* wq, const uint16_t* d,
                       const uint16_t* a, const uint16_t* b, int64_t r, int64_t M, int64_t N,
                       int64_t K, const int64_t* mi, const int64_t* ni, int64_t count,
                       double* out) {
  (void)M;
#pragma omp parallel
  {
    float* w = (float*)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
    for (int64_t s = 0; s < count; ++s) {
      int64_t m = mi[s], n = ni[s];
      if (w) oracle_q2_dequant(wq + n * (K / 4), d + n * (K / 128), 1, K, w);
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k)
        acc += (double)(w ? w[k] : 0.0f) * (double)oracle_bf16_to_f32(x[m * K + k]);
      if (a && b && r > 0) {
#ifndef ORACLE_PLANT_LORA_DROPPED
        double br = 0.0;
        for (int64_t i = 0; i < r; ++i) {
          double ui = 0.0;
          for (int64_t k = 0; k < K; ++k)
            ui += (double)oracle_bf16_to_f32(a[i * K + k]) * (double)oracle_bf16_to_f32(x[m * K + k]);
#ifdef ORACLE_PLANT_SAMPLED_B_TRANSPOSED
          /* the sampled path alone reads B as [r][N]; the index stays inside the buffer */
          br += (double)oracle_bf16_to_f32(b[i * N + n]) * ui;
#else
          br += (double)oracle_bf16_to_f32(b[n * r + i]) * ui;
#endif
        }
        acc += br;
#endif
      }
      out[s] = acc;
    }
    free(w);
  }
  (void)N;
}

void oracle_q2_dual_gemm_at(const uint16_t* x1, const uint8_t* wq1, const uint16_t* d1,
                            int64_t K1, const uint16_t* x2, const uint8_t* wq2,
                            const uint16_t* d2, int64_t K2, int64_t M, int64_t N,
                            const int64_t* mi, const int64_t* ni, int64_t count, double* out) {
  double* o2 = (double*)malloc((size_t)count * sizeof(double));
  if (!o2) return;
  oracle_q2_gemm_at(x1, wq1, d1, NULL, NULL, 0, M, N, K1, mi, ni, count, out);
  oracle_q2_gemm_at(x2, wq2, d2, NULL, NULL, 0, M, N, K2, mi, ni, count, o2);
#ifndef ORACLE_PLANT_DUAL_SECOND_DROPPED
  for (int64_t s = 0; s < count; ++s) out[s] += o2[s];
#endif
  free(o2);
}

void oracle_q4_gemm_at(const uint16_t* x, const uint8_t* wq, const uint16_t* sz, int64_t M,
                       int64_t N, int64_t K, const int64_t* mi, const int64_t* ni,
                       int64_t count, double* out) {
  (void)M; (void)N;
#pragma omp parallel
  {
    float* w = (float*)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
    for (int64_t s = 0; s < count; ++s) {
      int64_t m = mi[s], n = ni[s];
      if (w) oracle_q4_dequant(wq + n * (K / 2), sz + n * (K / 64) * 2, 1, K, w);
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k)
        acc += (double)(w ? w[k] : 0.0f) * (double)oracle_bf16_to_f32(x[m * K + k]);
      out[s] = acc;
    }
    free(w);
  }
}
