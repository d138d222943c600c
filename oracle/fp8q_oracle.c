/*
 * fp8q_oracle.c -- plain, slow, obviously-correct CPU oracle for fine-grained
 * FP8 quantization and the block-scaled FP8 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * loads this file.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark may use it.  It shares no code, header, table or
 * constant with the CUDA implementation.
 *
 * Sources (web pages, cited by title and passage):
 *   [P1] "The Insider Secrets Of Deepseek Discovered" -- the FP8 mixed-precision
 *        passage: per-tensor amax scaling to the FP8 maximum; Figure 7 (a) 1x128
 *        activation tiles and 128x128 weight blocks; limited (~14-bit) tensor-core
 *        accumulation and promotion to CUDA cores at intervals, Figure 7 (b).
 *   [P2] "Deepgemm lancado no dia 4 da semana de codigo aberto Deepseek" --
 *        section "O que e FP8?", the figure description of E4M3 (1 sign, 4
 *        exponent, 3 mantissa bits; the bullet list above it gives E5M2) and
 *        "Necessidade de DeepGemm" (dense GEMM, MoE grouped GEMMs with
 *        contiguous and masked layouts).
 *   [P3] "DeepSeek-V3 FP8 precision" (codingmall knowledge base, Korean) --
 *        sections on fine-grained quantization, online quantization, increased
 *        accumulation precision and the unified E4M3 format.
 *
 * Readings taken where the pages are silent (each also listed in the design
 * notes): OCP E4M3FN (bias 7, max 448, no infinities, NaN = S.1111.111);
 * scale = fl32(amax / 448), replaced by 1 when it is zero; q = RNE_sat(fl32(x / s))
 * with IEEE single-precision division; saturation to +-448; E4M3 subnormals
 * down to 2^-9; the sign of a zero result is kept; promotion interval 128.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no -ffast-math:
 * IEEE division, no flush-to-zero).
 *
 * Every entry point returns 0 on success and a negative number on a bad
 * argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_TILE 128

/* ---------------------------------------------------------------------------
 * bf16 bit pattern -> float.  bf16 is the upper half of an IEEE binary32.
 * ------------------------------------------------------------------------- */
static float bf16_to_float(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* ---------------------------------------------------------------------------
 * E4M3 decode, from the 1-4-3 bit layout ([P2] "O que e FP8?"; [P3] unified
 * E4M3).  Exponent field E (bias 7), mantissa M:
 *   E == 0            : (-1)^S * (M / 8) * 2^-6          (subnormal)
 *   E == 15, M == 7   : NaN
 *   otherwise         : (-1)^S * (1 + M / 8) * 2^(E - 7)
 * ------------------------------------------------------------------------- */
double orc_e4m3_decode(uint8_t code) {
  int sign = code >> 7;
  int e = (code >> 3) & 0xF;
  int m = code & 0x7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, -6);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

void orc_e4m3_decode_table(double* out256) {
  for (int c = 0; c < 256; ++c) out256[c] = orc_e4m3_decode((uint8_t)c);
}

/* ---------------------------------------------------------------------------
 * E4M3 encode: round-to-nearest-even onto the E4M3 grid, saturating at +-448,
 * written as integer manipulation of the binary32 pattern.
 *
 * binary32 = S | 8-bit exponent X (bias 127) | 23-bit fraction.
 * E4M3 normal numbers cover [2^-6, 448]; with bias 7 the E4M3 exponent field
 * is X - 120.  Keeping the top 3 fraction bits drops 20 bits, which decide
 * the rounding.  Below 2^-6 the grid is n * 2^-9, n = 0..7.
 * ------------------------------------------------------------------------- */
uint8_t orc_e4m3_encode(float v) {
  uint32_t bits;
  memcpy(&bits, &v, sizeof bits);
  uint8_t sign = (uint8_t)((bits >> 24) & 0x80u);
  uint32_t mag = bits & 0x7FFFFFFFu;

  if (mag > 0x7F800000u) return 0x7F;          /* NaN */
  if (mag >= 0x43E00000u) return sign | 0x7E;  /* |v| >= 448 (incl. inf): saturate */

  uint32_t xexp = mag >> 23;
  if (xexp >= 121u) {
    /* normal E4M3 result (rounding may carry into the next binade, which the
       integer increment handles; it cannot pass 448 because mag < 448). */
    uint32_t keep = mag >> 20;           /* X:8 | top 3 fraction bits */
    uint32_t rest = mag & 0xFFFFFu;      /* 20 dropped bits */
    const uint32_t half = 0x80000u;
    if (rest > half || (rest == half && (keep & 1u))) keep += 1u;
    return sign | (uint8_t)(keep - (120u << 3));
  }
  if (xexp == 0u) return sign;           /* binary32 zero/subnormal: far below 2^-10 */

  /* subnormal E4M3 region: n = RNE(|v| * 2^9), |v| = sig * 2^(X - 150) */
  {
    uint32_t sig = (mag & 0x7FFFFFu) | 0x800000u;
    uint32_t shift = 141u - xexp;        /* >= 21 here */
    uint32_t n, rest, half;
    if (shift > 25u) return sign;        /* |v| < 2^-11: rounds to zero */
    n = sig >> shift;
    rest = sig & ((1u << shift) - 1u);
    half = 1u << (shift - 1u);
    if (rest > half || (rest == half && (n & 1u))) n += 1u;
    /* n == 8 is exactly 2^-6, whose encoding 0x08 equals n. */
    return sign | (uint8_t)n;
  }
}

/* ---------------------------------------------------------------------------
 * Online scale of one group.  [P1] describes the usual practice of mapping a
 * tensor's largest magnitude onto the largest FP8 value; Figure 7 (a) of [P1]
 * and the fine-grained / online quantization sections of [P3] apply that rule
 * to each group separately, from the group's current values:
 * s = fl32(amax / 448); s == 0 -> 1.
 * ------------------------------------------------------------------------- */
static float group_scale(float amax) {
  float s = amax / 448.0f;
  if (s == 0.0f) s = 1.0f;
  return s;
}

/* Activation quantization, 1x128 tiles: for row m and tile kb the group is
 * x[m, 128*kb .. 128*kb+127]: one scale for each token and each run of 128
 * channels ([P1] Figure 7 (a), item 1).  q is [M, K] E4M3 bytes, s is [M, K/128] float32. */
int orc_quant_act_1x128(const uint16_t* x, int64_t M, int64_t K, uint8_t* q, float* s) {
  if (M < 0 || K < 0 || K % ORC_TILE) return -1;
  const int64_t nkb = K / ORC_TILE;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t kb = 0; kb < nkb; ++kb) {
      const uint16_t* xt = x + m * K + kb * ORC_TILE;
      float amax = 0.0f;
      for (int j = 0; j < ORC_TILE; ++j) {
        float a = fabsf(bf16_to_float(xt[j]));
        if (a > amax) amax = a;
      }
      float sc = group_scale(amax);
      s[m * nkb + kb] = sc;
      for (int j = 0; j < ORC_TILE; ++j) q[m * K + kb * ORC_TILE + j] = orc_e4m3_encode(bf16_to_float(xt[j]) / sc);
    }
  }
  return 0;
}

/* Activation quantization along the token axis (128x1 tiles): x is [M, K]
 * (tokens x channels); the group of (mb, k) is column k, rows 128*mb..+127
 * (fewer in a ragged last block).  s is [ceil(M/128), K].  The backward
 * GEMM that contracts over tokens (Wgrad, [P1] Figure 6: Fprop, Dgrad and
 * Wgrad all in FP8) needs its operands grouped along the contraction, so the
 * 1x128 rule is applied to the transposed tensor; the pages do not spell
 * this layout out, it is the reading that keeps every scale constant within
 * a 128-deep slab of the contraction. */
int orc_quant_act_128x1(const uint16_t* x, int64_t M, int64_t K, uint8_t* q, float* s) {
  if (M < 0 || K < 0) return -1;
  const int64_t nmb = (M + ORC_TILE - 1) / ORC_TILE;
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < K; ++k) {
    for (int64_t mb = 0; mb < nmb; ++mb) {
      const int64_t m0 = mb * ORC_TILE, m1 = m0 + ORC_TILE < M ? m0 + ORC_TILE : M;
      float amax = 0.0f;
      for (int64_t m = m0; m < m1; ++m) {
        float a = fabsf(bf16_to_float(x[m * K + k]));
        if (a > amax) amax = a;
      }
      float sc = group_scale(amax);
      s[mb * K + k] = sc;
      for (int64_t m = m0; m < m1; ++m) q[m * K + k] = orc_e4m3_encode(bf16_to_float(x[m * K + k]) / sc);
    }
  }
  return 0;
}

/* Weight quantization, 128x128 blocks: w is [G, N, K] (K fastest, i.e. the
 * usual [out_features, in_features] layout, G = 1 for one matrix).  The group
 * of block (g, nb, kb) is rows 128*nb..+127 and columns 128*kb..+127: one
 * scale per 128 output channels x 128 input channels ([P1] Figure 7 (a),
 * item 2).
 * q is [G, N, K], s is [G, N/128, K/128]. */
int orc_quant_w_128x128(const uint16_t* w, int64_t G, int64_t N, int64_t K, uint8_t* q, float* s) {
  if (G < 0 || N < 0 || K < 0 || N % ORC_TILE || K % ORC_TILE) return -1;
  const int64_t nnb = N / ORC_TILE, nkb = K / ORC_TILE;
  const int64_t nblocks = G * nnb * nkb;
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < nblocks; ++b) {
    int64_t g = b / (nnb * nkb), nb = (b / nkb) % nnb, kb = b % nkb;
    const uint16_t* wb = w + g * N * K + nb * ORC_TILE * K + kb * ORC_TILE;
    uint8_t* qb = q + g * N * K + nb * ORC_TILE * K + kb * ORC_TILE;
    float amax = 0.0f;
    for (int r = 0; r < ORC_TILE; ++r)
      for (int j = 0; j < ORC_TILE; ++j) {
        float a = fabsf(bf16_to_float(wb[r * K + j]));
        if (a > amax) amax = a;
      }
    float sc = group_scale(amax);
    s[b] = sc; /* b == (g * nnb + nb) * nkb + kb */
    for (int r = 0; r < ORC_TILE; ++r)
      for (int j = 0; j < ORC_TILE; ++j) qb[r * K + j] = orc_e4m3_encode(bf16_to_float(wb[r * K + j]) / sc);
  }
  return 0;
}

/* Per-tensor quantization (the standard practice [P1] contrasts with the
 * fine-grained scheme): one scale for all n elements.  Used by the
 * accumulation-drift diagnostic and the scaling-accuracy study. */
int orc_quant_tensor(const uint16_t* x, int64_t n, uint8_t* q, float* s_out) {
  if (n < 0) return -1;
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    float a = fabsf(bf16_to_float(x[i]));
    if (a > amax) amax = a;
  }
  float sc = group_scale(amax);
  *s_out = sc;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) q[i] = orc_e4m3_encode(bf16_to_float(x[i]) / sc);
  return 0;
}

/* Power-of-two (UE8M0) group scales: the microscaling direction the first
 * page names for Blackwell ([P1], fine-grained quantization in step with
 * microscaling formats).  s = 2^e with e the smallest integer such that
 * 448 * 2^e >= amax (so |x / s| <= 448 and no code saturates), clamped to the
 * E8M0 range [-127, 127]; amax == 0 gives s = 1.  With amax = m 2^p,
 * m in [0.5, 1) (frexp), 448 = 0.875 * 2^9 gives e = p - 9 when m <= 0.875
 * and p - 8 otherwise.  Division by a power of two is exact, so the codes
 * are E4M3_RNE(x * 2^-e). */
static int ue8m0_exponent(float amax) {
  if (amax == 0.0f) return 0;
  int p;
  const float m = frexpf(amax, &p);
  int e = m <= 0.875f ? p - 9 : p - 8;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

int orc_quant_act_1x128_ue8m0(const uint16_t* x, int64_t M, int64_t K, uint8_t* q, float* s) {
  if (M < 0 || K < 0 || K % ORC_TILE) return -1;
  const int64_t nkb = K / ORC_TILE;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t kb = 0; kb < nkb; ++kb) {
      const uint16_t* xt = x + m * K + kb * ORC_TILE;
      float amax = 0.0f;
      for (int j = 0; j < ORC_TILE; ++j) {
        float a = fabsf(bf16_to_float(xt[j]));
        if (a > amax) amax = a;
      }
      const float sc = ldexpf(1.0f, ue8m0_exponent(amax));
      s[m * nkb + kb] = sc;
      for (int j = 0; j < ORC_TILE; ++j) q[m * K + kb * ORC_TILE + j] = orc_e4m3_encode(bf16_to_float(xt[j]) / sc);
    }
  }
  return 0;
}

int orc_quant_w_128x128_ue8m0(const uint16_t* w, int64_t G, int64_t N, int64_t K, uint8_t* q, float* s) {
  if (G < 0 || N < 0 || K < 0 || N % ORC_TILE || K % ORC_TILE) return -1;
  const int64_t nnb = N / ORC_TILE, nkb = K / ORC_TILE;
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < G * nnb * nkb; ++b) {
    const int64_t kb = b % nkb, gnb = b / nkb;
    const uint16_t* wb = w + gnb * ORC_TILE * K + kb * ORC_TILE;
    uint8_t* qb = q + gnb * ORC_TILE * K + kb * ORC_TILE;
    float amax = 0.0f;
    for (int r = 0; r < ORC_TILE; ++r)
      for (int j = 0; j < ORC_TILE; ++j) {
        float a = fabsf(bf16_to_float(wb[r * K + j]));
        if (a > amax) amax = a;
      }
    const float sc = ldexpf(1.0f, ue8m0_exponent(amax));
    s[b] = sc;
    for (int r = 0; r < ORC_TILE; ++r)
      for (int j = 0; j < ORC_TILE; ++j) qb[r * K + j] = orc_e4m3_encode(bf16_to_float(wb[r * K + j]) / sc);
  }
  return 0;
}

/* Quantization with a given scale (delayed scaling, which the codingmall page
 * contrasts with online scaling: the scale comes from earlier iterations'
 * maxima, so values beyond 448 * s saturate at +-448).  Used only by the
 * scaling-accuracy study. */
int orc_quant_with_scale(const uint16_t* x, int64_t n, float s, uint8_t* q) {
  if (n < 0 || !(s > 0.0f)) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) q[i] = orc_e4m3_encode(bf16_to_float(x[i]) / s);
  return 0;
}

/* Round a double to the nearest bf16 (ties to even) in one step, without an
 * intermediate float (which could round twice).  Finite inputs only; values
 * beyond the bf16 range become +-inf. */
static uint16_t double_to_bf16_rne(double v) {
  if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
  const uint16_t sign = v < 0 ? 0x8000 : 0x0000;
  double a = fabs(v);
  int e;
  (void)frexp(a, &e);  /* a = m 2^e, m in [0.5, 1) */
  /* bf16 normal: 8 significant bits (1 + 7), exponents 2^-126 .. 2^127 */
  int ulp_exp = e - 8;      /* weight of the last kept bit for a normal */
  if (e - 1 < -126) ulp_exp = -126 - 7;  /* subnormal spacing 2^-133 */
  double q = ldexp(a, -ulp_exp);  /* value in units of the last kept bit (exact) */
  double r = floor(q);
  double frac = q - r;
  if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) == 1.0)) r += 1.0;
  double y = ldexp(r, ulp_exp);
  if (y > 3.3895313892515355e38) return sign | 0x7F80;  /* overflow: inf */
  float f = (float)y;  /* exact: y has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return sign | (uint16_t)(u >> 16);
}

/* A double array rounded once to bf16 bit patterns (RNE). */
void orc_round_bf16(const double* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16_rne(v[i]);
}

/* SwiGLU between the two MoE GEMMs (not on the pages: the configurations'
 * GEMM1 width N = 4096 = 2 x 2048 = GEMM2's K implies it): c1 holds
 * [gate | up] halves of each row, h = silu(gate) * up with silu(g) =
 * g / (1 + exp(-g)), computed in double from the bf16 inputs and rounded once
 * to bf16.  rows x (2 inter) in, rows x inter out. */
int orc_swiglu_bf16(const uint16_t* c1, int64_t rows, int64_t inter, uint16_t* h) {
  if (rows < 0 || inter < 0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t i = 0; i < inter; ++i) {
      const double g = bf16_to_float(c1[r * 2 * inter + i]);
      const double u = bf16_to_float(c1[r * 2 * inter + inter + i]);
      h[r * inter + i] = double_to_bf16_rne(g / (1.0 + exp(-g)) * u);
    }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Block-scaled GEMM, C = A * B^T with per-slab promotion ([P1] Figure 7 (b);
 * [P3] increased accumulation precision):
 *   C[m,n] = sum_kb sa[m,kb] * sb[n/128,kb] * sum_{k in slab kb} dA[m,k] * dB[n,k]
 * where dA, dB are the decoded E4M3 values.  Each slab sum is exact in double
 * (every product has <= 8 significant bits and lies in [2^-18, 2^18]; 128 of
 * them need < 53 bits), so the only roundings are the three-factor products
 * and the outer sum: the result is the dequantized-input product to ~1e-16.
 * ------------------------------------------------------------------------- */
static void gemm_one_row(const uint8_t* qa_row, const float* sa_row, const uint8_t* qb, const float* sb, int64_t N,
                         int64_t K, const double* dec, double* c_row) {
  const int64_t nkb = K / ORC_TILE;
  for (int64_t n = 0; n < N; ++n) {
    const uint8_t* qb_row = qb + n * K;
    const float* sb_row = sb + (n / ORC_TILE) * nkb;
    double acc = 0.0;
    for (int64_t kb = 0; kb < nkb; ++kb) {
      double part = 0.0;
      for (int64_t k = kb * ORC_TILE; k < (kb + 1) * ORC_TILE; ++k) part += dec[qa_row[k]] * dec[qb_row[k]];
      acc += (double)sa_row[kb] * (double)sb_row[kb] * part;
    }
    c_row[n] = acc;
  }
}

/* Dense: qa [M,K], sa [M,K/128], qb [N,K], sb [N/128,K/128].
 * rows == NULL: all M rows, C is [M,N].  Otherwise C is [nrows,N] holding
 * rows[0..nrows). */
int orc_gemm_blockscaled(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb, int64_t M, int64_t N,
                         int64_t K, const int64_t* rows, int64_t nrows, double* C) {
  if (M < 0 || N < 0 || K < 0 || N % ORC_TILE || K % ORC_TILE) return -1;
  double dec[256];
  orc_e4m3_decode_table(dec);
  const int64_t nkb = K / ORC_TILE;
  const int64_t count = rows ? nrows : M;
  for (int64_t i = 0; i < count; ++i)
    if (rows && (rows[i] < 0 || rows[i] >= M)) return -2;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < count; ++i) {
    int64_t m = rows ? rows[i] : i;
    gemm_one_row(qa + m * K, sa + m * nkb, qb, sb, N, K, dec, C + i * N);
  }
  return 0;
}

/* Both operands scaled per row and per 128-deep slab ("1D x 1D"): qa [M,K]
 * with sa [M,K/128], qb [N,K] with sb [N,K/128]:
 *   C[m,n] = sum_kb sa[m,kb] * sb[n,kb] * sum_{k in slab kb} dA[m,k] * dB[n,k]
 * This is the weight-gradient GEMM once both of its operands are grouped
 * along the token axis (each token-slab of a channel has its own scale).
 * Exact per slab in double, like orc_gemm_blockscaled. */
int orc_gemm_1d1d(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb, int64_t M, int64_t N,
                  int64_t K, const int64_t* rows, int64_t nrows, double* C) {
  if (M < 0 || N < 0 || K < 0 || K % ORC_TILE) return -1;
  double dec[256];
  orc_e4m3_decode_table(dec);
  const int64_t nkb = K / ORC_TILE;
  const int64_t count = rows ? nrows : M;
  for (int64_t i = 0; i < count; ++i)
    if (rows && (rows[i] < 0 || rows[i] >= M)) return -2;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < count; ++i) {
    const int64_t m = rows ? rows[i] : i;
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t kb = 0; kb < nkb; ++kb) {
        double part = 0.0;
        for (int64_t k = kb * ORC_TILE; k < (kb + 1) * ORC_TILE; ++k) part += dec[qa[m * K + k]] * dec[qb[n * K + k]];
        acc += (double)sa[m * nkb + kb] * (double)sb[n * nkb + kb] * part;
      }
      C[i * N + n] = acc;
    }
  }
  return 0;
}

/* Grouped, contiguous layout ([P2], the MoE grouped GEMM kinds): rows of all experts
 * are concatenated; every 128-row block b belongs to expert m_indices[b] and
 * is multiplied by that expert's weights qb[e] ([E,N,K]) with scales sb[e]
 * ([E,N/128,K/128]).  Blocks whose index lies outside [0,E) produce no output
 * (their C rows are left as they are).  rows: as for the dense call. */
int orc_grouped_contiguous(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb,
                           const int32_t* m_indices, int64_t M_tot, int64_t N, int64_t K, int64_t E,
                           const int64_t* rows, int64_t nrows, double* C) {
  if (M_tot < 0 || N < 0 || K < 0 || E < 0 || M_tot % ORC_TILE || N % ORC_TILE || K % ORC_TILE) return -1;
  double dec[256];
  orc_e4m3_decode_table(dec);
  const int64_t nkb = K / ORC_TILE, nnb = N / ORC_TILE;
  const int64_t count = rows ? nrows : M_tot;
  for (int64_t i = 0; i < count; ++i)
    if (rows && (rows[i] < 0 || rows[i] >= M_tot)) return -2;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < count; ++i) {
    int64_t m = rows ? rows[i] : i;
    int64_t e = m_indices[m / ORC_TILE];
    if (e < 0 || e >= E) continue;
    gemm_one_row(qa + m * K, sa + m * nkb, qb + e * N * K, sb + e * nnb * nkb, N, K, dec, C + i * N);
  }
  return 0;
}

/* Grouped, masked layout ([P2], the MoE grouped GEMM kinds): expert e owns rows
 * qa[e, 0..cap) of which only the first masked_m[e] are valid.  C is
 * [E,cap,N]; rows at or beyond masked_m[e] are left as they are.
 * rows (optional) are flat indices e*cap + m into [E*cap); with rows given,
 * C is [nrows, N] and invalid rows are left as they are. */
int orc_grouped_masked(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb,
                       const int32_t* masked_m, int64_t E, int64_t cap, int64_t N, int64_t K, const int64_t* rows,
                       int64_t nrows, double* C) {
  if (E < 0 || cap < 0 || N < 0 || K < 0 || N % ORC_TILE || K % ORC_TILE) return -1;
  double dec[256];
  orc_e4m3_decode_table(dec);
  const int64_t nkb = K / ORC_TILE, nnb = N / ORC_TILE;
  const int64_t count = rows ? nrows : E * cap;
  for (int64_t i = 0; i < count; ++i)
    if (rows && (rows[i] < 0 || rows[i] >= E * cap)) return -2;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < count; ++i) {
    int64_t r = rows ? rows[i] : i;
    int64_t e = r / cap, m = r % cap;
    if (m >= masked_m[e]) continue;
    gemm_one_row(qa + r * K, sa + r * nkb, qb + e * N * K, sb + e * nnb * nkb, N, K, dec, C + i * N);
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Limited-precision accumulation (the drift demonstration of [P1]: tensor
 * cores keep ~14 bits while accumulating; promotion to FP32 at intervals
 * repairs it, Figure 7 (b)).
 *
 * Model (a reading; the pages fix neither the width's meaning nor the
 * rounding): products are summed exactly in groups of `group` consecutive k
 * (one tensor-core instruction's worth); each group sum is added to the
 * running accumulator and the result is truncated toward zero to `p_bits`
 * significant bits.  Every `interval` values of k (a multiple of 128, or 0 =
 * all of K) the limited accumulator is scaled by that interval's scales,
 * added to a double-precision accumulator, and restarted at zero.
 * Within one interval all 128-slabs must carry the same scales (true for the
 * per-tensor inputs this is meant for); otherwise the call returns -3.
 * ------------------------------------------------------------------------- */
static double round_toward_zero_bits(double x, int p) {
  int e;
  if (x == 0.0 || !isfinite(x)) return x;
  frexp(x, &e); /* |x| = f * 2^e with f in [0.5, 1) */
  return trunc(ldexp(x, p - e)) * ldexp(1.0, e - p);
}

int orc_gemm_limited_acc(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb, int64_t M, int64_t N,
                         int64_t K, int p_bits, int64_t group, int64_t interval, const int64_t* rows, int64_t nrows,
                         double* C) {
  if (M < 0 || N < 0 || K <= 0 || N % ORC_TILE || K % ORC_TILE) return -1;
  if (p_bits < 1 || p_bits > 53 || group < 1 || ORC_TILE % group) return -1;
  if (interval == 0) interval = K;
  if (interval % ORC_TILE || K % interval) return -1;
  const int64_t nkb = K / ORC_TILE, spi = interval / ORC_TILE;
  const int64_t count = rows ? nrows : M;
  double dec[256];
  orc_e4m3_decode_table(dec);
  for (int64_t i = 0; i < count; ++i)
    if (rows && (rows[i] < 0 || rows[i] >= M)) return -2;
  /* uniform-scale check inside every interval */
  for (int64_t i = 0; i < count; ++i) {
    int64_t m = rows ? rows[i] : i;
    for (int64_t kb = 0; kb < nkb; ++kb)
      if (sa[m * nkb + kb] != sa[m * nkb + (kb / spi) * spi]) return -3;
  }
  for (int64_t nb = 0; nb < N / ORC_TILE; ++nb)
    for (int64_t kb = 0; kb < nkb; ++kb)
      if (sb[nb * nkb + kb] != sb[nb * nkb + (kb / spi) * spi]) return -3;

#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < count; ++i) {
    int64_t m = rows ? rows[i] : i;
    for (int64_t n = 0; n < N; ++n) {
      double hi = 0.0;
      for (int64_t k0 = 0; k0 < K; k0 += interval) {
        double lim = 0.0;
        for (int64_t g0 = k0; g0 < k0 + interval; g0 += group) {
          double t = 0.0;
          for (int64_t k = g0; k < g0 + group; ++k) t += dec[qa[m * K + k]] * dec[qb[n * K + k]];
          lim = round_toward_zero_bits(lim + t, p_bits);
        }
        int64_t kb = k0 / ORC_TILE;
        hi += (double)sa[m * nkb + kb] * (double)sb[(n / ORC_TILE) * nkb + kb] * lim;
      }
      C[i * N + n] = hi;
    }
  }
  return 0;
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Array form of the encoder (used by tests to compare many values at once). */
void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}
