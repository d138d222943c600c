// fp8q_quant.cuh -- online fine-grained E4M3 quantizers.
//
// Method: "The Insider Secrets Of Deepseek Discovered", FP8 mixed-precision
// passage, Figure 7 (a): activations get one scale per 1x128 tile (a token's
// run of 128 channels), weights one per 128x128 block; the scale maps the
// group's largest magnitude onto the largest E4M3 value (448).  The codingmall
// DeepSeek-V3 FP8 page (online quantization) fixes that the scale comes from
// the current values, with no history.
//
// Both kernels are HBM-bound streams (2 bytes read, 1 byte + scales written
// per element).  A lane owns 16 consecutive elements (one 256-bit
// non-allocating load, one 128-bit store of codes); eight lanes cover a
// 128-element row segment, so a warp reads 1 KB per load instruction.  The
// group amax is a warp-shuffle reduction (plus shared memory across the warps
// of a weight block); s = fl32(amax / 448) and the codes of fl32(x / s) are
// computed exactly without a division on the common path (below), and the
// hardware's saturating round-to-nearest-even conversion produces the codes.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "fp8q_ptx.cuh"

namespace fp8q {

// fl32(1 / 448).
constexpr float kInv448 = 0x1.24924ap-9f;

// s = fl32(amax / 448), or 1 when amax == 0.
//
// amax is a bf16 magnitude (8 significant bits).  q0 = RN(amax * RN(1/448))
// is within an ulp of the quotient; the FMA residual r = amax - 448 q0 is
// exact, and q0 + r RN(1/448), rounded once, is the correctly rounded
// quotient for every non-negative finite bf16 amax (checked exhaustively
// against the exact quotient, subnormal results included).  Non-finite
// inputs are outside the quantizers' contract.
__device__ __forceinline__ float group_scale(float amax) {
  const float q0 = __fmul_rn(amax, kInv448);
  const float r = __fmaf_rn(-q0, 448.0f, amax);
  const float s = __fmaf_rn(r, kInv448, q0);
  return s == 0.0f ? 1.0f : s;
}

// Division-free codes with an exactness filter.
//
// Each code must be E4M3_RNE(fl32(x / s)).  Given r_lo < 1/s < r_hi, for
// x > 0, x r_lo < x/s < x r_hi (reversed for x < 0), and by the monotonicity
// of rounding RN(x r_lo) <= fl32(x/s) <= RN(x r_hi).  Rounding to E4M3 is
// monotone too, so when the two products get the same code, fl32(x/s) gets
// that code.  When they differ (a quotient within ~2^-20 of an E4M3 rounding
// midpoint) that element's code comes from the IEEE quotient.  Products below
// the binary32 normal range are far below the first E4M3 midpoint (2^-10) and
// give +-0 on every path (each product keeps the sign of x).
//
// With bf16 data such quotients are not rare: x and amax both carry 8-bit
// significands, and 448 x / amax lands exactly on an E4M3 midpoint for about
// 0.5% of the elements of normally distributed data.  So most warps meet one
// in every step, but a lane seldom meets more than one: the fallback
// recomputes single elements, not the lane's whole run.
//
// The bracket comes from the hardware's approximate reciprocal r ~ 1/s
// (s a normal float), widened to r_lo = RN(r (1 - 2^-20)) and r_hi =
// RN(r (1 + 2^-20)).  Whether it really brackets 1/s is then checked exactly:
// fma(-s, r_lo, 1) is 1 - s r_lo rounded once, which keeps the sign of the
// exact residual, so it is > 0 exactly when r_lo < 1/s (and < 0 for r_hi
// exactly when r_hi > 1/s).  A bracket that fails the check sends its group
// to the division path, so the codes never depend on how accurate the
// approximate reciprocal is.
__device__ __forceinline__ bool recip_bracket(float s, float& lo, float& hi) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
  lo = __fmul_rn(r, 1.0f - 0x1p-20f);
  hi = __fmul_rn(r, 1.0f + 0x1p-20f);
  return __fmaf_rn(-s, lo, 1.0f) > 0.0f && __fmaf_rn(-s, hi, 1.0f) < 0.0f;
}

struct RecipPair {
  uint64_t lo2, hi2;  // {r_lo, r_lo} and {r_hi, r_hi}
  bool ok;            // the bracket holds (else: the division path)
};
__device__ __forceinline__ RecipPair recip_pair(float s) {
  float lo, hi;
  const bool ok = recip_bracket(s, lo, hi);
  return {pack_f32x2(lo), pack_f32x2(hi), ok};
}

// Scales below this are not safely normal for the reciprocal path.
constexpr float kMinFastScale = 0x1p-125f;

// The exact path: codes of the IEEE quotients fl32(x / s) for the 16 bf16 in
// w.  Out of line, so the rarely taken branch adds no work to the common path.
__device__ __noinline__ uint4 quantize16_exact(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, uint32_t w4,
                                               uint32_t w5, uint32_t w6, uint32_t w7, float s) {
  const uint32_t w[8] = {w0, w1, w2, w3, w4, w5, w6, w7};
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a0 = __fdiv_rn(__uint_as_float(w[2 * i] << 16), s);
    const float a1 = __fdiv_rn(__uint_as_float(w[2 * i] & 0xFFFF0000u), s);
    const float a2 = __fdiv_rn(__uint_as_float(w[2 * i + 1] << 16), s);
    const float a3 = __fdiv_rn(__uint_as_float(w[2 * i + 1] & 0xFFFF0000u), s);
    c[i] = cvt_e4m3x2(a0, a1) | (cvt_e4m3x2(a2, a3) << 16);
  }
  return make_uint4(c[0], c[1], c[2], c[3]);
}

// Bit 8j + 7 of the result is set when byte j of d is nonzero (the low seven
// bits of a byte plus 0x7F carry into its top bit, never into the next byte).
__device__ __forceinline__ uint32_t nonzero_bytes(uint32_t d) {
  return (((d & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | d) & 0x80808080u;
}

// The bf16 element j (0..3) of a code word's two source words: byte j of a
// word of four codes comes from word j / 2, half j % 2 (low half first).
__device__ __forceinline__ float bf16_of_pair(uint32_t w_even, uint32_t w_odd, int j) {
  const uint32_t word = (j & 2) ? w_odd : w_even;
  return __uint_as_float((j & 1) ? (word & 0xFFFF0000u) : (word << 16));
}

// Replaces byte j of c by the E4M3 code of fl32(x / s).
__device__ __forceinline__ uint32_t with_exact_code(uint32_t c, int j, float x, float s) {
  const uint32_t code = cvt_e4m3x2(__fdiv_rn(x, s), 0.0f) & 0xFFu;
  const int sh = 8 * j;
  return (c & ~(0xFFu << sh)) | (code << sh);
}

// 16 bf16 (eight words) -> 16 E4M3 codes of fl32(x / s), low byte first.
// `exact_only` forces the division (scales that are not safely normal).
__device__ __forceinline__ uint4 quantize16(const uint32_t (&w)[8], float s, const RecipPair& rp, bool exact_only) {
  if (exact_only || !rp.ok) return quantize16_exact(w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7], s);
  uint32_t lo[4], hi[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint64_t x0 = bf16x2_to_f32x2(w[2 * i]);
    const uint64_t x1 = bf16x2_to_f32x2(w[2 * i + 1]);
    lo[i] = e4m3x4_from_f32x2(mul_f32x2(x0, rp.lo2), mul_f32x2(x1, rp.lo2));
    hi[i] = e4m3x4_from_f32x2(mul_f32x2(x0, rp.hi2), mul_f32x2(x1, rp.hi2));
  }
  // elements whose bracket codes differ: the IEEE quotient, one at a time
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    for (uint32_t m = nonzero_bytes(lo[i] ^ hi[i]); m != 0u; m &= m - 1u) {
      const int j = (__ffs(m) - 1) >> 3;
      lo[i] = with_exact_code(lo[i], j, bf16_of_pair(w[2 * i], w[2 * i + 1], j), s);
    }
  }
  return make_uint4(lo[0], lo[1], lo[2], lo[3]);
}

// Largest magnitude of the 16 bf16 in w, as a float: packed bf16 maxima of
// the magnitudes (sign bits cleared; exact, no rounding), then the larger
// half widened to binary32.
__device__ __forceinline__ float abs_max16(const uint32_t (&w)[8]) {
  uint32_t m[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = max_bf16x2(w[2 * i] & 0x7FFF7FFFu, w[2 * i + 1] & 0x7FFF7FFFu);
  const uint32_t a = max_bf16x2(max_bf16x2(m[0], m[1]), max_bf16x2(m[2], m[3]));
  return fmaxf(__uint_as_float(a & 0xFFFF0000u), __uint_as_float(a << 16));
}

__device__ __forceinline__ void zero8(uint32_t (&w)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = 0u;
}

// Power-of-two (UE8M0) group scales, the microscaling form the first page
// names for Blackwell: s = 2^e with e the least integer such that
// 448 * 2^e >= amax (so no code saturates), clamped to E8M0's [-127, 127];
// amax == 0 gives 1.  With amax = 1.f * 2^(E-127) (E the biased exponent),
// 448 = 1.75 * 2^8 gives e = E - 135 when 1.f <= 1.75 and E - 134 otherwise;
// a subnormal amax clamps to e = -127.  Returns 2^-e (the exact multiplier).
__device__ __forceinline__ float pow2_scale(float amax, float* inv) {
  const uint32_t b = __float_as_uint(amax);
  const int E = static_cast<int>(b >> 23);
  int e = E == 0 ? -127 : ((b & 0x7FFFFFu) <= 0x600000u ? E - 135 : E - 134);
  if (amax == 0.0f) e = 0;
  e = e < -127 ? -127 : (e > 127 ? 127 : e);
  *inv = e <= 126 ? __uint_as_float(static_cast<uint32_t>(127 - e) << 23) : 0x1p-127f;  // 2^-e
  return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23) : 0x1p-127f;
}

// 16 bf16 -> 16 codes of x * 2^-e (exact products: one conversion each).
__device__ __forceinline__ uint4 quantize16_pow2(const uint32_t (&w)[8], float inv) {
  const uint64_t inv2 = pack_f32x2(inv);
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    c[i] = e4m3x4_from_f32x2(mul_f32x2(bf16x2_to_f32x2(w[2 * i]), inv2), mul_f32x2(bf16x2_to_f32x2(w[2 * i + 1]), inv2));
  return make_uint4(c[0], c[1], c[2], c[3]);
}

// ---------------------------------------------------------------------------
// 1x128 activation tiles.  A tile is 128 bf16 = 256 contiguous bytes; eight
// lanes (32 bytes each) own one tile per step, so a warp covers four tiles.
// Tile t = m * (K/128) + kb, which is also the index of its scale in
// s[M, K/128].  Each lane group handles kUnroll tiles per iteration (loads
// issued together) in a grid-stride loop; five CTAs fit per SM.
// ---------------------------------------------------------------------------
template <int kUnroll, bool kPow2>
__global__ void __launch_bounds__(256, 5) quant_act_1x128_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ q,
                                                              float* __restrict__ s, int64_t num_tiles) {
  const int sub = threadIdx.x & 7;
  const int64_t grp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 3;
  const int64_t ngrp = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 3;
  // The trip count is the same for every lane of a warp (the shuffles below
  // need all 32); tiles past the end load zeros and store nothing.
  for (int64_t t0 = grp; t0 - grp < num_tiles; t0 += ngrp * kUnroll) {
    uint32_t v[kUnroll][8];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t t = t0 + u * ngrp;
      if (t < num_tiles)
        ld_nc_v8(x + t * 256 + sub * 32, v[u]);
      else
        zero8(v[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t t = t0 + u * ngrp;
      float amax = abs_max16(v[u]);
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
      if constexpr (kPow2) {
        float inv;
        const float sc = pow2_scale(amax, &inv);
        if (t < num_tiles) {
          *reinterpret_cast<uint4*>(q + t * 128 + sub * 16) = quantize16_pow2(v[u], inv);
          if (sub == 0) s[t] = sc;
        }
      } else {
        const float sc = group_scale(amax);
        const RecipPair rp = recip_pair(sc);
        if (t < num_tiles) {
          *reinterpret_cast<uint4*>(q + t * 128 + sub * 16) = quantize16(v[u], sc, rp, sc < kMinFastScale);
          if (sub == 0) s[t] = sc;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// 128x128 weight blocks.  One 256-thread CTA per block: eight lanes cover one
// 256-byte row segment, 32 rows per pass, 4 passes; the block (32 KB) stays in
// registers between the amax reduction and the quantization, so it is read
// from HBM once (four CTAs per SM, 59 registers).  Block b = (g * N/128 + nb)
// * K/128 + kb, also the index of its scale in s[G, N/128, K/128].
// `warp_max` is 8 floats of shared memory; consecutive blocks of one CTA
// alternate between two such halves, so one CTA barrier per block suffices.
// ---------------------------------------------------------------------------
template <bool kPow2>
__device__ __forceinline__ void quant_w_block(const uint8_t* __restrict__ w, uint8_t* __restrict__ q,
                                              float* __restrict__ s, int64_t K, int64_t b, float* warp_max) {
  const int tid = threadIdx.x;
  const int sub = tid & 7;    // 32-byte chunk within the 256-byte row segment
  const int rsub = tid >> 3;  // row within a pass of 32 rows
  const int64_t nkb = K >> 7;
  const int64_t kb = b % nkb;
  const int64_t row0 = (b / nkb) * 128;  // first row in the [G*N, K] view
  const uint8_t* src = w + (row0 * K + kb * 128) * 2 + sub * 32;
  uint32_t v[4][8];
#pragma unroll
  for (int p = 0; p < 4; ++p) ld_nc_v8(src + (p * 32 + rsub) * K * 2, v[p]);
  float amax = 0.0f;
#pragma unroll
  for (int p = 0; p < 4; ++p) amax = fmaxf(amax, abs_max16(v[p]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  if ((tid & 31) == 0) warp_max[tid >> 5] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, warp_max[i]);
  uint8_t* dst = q + row0 * K + kb * 128 + sub * 16;
  float sc;
  if constexpr (kPow2) {
    float inv;
    sc = pow2_scale(amax, &inv);
#pragma unroll
    for (int p = 0; p < 4; ++p) *reinterpret_cast<uint4*>(dst + (p * 32 + rsub) * K) = quantize16_pow2(v[p], inv);
  } else {
    sc = group_scale(amax);
    const RecipPair rp = recip_pair(sc);
    const bool exact_only = sc < kMinFastScale;
#pragma unroll
    for (int p = 0; p < 4; ++p)
      *reinterpret_cast<uint4*>(dst + (p * 32 + rsub) * K) = quantize16(v[p], sc, rp, exact_only);
  }
  if (tid == 0) s[b] = sc;
}

// Grid-stride over weight blocks.
template <bool kPow2>
__global__ void __launch_bounds__(256, 4) quant_w_128x128_kernel(const uint8_t* __restrict__ w,
                                                                 uint8_t* __restrict__ q, float* __restrict__ s,
                                                                 int64_t K, int64_t num_blocks) {
  __shared__ float warp_max[2][8];
  int half = 0;
  for (int64_t b = blockIdx.x; b < num_blocks; b += gridDim.x, half ^= 1)
    quant_w_block<kPow2>(w, q, s, K, b, warp_max[half]);
}

// ---------------------------------------------------------------------------
// Both operands of a GEMM in one launch: the 1x128 activation quantization
// and the 128x128 weight quantization, the same codes and scales as the two
// kernels above, bit for bit.  Every CTA quantizes one 32 KB unit: CTAs
// below `act_ctas` take 128 consecutive activation tiles (four per lane
// group, all loaded before any is reduced), the others one weight block.
// One launch instead of two: the ramp-up and the last partial wave are paid
// once, and the two streams share the device.
// ---------------------------------------------------------------------------
constexpr int kActTilesPerCta = 128;

__global__ void __launch_bounds__(256, 4) quant_act_w_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ qa,
                                                             float* __restrict__ sa, int64_t num_tiles,
                                                             int64_t act_ctas, const uint8_t* __restrict__ w,
                                                             uint8_t* __restrict__ qw, float* __restrict__ sw,
                                                             int64_t Kw) {
  __shared__ float warp_max[8];
  if (static_cast<int64_t>(blockIdx.x) >= act_ctas) {
    quant_w_block<false>(w, qw, sw, Kw, static_cast<int64_t>(blockIdx.x) - act_ctas, warp_max);
    return;
  }
  const int sub = threadIdx.x & 7;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kActTilesPerCta + (threadIdx.x >> 3);
  constexpr int kPer = kActTilesPerCta / 32;  // tiles per lane group
  uint32_t v[kPer][8];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int64_t t = t0 + u * 32;
    if (t < num_tiles)
      ld_nc_v8(x + t * 256 + sub * 32, v[u]);
    else
      zero8(v[u]);
  }
  // every lane runs every step (the shuffles need all 32); tiles past the end store nothing
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int64_t t = t0 + u * 32;
    float amax = abs_max16(v[u]);
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    const float sc = group_scale(amax);
    const RecipPair rp = recip_pair(sc);
    if (t < num_tiles) {
      *reinterpret_cast<uint4*>(qa + t * 128 + sub * 16) = quantize16(v[u], sc, rp, sc < kMinFastScale);
      if (sub == 0) sa[t] = sc;
    }
  }
}

// ---------------------------------------------------------------------------
// Token-axis tiles (128x1) for the weight-gradient GEMM, which contracts over
// tokens: the group of (mb, k) is channel k over tokens 128*mb..+127 (fewer in
// a ragged last block).  A 256-thread CTA quantizes one 128-token x
// 128-channel block at a time: thread t owns channels 8*(t%16)..+7 of tokens
// 8*(t/16)..+7.  The per-channel amax is reduced over the 16 token groups (a
// shuffle, then shared memory across the 8 warps); each channel's codes use
// its own scale, with the same exact division-free filter as the other
// quantizers.  s is [ceil(M/128), K].
//
// The kernel is persistent: a CTA takes blocks at a stride of the grid, and
// while it quantizes one block the next two blocks' bf16 (32 KB each) are
// being copied into the other stages of a three-stage shared buffer (16-byte
// cp.async per thread through the L2), so every CTA keeps loads in flight; a
// block read straight into registers would leave the memory system idle while
// its codes are computed.
// ---------------------------------------------------------------------------

// Codes of fl32(x / s_c) for the 8 bf16 in w (4 words; element i uses column
// scale sc[i]) by IEEE division: the exact path.
__device__ __noinline__ uint2 quantize8_cols_exact(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float s0,
                                                   float s1, float s2, float s3, float s4, float s5, float s6,
                                                   float s7) {
  const uint32_t w[4] = {w0, w1, w2, w3};
  const float sc[8] = {s0, s1, s2, s3, s4, s5, s6, s7};
  uint32_t c[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float a0 = __fdiv_rn(__uint_as_float(w[2 * h] << 16), sc[4 * h]);
    const float a1 = __fdiv_rn(__uint_as_float(w[2 * h] & 0xFFFF0000u), sc[4 * h + 1]);
    const float a2 = __fdiv_rn(__uint_as_float(w[2 * h + 1] << 16), sc[4 * h + 2]);
    const float a3 = __fdiv_rn(__uint_as_float(w[2 * h + 1] & 0xFFFF0000u), sc[4 * h + 3]);
    c[h] = cvt_e4m3x2(a0, a1) | (cvt_e4m3x2(a2, a3) << 16);
  }
  return make_uint2(c[0], c[1]);
}

// 4x4 byte transpose: w[i] holds row i (byte j = column j); afterwards w[j]
// holds column j (byte i = row i).
__device__ __forceinline__ void transpose4x4_bytes(uint32_t& w0, uint32_t& w1, uint32_t& w2, uint32_t& w3) {
  const uint32_t x0 = __byte_perm(w0, w2, 0x5410), x2 = __byte_perm(w0, w2, 0x7632);
  const uint32_t x1 = __byte_perm(w1, w3, 0x5410), x3 = __byte_perm(w1, w3, 0x7632);
  w0 = __byte_perm(x0, x1, 0x6240);
  w1 = __byte_perm(x0, x1, 0x7351);
  w2 = __byte_perm(x2, x3, 0x6240);
  w3 = __byte_perm(x2, x3, 0x7351);
}

// 8x8 byte transpose of rows (lo[r]: bytes 0-3, hi[r]: bytes 4-7): as 2x2
// blocks of 4x4, [[A, B], [C, D]]^T = [[A^T, C^T], [B^T, D^T]].
__device__ __forceinline__ void transpose8x8_bytes(uint32_t (&lo)[8], uint32_t (&hi)[8]) {
  transpose4x4_bytes(lo[0], lo[1], lo[2], lo[3]);  // A
  transpose4x4_bytes(lo[4], lo[5], lo[6], lo[7]);  // C
  transpose4x4_bytes(hi[0], hi[1], hi[2], hi[3]);  // B
  transpose4x4_bytes(hi[4], hi[5], hi[6], hi[7]);  // D
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t b = hi[i];  // B^T row i becomes row 4 + i, low half
    hi[i] = lo[4 + i];         // C^T row i: row i, high half
    lo[4 + i] = b;
  }
}

// One 128-token x 128-channel block of bf16, as staged in shared memory
// ([token][channel], 256 bytes per token), and the stages of a CTA: while one
// is quantized the next two are being filled.
constexpr int kTokBlockBytes = 128 * 128 * 2;
constexpr int kTokStages = 3;
constexpr int kTokSmemBytes = kTokStages * kTokBlockBytes;
// CTAs per SM the kernel is fitted to: 128 registers, 100 KB of shared memory each.
constexpr int kTokCtasPerSm = 2;

// kTokenContiguous = false: codes q [M, K], laid out like x.
//
// kTokenContiguous = true: the weight gradient dW = dY^T X, written as
// C = A * B^T, contracts over tokens: A = dY^T [N, Mp] and B = X^T [K, Mp],
// each row carrying one scale per 128-token slab.  The codes are then written
// transposed, q = qt [K, Mp] for a padded token count Mp >= M (a multiple of
// 128); tokens past M get code 0 and whole padding groups scale 1.  The scales
// s [Mp/128, K] are the slab-major layout the GEMM stages.  A thread's 8x8
// code bytes are transposed in registers (byte permutes) and written to a
// [channel][token] tile in the block's spent stage, whose 8-byte slots are
// XOR-swizzled by channel / 8 (two wavefronts per warp store); each channel
// row then leaves as eight coalesced 16-byte stores.
//
// Blocks are numbered b = mb * (K/128) + kc over Mp/128 token blocks (Mp =
// 128 * ceil(M/128) for the row-major form).
template <bool kTokenContiguous>
__global__ void __launch_bounds__(256, kTokCtasPerSm) quant_act_128x1_kernel(const uint8_t* __restrict__ x,
                                                                             uint8_t* __restrict__ q,
                                                                             float* __restrict__ s, int64_t M,
                                                                             int64_t K, int64_t Mp,
                                                                             int64_t num_blocks) {
  extern __shared__ __align__(128) uint8_t stage_buf[];  // [kTokStages][128 tokens][256 bytes]
  __shared__ __align__(16) uint32_t col_max[8][16][4];   // [warp][channel group][word]: bf16 maxima, packed
  // per channel of the block: scale, bracketing reciprocals, whether its codes take the division path
  __shared__ __align__(16) float ch_scale[128];
  __shared__ __align__(16) float ch_rlo[128];
  __shared__ __align__(16) float ch_rhi[128];
  __shared__ __align__(8) uint8_t ch_exact[128];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cg = tid & 15, rg = tid >> 4;
  // block b = mb * nkc + kc; a CTA's blocks are gridDim.x apart, i.e. step_mb
  // token blocks and step_kc channel blocks (with a carry)
  const int nkc = static_cast<int>(K >> 7);
  const int step_mb = static_cast<int>(gridDim.x) / nkc, step_kc = static_cast<int>(gridDim.x) % nkc;
  auto advance = [&](int& mb, int& kc) {
    kc += step_kc;
    mb += step_mb;
    if (kc >= nkc) {
      kc -= nkc;
      ++mb;
    }
  };
  // Copies of block (mb, kc) into stage st: 16-byte chunk c = tid + 256 i is
  // token c / 16, channels 8 (c % 16) .. +7, so a warp copies two 256-byte
  // token rows per instruction.  Tokens past M are zero-filled (nothing is read).
  auto fetch = [&](int mb, int kc, int st) {
    const uint32_t dst = smem_u32(stage_buf + st * kTokBlockBytes);
    const uint8_t* src = x + static_cast<int64_t>(kc) * 256;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = tid + 256 * i, row = c >> 4, ch = c & 15;
      const int64_t grow = static_cast<int64_t>(mb) * 128 + row;
      const bool in = grow < M;
      cp_async_16(dst + row * 256 + ch * 16, in ? src + grow * K * 2 + ch * 16 : x, in ? 16u : 0u);
    }
  };
  // the CTA's i-th block b = blockIdx.x + i * gridDim.x lives in stage i % kTokStages;
  // (fmb, fkc) is the next block to copy, fb its number
  int fmb = static_cast<int>(blockIdx.x) / nkc, fkc = static_cast<int>(blockIdx.x) % nkc;
  int64_t fb = blockIdx.x;
#pragma unroll
  for (int j = 0; j < kTokStages - 1; ++j) {
    if (fb < num_blocks) fetch(fmb, fkc, j);
    cp_async_commit();
    fb += gridDim.x;
    advance(fmb, fkc);
  }
  int st = 0, mb = static_cast<int>(blockIdx.x) / nkc, kc = static_cast<int>(blockIdx.x) % nkc;
  for (int64_t b = blockIdx.x; b < num_blocks;
       b += gridDim.x, advance(mb, kc), st = st + 1 == kTokStages ? 0 : st + 1) {
    // refill the stage the previous block used (every thread is past it: the
    // barrier at the end of the previous iteration)
    if (fb < num_blocks) fetch(fmb, fkc, st == 0 ? kTokStages - 1 : st - 1);
    cp_async_commit();
    fb += gridDim.x;
    advance(fmb, fkc);
    cp_async_wait<kTokStages - 1>();  // this block's copies have landed; the later blocks' may be in flight
    __syncthreads();                  // ... every thread's
    const int64_t col0 = static_cast<int64_t>(kc) * 128 + cg * 8;
    const int64_t row0 = static_cast<int64_t>(mb) * 128 + rg * 8;
    uint8_t* buf = stage_buf + st * kTokBlockBytes;
    // this thread's 8 tokens x 8 channels (a warp reads two 256-byte rows per load)
    uint4 v[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) v[r] = *reinterpret_cast<const uint4*>(buf + (rg * 8 + r) * 256 + cg * 16);
    // per-channel maxima of |x| over this thread's 8 tokens, as packed bf16 pairs
    // (word i: channels 2i and 2i + 1; a maximum of bf16 values is exact)
    uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      m[0] = max_bf16x2(m[0], v[r].x & 0x7FFF7FFFu);
      m[1] = max_bf16x2(m[1], v[r].y & 0x7FFF7FFFu);
      m[2] = max_bf16x2(m[2], v[r].z & 0x7FFF7FFFu);
      m[3] = max_bf16x2(m[3], v[r].w & 0x7FFF7FFFu);
    }
    // lanes l and l ^ 16 hold the same channels (two token groups of the warp)
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = max_bf16x2(m[i], __shfl_xor_sync(0xFFFFFFFFu, m[i], 16));
    if (lane < 16) *reinterpret_cast<uint4*>(&col_max[warp][cg][0]) = make_uint4(m[0], m[1], m[2], m[3]);
    __syncthreads();  // col_max is complete, and the stage has been read by every thread
    // one thread per channel: its amax over the 8 warps, scale and bracket, once for the block
    if (tid < 128) {
      uint32_t a = 0u;
#pragma unroll
      for (int w = 0; w < 8; ++w) a = max_bf16x2(a, col_max[w][tid >> 3][(tid & 7) >> 1]);
      const float amax = __uint_as_float((tid & 1) ? (a & 0xFFFF0000u) : (a << 16));
      const float sc = group_scale(amax);
      float lo, hi;
      const bool ok = recip_bracket(sc, lo, hi);
      ch_scale[tid] = sc;
      ch_rlo[tid] = lo;
      ch_rhi[tid] = hi;
      ch_exact[tid] = static_cast<uint8_t>(sc < kMinFastScale || !ok);
      s[mb * K + static_cast<int64_t>(kc) * 128 + tid] = sc;
    }
    __syncthreads();
    // this thread's 8 channels' bracketing reciprocals, paired as the packed products need them
    uint64_t lo2[4], hi2[4];
    {
      const float4 l0 = *reinterpret_cast<const float4*>(&ch_rlo[cg * 8]);
      const float4 l1 = *reinterpret_cast<const float4*>(&ch_rlo[cg * 8 + 4]);
      const float4 h0 = *reinterpret_cast<const float4*>(&ch_rhi[cg * 8]);
      const float4 h1 = *reinterpret_cast<const float4*>(&ch_rhi[cg * 8 + 4]);
      asm("mov.b64 %0, {%1, %2};" : "=l"(lo2[0]) : "f"(l0.x), "f"(l0.y));
      asm("mov.b64 %0, {%1, %2};" : "=l"(lo2[1]) : "f"(l0.z), "f"(l0.w));
      asm("mov.b64 %0, {%1, %2};" : "=l"(lo2[2]) : "f"(l1.x), "f"(l1.y));
      asm("mov.b64 %0, {%1, %2};" : "=l"(lo2[3]) : "f"(l1.z), "f"(l1.w));
      asm("mov.b64 %0, {%1, %2};" : "=l"(hi2[0]) : "f"(h0.x), "f"(h0.y));
      asm("mov.b64 %0, {%1, %2};" : "=l"(hi2[1]) : "f"(h0.z), "f"(h0.w));
      asm("mov.b64 %0, {%1, %2};" : "=l"(hi2[2]) : "f"(h1.x), "f"(h1.y));
      asm("mov.b64 %0, {%1, %2};" : "=l"(hi2[3]) : "f"(h1.z), "f"(h1.w));
    }
    const uint2 ex = *reinterpret_cast<const uint2*>(&ch_exact[cg * 8]);
    const bool exact_only = (ex.x | ex.y) != 0u;
    const float* my_scale = &ch_scale[cg * 8];
    // codes of the 8 tokens (zero tokens past M give code 0)
    uint32_t clo[8], chi[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const uint32_t w[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
      uint32_t lo[2], hi[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint64_t x0 = bf16x2_to_f32x2(w[2 * h]), x1 = bf16x2_to_f32x2(w[2 * h + 1]);
        lo[h] = e4m3x4_from_f32x2(mul_f32x2(x0, lo2[2 * h]), mul_f32x2(x1, lo2[2 * h + 1]));
        hi[h] = e4m3x4_from_f32x2(mul_f32x2(x0, hi2[2 * h]), mul_f32x2(x1, hi2[2 * h + 1]));
      }
      if (exact_only) {
        const uint2 out = quantize8_cols_exact(w[0], w[1], w[2], w[3], my_scale[0], my_scale[1], my_scale[2],
                                               my_scale[3], my_scale[4], my_scale[5], my_scale[6], my_scale[7]);
        lo[0] = out.x;
        lo[1] = out.y;
      } else {
        // elements whose bracket codes differ: the IEEE quotient, one at a time
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          for (uint32_t mk = nonzero_bytes(lo[h] ^ hi[h]); mk != 0u; mk &= mk - 1u) {
            const int j = (__ffs(mk) - 1) >> 3;
            lo[h] = with_exact_code(lo[h], j, bf16_of_pair(w[2 * h], w[2 * h + 1], j), my_scale[4 * h + j]);
          }
        }
      }
      clo[r] = lo[0];
      chi[r] = lo[1];
    }
    if constexpr (kTokenContiguous) {
      transpose8x8_bytes(clo, chi);  // now channel c: tokens 0-3 in clo[c], 4-7 in chi[c]
      // channel row cg*8 + c of the tile, logical 8-byte slot rg, physical slot rg ^ cg
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint2*>(buf + (cg * 8 + c) * 128 + ((rg ^ cg) << 3)) = make_uint2(clo[c], chi[c]);
      __syncthreads();
      uint8_t* dst = q + (static_cast<int64_t>(kc) * 128) * Mp + static_cast<int64_t>(mb) * 128;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = tid + 256 * i, row = c >> 3, ch = c & 7;
        const int swz = row >> 3;  // the row's channel group, 0..15
        // logical slots 2ch, 2ch+1 sit in physical 16-byte chunk ch ^ (swz / 2),
        // their halves swapped when swz is odd
        uint4 o = *reinterpret_cast<const uint4*>(buf + row * 128 + ((ch ^ (swz >> 1)) << 4));
        if (swz & 1) o = make_uint4(o.z, o.w, o.x, o.y);
        *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(row) * Mp + ch * 16) = o;
      }
    } else {
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int64_t row = row0 + r;
        if (row < M) *reinterpret_cast<uint2*>(q + row * K + col0) = make_uint2(clo[r], chi[r]);
      }
    }
    __syncthreads();  // col_max, and this stage (refilled by the next iteration's copies), are reused
  }
  cp_async_wait<0>();  // only empty groups can be pending here
}

// ---------------------------------------------------------------------------
// Transposition of 128x128-block-quantized weights: codes [G, N, K] -> [G, K, N]
// and block scales [G, N/128, K/128] -> [G, K/128, N/128].  A 128x128 block of
// W^T is the transpose of W's block (same amax, same scale, the same codes),
// so the forward GEMM on the transposed codes computes dY * W (the
// activation-gradient GEMM).
//
// One 256-thread CTA per block.  The 16 KB block is read with coalesced
// 16-byte loads (eight lanes per 128-byte row) into a shared tile whose
// 8-byte slots are XOR-swizzled by row group (slot s of row R sits at
// s ^ (R / 8)); thread (l = t % 16, j = t / 16) then takes the 8x8 bytes at
// rows 8l.., columns 8j.. (eight 8-byte shared loads, one wavefront per half
// warp), transposes them in registers and stores eight 8-byte pieces at rows
// 8j.., columns 8l.. of the output: each warp store writes two full 128-byte
// rows.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) transpose_w_128x128_kernel(const uint8_t* __restrict__ qw,
                                                                  const float* __restrict__ sw,
                                                                  uint8_t* __restrict__ qt, float* __restrict__ st,
                                                                  int64_t N, int64_t K, int64_t num_blocks) {
  __shared__ __align__(16) uint8_t tile[128 * 128];
  const int tid = threadIdx.x;
  const int l = tid & 15, j = tid >> 4;
  const int64_t nkb = K >> 7, nnb = N >> 7;
  for (int64_t b = blockIdx.x; b < num_blocks; b += gridDim.x) {
    const int64_t g = b / (nnb * nkb), rem = b % (nnb * nkb);
    const int64_t nb = rem / nkb, kb = rem % nkb;
    const uint8_t* src = qw + (g * N + nb * 128) * K + kb * 128;
    // rows tid / 8 + 32 i, 16-byte chunk tid % 8 (slots 2c, 2c + 1)
    uint4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = (tid >> 3) + 32 * i, c = tid & 7;
      v[i] = ld_nc_v4(src + static_cast<int64_t>(row) * K + c * 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = (tid >> 3) + 32 * i, c = tid & 7, x = (row >> 3) & 15;
      *reinterpret_cast<uint2*>(tile + row * 128 + (((2 * c) ^ x) << 3)) = make_uint2(v[i].x, v[i].y);
      *reinterpret_cast<uint2*>(tile + row * 128 + (((2 * c + 1) ^ x) << 3)) = make_uint2(v[i].z, v[i].w);
    }
    __syncthreads();
    uint32_t lo[8], hi[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int row = 8 * l + r;  // row group l
      const uint2 w = *reinterpret_cast<const uint2*>(tile + row * 128 + ((j ^ l) << 3));
      lo[r] = w.x;
      hi[r] = w.y;
    }
    __syncthreads();  // the tile is reused by the next block
    transpose8x8_bytes(lo, hi);  // lo[c], hi[c]: column 8j + c, rows 8l .. 8l + 7
    uint8_t* dst = qt + (g * K + kb * 128 + 8 * j) * N + nb * 128 + 8 * l;
#pragma unroll
    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint2*>(dst + static_cast<int64_t>(c) * N) = make_uint2(lo[c], hi[c]);
    if (tid == 0) st[(g * nkb + kb) * nnb + nb] = sw[(g * nnb + nb) * nkb + kb];
  }
}

// ---------------------------------------------------------------------------
// SwiGLU between the two MoE GEMMs, fused with the 1x128 requantization of its
// output.  Each row of GEMM1's bf16 output is [gate | up] (inter columns each);
// the next GEMM's activation is h = silu(gate) * up, silu(g) = g / (1 +
// exp(-g)), rounded once to bf16, then quantized per 1x128 tile exactly as
// quant_act_1x128_kernel does.  (The SwiGLU is not on the pages: the MoE
// configurations' GEMM1 width, twice GEMM2's depth, implies it.)
//
// h is the correctly rounded bf16 of the expression.  The FP32 evaluation
// (expf within 2 ulp, the quotient by div.full.f32 within 2 ulp, one rounded
// add and one rounded multiply: relative error below 2.5 * 2^-22) is
// bracketed by h (1 -+ 2^-20); when both ends round to the same bf16, that is
// the result (rounding is monotone).  Otherwise -- a value within ~2^-20 of a
// bf16 rounding midpoint, or outside the range where the bound holds -- the
// expression is evaluated in double and rounded to bf16 through round-to-odd
// FP32 (16 spare bits, so the two steps round once).  The FP32 evaluation and
// the bracket are branch-free; the elements the bracket leaves open (about one
// in 2^11) are redone afterwards.
// ---------------------------------------------------------------------------
__device__ __noinline__ uint32_t swiglu_bf16_exact(float g, float u) {
  const double hd = static_cast<double>(g) / (1.0 + exp(-static_cast<double>(g))) * static_cast<double>(u);
  float f = __double2float_rz(hd);
  if (isfinite(hd) && static_cast<double>(f) != hd) f = __uint_as_float(__float_as_uint(f) | 1u);
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// a / b within 2 ulp for all finite a, b (PTX div.full.f32): no branch.
__device__ __forceinline__ float div_full(float a, float b) {
  float r;
  asm("div.full.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// Two floats rounded to nearest-even bf16, packed (lo in the low half).
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// FP32 g / (1 + exp(-g)) * u; `ok` when exp did not overflow and |h| lies in
// [2^-100, 2^120], where the relative error bound holds.
__device__ __forceinline__ float swiglu_f32(float g, float u, bool& ok) {
  const float e = expf(-g);
  const float h = __fmul_rn(div_full(g, __fadd_rn(1.0f, e)), u);
  const float a = fabsf(h);
  ok = e <= 0x1.fffffep+127f && a >= 0x1p-100f && a <= 0x1p+120f;
  return h;
}

// Eight words of bf16 pairs (gate) and (up) -> eight words of bf16 pairs of h.
// gp, up: where gw and uw were loaded from; the rare redo path reads its
// word there again rather than keeping all sixteen words live.
__device__ __forceinline__ void swiglu16(const uint32_t (&gw)[8], const uint32_t (&uw)[8], uint32_t (&hw)[8],
                                         const uint8_t* gp, const uint8_t* up) {
  uint32_t redo = 0u;  // bit 2i + j: the half j of word i is left open by its bracket
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    bool ok0, ok1;
    const float h0 = swiglu_f32(__uint_as_float(gw[i] << 16), __uint_as_float(uw[i] << 16), ok0);
    const float h1 = swiglu_f32(__uint_as_float(gw[i] & 0xFFFF0000u), __uint_as_float(uw[i] & 0xFFFF0000u), ok1);
    const uint32_t lo = bf16x2_rn(__fmul_rn(h0, 1.0f - 0x1p-20f), __fmul_rn(h1, 1.0f - 0x1p-20f));
    const uint32_t hi = bf16x2_rn(__fmul_rn(h0, 1.0f + 0x1p-20f), __fmul_rn(h1, 1.0f + 0x1p-20f));
    hw[i] = lo;
    const uint32_t d = lo ^ hi;
    redo |= static_cast<uint32_t>(!ok0 || (d & 0xFFFFu) != 0u) << (2 * i);
    redo |= static_cast<uint32_t>(!ok1 || (d >> 16) != 0u) << (2 * i + 1);
  }
  for (; redo != 0u; redo &= redo - 1u) {
    const int b = __ffs(redo) - 1, i = b >> 1;
    const uint32_t g = __ldg(reinterpret_cast<const uint32_t*>(gp) + i);
    const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(up) + i);
    if (b & 1) {
      const uint32_t x = swiglu_bf16_exact(__uint_as_float(g & 0xFFFF0000u), __uint_as_float(u & 0xFFFF0000u));
#pragma unroll
      for (int k = 0; k < 8; ++k) hw[k] = i == k ? (hw[k] & 0xFFFFu) | (x << 16) : hw[k];
    } else {
      const uint32_t x = swiglu_bf16_exact(__uint_as_float(g << 16), __uint_as_float(u << 16));
#pragma unroll
      for (int k = 0; k < 8; ++k) hw[k] = i == k ? (hw[k] & 0xFFFF0000u) | x : hw[k];
    }
  }
}

// c1 [rows, 2 * inter] bf16 -> qh [rows, inter] E4M3 codes, sh [rows, inter/128]
// scales.  Tile t = row * (inter/128) + kb, as in quant_act_1x128_kernel.  With
// masked_m, row = e * cap + r is valid when r < clamp(masked_m[e], 0, cap);
// other rows are neither read nor written.
__global__ void __launch_bounds__(256, 5) swiglu_quant_1x128_kernel(const uint8_t* __restrict__ c1,
                                                                    uint8_t* __restrict__ qh, float* __restrict__ sh,
                                                                    int64_t inter, int64_t num_tiles,
                                                                    const int32_t* __restrict__ masked_m,
                                                                    int64_t cap) {
  const int sub = threadIdx.x & 7;
  const int64_t grp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 3;
  const int64_t ngrp = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 3;
  const int64_t per_row = inter >> 7;
  // same trip count for every lane of a warp (the shuffles need all 32)
  for (int64_t t = grp; t - grp < num_tiles; t += ngrp) {
    bool valid = t < num_tiles;
    const int64_t row = valid ? t / per_row : 0, kb = valid ? t - row * per_row : 0;
    if (valid && masked_m != nullptr) {
      const int64_t e = row / cap;
      int64_t m = masked_m[e];
      m = m < 0 ? 0 : (m > cap ? cap : m);
      valid = row - e * cap < m;
    }
    uint32_t hw[8];
    if (valid) {
      uint32_t gw[8], uw[8];
      const uint8_t* src = c1 + ((row * 2 * inter) + kb * 128 + sub * 16) * 2;
      ld_nc_v8(src, gw);
      ld_nc_v8(src + inter * 2, uw);
      swiglu16(gw, uw, hw, src, src + inter * 2);
    } else {
      zero8(hw);
    }
    float amax = abs_max16(hw);
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    const float sc = group_scale(amax);
    const RecipPair rp = recip_pair(sc);
    if (valid) {
      *reinterpret_cast<uint4*>(qh + t * 128 + sub * 16) = quantize16(hw, sc, rp, sc < kMinFastScale);
      if (sub == 0) sh[t] = sc;
    }
  }
}

}  // namespace fp8q
