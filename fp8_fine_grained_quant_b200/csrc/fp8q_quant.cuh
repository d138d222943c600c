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
// per element): 16-byte non-allocating vector loads, several loads in flight
// per thread, amax by warp shuffles, IEEE division for s and x/s (no fast
// math, no flush-to-zero), and the hardware saturating RNE conversion to E4M3.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "fp8q_ptx.cuh"

namespace fp8q {

// 8 bf16 (one 16-byte vector) -> floats.  bf16 is the top half of a binary32.
__device__ __forceinline__ void bf16x8_to_float(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float abs_max8(const float (&f)[8]) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
  return m;
}

// s = fl32(amax / 448), 1 when zero.  __fdiv_rn is IEEE round-to-nearest.
__device__ __forceinline__ float group_scale(float amax) {
  float s = __fdiv_rn(amax, 448.0f);
  return s == 0.0f ? 1.0f : s;
}

// Division-free quantization with an exactness filter.
//
// The code must be E4M3_RNE(fl32(x / s)).  With r = RN(1/s) (s a normal
// float), r_lo = RN(r (1 - 2^-20)) and r_hi = RN(r (1 + 2^-20)):
//   x r_lo = (x/s)(1 - 2^-20)(1 + d), |d| <= 4 * 2^-24, so x r_lo < fl32(x/s)
//   (and symmetrically x r_hi > fl32(x/s)) for x > 0; the order flips for
//   x < 0.  So fl32(x/s) lies between the two products y_lo = RN(x r_lo) and
//   y_hi = RN(x r_hi).  Rounding to E4M3 is monotone, so when y_lo and y_hi get
//   the same code, fl32(x/s) gets that code too.  When they differ (a quotient
//   within ~2^-20 of a rounding midpoint, a few in 10^5) the IEEE quotient is
//   used.  Results below the binary32 normal range are far below the first
//   E4M3 midpoint (2^-10) and encode to +-0 on every path (the sign of x is
//   kept by each multiplication).
// 8 values -> 8 E4M3 codes of fl32(x / s), packed little-endian in two words.
// `exact_only` forces the division (scales that are not safely normal).
__device__ __forceinline__ uint2 quantize8(const float (&f)[8], float s, float r_lo, float r_hi, bool exact_only) {
  uint32_t lo[4], hi[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    lo[i] = cvt_e4m3x2(__fmul_rn(f[2 * i], r_lo), __fmul_rn(f[2 * i + 1], r_lo));
    hi[i] = cvt_e4m3x2(__fmul_rn(f[2 * i], r_hi), __fmul_rn(f[2 * i + 1], r_hi));
  }
  uint2 out = make_uint2(lo[0] | (lo[1] << 16), lo[2] | (lo[3] << 16));
  const uint2 chk = make_uint2(hi[0] | (hi[1] << 16), hi[2] | (hi[3] << 16));
  if (exact_only || out.x != chk.x || out.y != chk.y) {
    uint32_t p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = cvt_e4m3x2(__fdiv_rn(f[2 * i], s), __fdiv_rn(f[2 * i + 1], s));
    out = make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
  }
  return out;
}

// The two bracketing reciprocals of a group scale.
struct RecipPair {
  float lo, hi;
};
__device__ __forceinline__ RecipPair recip_pair(float s) {
  const float r = __frcp_rn(s);
  return {__fmul_rn(r, 1.0f - 0x1p-20f), __fmul_rn(r, 1.0f + 0x1p-20f)};
}

// Scales below this are not safely normal for the reciprocal path.
constexpr float kMinFastScale = 0x1p-125f;

// ---------------------------------------------------------------------------
// 1x128 activation tiles.  A tile is 128 bf16 = 256 contiguous bytes; a
// half-warp (16 lanes x 16 bytes) owns one tile per step, so a warp reads 512
// contiguous bytes per load.  Tile t = m * (K/128) + kb, which is also the
// index of its scale in s[M, K/128].  Each half-warp handles kUnroll tiles
// per iteration (loads issued together) in a grid-stride loop.
// ---------------------------------------------------------------------------
template <int kUnroll>
__global__ void __launch_bounds__(256) quant_act_1x128_kernel(const uint4* __restrict__ x, uint2* __restrict__ q,
                                                              float* __restrict__ s, int64_t num_tiles) {
  const int sub = threadIdx.x & 15;
  const int64_t hw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  const int64_t nhw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 4;
  for (int64_t t0 = hw; t0 - hw < num_tiles; t0 += nhw * kUnroll) {
    // Every lane runs the shuffles below (the two half-warps may differ in
    // validity at the tail), so out-of-range tiles load zeros instead.
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t t = t0 + u * nhw;
      v[u] = t < num_tiles ? ld_nc_v4(x + t * 16 + sub) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t t = t0 + u * nhw;
      float f[8];
      bf16x8_to_float(v[u], f);
      float amax = abs_max8(f);
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
      const float sc = group_scale(amax);
      const RecipPair rp = recip_pair(sc);
      if (t < num_tiles) {
        q[t * 16 + sub] = quantize8(f, sc, rp.lo, rp.hi, sc < kMinFastScale);
        if (sub == 0) s[t] = sc;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// 128x128 weight blocks.  One 256-thread CTA per block: 16 threads cover one
// 256-byte row segment, 16 rows per pass, 8 passes; the block (32 KB) stays in
// registers between the amax reduction and the quantization, so it is read
// from HBM once.  Block b = (g * N/128 + nb) * K/128 + kb, also the index of
// its scale in s[G, N/128, K/128].  Grid-stride over blocks.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256, 3) quant_w_128x128_kernel(const uint8_t* __restrict__ w, uint8_t* __restrict__ q,
                                                              float* __restrict__ s, int64_t N, int64_t K,
                                                              int64_t num_blocks) {
  __shared__ float warp_max[8];
  const int tid = threadIdx.x;
  const int sub = tid & 15;   // 16-byte column chunk within the 256-byte row segment
  const int rsub = tid >> 4;  // row within a pass of 16 rows
  const int64_t nkb = K >> 7, nnb = N >> 7;
  for (int64_t b = blockIdx.x; b < num_blocks; b += gridDim.x) {
    const int64_t kb = b % nkb;
    const int64_t gnb = b / nkb;  // g * nnb + nb
    const int64_t row0 = gnb * 128;  // row in the [G*N, K] view
    (void)nnb;
    const uint8_t* src = w + (row0 * K + kb * 128) * 2;
    uint4 v[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) v[p] = ld_nc_v4(src + ((p * 16 + rsub) * K) * 2 + sub * 16);
    float amax = 0.0f;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      float f[8];
      bf16x8_to_float(v[p], f);
      amax = fmaxf(amax, abs_max8(f));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    if ((tid & 31) == 0) warp_max[tid >> 5] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, warp_max[i]);
    const float sc = group_scale(amax);
    const RecipPair rp = recip_pair(sc);
    const bool exact_only = sc < kMinFastScale;
    uint8_t* dst = q + row0 * K + kb * 128;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      float f[8];
      bf16x8_to_float(v[p], f);
      *reinterpret_cast<uint2*>(dst + (p * 16 + rsub) * K + sub * 8) = quantize8(f, sc, rp.lo, rp.hi, exact_only);
    }
    if (tid == 0) s[b] = sc;
    __syncthreads();  // warp_max is reused by the next block
  }
}

}  // namespace fp8q
