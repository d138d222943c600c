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
// The code must be E4M3_RNE(fl32(x / s)).  With r = RN(1/s) (s a normal float)
// and y = RN(x * r), |y - x/s| <= (2^-23 + 2^-48)|x/s| and fl32(x/s) is within
// 2^-24 |x/s| of x/s, so y and fl32(x/s) are at most ~3 ulps of y apart.  The
// E4M3 code changes only across a rounding midpoint, so whenever y is more
// than 16 ulps from every midpoint both round to the same code.  Otherwise
// (about 3e-5 of values) the exact IEEE quotient is used.
//
// Midpoints: for |y| >= 2^-6 the E4M3 grid keeps 3 fraction bits, so a midpoint
// is a binary32 whose 20 dropped bits equal 0x80000; below 2^-6 the grid is
// n * 2^-9 and the midpoints are (n + 1/2) * 2^-9.  Values that underflow in
// the product are far below 2^-10 and give +-0 either way (the sign of x is
// kept by the multiplication).
__device__ __forceinline__ bool e4m3_code_is_stable(float y) {
  const uint32_t b = __float_as_uint(y) & 0x7FFFFFFFu;
  if (b >= 0x3C800000u) {  // |y| >= 2^-6
    const int32_t rem = static_cast<int32_t>(b & 0xFFFFFu) - 0x80000;
    return rem > 16 || rem < -16;
  }
  const float t = __uint_as_float(b) * 512.0f;  // exact: grid -> integers
  return fabsf(t - truncf(t) - 0.5f) > (1.0f / 4096.0f);
}

// 8 values -> 8 E4M3 codes of fl32(x / s), packed little-endian in two words.
// `r` = RN(1/s); `exact_only` forces the division (scales that are not normal).
__device__ __forceinline__ uint2 quantize8(const float (&f)[8], float s, float r, bool exact_only) {
  float y[8];
  bool stable = !exact_only;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    y[i] = __fmul_rn(f[i], r);
    stable = stable && e4m3_code_is_stable(y[i]);
  }
  if (!stable) {
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = __fdiv_rn(f[i], s);
  }
  uint32_t p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = cvt_e4m3x2(y[2 * i], y[2 * i + 1]);
  return make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
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
      const float rc = __frcp_rn(sc);
      if (t < num_tiles) {
        q[t * 16 + sub] = quantize8(f, sc, rc, sc < kMinFastScale);
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
__global__ void __launch_bounds__(256) quant_w_128x128_kernel(const uint8_t* __restrict__ w, uint8_t* __restrict__ q,
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
    const float rc = __frcp_rn(sc);
    const bool exact_only = sc < kMinFastScale;
    uint8_t* dst = q + row0 * K + kb * 128;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      float f[8];
      bf16x8_to_float(v[p], f);
      *reinterpret_cast<uint2*>(dst + (p * 16 + rsub) * K + sub * 8) = quantize8(f, sc, rc, exact_only);
    }
    if (tid == 0) s[b] = sc;
    __syncthreads();  // warp_max is reused by the next block
  }
}

}  // namespace fp8q
