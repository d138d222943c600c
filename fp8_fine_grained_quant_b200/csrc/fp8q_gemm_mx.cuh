// fp8q_gemm_mx.cuh -- block-scaled FP8 GEMM with power-of-two (UE8M0)
// scales applied by the tensor cores (tcgen05.mma.kind::mxf8f6f4.block_scale).
//
// Method: the microscaling variant of the fine-grained scheme ("The Insider
// Secrets Of Deepseek Discovered", FP8 passage: Blackwell's tensor cores take
// per-group scales in hardware).  With power-of-two scales (the _ue8m0
// quantizers: one 2^e per 1x128 activation tile and per 128x128 weight block)
// the tensor cores scale each 32-element block of A's rows and B's rows by
// 2^(sf - 127), so the whole K accumulates in one TMEM accumulator and the
// epilogue only converts it to bf16 -- no per-slab promotion on the CUDA
// cores.  Each 128-deep slab's four K = 32 steps share one scale per row.
//
// Scale factors in TMEM: per slab, a 128-row x 4-block atom of E8M0 bytes for
// A and one for B (512 bytes each), staged to shared memory by bulk copies
// with the slab's operands, then copied to TMEM by the MMA thread
// (tcgen05.cp 32x128b.warpx4): TMEM lane l, column c holds rows l + 32 c of
// the tile, byte j the scale of K block j.  The MMA's scale-factor id j picks
// the byte.  tcgen05.cp and tcgen05.mma of one thread execute in order, so
// the same eight TMEM columns serve every slab.
//
// Global scale layout (written by mx_scales_*_kernel): atoms [tile][slab][512]
// with byte 16 m0 + 4 m1 + j = the scale of tile row 32 m1 + m0 (all four j
// equal here).
#pragma once

#include "fp8q_gemm.cuh"

namespace fp8q {

constexpr int kMxStages = 6;
constexpr uint32_t kMxAtomBytes = 512;

// Scheduling, output and status as for the promoted GEMM (GemmArgs: the
// dense, contiguous and masked layouts, get_tile); the scale atoms instead of
// f32 scales.
struct MxArgs {
  GemmArgs g;
  const uint8_t* sfa;   // [rows of A / 128][nkb][512] E8M0
  const uint8_t* sfb;   // [E*N/128][nkb][512] E8M0
};

struct MxSmem {
  static constexpr uint32_t kABytes = kBlockM * kSlabK;  // 16 KB
  static constexpr uint32_t kBBytes = 128 * kSlabK;      // 16 KB (BN = 128)
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffB = kMxStages * kABytes;
  static constexpr uint32_t kOffSf = kMxStages * kStageBytes;              // per stage: SFA atom, SFB atom
  static constexpr uint32_t kOffBars = kOffSf + kMxStages * 2 * kMxAtomBytes;
  // full[S], empty[S], tfull[2], tempty[2], drain
  static constexpr uint32_t kNumBars = 2 * kMxStages + 2 + 2 + 1;
  static constexpr uint32_t kOffMisc = kOffBars + 8 * kNumBars;  // tmem slot, abort flag, total tiles
  static constexpr uint32_t kOffPrefix = (kOffMisc + 16 + 15) / 16 * 16;  // masked layout: tile prefix
  static constexpr uint32_t kBytes = kOffPrefix + 4 * (kMaxMaskedExperts + 1);
  static constexpr uint32_t kDynamicBytes = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;    // 2 accumulators x 128 + scale factors
  static constexpr uint32_t kTmemSfa = 256;     // 4 columns
  static constexpr uint32_t kTmemSfb = 260;     // 4 columns
  static_assert(kDynamicBytes <= 227u * 1024u, "shared memory per CTA");
};

struct MxBars {
  uint32_t base;
  __device__ uint32_t full(int s) const { return base + 8u * s; }
  __device__ uint32_t empty(int s) const { return base + 8u * (kMxStages + s); }
  __device__ uint32_t tfull(int b) const { return base + 8u * (2 * kMxStages + b); }
  __device__ uint32_t tempty(int b) const { return base + 8u * (2 * kMxStages + 2 + b); }
  __device__ uint32_t drain() const { return base + 8u * (2 * kMxStages + 4); }
};

template <Sched S>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_mx_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                   const MxArgs args) {
  using L = MxSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const MxBars bars{s_base + L::kOffBars};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  int32_t* total_slot = reinterpret_cast<int32_t*>(smem + L::kOffMisc + 8);
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + L::kOffPrefix);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const GemmArgs& ga = args.g;
  const WaitCtl wc{ga.timeout_ns, ga.status, abort_flag};
  const int nkb = ga.nkb;

  if (threadIdx.x == 0) {
    for (int st = 0; st < kMxStages; ++st) {
      mbar_init(bars.full(st), 1);
      mbar_init(bars.empty(st), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bars.tfull(b), 1);
      mbar_init(bars.tempty(b), 8);  // one arrival per epilogue warp
    }
    mbar_init(bars.drain(), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tma_a);
    tma_prefetch_map(&tma_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  if constexpr (S == Sched::kMasked) {
    if (warp == 2) build_masked_prefix(ga, prefix, lane);
  } else {
    if (threadIdx.x == 64) *total_slot = ga.m_tiles * ga.n_tiles;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (S == Sched::kMasked) {
    if (threadIdx.x == 64) *total_slot = prefix[ga.E];
    __syncthreads();
  }
  const uint32_t tmem_base = *tmem_slot;
  const int32_t total = *total_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;
    bool ok = true;
    for (int32_t t = blockIdx.x; ok && t < total && !*wc.abort; t += gridDim.x) {
      Tile tile;
      if (!get_tile<S, 128>(ga, prefix, t, tile)) continue;
      // scale atoms of this tile's 128 A rows and 128 B rows (both multiples of 128)
      const uint8_t* sfa_t = args.sfa + static_cast<int64_t>(tile.a_row / kBlockM) * nkb * kMxAtomBytes;
      const uint8_t* sfb_t = args.sfb + static_cast<int64_t>(tile.b_row / 128) * nkb * kMxAtomBytes;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(bars.empty(stage), phase ^ 1u, wc, 0x11)) { ok = false; break; }
        mbar_arrive_expect_tx(bars.full(stage), L::kStageBytes + 2 * kMxAtomBytes);
        tma_load_2d(s_base + L::kOffA + stage * L::kABytes, &tma_a, bars.full(stage), kb * kSlabK, tile.a_row);
        tma_load_2d(s_base + L::kOffB + stage * L::kBBytes, &tma_b, bars.full(stage), kb * kSlabK, tile.b_row);
        const uint32_t sf = s_base + L::kOffSf + stage * 2 * kMxAtomBytes;
        bulk_load_g2s(sf, sfa_t + kb * kMxAtomBytes, kMxAtomBytes, bars.full(stage));
        bulk_load_g2s(sf + kMxAtomBytes, sfb_t + kb * kMxAtomBytes, kMxAtomBytes, bars.full(stage));
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == kMxStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (*wc.abort) {
      // every armed stage completes once its bytes land (the producer is its
      // only arrival): wait for that before the CTA exits (fixed bound)
      for (int st = 0; st < kMxStages; ++st)
        if (armed & (1u << st)) mbar_drain(bars.full(st), (armed_parity >> st) & 1u, wc.status);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    int stage = 0, buf = 0;
    uint32_t phase = 0, tphase = 0;
    bool ok = true;
    const uint32_t sfa_t = tmem_base + L::kTmemSfa, sfb_t = tmem_base + L::kTmemSfb;
    for (int32_t t = blockIdx.x; ok && t < total && !*wc.abort; t += gridDim.x) {
      Tile tile;
      if (!get_tile<S, 128>(ga, prefix, t, tile)) continue;
      if (!mbar_wait(bars.tempty(buf), tphase ^ 1u, wc, 0x12)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + buf * 128;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(bars.full(stage), phase, wc, 0x13)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sf = s_base + L::kOffSf + stage * 2 * kMxAtomBytes;
        tmem_cp_32x128b_warpx4(sfa_t, smem_desc_k_none(sf, 128));
        tmem_cp_32x128b_warpx4(sfb_t, smem_desc_k_none(sf + kMxAtomBytes, 128));
        const uint64_t adesc = smem_desc_k_sw128(s_base + L::kOffA + stage * L::kABytes);
        const uint64_t bdesc = smem_desc_k_sw128(s_base + L::kOffB + stage * L::kBBytes);
#pragma unroll
        for (int k = 0; k < kSlabK / 32; ++k) {
          const uint32_t j = static_cast<uint32_t>(k);
          mma_mx_e4m3(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc_mx_e4m3(kBlockM, 128, j, j), sfa_t | (j << 30),
                      sfb_t | (j << 30), (kb > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(bars.empty(stage));
        if (++stage == kMxStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      mma_commit(bars.tfull(buf));
      if (++buf == 2) {
        buf = 0;
        tphase ^= 1u;
      }
    }
    // every MMA issued completes before TMEM is released (fixed bound, not the caller's wait limit)
    mma_commit(bars.drain());
    mbar_drain(bars.drain(), 0, wc.status);
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3, half = (warp - 4) >> 2;
    const int r = quad * 32 + lane;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    int buf = 0;
    uint32_t tphase = 0;
    for (int32_t t = blockIdx.x; t < total && !*wc.abort; t += gridDim.x) {
      Tile tile;
      if (!get_tile<S, 128>(ga, prefix, t, tile)) continue;
      const bool got = mbar_wait(bars.tfull(buf), tphase, wc, 0x14);
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      tc_fence_after();
      uint64_t v[32];
      tmem_ld_32x32b_x64_pairs(t_lane + buf * 128 + half * 64, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.tempty(buf));
      if (r < tile.rows) {
        __nv_bfloat16* crow = ga.c + static_cast<int64_t>(tile.a_row + r) * ga.N + tile.n0 + half * 64;
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
          uint4 o;
          o.x = bf16x2_from_pair(v[c / 2]);
          o.y = bf16x2_from_pair(v[c / 2 + 1]);
          o.z = bf16x2_from_pair(v[c / 2 + 2]);
          o.w = bf16x2_from_pair(v[c / 2 + 3]);
          *reinterpret_cast<uint4*>(crow + c) = o;
        }
      }
      if (++buf == 2) {
        buf = 0;
        tphase ^= 1u;
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ---------------------------------------------------------------- scale layouts
// E8M0 byte of a power-of-two binary32 scale 2^e, e in [-127, 127]: the
// biased exponent field (2^-127, the binary32 subnormal 0x00400000, has
// field 0, which is E8M0's 2^-127).
__device__ __forceinline__ uint32_t e8m0_of(float s) { return (__float_as_uint(s) >> 23) & 0xFFu; }

// sa [M][nkb] (1x128 activation scales) -> atoms [m_tiles][nkb][512]: thread
// (mt, kb, m0) writes the 16 bytes at 16 m0: rows 32 m1 + m0, m1 = 0..3, each
// byte repeated for the four K blocks; rows past M get 127 (2^0).
__global__ void __launch_bounds__(256) mx_scales_act_kernel(const float* __restrict__ sa, uint8_t* __restrict__ out,
                                                            int64_t M, int64_t nkb, int64_t total) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m0 = i & 31, atom = i >> 5;  // atom = mt * nkb + kb
    const int64_t mt = atom / nkb, kb = atom - mt * nkb;
    uint32_t w[4];
#pragma unroll
    for (int m1 = 0; m1 < 4; ++m1) {
      const int64_t row = mt * 128 + 32 * m1 + m0;
      const uint32_t b = row < M ? e8m0_of(sa[row * nkb + kb]) : 127u;
      w[m1] = b * 0x01010101u;
    }
    *reinterpret_cast<uint4*>(out + atom * kMxAtomBytes + m0 * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// sb [NB][nkb] (128x128 weight-block scales) -> atoms [NB][nkb][512], every
// byte of an atom the block's scale: one thread per 16 bytes.
__global__ void __launch_bounds__(256) mx_scales_w_kernel(const float* __restrict__ sb, uint8_t* __restrict__ out,
                                                          int64_t total) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t atom = i >> 5;  // = nb * nkb + kb, the index of its scale in sb
    const uint32_t w = e8m0_of(sb[atom]) * 0x01010101u;
    *reinterpret_cast<uint4*>(out + i * 16) = make_uint4(w, w, w, w);
  }
}

}  // namespace fp8q
