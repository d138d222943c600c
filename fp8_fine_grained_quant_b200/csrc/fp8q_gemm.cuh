// fp8q_gemm.cuh -- block-scaled FP8 GEMM for sm_100a with per-slab promotion.
//
// Method ("The Insider Secrets Of Deepseek Discovered", Figure 7 (b); the
// codingmall DeepSeek-V3 FP8 page, increased accumulation precision): the
// tensor cores produce one 128-deep K slab's partial sum at a time; each
// partial is moved to FP32 registers on the CUDA cores, multiplied by the two
// dequantization scales of that slab (the activation tile's and the weight
// block's) and added to the running FP32 sum.  The output is rounded to bf16
// once at the end.  Dense and the two MoE grouped layouts of the DeepGEMM
// announcement ("Deepgemm lancado ...", contiguous and masked) share one
// kernel; only the tile scheduler differs.
//
// Design (B200):
//   * persistent CTAs, one per SM, walking a static tile sequence;
//   * warps 0 and 3: TMA producers for alternate slabs (one 128-deep K slab
//     of A [128 x 128 B] and B [BN x 128 B] per pipeline stage, 128-byte
//     swizzle, mbarrier tx count); when the scale rows allow it (K % 512 ==
//     0, 16-byte-aligned scale tensors) the scales of every 4 slabs come by
//     TMA with the first of them, into a small shared ring;
//   * warp 1 allocates TMEM; warps 1 and 2 issue tcgen05.mma.kind::f8f6f4
//     (M = 128, N = BN, K = 32, four per slab) for alternate slabs into four
//     TMEM slab buffers; the first MMA of every slab overwrites, so each
//     buffer holds exactly one slab's partial;
//   * warp 2 also builds the masked-layout tile table before the main loop;
//   * warps 4-11: epilogue; warp w reads TMEM lanes 32*(w%4)..+31 (the rows the
//     hardware lets it access) and half of the BN columns, applies
//     acc += (sa * sb) * partial with packed FP32 FMAs, releases the buffer,
//     and after the last slab stores bf16.  The MMAs of slabs k+1..k+3 run
//     while slab k is being promoted;
//   * promotion is a compile-time parameter: the unpromoted build (all of K
//     accumulated in TMEM, a diagnostic of accumulation precision) is a
//     separate instance;
//   * every mbarrier wait is bounded; a wait that runs out records a timeout
//     in the device status word and all roles drain and return.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "fp8q_ptx.cuh"

namespace fp8q {

enum class Sched : int { kDense = 0, kContiguous = 1, kMasked = 2 };

constexpr int kBlockM = 128;
constexpr int kSlabK = 128;  // promotion interval = scale slab
constexpr int kGemmThreads = 384;  // warpgroup 0: TMA + MMA (+ scheduler set-up); 1-2: epilogue
// Register split of the wide-tile (BN = 256) instances: launched at
// kLaunchRegs per thread (the most __launch_bounds__(384, 1) allows), the
// control warpgroup drops to kCtlRegs and the epilogue warpgroups rise to
// kEpiRegs.  The host checks the launch count before the first launch.
constexpr uint32_t kLaunchRegs = 168;
constexpr uint32_t kCtlRegs = 56;
constexpr uint32_t kEpiRegs = 224;
static_assert(128 * kCtlRegs + 256 * kEpiRegs <= kGemmThreads * kLaunchRegs, "register split exceeds the launch");
constexpr int kMaxMaskedExperts = 1024;


struct GemmArgs {
  const float* sa;           // [rows of A][nkb]
  const float* sb;           // [E][N/128][nkb]
  __nv_bfloat16* c;          // [rows of A][N]: C row r belongs to A row r in every layout
  const int32_t* m_indices;  // contiguous: expert of each 128-row block
  const int32_t* masked_m;   // masked: valid rows per expert
  uint32_t* status;          // device status word
  uint64_t timeout_ns;
  int32_t M;                 // dense: rows of A; contiguous: M_tot; masked: cap
  int32_t N;
  int32_t nkb;               // K / 128
  int32_t E;
  int32_t m_tiles;           // dense: ceil(M/128); contiguous: M_tot/128; masked: cap/128
  int32_t n_tiles;           // ceil(N / BN)
};

struct Tile {
  int32_t a_row;  // first row in A's [rows, K] view (and in C)
  int32_t b_row;  // first row in B's [E*N, K] view
  int32_t n0;     // first output column
  int32_t e;      // expert (0 for dense)
  int32_t rows;   // valid rows in this tile (<= 128)
};

template <int BN, int STAGES, bool k1D1D = false>
struct GemmSmem {
  static constexpr uint32_t kABytes = kBlockM * kSlabK;  // 16 KB
  static constexpr uint32_t kBBytes = BN * kSlabK;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTmemStride = BN <= 128 ? 128 : 256;  // columns per TMEM slab buffer
  static constexpr uint32_t kTmemCols = 512;                      // all of TMEM (one CTA per SM)
  static constexpr int kAccBufs = kTmemCols / kTmemStride;        // slab buffers in flight
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffB = STAGES * kABytes;
  // full[S], empty[S], tfull[B], tempty[B], drain[2]
  static constexpr uint32_t kOffBars = STAGES * kStageBytes;
  static constexpr uint32_t kNumBars = 2 * STAGES + 2 * kAccBufs + 2;
  // misc: tmem slot, abort flag, total tiles, epilogue warps finished, and
  // each epilogue warp's count of TMEM-buffer releases (8 words)
  static constexpr uint32_t kOffMisc = kOffBars + 8 * kNumBars;
  static constexpr uint32_t kMiscBytes = 16 + 4 * 8;
  static constexpr uint32_t kOffPrefix = (kOffMisc + kMiscBytes + 15) / 16 * 16;
  // Scale ring (TMA-staged scales): per group of kScaleGroup slabs, the 128
  // tile rows' activation scales as a [128][kScaleGroup] f32 box and the
  // weight block's kScaleGroup scales.  With per-row scales on both operands
  // (k1D1D, the weight-gradient GEMM) both boxes are slab-major,
  // [kScaleGroup][128] and [kScaleGroup][BN].
  static constexpr int kScaleGroup = 4;
  static constexpr int kScaleSlots = 4;
  static constexpr uint32_t kSaSlotBytes = kBlockM * kScaleGroup * 4;  // 2 KB
  // (block scales: one row of kScaleGroup per 128-column weight block the tile spans)
  static constexpr uint32_t kSbBlocks = BN >= 128 ? BN / 128 : 1;
  static constexpr uint32_t kSbSlotBytes = k1D1D ? BN * kScaleGroup * 4 : kSbBlocks * kScaleGroup * 4;
  static constexpr uint32_t kSbSlotStride = k1D1D ? kSbSlotBytes : 128;  // TMA destinations 128-byte aligned
  // the masked layout's tile prefix (the weight-gradient instance is dense-only and has none)
  static constexpr uint32_t kPrefixBytes = k1D1D ? 0u : 4u * (kMaxMaskedExperts + 1);
  static constexpr uint32_t kOffSa = (kOffPrefix + kPrefixBytes + 127) / 128 * 128;
  static constexpr uint32_t kOffSb = kOffSa + kScaleSlots * kSaSlotBytes;
  static constexpr uint32_t kBytes = kOffSb + kScaleSlots * kSbSlotStride;
  static constexpr uint32_t kDynamicBytes = kBytes + 1024;  // slack for 1024-byte alignment
  static_assert(kDynamicBytes <= 227u * 1024u, "shared memory per CTA");
};

// ----------------------------------------------------------------- scheduler
// Masked layout: per-expert counts of 128-row tiles are turned into a prefix
// over (expert, n-tile, m-tile) once per CTA, in shared memory.
__device__ __forceinline__ int32_t masked_rows(const GemmArgs& a, int e) {
  int32_t m = a.masked_m[e];
  return m < 0 ? 0 : (m > a.M ? a.M : m);
}

__device__ void build_masked_prefix(const GemmArgs& a, int32_t* prefix, int lane) {
  // one warp: lane l sums a contiguous chunk of experts, then a warp scan
  const int chunk = (a.E + 31) / 32;
  const int e0 = lane * chunk, e1 = min(a.E, e0 + chunk);
  int32_t local = 0;
  for (int e = e0; e < e1; ++e) local += ((masked_rows(a, e) + kBlockM - 1) / kBlockM) * a.n_tiles;
  int32_t incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += v;
  }
  int32_t run = incl - local;
  for (int e = e0; e < e1; ++e) {
    prefix[e] = run;
    run += ((masked_rows(a, e) + kBlockM - 1) / kBlockM) * a.n_tiles;
  }
  if (lane == 31) prefix[a.E] = incl;
}

template <Sched S, int BN>
__device__ __forceinline__ bool get_tile(const GemmArgs& a, const int32_t* prefix, int32_t t, Tile& tile) {
  if constexpr (S == Sched::kMasked) {
    int lo = 0, hi = a.E;  // largest e with prefix[e] <= t
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (prefix[mid] <= t) lo = mid; else hi = mid;
    }
    const int e = lo;
    const int32_t rows_e = masked_rows(a, e);
    const int32_t mt_count = (rows_e + kBlockM - 1) / kBlockM;
    const int32_t local = t - prefix[e];
    const int32_t nt = local / mt_count, mt = local - nt * mt_count;  // m-tile fastest: siblings share B
    tile.e = e;
    tile.a_row = e * a.M + mt * kBlockM;
    tile.rows = min(kBlockM, rows_e - mt * kBlockM);
    tile.n0 = nt * BN;
    tile.b_row = e * a.N + tile.n0;
    return true;
  } else {
    const int32_t mt = t / a.n_tiles, nt = t - mt * a.n_tiles;
    tile.a_row = mt * kBlockM;
    tile.n0 = nt * BN;
    if constexpr (S == Sched::kContiguous) {
      const int32_t e = a.m_indices[mt];
      if (e < 0 || e >= a.E) return false;
      tile.e = e;
      tile.rows = kBlockM;
    } else {
      tile.e = 0;
      tile.rows = min(kBlockM, a.M - tile.a_row);
    }
    tile.b_row = tile.e * a.N + tile.n0;
    return true;
  }
}

// ----------------------------------------------------------------- roles
//
// Barrier protocol.  Slabs are numbered j = 0, 1, ... in the order this CTA
// processes them (tiles of its static sequence, then 128-deep K slabs within
// a tile).  Slab j uses pipeline stage s = j % STAGES and, with promotion,
// TMEM slab buffer j % kAccBufs.
//   full[s]  : slab j's operands have landed (TMA transaction bytes) and, with
//              promotion, TMEM buffer j % kAccBufs is free again: the eight
//              epilogue warps arrive once they have read slab j - kAccBufs out
//              of it (for the first kAccBufs slabs they arrive up front).
//              Arrivals: 1 (producer) + 256 (every epilogue lane, once its
//              own TMEM loads are complete) with promotion, else 1.
//   empty[s] : the four MMAs of slab j have completed (one tcgen05.commit):
//              stage s may be refilled (producer, for slab j + STAGES) and,
//              with promotion, the partial in buffer j % kAccBufs is final
//              (epilogue, for slab j).
//   tfull/tempty[b] : only without promotion (the accumulation diagnostic),
//              where a whole tile accumulates in buffer b.
// Every role consumes in slab order, so no phase is re-armed before all its
// waiters have passed it: the MMAs of slab j + STAGES wait for the epilogue's
// release of slab j + STAGES - kAccBufs >= j, which it gives only after it has
// observed empty[s] for slab j, and the producer observes empty[s] for slab j
// before it loads slab j + STAGES.
//
// TMA-staged scales: the scales of slabs 4g..4g+3 of a tile (group g) arrive
// with slab 4g's stage (same full[] barrier) in scale slot g % 4.  The slot is
// rewritten for group g + 4, by the producer of slab 4g + 16, only after
// empty[] of slab 4g + 10, which needs the epilogue's releases of slab 4g + 6:
// by then every epilogue warp has read the scales of slabs <= 4g + 5.  The
// epilogue reads a slab's scales after observing that slab's MMAs complete,
// and those MMAs were issued after full[] of slab 4g (the copies landed).
// Visibility of those bytes to the epilogue threads follows one causality
// chain: the copies' complete-tx on full[] releases the async proxy's writes,
// the MMA thread's wait on full[] acquires them, its tcgen05.commit arrives on
// empty[] after that wait in program order (an arrive-on with release
// semantics at CTA scope), and the epilogue's wait on empty[] acquires.  The
// epilogue never waits on full[] itself.
//
// Each waiting role costs its thread ~150 cycles per barrier probe, and an MMA
// instruction is accepted only as the tensor pipe frees up, so the TMA and MMA
// roles are split over two threads each (slabs alternate between them) and
// each issues one probe and one commit per slab.

template <int STAGES, int ACC>
struct Bars {
  uint32_t base;
  __device__ uint32_t full(int s) const { return base + 8u * s; }
  __device__ uint32_t empty(int s) const { return base + 8u * (STAGES + s); }
  __device__ uint32_t tfull(int b) const { return base + 8u * (2 * STAGES + b); }
  __device__ uint32_t tempty(int b) const { return base + 8u * (2 * STAGES + ACC + b); }
  __device__ uint32_t drain(int i) const { return base + 8u * (2 * STAGES + 2 * ACC + i); }
};

// What the epilogue warps leave for the producers' abort path: where each
// warp stopped, as (stage + STAGES * phase) of the next slab it had not yet
// read (its slab index modulo 2 * STAGES), and how many warps have published.
struct EpiRecord {
  volatile int* done;        // shared: warps that have published
  volatile uint32_t* pos;    // shared: [8] stopping position per epilogue warp
};

// The producers' abort path (see produce).
template <int STAGES, int ACC>
__device__ __noinline__ void producer_abort_drain(Bars<STAGES, ACC> bars, WaitCtl wc, uint32_t armed,
                                                  uint32_t armed_parity, bool promote, EpiRecord epi) {
  bool published = true;
  if (promote) {
    const uint64_t t0 = globaltimer_ns();
    while (*epi.done < 8) {
      if (globaltimer_ns() - t0 > kDrainNs) {
        atomicOr(wc.status, kDevErrTimeout | kDevErrDrain);
        published = false;
        break;
      }
    }
    __threadfence_block();
  }
  for (int st = 0; st < STAGES; ++st) {
    if (!(armed & (1u << st))) continue;
    const uint32_t par = (armed_parity >> st) & 1u;
    if (promote && published && !mbar_test_wait(bars.full(st), par)) {
      // The stage's pending slab js (js mod 2 STAGES = st + STAGES par) needs
      // the release of slab js - ACC from every warp.  A warp that stopped
      // before slab je (je mod 2 STAGES published) has released the slabs
      // below je.  0 <= js - je: js's MMAs have not run, so no warp read it.
      // js - je < STAGES + ACC <= 2 STAGES: js was armed after the MMAs of
      // js - STAGES completed, which needed every warp's release of slab
      // js - STAGES - ACC.  So js - je is their difference modulo 2 STAGES,
      // and the warp's release is missing when js - je >= ACC.
      const uint32_t js = static_cast<uint32_t>(st) + STAGES * par;
      uint32_t missing = 0;
      for (int w = 0; w < 8; ++w) {
        const uint32_t d = (js + 2 * STAGES - epi.pos[w]) % (2 * STAGES);
        if (d >= static_cast<uint32_t>(ACC)) missing += 32;
      }
      if (missing) mbar_arrive_cnt(bars.full(st), missing);
    }
    if (!published) {
      // without the positions the phase may never complete: a short look only
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bars.full(st), par) && globaltimer_ns() - t0 < 1000000ull) {
      }
    } else {
      mbar_drain(bars.full(st), par, wc.status);
    }
  }
}

// TMA producer `who` of two: loads the slabs j with j % 2 == who.
//
// Abort path: before the CTA exits, every copy this thread issued must have
// landed in shared memory.  A stage's phase completes when its bytes have
// landed and its TMEM-buffer releases have arrived, and after an abort some
// releases never come, so the producer first adds, from the stopping
// positions the epilogue warps publish, exactly the releases that are missing,
// then waits for each armed phase (fixed bound kDrainNs).  The stage barrier
// of slab j takes the release of slab j - kAccBufs (the first kAccBufs slabs'
// are posted up front), and stage s is only ever armed by producer s % 2
// (STAGES is even).
template <int BN, int STAGES, Sched S, bool kTmaScales, bool k1D1D>
__device__ __forceinline__ void produce(const CUtensorMap* tma_a, const CUtensorMap* tma_b,
                                        const CUtensorMap* tma_sa, const CUtensorMap* tma_sb, const GemmArgs& args,
                                        const int32_t* prefix, uint32_t s_base,
                                        Bars<STAGES, GemmSmem<BN, STAGES>::kAccBufs> bars, WaitCtl wc,
                                        int32_t total, uint32_t who, bool promote, EpiRecord epi) {
  using L = GemmSmem<BN, STAGES, k1D1D>;
  const int nnb = args.N / 128;
  int stage = 0;
  uint32_t phase = 0, j = 0;
  uint32_t group = 0;  // scale groups so far (kTmaScales)
  uint32_t armed = 0, armed_parity = 0;  // per stage: ever armed / parity of its last phase
  bool ok = true;
  for (int32_t t = blockIdx.x; ok && t < total && !*wc.abort; t += gridDim.x) {
    Tile tile;
    if (!get_tile<S, BN>(args, prefix, t, tile)) continue;
    for (int kb = 0; kb < args.nkb; ++kb, ++j) {
      const bool group_start = kTmaScales && (kb % L::kScaleGroup) == 0;
      if ((j & 1u) == who) {
        if (!mbar_wait(bars.empty(stage), phase ^ 1u, wc, 1)) { ok = false; break; }
        mbar_arrive_expect_tx(bars.full(stage),
                              L::kStageBytes + (group_start ? L::kSaSlotBytes + L::kSbSlotBytes : 0u));
        tma_load_2d(s_base + L::kOffA + stage * L::kABytes, tma_a, bars.full(stage), kb * kSlabK, tile.a_row);
        tma_load_2d(s_base + L::kOffB + stage * L::kBBytes, tma_b, bars.full(stage), kb * kSlabK, tile.b_row);
        if (group_start) {
          const uint32_t slot = group % L::kScaleSlots;
          if constexpr (k1D1D) {
            // slab-major [nkb, rows] scales: x = the tile's first row, a
            // multiple of 128 f32 (16-byte aligned); slabs past nkb read as 0
            tma_load_2d(s_base + L::kOffSa + slot * L::kSaSlotBytes, tma_sa, bars.full(stage), tile.a_row, kb);
            tma_load_2d(s_base + L::kOffSb + slot * L::kSbSlotStride, tma_sb, bars.full(stage), tile.b_row, kb);
          } else {
            // x = kb is a multiple of 4 f32: a 16-byte-aligned start
            tma_load_2d(s_base + L::kOffSa + slot * L::kSaSlotBytes, tma_sa, bars.full(stage), kb, tile.a_row);
            tma_load_2d(s_base + L::kOffSb + slot * L::kSbSlotStride, tma_sb, bars.full(stage), kb,
                        tile.e * nnb + tile.n0 / 128);
          }
        }
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
      }
      if (group_start) ++group;
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  if (*wc.abort && armed) producer_abort_drain<STAGES>(bars, wc, armed, armed_parity, promote, epi);
}

// MMA issuer `who` of `n`: four K = 32 MMAs per slab.  With promotion every
// slab starts a fresh accumulator in its own TMEM buffer, so slabs are
// independent and two issuers take alternate slabs.  Without promotion a tile
// accumulates in one buffer and one issuer (n = 1) does all of it.
template <int BN, int STAGES, Sched S, bool kPromote>
__device__ __forceinline__ void issue_mma(const GemmArgs& args, const int32_t* prefix, uint32_t s_base,
                                          Bars<STAGES, GemmSmem<BN, STAGES>::kAccBufs> bars, WaitCtl wc,
                                          int32_t total, uint32_t tmem_base, uint32_t who, uint32_t n) {
  using L = GemmSmem<BN, STAGES>;
  constexpr uint32_t kIdesc = idesc_e4m3_f32(kBlockM, BN);
  constexpr bool promote = kPromote;
  const uint32_t mask = n - 1;  // n is 1 or 2
  int stage = 0, buf = 0;
  uint32_t phase = 0, tphase = 0, j = 0;
  bool ok = true;
  for (int32_t t = blockIdx.x; ok && t < total && !*wc.abort; t += gridDim.x) {
    Tile tile;
    if (!get_tile<S, BN>(args, prefix, t, tile)) continue;
    for (int kb = 0; kb < args.nkb; ++kb, ++j) {
      if ((j & mask) == who) {
        if (!promote && kb == 0) {
          if (!mbar_wait(bars.tempty(buf), tphase ^ 1u, wc, 2)) { ok = false; break; }
        }
        if (!mbar_wait(bars.full(stage), phase, wc, 3)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * L::kTmemStride;
        const uint64_t adesc = smem_desc_k_sw128(s_base + L::kOffA + stage * L::kABytes);
        const uint64_t bdesc = smem_desc_k_sw128(s_base + L::kOffB + stage * L::kBBytes);
        const uint32_t fresh = (promote || kb == 0) ? 0u : 1u;
        mma_e4m3(d_tmem, adesc, bdesc, kIdesc, fresh);
#pragma unroll
        for (int k = 1; k < kSlabK / 32; ++k) mma_e4m3(d_tmem, adesc + 2u * k, bdesc + 2u * k, kIdesc, 1u);
        mma_commit(bars.empty(stage));
        if (!promote && kb == args.nkb - 1) mma_commit(bars.tfull(buf));
      }
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
      if (promote || kb == args.nkb - 1) {
        if (++buf == L::kAccBufs) {
          buf = 0;
          tphase ^= 1u;
        }
      }
    }
  }
  // Every MMA this thread issued completes before TMEM is released.  The
  // bound is fixed (kDrainNs), not the caller's wait limit: MMAs already
  // issued finish in microseconds.  If it still runs out the status word
  // records a drain timeout; TMEM is freed all the same, since a CTA that
  // exits holding it would leave the next kernel's allocation on this SM
  // waiting forever.
  mma_commit(bars.drain(who));
  mbar_drain(bars.drain(who), 0, wc.status);
}

// Epilogue warp: promotion of every slab partial into FP32 registers, then the
// bf16 store of the finished tile.  Warp w owns TMEM lanes 32*(w%4)..+31 (tile
// rows) and kCols = BN/2 columns; for BN in {128, 256} each half lies inside
// one 128-column weight block, so one sb value per slab.  Per slab the warp
// loads its columns (two 32-column TMEM loads, one wait), hands the buffer
// back as soon as the values are in registers, then applies
// acc += (sa * sb) * partial.  The completion probe of the next slab is issued
// before this slab's work and read after it.
// At its end the warp publishes where it stopped (EpiRecord).
template <int BN, int STAGES, Sched S, bool kPromote, bool kTmaScales, bool k1D1D>
__device__ __forceinline__ void epilogue(uint32_t s_base, const GemmArgs& args, EpiRecord epi, const int32_t* prefix,
                                         Bars<STAGES, GemmSmem<BN, STAGES>::kAccBufs> bars, WaitCtl wc,
                                         int32_t total, uint32_t tmem_base, int warp, int lane) {
  using L = GemmSmem<BN, STAGES, k1D1D>;
  constexpr int kCols = BN / 2;
  constexpr int kGroup = kCols < 64 ? kCols : 64;
  constexpr int kGroups = kCols / kGroup;
  constexpr int kAcc = L::kAccBufs;
  static_assert(kCols <= 128 && 128 % kCols == 0 && kGroup % 32 == 0, "each half must sit in one scale block");
  static_assert(kAcc < STAGES, "buffer releases are posted on the stage barrier of a later slab");
  static_assert(L::kScaleSlots * L::kScaleGroup >= STAGES + kAcc + L::kScaleGroup - 1,
                "a scale slot is rewritten only after every epilogue warp has read its previous group");
  static_assert(STAGES % 2 == 0,
                "two threads take alternate slabs per role; with an even stage count each waits only on its "
                "own stages, so no parity wait can pass on an earlier phase");
  static_assert(kPromote || !kTmaScales, "staged scales serve the per-slab promotion only");
  // k1D1D also needs whole scale groups (nkb % 4 == 0, checked by the host):
  // the slot bound above counts four slabs per group
  static_assert(!k1D1D || (kTmaScales && S == Sched::kDense), "per-row B scales come staged, dense layout only");
  constexpr bool promote = kPromote;
  const int quad = warp & 3;
  const int half = (warp - 4) >> 2;
  const int r = quad * 32 + lane;
  const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
  const int nkb = args.nkb;
  const int nnb = args.N / 128;
  int buf = 0, stage = 0;
  uint32_t tphase = 0, phase = 0;
  bool ready = false;  // the current slab (or tile, without promotion) is known complete
  uint32_t group = 0;  // scale groups so far (kTmaScales)
  for (int32_t t = blockIdx.x; t < total && !*wc.abort; t += gridDim.x) {
    Tile tile;
    if (!get_tile<S, BN>(args, prefix, t, tile)) continue;
    const bool row_ok = r < tile.rows;
    const int col0 = tile.n0 + half * kCols;
    const bool col_ok = col0 < args.N;
    const float* sa_row = args.sa + static_cast<int64_t>(tile.a_row + (row_ok ? r : 0)) * nkb;
    const float* sb_row = args.sb + (static_cast<int64_t>(tile.e) * nnb + (col_ok ? col0 / 128 : 0)) * nkb;
    uint64_t acc[kCols / 2];  // packed pairs of FP32 running sums
#pragma unroll
    for (int i = 0; i < kCols / 2; ++i) acc[i] = 0ull;

    const int n_reads = promote ? nkb : 1;
    // the next slab's scales are fetched one slab ahead (rows past the valid
    // ones read row 0's scales: their sums are never stored)
    float sa_next = kTmaScales ? 0.0f : __ldg(sa_row);
    float sb_next = kTmaScales ? 0.0f : __ldg(sb_row);
    bool ok = true;
    for (int it = 0; it < n_reads; ++it) {
      uint64_t scale2;
      // Warp-uniform outcome: the tcgen05.ld below must be executed by all 32 lanes.
      if (!ready) {
        const bool got = promote ? mbar_wait_inl(bars.empty(stage), phase, wc, 4)
                                 : mbar_wait_inl(bars.tfull(buf), tphase, wc, 4);
        if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
      }
      float sa_smem = 0.0f, sb_smem = 0.0f;
      uint32_t sb_cols = 0;  // k1D1D: shared address of this half's column scales for the slab
      if constexpr (kTmaScales) {
        // this slab's scales, staged with its group's first stage
        const uint32_t slot = group % L::kScaleSlots;
        const uint32_t k = static_cast<uint32_t>(it % L::kScaleGroup);
        if constexpr (k1D1D) {
          sa_smem = lds_f32(s_base + L::kOffSa + slot * L::kSaSlotBytes + k * (kBlockM * 4) + r * 4);
          sb_cols = s_base + L::kOffSb + slot * L::kSbSlotStride + k * (BN * 4) + half * (kCols * 4);
        } else {
          sa_smem = lds_f32(s_base + L::kOffSa + slot * L::kSaSlotBytes + r * (L::kScaleGroup * 4) + k * 4);
          sb_smem = lds_f32(s_base + L::kOffSb + slot * L::kSbSlotStride +
                            ((half * kCols) / 128) * (L::kScaleGroup * 4) + k * 4);
        }
        if (k == L::kScaleGroup - 1) ++group;
      }
      tc_fence_after();
      const uint32_t t_buf = t_lane + buf * L::kTmemStride + half * kCols;
      // position of the next slab (promotion) or tile (no promotion)
      const int nbuf = buf + 1 == kAcc ? 0 : buf + 1;
      const uint32_t ntphase = nbuf == 0 ? (tphase ^ 1u) : tphase;
      const int nstage = stage + 1 == STAGES ? 0 : stage + 1;
      const uint32_t nphase = nstage == 0 ? (phase ^ 1u) : phase;
      const bool next_done = promote ? mbar_test_wait(bars.empty(nstage), nphase)
                                     : mbar_test_wait(bars.tfull(nbuf), ntphase);
      static_assert(kGroup == 64, "the promotion loads 64 columns per group");
#pragma unroll
      for (int g = 0; g < kGroups; ++g) {
        uint64_t v[32];
        tmem_ld_32x32b_x64_pairs(t_buf + g * kGroup, v);
        if (g == kGroups - 1) {
          // buffer free: with promotion it serves slab j + kAcc, whose stage barrier takes the arrival
          tc_fence_before();
          if (promote) {
            int rs = stage + kAcc;
            if (rs >= STAGES) rs -= STAGES;
            mbar_arrive(bars.full(rs));
          } else {
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.tempty(buf));
          }
        }
        if (g == 0) {
          if constexpr (kTmaScales) {
            scale2 = pack_f32x2(sa_smem * sb_smem);
          } else {
            // The slab's scales are consumed here, after its TMEM load and
            // buffer release, and the next slab's are requested right after:
            // each load has a whole slab to arrive, and no buffer release (a
            // release-ordered arrival) waits behind an outstanding load.
            scale2 = pack_f32x2(sa_next * sb_next);
            if (it + 1 < n_reads) {
              sa_next = __ldg(sa_row + it + 1);
              sb_next = __ldg(sb_row + it + 1);
            }
          }
        }
        if constexpr (k1D1D) {
          // acc += (sa_r * sb_c) * partial, column by column: the B scales of
          // 4 columns per (broadcast) shared load
          const uint64_t sa2 = pack_f32x2(sa_smem);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            uint64_t sb01, sb23;
            lds_v2_b64(sb_cols + (g * kGroup + 2 * i) * 4, sb01, sb23);
            ffma2(acc[g * 32 + i], v[i], mul_f32x2(sa2, sb01));
            ffma2(acc[g * 32 + i + 1], v[i + 1], mul_f32x2(sa2, sb23));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ffma2(acc[g * 32 + i], v[i], scale2);
        }
      }
      ready = __all_sync(0xFFFFFFFFu, next_done);
      if (promote) {
        buf = nbuf;
        stage = nstage;
        phase = nphase;
      } else {
        buf = nbuf;
        tphase = ntphase;
      }
    }
    if (!ok) break;
    // The bf16 result: each lane stores its row's columns (rows past the
    // valid ones are never written).
    if (row_ok && col_ok) {
      __nv_bfloat16* crow = args.c + static_cast<int64_t>(tile.a_row + r) * args.N + col0;
#pragma unroll
      for (int c = 0; c < kCols; c += 8) {
        uint4 o;
        o.x = bf16x2_from_pair(acc[c / 2]);
        o.y = bf16x2_from_pair(acc[c / 2 + 1]);
        o.z = bf16x2_from_pair(acc[c / 2 + 2]);
        o.w = bf16x2_from_pair(acc[c / 2 + 3]);
        *reinterpret_cast<uint4*>(crow + c) = o;
      }
    }
  }
  // where this warp stopped, for the producers' abort path
  if (lane == 0) {
    epi.pos[warp - 4] = static_cast<uint32_t>(stage) + STAGES * phase;
    __threadfence_block();
    atomicAdd(const_cast<int*>(epi.done), 1);
  }
  __syncwarp();
}


// ----------------------------------------------------------------- kernel
template <int BN, int STAGES, Sched S, bool kPromote, bool kTmaScales, bool k1D1D>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_blockscaled_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                            const __grid_constant__ CUtensorMap tma_sa, const __grid_constant__ CUtensorMap tma_sb,
                            const GemmArgs args) {
  using L = GemmSmem<BN, STAGES, k1D1D>;
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "UMMA N for M=128 must be a multiple of 16 in [16,256]");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const Bars<STAGES, L::kAccBufs> bars{s_base + L::kOffBars};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  int32_t* total_slot = reinterpret_cast<int32_t*>(smem + L::kOffMisc + 8);
  const EpiRecord epi{reinterpret_cast<volatile int*>(smem + L::kOffMisc + 12),
                      reinterpret_cast<volatile uint32_t*>(smem + L::kOffMisc + 16)};  // 8 positions
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + L::kOffPrefix);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtl wc{args.timeout_ns, args.status, abort_flag};
  constexpr bool promote = kPromote;

  if (threadIdx.x == 0) {
    for (int st = 0; st < STAGES; ++st) {
      mbar_init(bars.full(st), promote ? 1 + 8 * 32 : 1);  // producer (+ every lane of the eight epilogue warps)
      mbar_init(bars.empty(st), 1);
    }
    for (int b = 0; b < L::kAccBufs; ++b) {
      mbar_init(bars.tfull(b), 1);
      mbar_init(bars.tempty(b), 8);  // one arrival per epilogue warp
    }
    mbar_init(bars.drain(0), 1);
    mbar_init(bars.drain(1), 1);
    *abort_flag = 0;
    *epi.done = 0;
    fence_barrier_init();
    tma_prefetch_map(&tma_a);
    tma_prefetch_map(&tma_b);
    if constexpr (kTmaScales) {
      tma_prefetch_map(&tma_sa);
      tma_prefetch_map(&tma_sb);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  if constexpr (S == Sched::kMasked) {
    if (warp == 2) build_masked_prefix(args, prefix, lane);
  } else {
    if (threadIdx.x == 64) *total_slot = args.m_tiles * args.n_tiles;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (S == Sched::kMasked) {
    if (threadIdx.x == 64) *total_slot = prefix[args.E];
    __syncthreads();
  }
  const uint32_t tmem_base = *tmem_slot;
  const int32_t total = *total_slot;

  // Wide tiles hold 128 FP32 sums per epilogue thread: the control
  // warpgroup hands registers to the two epilogue warpgroups
  // (128 x kCtlRegs + 256 x kEpiRegs = 384 x kLaunchRegs).  Each role then
  // finishes on its own path, and the epilogue calls no out-of-line function.
  constexpr bool kSplitRegs = BN > 128;
  if (warp < 4) {
    if constexpr (kSplitRegs) setmaxnreg_dec<kCtlRegs>();
    // warps 0 and 3: TMA producers; warps 1 and 2: MMA issuers (one issuer
    // when a tile accumulates in a single buffer)
    const uint32_t n_mma = promote ? 2u : 1u;
    if (lane == 0) {
      if (warp == 0 || warp == 3)
        produce<BN, STAGES, S, kTmaScales, k1D1D>(&tma_a, &tma_b, &tma_sa, &tma_sb, args, prefix, s_base, bars, wc,
                                                  total, warp == 0 ? 0u : 1u, promote, epi);
      else if (static_cast<uint32_t>(warp - 1) < n_mma)
        issue_mma<BN, STAGES, S, kPromote>(args, prefix, s_base, bars, wc, total, tmem_base, warp - 1, n_mma);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem_base, L::kTmemCols);
    }
  } else {
    if constexpr (kSplitRegs) setmaxnreg_inc<kEpiRegs>();
    // all TMEM slab buffers start free: every lane releases them for the first slabs
    if (promote)
      for (int b = 0; b < L::kAccBufs; ++b) mbar_arrive(bars.full(b));
    epilogue<BN, STAGES, S, kPromote, kTmaScales, k1D1D>(s_base, args, epi, prefix, bars, wc, total, tmem_base,
                                                         warp, lane);
    __syncwarp();
    tc_fence_before();
    __syncthreads();
  }
}

}  // namespace fp8q
