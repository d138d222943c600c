// fp8q_api.cu -- the C ABI declared in include/fp8q.h: argument validation,
// TMA descriptor encoding, kernel-instance choice and launches on the caller's
// stream.  One translation unit holds every kernel so the device status word
// is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "fp8q.h"
#include "fp8q_gemm.cuh"
#include "fp8q_gemm_mx.cuh"
#include "fp8q_ptx.cuh"
#include "fp8q_quant.cuh"

namespace fp8q {

__device__ uint32_t g_device_status;
// Where fp8q_get_device_error's exchange kernel leaves the word it took: one
// slot per query, taken round-robin, so queries that overlap on different
// streams do not read each other's result.
constexpr int kTakeSlots = 64;
__device__ uint32_t g_device_status_taken[kTakeSlots];

namespace {

constexpr uint64_t kDefaultTimeoutNs = 4000000000ull;
constexpr int kMaxDevices = 64;

std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<uint64_t> g_launches{0};
std::atomic<uint32_t> g_take_slot{0};

struct DeviceInfo {
  // set (release) once every other field is final; read (acquire) without the lock
  std::atomic<bool> ready{false};
  bool supported = false;
  int num_sms = 0;
  uint32_t* status = nullptr;  // device address of g_device_status
  bool wide_ok = false;        // the wide-tile instances were built with the register count their split needs
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Per-device set-up, done once: SM count, arch check, status-word address,
// and the dynamic shared-memory opt-in of every GEMM instantiation (and of
// the token-axis quantizer).
template <int BN, int STAGES, Sched S, bool kPromote, bool kTmaScales, bool k1D1D = false>
cudaError_t opt_in_smem() {
  return cudaFuncSetAttribute(gemm_blockscaled_kernel<BN, STAGES, S, kPromote, kTmaScales, k1D1D>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              GemmSmem<BN, STAGES, k1D1D>::kDynamicBytes);
}

// The token-axis quantizer's two 32 KB stages (dynamic shared memory), with
// the carveout that lets kTokCtasPerSm of its CTAs share an SM.
template <bool kTokenContiguous>
cudaError_t opt_in_token_axis_smem() {
  cudaError_t e = cudaFuncSetAttribute(quant_act_128x1_kernel<kTokenContiguous>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kTokSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(quant_act_128x1_kernel<kTokenContiguous>,
                             cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  return e;
}

// Whether an instance that splits registers between its warpgroups was
// built with the launch count the split assumes (a split larger than the
// launch's allocation would never be granted).
template <int BN, int STAGES, Sched S, bool kPromote, bool kTmaScales, bool k1D1D = false>
bool split_regs_ok() {
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, gemm_blockscaled_kernel<BN, STAGES, S, kPromote, kTmaScales, k1D1D>) != cudaSuccess)
    return false;
  return static_cast<uint32_t>(fa.numRegs) * kGemmThreads >= 128 * kCtlRegs + 256 * kEpiRegs;
}

// Output tile 128 x kTileN: 64 FP32 accumulators per epilogue thread, four
// TMEM slab buffers, six 32 KB pipeline stages.
constexpr int kTileN = 128;
constexpr int kStages128 = 6;
// Wide output tile 128 x 256: 128 FP32 accumulators per epilogue thread
// (registers split between the warpgroups), two TMEM slab buffers of 256
// columns, four 48 KB stages.  Each A slab loaded serves twice the columns.
constexpr int kTileWide = 256;
constexpr int kStagesWide = 4;

int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8Q_ERR_CUDA;
  DeviceInfo& d = g_dev[dev];
  if (!d.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (!d.ready.load(std::memory_order_relaxed)) {
      int major = 0, minor = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return FP8Q_ERR_CUDA;
      d.supported = (major == 10 && minor == 0);
      d.num_sms = sms;
      if (d.supported) {
        if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.status), g_device_status) != cudaSuccess)
          return FP8Q_ERR_CUDA;
        cudaError_t e = cudaSuccess;
        if (e == cudaSuccess) e = opt_in_smem<kTileN, kStages128, Sched::kDense, true, true>();
        if (e == cudaSuccess) e = opt_in_smem<kTileN, kStages128, Sched::kDense, true, false>();
        if (e == cudaSuccess) e = opt_in_smem<kTileN, kStages128, Sched::kDense, false, false>();
        if (e == cudaSuccess) e = opt_in_smem<kTileN, kStages128, Sched::kContiguous, true, true>();
        if (e == cudaSuccess) e = opt_in_smem<kTileN, kStages128, Sched::kContiguous, true, false>();
        if (e == cudaSuccess) e = opt_in_smem<kTileN, kStages128, Sched::kMasked, true, true>();
        if (e == cudaSuccess) e = opt_in_smem<kTileN, kStages128, Sched::kMasked, true, false>();
        if (e == cudaSuccess) e = opt_in_smem<kTileN, kStages128, Sched::kDense, true, true, true>();
        if (e == cudaSuccess) e = opt_in_smem<kTileWide, kStagesWide, Sched::kDense, true, true>();
        if (e == cudaSuccess) e = opt_in_smem<kTileWide, kStagesWide, Sched::kContiguous, true, true>();
        if (e == cudaSuccess) e = opt_in_smem<kTileWide, kStagesWide, Sched::kMasked, true, true>();
        d.wide_ok = split_regs_ok<kTileWide, kStagesWide, Sched::kDense, true, true>() &&
                    split_regs_ok<kTileWide, kStagesWide, Sched::kContiguous, true, true>() &&
                    split_regs_ok<kTileWide, kStagesWide, Sched::kMasked, true, true>();
        if (e == cudaSuccess)
          e = cudaFuncSetAttribute(gemm_mx_kernel<Sched::kDense>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   MxSmem::kDynamicBytes);
        if (e == cudaSuccess)
          e = cudaFuncSetAttribute(gemm_mx_kernel<Sched::kContiguous>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   MxSmem::kDynamicBytes);
        if (e == cudaSuccess)
          e = cudaFuncSetAttribute(gemm_mx_kernel<Sched::kMasked>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   MxSmem::kDynamicBytes);
        if (e == cudaSuccess) e = opt_in_token_axis_smem<false>();
        if (e == cudaSuccess) e = opt_in_token_axis_smem<true>();
        if (e != cudaSuccess) return FP8Q_ERR_CUDA;
      }
      d.ready.store(true, std::memory_order_release);
    }
  }
  if (!d.supported) return FP8Q_ERR_UNSUPPORTED;
  *out = &d;
  return FP8Q_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// ---------------------------------------------------------------- TMA maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// [rows, K] bytes, row stride K, box = 128 bytes x box_rows, 128-byte swizzle.
// Rows past `rows` read as zero.
int make_operand_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FP8Q_ERR_CUDA;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kSlabK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// Scale tensor [rows, nkb] f32 as a 2-D map with a box of 4 slabs x box_rows
// rows (the GEMM stages a group of 4 slabs' scales at once).  Needs nkb % 4 ==
// 0 and a 16-byte-aligned base; rows past the end read as zero.
int make_scale_map(CUtensorMap* map, const float* base, uint64_t rows, uint64_t nkb, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FP8Q_ERR_CUDA;
  const cuuint64_t dims[2] = {nkb, rows};
  const cuuint64_t strides[1] = {nkb * 4};
  const cuuint32_t box[2] = {4, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// Slab-major scale tensor [nkb, rows] f32 (one row per 128-deep slab) with a
// box of 4 slabs x box_rows: the per-row scales of both weight-gradient
// operands.  rows % 4 == 0 and a 16-byte-aligned base; slabs past nkb read as
// zero.
int make_row_scale_map(CUtensorMap* map, const float* base, uint64_t rows, uint64_t nkb, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FP8Q_ERR_CUDA;
  const cuuint64_t dims[2] = {rows, nkb};
  const cuuint64_t strides[1] = {rows * 4};
  const cuuint32_t box[2] = {box_rows, 4};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// ---------------------------------------------------------------- GEMM launch
struct GemmCall {
  const uint8_t* qa;
  const float* sa;
  const uint8_t* qb;
  const float* sb;
  void* c;
  const int32_t* m_indices;
  const int32_t* masked_m;
  int64_t a_rows;   // rows of A's 2-D view
  int64_t M;        // dense M, M_tot, or cap
  int64_t N, K, E;
  int64_t m_tiles;  // per expert for masked
  int64_t expected_m;
  int promote;
};

// Output tiles of one GEMM launch: the kernels number them (and walk them,
// t += gridDim.x) in 32-bit integers.
constexpr int64_t kMaxTiles = (int64_t(1) << 31) - (int64_t(1) << 16);

// One launch of one kernel instance.
template <int BN, int STAGES, Sched S, bool kPromote, bool kTmaScales, bool k1D1D>
int launch_instance(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& msa, const CUtensorMap& msb,
                    const GemmArgs& a, int64_t grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = GemmSmem<BN, STAGES, k1D1D>::kDynamicBytes;
  cfg.stream = stream;
  cudaError_t e =
      cudaLaunchKernelEx(&cfg, gemm_blockscaled_kernel<BN, STAGES, S, kPromote, kTmaScales, k1D1D>, ma, mb, msa, msb,
                         a);
  if (e != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

template <int BN, int STAGES, Sched S, bool kPromote, bool kTmaScales, bool k1D1D = false>
int launch_gemm(const GemmCall& g, const DeviceInfo& dev, cudaStream_t stream) {
  CUtensorMap ma, mb, msa, msb;
  std::memset(&msa, 0, sizeof msa);
  std::memset(&msb, 0, sizeof msb);
  int rc = make_operand_map(&ma, g.qa, static_cast<uint64_t>(g.a_rows), static_cast<uint64_t>(g.K), kBlockM);
  if (rc) return rc;
  rc = make_operand_map(&mb, g.qb, static_cast<uint64_t>(g.E * g.N), static_cast<uint64_t>(g.K), BN);
  if (rc) return rc;
  if constexpr (k1D1D) {
    const uint64_t nkb = static_cast<uint64_t>(g.K / kSlabK);
    rc = make_row_scale_map(&msa, g.sa, static_cast<uint64_t>(g.a_rows), nkb, kBlockM);
    if (rc) return rc;
    rc = make_row_scale_map(&msb, g.sb, static_cast<uint64_t>(g.N), nkb, BN);
    if (rc) return rc;
  } else if constexpr (kTmaScales) {
    const uint64_t nkb = static_cast<uint64_t>(g.K / kSlabK);
    rc = make_scale_map(&msa, g.sa, static_cast<uint64_t>(g.a_rows), nkb, kBlockM);
    if (rc) return rc;
    rc = make_scale_map(&msb, g.sb, static_cast<uint64_t>(g.E * (g.N / 128)), nkb,
                        GemmSmem<BN, STAGES, k1D1D>::kSbBlocks);
    if (rc) return rc;
  }
  GemmArgs a;
  std::memset(&a, 0, sizeof a);
  a.sa = g.sa;
  a.sb = g.sb;
  a.c = static_cast<__nv_bfloat16*>(g.c);
  a.m_indices = g.m_indices;
  a.masked_m = g.masked_m;
  a.status = dev.status;
  a.timeout_ns = g_timeout_ns.load();
  a.M = static_cast<int32_t>(g.M);
  a.N = static_cast<int32_t>(g.N);
  a.nkb = static_cast<int32_t>(g.K / kSlabK);
  a.E = static_cast<int32_t>(g.E);
  a.m_tiles = static_cast<int32_t>(g.m_tiles);
  a.n_tiles = static_cast<int32_t>((g.N + BN - 1) / BN);
  const int64_t max_tiles = g.m_tiles * a.n_tiles * (S == Sched::kMasked ? g.E : 1);
  if (max_tiles >= kMaxTiles) return FP8Q_ERR_SHAPE;  // the kernel numbers tiles in 32 bits
  const int64_t grid = max_tiles < dev.num_sms ? max_tiles : dev.num_sms;
  if (grid <= 0) return FP8Q_OK;
  return launch_instance<BN, STAGES, S, kPromote, kTmaScales, k1D1D>(ma, mb, msa, msb, a, grid, stream);
}

// Tile width.  Wide tiles need N to be a multiple of 256 (no half-empty tile
// column).  A wide tile does the work of two 128-column tiles in about 0.95
// of their time, but there are half as many, so the last partial round of
// tiles over the SMs can cost more than that gains: for the dense and
// contiguous layouts (tile count known on the host) wide tiles are taken
// only when 2 x 0.95 x (rounds of wide tiles) <= rounds of 128-column tiles.
// The masked layout's tile count is known on the device only; it takes wide
// tiles whenever N allows.
template <Sched S>
bool use_wide_tiles(const GemmCall& g, int64_t sms) {
  if (g.N % kTileWide != 0) return false;
  if constexpr (S == Sched::kMasked) return true;
  const int64_t narrow = g.m_tiles * (g.N / kTileN), wide = g.m_tiles * (g.N / kTileWide);
  const int64_t r_narrow = (narrow + sms - 1) / sms, r_wide = (wide + sms - 1) / sms;
  return 19 * r_wide <= 10 * r_narrow;
}

template <Sched S>
int run_gemm(const GemmCall& g, cudaStream_t stream) {
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  if (g.promote) {
    // scales staged by TMA with the operands when their rows are 16-byte
    // multiples (K % 512 == 0) and both scale tensors are 16-byte aligned
    if ((g.K / kSlabK) % 4 == 0 && aligned(g.sa, 16) && aligned(g.sb, 16)) {
      if (dev->wide_ok && use_wide_tiles<S>(g, dev->num_sms))
        return launch_gemm<kTileWide, kStagesWide, S, true, true>(g, *dev, stream);
      return launch_gemm<kTileN, kStages128, S, true, true>(g, *dev, stream);
    }
    return launch_gemm<kTileN, kStages128, S, true, false>(g, *dev, stream);
  }
  // only the dense form has the unpromoted (accumulation diagnostic) build
  if constexpr (S == Sched::kDense) return launch_gemm<kTileN, kStages128, S, false, false>(g, *dev, stream);
  return FP8Q_ERR_UNSUPPORTED;
}

int check_operands(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb, const void* c) {
  if (!qa || !sa || !qb || !sb || !c) return FP8Q_ERR_NULL;
  if (!aligned(qa, 16) || !aligned(qb, 16) || !aligned(c, 16) || !aligned(sa, 4) || !aligned(sb, 4))
    return FP8Q_ERR_ALIGN;
  return FP8Q_OK;
}

constexpr int64_t kMaxRows = int64_t(1) << 31;

// Persistent: at most kTokCtasPerSm CTAs per SM, each walking its blocks.
template <bool kTokenContiguous>
void launch_quant_act_128x1(const uint8_t* x, uint8_t* q, float* s, int64_t M, int64_t K, int64_t Mp, int num_sms,
                            cudaStream_t stream) {
  const int64_t blocks = (Mp / 128) * (K / 128);
  const int64_t cap = static_cast<int64_t>(num_sms) * kTokCtasPerSm;
  const int64_t grid = blocks < cap ? blocks : cap;
  quant_act_128x1_kernel<kTokenContiguous>
      <<<static_cast<unsigned>(grid), 256, kTokSmemBytes, stream>>>(x, q, s, M, K, Mp, blocks);
}

}  // namespace

// Reads and clears the status word in one atomic step, after the work queued
// before it on the caller's stream.
__global__ void status_take_kernel(uint32_t* status, uint32_t* taken) { *taken = atomicExch(status, 0u); }

// Bounded-wait self-test kernel: waits on a barrier nobody completes.
__global__ void wait_selftest_kernel(uint32_t* status, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtl w{timeout_ns, status, &abort_flag};
    mbar_wait(smem_u32(&bar), 0, w, 0x7F);
  }
}

}  // namespace fp8q

using namespace fp8q;

// An NVTX range named after the entry point around each call that launches
// work, so profilers show the library's calls on the host timeline (a no-op
// when no tool is attached).
namespace {
struct ApiRange {
  explicit ApiRange(const char* name) { nvtxRangePushA(name); }
  ~ApiRange() { nvtxRangePop(); }
  ApiRange(const ApiRange&) = delete;
  ApiRange& operator=(const ApiRange&) = delete;
};
}  // namespace
#define FP8Q_API_RANGE() ApiRange fp8q_api_range_(__func__)

template <bool kPow2>
static int quant_act_1x128(const void* x_bf16, int64_t M, int64_t K, uint8_t* q, float* s, cudaStream_t stream) {
  if (M < 0 || K < 0 || K % 128 || M >= kMaxRows || K >= kMaxRows) return FP8Q_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (!x_bf16 || !q || !s) return FP8Q_ERR_NULL;
  if (!aligned(x_bf16, 32) || !aligned(q, 16) || !aligned(s, 4)) return FP8Q_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  const int64_t tiles = M * (K / 128);
  constexpr int kUnroll = 2;  // tiles per lane group in flight (64 bytes of loads per lane)
  const int64_t per_cta = (256 / 8) * kUnroll;
  int64_t grid = (tiles + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(dev->num_sms) * 10;  // two full waves of 5 resident CTAs per SM
  if (grid > cap) grid = cap;
  quant_act_1x128_kernel<kUnroll, kPow2><<<static_cast<unsigned>(grid), 256, 0, stream>>>(
      static_cast<const uint8_t*>(x_bf16), q, s, tiles);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

template <bool kPow2>
static int quant_w_128x128(const void* w_bf16, int64_t G, int64_t N, int64_t K, uint8_t* q, float* s,
                           cudaStream_t stream) {
  if (G < 0 || N < 0 || K < 0 || N % 128 || K % 128 || G >= kMaxRows || N >= kMaxRows || G * N >= kMaxRows ||
      K >= kMaxRows)
    return FP8Q_ERR_SHAPE;
  if (G == 0 || N == 0 || K == 0) return FP8Q_OK;
  if (!w_bf16 || !q || !s) return FP8Q_ERR_NULL;
  if (!aligned(w_bf16, 32) || !aligned(q, 16) || !aligned(s, 4)) return FP8Q_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  const int64_t blocks = G * (N / 128) * (K / 128);
  const int64_t cap = static_cast<int64_t>(dev->num_sms) * 64;
  const int64_t grid = blocks < cap ? blocks : cap;
  quant_w_128x128_kernel<kPow2><<<static_cast<unsigned>(grid), 256, 0, stream>>>(static_cast<const uint8_t*>(w_bf16), q, s,
                                                                           K, blocks);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

// Launch of the block-scaled GEMM for one layout; g carries the GemmCall
// shapes (a_rows, M, N, K, E, m_tiles) and layout arrays.
template <Sched S>
static int launch_mx(const GemmCall& g, const uint8_t* sfa_mx, const uint8_t* sfb_mx, cudaStream_t stream) {
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  CUtensorMap ma, mb;
  rc = make_operand_map(&ma, g.qa, static_cast<uint64_t>(g.a_rows), static_cast<uint64_t>(g.K), kBlockM);
  if (rc) return rc;
  rc = make_operand_map(&mb, g.qb, static_cast<uint64_t>(g.E * g.N), static_cast<uint64_t>(g.K), 128);
  if (rc) return rc;
  MxArgs a;
  std::memset(&a, 0, sizeof a);
  a.g.c = static_cast<__nv_bfloat16*>(g.c);
  a.g.m_indices = g.m_indices;
  a.g.masked_m = g.masked_m;
  a.g.status = dev->status;
  a.g.timeout_ns = g_timeout_ns.load();
  a.g.M = static_cast<int32_t>(g.M);
  a.g.N = static_cast<int32_t>(g.N);
  a.g.nkb = static_cast<int32_t>(g.K / kSlabK);
  a.g.E = static_cast<int32_t>(g.E);
  a.g.m_tiles = static_cast<int32_t>(g.m_tiles);
  a.g.n_tiles = static_cast<int32_t>(g.N / 128);
  a.sfa = sfa_mx;
  a.sfb = sfb_mx;
  const int64_t max_tiles = g.m_tiles * (g.N / 128) * (S == Sched::kMasked ? g.E : 1);
  if (max_tiles >= kMaxTiles) return FP8Q_ERR_SHAPE;  // the kernel numbers tiles in 32 bits
  const int grid = static_cast<int>(max_tiles < dev->num_sms ? max_tiles : dev->num_sms);
  if (grid <= 0) return FP8Q_OK;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = MxSmem::kDynamicBytes;
  cfg.stream = stream;
  if (cudaLaunchKernelEx(&cfg, gemm_mx_kernel<S>, ma, mb, a) != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

static int check_mx_operands(const uint8_t* qa, const uint8_t* sfa_mx, const uint8_t* qb, const uint8_t* sfb_mx,
                             const void* c) {
  if (!qa || !sfa_mx || !qb || !sfb_mx || !c) return FP8Q_ERR_NULL;
  if (!aligned(qa, 16) || !aligned(qb, 16) || !aligned(c, 16) || !aligned(sfa_mx, 16) || !aligned(sfb_mx, 16))
    return FP8Q_ERR_ALIGN;
  return FP8Q_OK;
}

extern "C" {

int fp8_quant_act_w(const void* x_bf16, int64_t M, int64_t K, uint8_t* qa, float* sa, const void* w_bf16, int64_t G,
                    int64_t N, int64_t Kw, uint8_t* qw, float* sw, cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (M < 0 || K < 0 || K % 128 || M >= kMaxRows || K >= kMaxRows) return FP8Q_ERR_SHAPE;
  if (G < 0 || N < 0 || Kw < 0 || N % 128 || Kw % 128 || G >= kMaxRows || N >= kMaxRows || G * N >= kMaxRows ||
      Kw >= kMaxRows)
    return FP8Q_ERR_SHAPE;
  const bool act = M > 0 && K > 0, wt = G > 0 && N > 0 && Kw > 0;
  if (act && (!x_bf16 || !qa || !sa)) return FP8Q_ERR_NULL;
  if (wt && (!w_bf16 || !qw || !sw)) return FP8Q_ERR_NULL;
  if (act && (!aligned(x_bf16, 32) || !aligned(qa, 16) || !aligned(sa, 4))) return FP8Q_ERR_ALIGN;
  if (wt && (!aligned(w_bf16, 32) || !aligned(qw, 16) || !aligned(sw, 4))) return FP8Q_ERR_ALIGN;
  const int64_t tiles = act ? M * (K / 128) : 0;
  const int64_t act_ctas = (tiles + kActTilesPerCta - 1) / kActTilesPerCta;
  const int64_t blocks = wt ? G * (N / 128) * (Kw / 128) : 0;
  if (act_ctas + blocks >= kMaxRows) return FP8Q_ERR_SHAPE;  // one CTA per 32 KB unit: the grid's x limit
  if (act_ctas + blocks == 0) return FP8Q_OK;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  quant_act_w_kernel<<<static_cast<unsigned>(act_ctas + blocks), 256, 0, stream>>>(
      static_cast<const uint8_t*>(x_bf16), qa, sa, tiles, act_ctas, static_cast<const uint8_t*>(w_bf16), qw, sw, Kw);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

int fp8_quant_act_1x128(const void* x_bf16, int64_t M, int64_t K, uint8_t* q, float* s, cudaStream_t stream) {
  FP8Q_API_RANGE();
  return quant_act_1x128<false>(x_bf16, M, K, q, s, stream);
}

int fp8_quant_act_1x128_ue8m0(const void* x_bf16, int64_t M, int64_t K, uint8_t* q, float* s, cudaStream_t stream) {
  FP8Q_API_RANGE();
  return quant_act_1x128<true>(x_bf16, M, K, q, s, stream);
}

int fp8_quant_w_128x128(const void* w_bf16, int64_t G, int64_t N, int64_t K, uint8_t* q, float* s,
                        cudaStream_t stream) {
  FP8Q_API_RANGE();
  return quant_w_128x128<false>(w_bf16, G, N, K, q, s, stream);
}

int fp8_quant_w_128x128_ue8m0(const void* w_bf16, int64_t G, int64_t N, int64_t K, uint8_t* q, float* s,
                              cudaStream_t stream) {
  FP8Q_API_RANGE();
  return quant_w_128x128<true>(w_bf16, G, N, K, q, s, stream);
}

int fp8_quant_act_128x1(const void* x_bf16, int64_t M, int64_t K, uint8_t* q, float* s, cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (M < 0 || K < 0 || K % 128 || M >= kMaxRows || K >= kMaxRows) return FP8Q_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (!x_bf16 || !q || !s) return FP8Q_ERR_NULL;
  if (!aligned(x_bf16, 16) || !aligned(q, 16) || !aligned(s, 16)) return FP8Q_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  const int64_t Mp = (M + 127) / 128 * 128;
  launch_quant_act_128x1<false>(static_cast<const uint8_t*>(x_bf16), q, s, M, K, Mp, dev->num_sms, stream);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

int fp8_swiglu_quant_1x128(const void* c1_bf16, int64_t rows, int64_t inter, const int32_t* masked_m, int64_t cap,
                           uint8_t* qh, float* sh, cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (rows < 0 || inter < 0 || inter % 128 || rows >= kMaxRows || inter >= kMaxRows / 2) return FP8Q_ERR_SHAPE;
  if (masked_m && (cap <= 0 || rows % cap)) return FP8Q_ERR_SHAPE;
  if (rows == 0 || inter == 0) return FP8Q_OK;
  if (!c1_bf16 || !qh || !sh) return FP8Q_ERR_NULL;
  if (!aligned(c1_bf16, 32) || !aligned(qh, 16) || !aligned(sh, 4) || (masked_m && !aligned(masked_m, 4)))
    return FP8Q_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  const int64_t tiles = rows * (inter / 128);
  int64_t grid = (tiles + 31) / 32;  // 32 tiles per CTA pass
  const int64_t cap_grid = static_cast<int64_t>(dev->num_sms) * 8;
  if (grid > cap_grid) grid = cap_grid;
  swiglu_quant_1x128_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
      static_cast<const uint8_t*>(c1_bf16), qh, sh, inter, tiles, masked_m, masked_m ? cap : 1);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

int fp8_quant_act_128x1_t(const void* x_bf16, int64_t M, int64_t K, int64_t Mp, uint8_t* qt, float* s,
                          cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (M < 0 || K < 0 || K % 128 || Mp < M || Mp % 128 || Mp >= kMaxRows || K >= kMaxRows) return FP8Q_ERR_SHAPE;
  if (Mp == 0 || K == 0) return FP8Q_OK;
  if (!x_bf16 || !qt || !s) return FP8Q_ERR_NULL;
  if (!aligned(x_bf16, 16) || !aligned(qt, 16) || !aligned(s, 16)) return FP8Q_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  launch_quant_act_128x1<true>(static_cast<const uint8_t*>(x_bf16), qt, s, M, K, Mp, dev->num_sms, stream);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

int fp8_mx_scales_act(const float* sa, int64_t M, int64_t K, uint8_t* sfa_mx, cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (M < 0 || K < 0 || K % 128 || M >= kMaxRows || K >= kMaxRows) return FP8Q_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (!sa || !sfa_mx) return FP8Q_ERR_NULL;
  if (!aligned(sa, 4) || !aligned(sfa_mx, 16)) return FP8Q_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  const int64_t nkb = K / 128, total = ((M + 127) / 128) * nkb * 32;
  int64_t grid = (total + 255) / 256;
  if (grid > dev->num_sms * 8) grid = dev->num_sms * 8;
  mx_scales_act_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(sa, sfa_mx, M, nkb, total);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

int fp8_mx_scales_w(const float* sb, int64_t G, int64_t N, int64_t K, uint8_t* sfb_mx, cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (G < 0 || N < 0 || K < 0 || N % 128 || K % 128 || G >= kMaxRows || N >= kMaxRows || G * N >= kMaxRows ||
      K >= kMaxRows)
    return FP8Q_ERR_SHAPE;
  if (G == 0 || N == 0 || K == 0) return FP8Q_OK;
  if (!sb || !sfb_mx) return FP8Q_ERR_NULL;
  if (!aligned(sb, 4) || !aligned(sfb_mx, 16)) return FP8Q_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  const int64_t total = G * (N / 128) * (K / 128) * 32;
  int64_t grid = (total + 255) / 256;
  if (grid > dev->num_sms * 8) grid = dev->num_sms * 8;
  mx_scales_w_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(sb, sfb_mx, total);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

int fp8_gemm_mx(const uint8_t* qa, const uint8_t* sfa_mx, const uint8_t* qb, const uint8_t* sfb_mx, void* c_bf16,
                int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (M < 0 || N < 0 || K < 128 || K % 128 || N % 128 || M >= kMaxRows || N >= kMaxRows || K >= kMaxRows)
    return FP8Q_ERR_SHAPE;
  if (M == 0 || N == 0) return FP8Q_OK;
  int rc = check_mx_operands(qa, sfa_mx, qb, sfb_mx, c_bf16);
  if (rc) return rc;
  GemmCall g{qa, nullptr, qb, nullptr, c_bf16, nullptr, nullptr, M, M, N, K, 1, (M + kBlockM - 1) / kBlockM, 0, 1};
  return launch_mx<Sched::kDense>(g, sfa_mx, sfb_mx, stream);
}

int fp8_grouped_gemm_mx_contiguous(const uint8_t* qa, const uint8_t* sfa_mx, const uint8_t* qb,
                                   const uint8_t* sfb_mx, const int32_t* m_indices, void* c_bf16, int64_t M_tot,
                                   int64_t N, int64_t K, int64_t E, cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (M_tot < 0 || N < 0 || E < 0 || K < 128 || K % 128 || N % 128 || M_tot % 128 || M_tot >= kMaxRows ||
      K >= kMaxRows || E * N >= kMaxRows)
    return FP8Q_ERR_SHAPE;
  if (M_tot == 0 || N == 0 || E == 0) return FP8Q_OK;
  int rc = check_mx_operands(qa, sfa_mx, qb, sfb_mx, c_bf16);
  if (rc) return rc;
  if (!m_indices) return FP8Q_ERR_NULL;
  if (!aligned(m_indices, 4)) return FP8Q_ERR_ALIGN;
  GemmCall g{qa, nullptr, qb, nullptr, c_bf16, m_indices, nullptr, M_tot, M_tot, N, K, E, M_tot / kBlockM, 0, 1};
  return launch_mx<Sched::kContiguous>(g, sfa_mx, sfb_mx, stream);
}

int fp8_grouped_gemm_mx_masked(const uint8_t* qa, const uint8_t* sfa_mx, const uint8_t* qb, const uint8_t* sfb_mx,
                               const int32_t* masked_m, void* c_bf16, int64_t E, int64_t cap, int64_t N, int64_t K,
                               cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (E < 0 || cap < 0 || N < 0 || K < 128 || K % 128 || N % 128 || cap % 128 || E > kMaxMaskedExperts ||
      E * cap >= kMaxRows || E * N >= kMaxRows || K >= kMaxRows)
    return FP8Q_ERR_SHAPE;
  if (E == 0 || cap == 0 || N == 0) return FP8Q_OK;
  int rc = check_mx_operands(qa, sfa_mx, qb, sfb_mx, c_bf16);
  if (rc) return rc;
  if (!masked_m) return FP8Q_ERR_NULL;
  if (!aligned(masked_m, 4)) return FP8Q_ERR_ALIGN;
  GemmCall g{qa, nullptr, qb, nullptr, c_bf16, nullptr, masked_m, E * cap, cap, N, K, E, cap / kBlockM, 0, 1};
  return launch_mx<Sched::kMasked>(g, sfa_mx, sfb_mx, stream);
}

int fp8_transpose_w_128x128(const uint8_t* q, const float* s, int64_t G, int64_t N, int64_t K, uint8_t* qt,
                            float* st, cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (G < 0 || N < 0 || K < 0 || N % 128 || K % 128 || G >= kMaxRows || N >= kMaxRows || G * N >= kMaxRows ||
      K >= kMaxRows)
    return FP8Q_ERR_SHAPE;
  if (G == 0 || N == 0 || K == 0) return FP8Q_OK;
  if (!q || !s || !qt || !st) return FP8Q_ERR_NULL;
  if (!aligned(q, 16) || !aligned(qt, 16) || !aligned(s, 4) || !aligned(st, 4)) return FP8Q_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  const int64_t blocks = G * (N / 128) * (K / 128);
  const int64_t cap = static_cast<int64_t>(dev->num_sms) * 16;
  const int64_t grid = blocks < cap ? blocks : cap;
  transpose_w_128x128_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(q, s, qt, st, N, K, blocks);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

static int dense_common(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb, void* c, int64_t M,
                        int64_t N, int64_t K, int promote, cudaStream_t stream) {
  if (M < 0 || N < 0 || K < 128 || K % 128 || N % 128 || M >= kMaxRows || N >= kMaxRows || K >= kMaxRows)
    return FP8Q_ERR_SHAPE;
  if (M == 0 || N == 0) return FP8Q_OK;
  int rc = check_operands(qa, sa, qb, sb, c);
  if (rc) return rc;
  GemmCall g{qa, sa, qb, sb, c, nullptr, nullptr, M, M, N, K, 1, (M + kBlockM - 1) / kBlockM, 0, promote};
  return run_gemm<Sched::kDense>(g, stream);
}

int fp8_gemm_blockscaled(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb, void* c_bf16,
                         int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
  FP8Q_API_RANGE();
  return dense_common(qa, sa, qb, sb, c_bf16, M, N, K, 1, stream);
}

int fp8_gemm_unpromoted_diag(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb, void* c_bf16,
                             int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
  FP8Q_API_RANGE();
  return dense_common(qa, sa, qb, sb, c_bf16, M, N, K, 0, stream);
}

int fp8_grouped_gemm_contiguous(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb,
                                const int32_t* m_indices, void* c_bf16, int64_t M_tot, int64_t N, int64_t K,
                                int64_t E, cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (M_tot < 0 || N < 0 || E < 0 || K < 128 || K % 128 || N % 128 || M_tot % 128 || M_tot >= kMaxRows ||
      K >= kMaxRows || E * N >= kMaxRows)
    return FP8Q_ERR_SHAPE;
  if (M_tot == 0 || N == 0) return FP8Q_OK;
  if (E == 0) return FP8Q_OK;  // every block index is out of range: nothing is written
  int rc = check_operands(qa, sa, qb, sb, c_bf16);
  if (rc) return rc;
  if (!m_indices) return FP8Q_ERR_NULL;
  if (!aligned(m_indices, 4)) return FP8Q_ERR_ALIGN;
  GemmCall g{qa, sa, qb, sb, c_bf16, m_indices, nullptr, M_tot, M_tot, N, K, E, M_tot / kBlockM, 0, 1};
  return run_gemm<Sched::kContiguous>(g, stream);
}

int fp8_grouped_gemm_masked(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb,
                            const int32_t* masked_m, void* c_bf16, int64_t E, int64_t cap, int64_t N, int64_t K,
                            int64_t expected_m, cudaStream_t stream) {
  FP8Q_API_RANGE();
  if (E < 0 || cap < 0 || N < 0 || K < 128 || K % 128 || N % 128 || cap % 128 || E > kMaxMaskedExperts ||
      E * cap >= kMaxRows || E * N >= kMaxRows || K >= kMaxRows || expected_m < 0)
    return FP8Q_ERR_SHAPE;
  if (E == 0 || cap == 0 || N == 0) return FP8Q_OK;
  int rc = check_operands(qa, sa, qb, sb, c_bf16);
  if (rc) return rc;
  if (!masked_m) return FP8Q_ERR_NULL;
  if (!aligned(masked_m, 4)) return FP8Q_ERR_ALIGN;
  GemmCall g{qa, sa, qb, sb, c_bf16, nullptr, masked_m, E * cap, cap, N, K, E, cap / kBlockM, expected_m, 1};
  return run_gemm<Sched::kMasked>(g, stream);
}

int fp8_gemm_wgrad(const uint8_t* q_dy_t, const float* s_dy, const uint8_t* q_x_t, const float* s_x, void* dw_bf16,
                   int64_t N, int64_t K, int64_t Mp, cudaStream_t stream) {
  FP8Q_API_RANGE();
  // the contraction runs over Mp tokens in whole groups of four 128-token
  // slabs: the per-row scales of both operands are staged a group at a time
  if (N < 0 || K < 0 || Mp < 512 || N % 128 || K % 128 || Mp % 512 || N >= kMaxRows || K >= kMaxRows ||
      Mp >= kMaxRows)
    return FP8Q_ERR_SHAPE;
  if (N == 0 || K == 0) return FP8Q_OK;
  if (!q_dy_t || !s_dy || !q_x_t || !s_x || !dw_bf16) return FP8Q_ERR_NULL;
  if (!aligned(q_dy_t, 16) || !aligned(q_x_t, 16) || !aligned(dw_bf16, 16) || !aligned(s_dy, 16) ||
      !aligned(s_x, 16))
    return FP8Q_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  // C [N, K] = A [N, Mp] * B [K, Mp]^T: GEMM rows N, columns K, depth Mp
  GemmCall g{q_dy_t, s_dy, q_x_t, s_x, dw_bf16, nullptr, nullptr, N, N, K, Mp, 1, N / kBlockM, 0, 1};
  return launch_gemm<kTileN, kStages128, Sched::kDense, true, true, true>(g, *dev, stream);
}

const char* fp8q_status_string(int status) {
  switch (status) {
    case FP8Q_OK: return "ok";
    case FP8Q_ERR_NULL: return "null pointer";
    case FP8Q_ERR_SHAPE: return "invalid shape";
    case FP8Q_ERR_ALIGN: return "misaligned pointer";
    case FP8Q_ERR_CUDA: return "CUDA error";
    case FP8Q_ERR_TIMEOUT: return "device wait timed out";
    case FP8Q_ERR_UNSUPPORTED: return "unsupported device or limit";
    default: return "unknown status";
  }
}

int fp8q_get_device_error(cudaStream_t stream) {
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  uint32_t* taken = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&taken), g_device_status_taken) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  taken += g_take_slot.fetch_add(1) % kTakeSlots;
  status_take_kernel<<<1, 1, 0, stream>>>(dev->status, taken);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, taken, sizeof v, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  if (v == 0) return FP8Q_OK;
  return (v & kDevErrTimeout) ? FP8Q_ERR_TIMEOUT : FP8Q_ERR_CUDA;
}

int fp8q_set_wait_timeout_ns(uint64_t timeout_ns) {
  g_timeout_ns.store(timeout_ns ? timeout_ns : kDefaultTimeoutNs);
  return FP8Q_OK;
}

int fp8q_selftest_wait_timeout(uint64_t timeout_ns, cudaStream_t stream) {
  FP8Q_API_RANGE();
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  wait_selftest_kernel<<<1, 32, 0, stream>>>(dev->status, timeout_ns);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FP8Q_OK;
}

uint64_t fp8q_launch_count(void) { return g_launches.load(); }

}  // extern "C"
