/*
 * fp8q.h -- C ABI of the fine-grained FP8 quantization + block-scaled FP8 GEMM
 * library for NVIDIA B200 (sm_100a).
 *
 * The method (sources cited by page title and passage):
 *  - "The Insider Secrets Of Deepseek Discovered", FP8 mixed-precision passage:
 *    activations are scaled per 1x128 tile (one scale per token per 128
 *    channels) and weights per 128x128 block, Figure 7 (a); the group's largest
 *    magnitude is mapped onto the largest FP8 value; tensor-core partial sums
 *    are promoted to FP32 on CUDA cores at fixed K intervals, where the
 *    dequantization scales are applied, Figure 7 (b).
 *  - codingmall "DeepSeek-V3 FP8" page (Korean), sections on online
 *    quantization (scales computed from the current tile), increased
 *    accumulation precision, and the unified E4M3 format.
 *  - "Deepgemm lancado no dia 4 da semana de codigo aberto Deepseek", sections
 *    "O que e FP8?" (E4M3: 1 sign, 4 exponent, 3 mantissa bits) and
 *    "Necessidade de DeepGemm" / "Principais caracteristicas" (dense GEMM plus
 *    two MoE grouped layouts, contiguous and masked).
 *
 * Conventions shared by every entry point:
 *  - All data pointers are DEVICE pointers on the current CUDA device; the
 *    caller owns and allocates every buffer.  No call allocates memory.
 *  - Every call is asynchronous on `stream` and never synchronizes the host.
 *  - All tensors are dense and row-major (last index fastest).  FP8 tensors
 *    hold E4M3FN codes (bias 7, largest finite 448 = 0x7E, NaN = 0x7F/0xFF, no
 *    infinities; byte-compatible with torch.float8_e4m3fn).  bf16 tensors hold
 *    IEEE bfloat16.  Scale tensors are float32.
 *  - Quantization rule (per group): s = fl32(amax / 448) with IEEE division,
 *    s = 1 when that is zero; q = E4M3(fl32(x / s)) rounded to nearest even,
 *    saturating at +-448, subnormal E4M3 codes down to 2^-9, sign of zero kept.
 *  - Argument errors return a non-zero status before anything is launched
 *    (no side effects).  A failed launch returns FP8Q_ERR_CUDA.
 *  - Pointer alignment: the quantizers' bf16 inputs 32 bytes; every other
 *    bf16 / FP8 / output pointer 16 bytes; scale and index pointers 4 bytes.
 *  - Size limits: every row count, column count and K below 2^31, and so are
 *    the stacked row counts E*N, G*N and E*cap; a GEMM's count of 128-row
 *    output tiles times its column tiles (times E for the masked layout) stays
 *    below 2^31 - 2^16; larger shapes return FP8Q_ERR_SHAPE.
 *  - Non-finite inputs are outside the contract (results unspecified, no fault).
 *  - Every on-device wait is bounded (default 4 s, see fp8q_set_wait_timeout_ns);
 *    a wait that runs out records FP8Q_ERR_TIMEOUT in a device status word
 *    (one per device), the kernel lets its copies and MMAs in flight finish
 *    (a fixed bound, independent of the wait limit), releases its resources
 *    and returns, and the host reads the word with fp8q_get_device_error.
 */
#ifndef FP8Q_H_
#define FP8Q_H_

#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define FP8Q_API __attribute__((visibility("default")))
#else
#define FP8Q_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP8Q_OK = 0,
  FP8Q_ERR_NULL = 1,        /* a required pointer is NULL */
  FP8Q_ERR_SHAPE = 2,       /* a size is negative, not a multiple of 128 where required, or too large */
  FP8Q_ERR_ALIGN = 3,       /* a pointer is not aligned as required */
  FP8Q_ERR_CUDA = 4,        /* the CUDA runtime/driver reported an error */
  FP8Q_ERR_TIMEOUT = 5,     /* a bounded on-device wait ran out (read via fp8q_get_device_error) */
  FP8Q_ERR_UNSUPPORTED = 6  /* device is not sm_100 or a limit of this build is exceeded */
} fp8q_status;

/*
 * Activation quantization, 1x128 tiles ("The Insider Secrets Of Deepseek
 * Discovered", Figure 7 (a), item 1; codingmall page, online quantization).
 *   x_bf16 : [M, K] bf16, read only.
 *   q      : [M, K] E4M3 codes, written.
 *   s      : [M, K/128] float32, written; s[m, kb] is the scale of
 *            x[m, 128*kb .. 128*kb+127].
 * K must be a multiple of 128.  M == 0 or K == 0 is a no-op.
 */
FP8Q_API int fp8_quant_act_1x128(const void* x_bf16, int64_t M, int64_t K, uint8_t* q, float* s, cudaStream_t stream);

/*
 * Weight quantization, 128x128 blocks (same passage, item 2).
 *   w_bf16 : [G, N, K] bf16 (G stacked [out_features, in_features] matrices;
 *            G = 1 for one matrix), read only.
 *   q      : [G, N, K] E4M3 codes, written.
 *   s      : [G, N/128, K/128] float32, written; s[g, nb, kb] is the scale of
 *            rows 128*nb..+127, columns 128*kb..+127 of matrix g.
 * N and K must be multiples of 128.  Any zero size is a no-op.
 */
FP8Q_API int fp8_quant_w_128x128(const void* w_bf16, int64_t G, int64_t N, int64_t K, uint8_t* q, float* s,
                        cudaStream_t stream);

/*
 * Both operands of one GEMM in a single launch: exactly the codes and scales
 * of fp8_quant_act_1x128(x) and fp8_quant_w_128x128(w), bit for bit (the
 * same per-group rule: "The Insider Secrets Of Deepseek Discovered", FP8
 * passage, Figure 7 (a)).  One launch instead of two, so the ramp-up and the
 * last partial wave of a launch are paid once per GEMM step.
 *   x_bf16, M, K, qa, sa     : as fp8_quant_act_1x128 (M = 0 or K = 0: no activations)
 *   w_bf16, G, N, Kw, qw, sw : as fp8_quant_w_128x128 (G, N or Kw = 0: no weights)
 * Same requirements and errors as the two calls; the argument checks of both
 * run before anything is launched.
 */
FP8Q_API int fp8_quant_act_w(const void* x_bf16, int64_t M, int64_t K, uint8_t* qa, float* sa, const void* w_bf16,
                             int64_t G, int64_t N, int64_t Kw, uint8_t* qw, float* sw, cudaStream_t stream);

/*
 * The same two quantizers with power-of-two (UE8M0) group scales: the
 * microscaling form the first page names for Blackwell ("The Insider Secrets
 * Of Deepseek Discovered", fine-grained quantization in step with
 * microscaling formats).  s = 2^e with e the least integer such that
 * 448 * 2^e >= amax, clamped to [-127, 127] (amax == 0: s = 1), so no code
 * saturates and q = E4M3_RNE(x * 2^-e) exactly.  Scales are written as
 * float32 powers of two, in the same layouts as above, so the GEMMs accept
 * them unchanged.  Same shapes, alignment and errors as the entry points
 * above.
 */
FP8Q_API int fp8_quant_act_1x128_ue8m0(const void* x_bf16, int64_t M, int64_t K, uint8_t* q, float* s,
                                       cudaStream_t stream);
FP8Q_API int fp8_quant_w_128x128_ue8m0(const void* w_bf16, int64_t G, int64_t N, int64_t K, uint8_t* q, float* s,
                                       cudaStream_t stream);

/*
 * Activation quantization along the token axis, 128x1 tiles (for the weight
 * gradient dW = dY^T X, which contracts over tokens; "The Insider Secrets Of
 * Deepseek Discovered", Figure 6: Fprop, Dgrad and Wgrad all run in FP8).
 * Same per-group rule as fp8_quant_act_1x128, over a channel's run of 128
 * tokens instead of a token's run of 128 channels.
 *   x_bf16 : [M, K] bf16 (tokens x channels), read only.
 *   q      : [M, K] E4M3 codes, written.
 *   s      : [ceil(M/128), K] float32, written; s[mb, k] is the scale of
 *            x[128*mb .. min(M, 128*mb+128) - 1, k] (a ragged last group of
 *            tokens takes its own scale).
 * K must be a multiple of 128; any M >= 0.  x, q and s 16-byte aligned.
 */
FP8Q_API int fp8_quant_act_128x1(const void* x_bf16, int64_t M, int64_t K, uint8_t* q, float* s, cudaStream_t stream);

/*
 * SwiGLU between the two MoE GEMMs fused with the 1x128 requantization of its
 * output (the chained MoE decode; the SwiGLU is not on the pages: the MoE
 * configurations' GEMM1 width, twice GEMM2's depth, implies it):
 *   h[r, i] = bf16_rne( g / (1 + exp(-g)) * u ),  g = c1[r, i], u = c1[r, inter + i]
 * (the correctly rounded bf16 of the real-valued expression), then qh, sh =
 * the fp8_quant_act_1x128 quantization of h.
 *   c1_bf16  : [rows, 2*inter] bf16 (GEMM1's output, [gate | up] halves), read only.
 *   masked_m : NULL (every row valid), or the masked layout's [rows/cap] int32
 *              counts: row e*cap + r is valid when r < clamp(masked_m[e], 0, cap);
 *              invalid rows of qh and sh are left unwritten (their c1 rows are
 *              not read).
 *   qh       : [rows, inter] E4M3, sh : [rows, inter/128] f32, written.
 * inter a multiple of 128; with masked_m, cap > 0 divides rows.  c1 32-byte,
 * qh 16-byte, sh and masked_m 4-byte aligned.
 */
FP8Q_API int fp8_swiglu_quant_1x128(const void* c1_bf16, int64_t rows, int64_t inter, const int32_t* masked_m,
                                    int64_t cap, uint8_t* qh, float* sh, cudaStream_t stream);

/*
 * The same token-axis quantization with the codes written token-contiguous,
 * the operand layout of the weight-gradient GEMM fp8_gemm_wgrad:
 *   x_bf16 : [M, K] bf16 (tokens x channels), read only.
 *   Mp     : padded token count, a multiple of 128 with Mp >= M
 *            (fp8_gemm_wgrad takes multiples of 512).
 *   qt     : [K, Mp] E4M3 codes, written; qt[k, m] is the code of x[m, k],
 *            and 0 for m >= M.
 *   s      : [Mp/128, K] float32, written; rows below ceil(M/128) are the
 *            scales of fp8_quant_act_128x1, the rows of groups made only of
 *            padding are 1 (the zero-group rule).
 * K a multiple of 128; any M >= 0.  x, qt and s 16-byte aligned.
 */
FP8Q_API int fp8_quant_act_128x1_t(const void* x_bf16, int64_t M, int64_t K, int64_t Mp, uint8_t* qt, float* s,
                                   cudaStream_t stream);

/*
 * Transposition of 128x128-block-quantized weights (for the activation
 * gradient dX = dY W, the Dgrad GEMM of the same Figure 6): a 128x128 block
 * of W^T has the same amax, scale and codes as W's block, transposed.
 *   q  : [G, N, K] E4M3 codes, s : [G, N/128, K/128] (from fp8_quant_w_128x128)
 *   qt : [G, K, N] E4M3 codes, st : [G, K/128, N/128], written.
 * Then fp8_gemm_blockscaled(q_dy, s_dy, qt, st, dX, M, K, N) computes
 * dX = dY W with dY 1x128-quantized (fp8_quant_act_1x128 of dY [M, N]).
 * N, K multiples of 128.  q, qt 16-byte aligned; s, st 4-byte aligned.
 */
FP8Q_API int fp8_transpose_w_128x128(const uint8_t* q, const float* s, int64_t G, int64_t N, int64_t K, uint8_t* qt,
                                     float* st, cudaStream_t stream);

/*
 * Dense block-scaled FP8 GEMM, C = A * B^T, with promotion at every 128-wide
 * K slab ("The Insider Secrets Of Deepseek Discovered", Figure 7 (b); codingmall
 * page, increased accumulation precision):
 *   C[m,n] = bf16_rne( sum_kb sa[m,kb] * sb[n/128,kb] * sum_{k in slab kb} A[m,k] * B[n,k] )
 * where each slab's partial sum comes from the tensor cores in FP32 and the
 * scaled sum over slabs is kept in FP32 registers.
 *   qa : [M, K] E4M3, sa : [M, K/128] f32   (from fp8_quant_act_1x128)
 *   qb : [N, K] E4M3, sb : [N/128, K/128] f32 (from fp8_quant_w_128x128, G = 1)
 *   c_bf16 : [M, N] bf16, written (every element).
 * K >= 128 and K, N multiples of 128; any M >= 0 (M == 0 or N == 0: no-op).
 * Performance note (all three GEMM forms): when K is a multiple of 512 and
 * sa, sb are 16-byte aligned, the scales travel to the SM with the operand
 * tiles (TMA); otherwise each is fetched from global memory.  The results
 * are bit-identical either way.
 */
FP8Q_API int fp8_gemm_blockscaled(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb, void* c_bf16,
                         int64_t M, int64_t N, int64_t K, cudaStream_t stream);

/*
 * Grouped GEMM, contiguous layout ("Deepgemm lancado ...", MoE grouped GEMM
 * kinds): the rows of all experts are concatenated, each expert's run padded
 * to a multiple of 128 rows.
 *   qa : [M_tot, K], sa : [M_tot, K/128]
 *   qb : [E, N, K], sb : [E, N/128, K/128]
 *   m_indices : [M_tot/128] int32 (device): expert of each 128-row block.
 *   c_bf16 : [M_tot, N] bf16.  Rows of block b are A[b]*B[m_indices[b]]^T.
 *   A block whose index is outside [0, E) is skipped and its C rows are left
 *   unwritten.  Padding rows are computed like any row (zero rows give zero).
 * M_tot, N, K multiples of 128, K >= 128.
 */
FP8Q_API int fp8_grouped_gemm_contiguous(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb,
                                const int32_t* m_indices, void* c_bf16, int64_t M_tot, int64_t N, int64_t K,
                                int64_t E, cudaStream_t stream);

/*
 * Grouped GEMM, masked layout (same page): expert e owns a fixed capacity of
 * `cap` rows of which only the first masked_m[e] are valid; the counts stay on
 * the device, so the call never synchronizes and can sit in a CUDA graph.
 *   qa : [E, cap, K], sa : [E, cap, K/128]
 *   qb : [E, N, K],   sb : [E, N/128, K/128]
 *   masked_m : [E] int32 (device); values are clamped to [0, cap].
 *   c_bf16 : [E, cap, N] bf16; rows m >= masked_m[e] are left unwritten.
 *   expected_m : hint of the typical valid count (may be 0); results never
 *   depend on it.
 * cap, N, K multiples of 128, K >= 128, E <= 1024.
 */
FP8Q_API int fp8_grouped_gemm_masked(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb,
                            const int32_t* masked_m, void* c_bf16, int64_t E, int64_t cap, int64_t N, int64_t K,
                            int64_t expected_m, cudaStream_t stream);

/*
 * Weight-gradient GEMM dW = dY^T X over tokens ("The Insider Secrets Of
 * Deepseek Discovered", Figure 6, Wgrad in FP8), with both operands
 * quantized along tokens (fp8_quant_act_128x1_t of dY [M, N] and of X [M, K]):
 *   dW[n,k] = bf16_rne( sum_mb s_dy[mb,n] * s_x[mb,k] * sum_{m in slab mb} dY[m,n] * X[m,k] )
 * with the same per-slab FP32 promotion as fp8_gemm_blockscaled, each slab's
 * partial scaled by one A-row scale and one scale per output column.
 *   q_dy_t : [N, Mp] E4M3, s_dy : [Mp/128, N] f32
 *   q_x_t  : [K, Mp] E4M3, s_x  : [Mp/128, K] f32
 *   dw_bf16: [N, K] bf16, written.
 * N, K multiples of 128; Mp a multiple of 512 (whole groups of four token
 * slabs), Mp >= 512.  Every pointer 16-byte aligned.
 */
FP8Q_API int fp8_gemm_wgrad(const uint8_t* q_dy_t, const float* s_dy, const uint8_t* q_x_t, const float* s_x,
                            void* dw_bf16, int64_t N, int64_t K, int64_t Mp, cudaStream_t stream);

/*
 * Block-scaled FP8 GEMM with power-of-two (UE8M0) scales applied by the
 * tensor cores ("The Insider Secrets Of Deepseek Discovered", FP8 passage:
 * the microscaling form Blackwell's tensor cores support):
 *   C[m,n] = bf16_rne( sum_kb sa[m,kb] * sb[n/128,kb] * sum_{k in slab kb} A[m,k] * B[n,k] )
 * with every sa, sb a power of two (fp8_quant_act_1x128_ue8m0,
 * fp8_quant_w_128x128_ue8m0), the whole K accumulated in FP32 in the tensor
 * cores, no CUDA-core promotion.  The scales go in as E8M0 atoms:
 *   fp8_mx_scales_act: sa [M, K/128] f32 -> sfa_mx [ceil(M/128), K/128, 512] bytes
 *   fp8_mx_scales_w  : sb [G, N/128, K/128] f32 -> sfb_mx [G*N/128, K/128, 512] bytes
 * (one 512-byte atom per 128-row tile and 128-deep K slab: byte
 * 16*m0 + 4*m1 + j = E8M0 of row 32*m1 + m0 of the tile for the slab's
 * 32-element K block j, the four j equal; a normal scale that is not a
 * power of two is truncated to the power of two below it).
 *   qa : [M, K] E4M3, qb : [N, K] E4M3, c_bf16 : [M, N] bf16.
 * N, K multiples of 128; any M >= 0.  sfa_mx, sfb_mx and every code/output
 * pointer 16-byte aligned; sa, sb 4-byte aligned.
 */
FP8Q_API int fp8_mx_scales_act(const float* sa, int64_t M, int64_t K, uint8_t* sfa_mx, cudaStream_t stream);
FP8Q_API int fp8_mx_scales_w(const float* sb, int64_t G, int64_t N, int64_t K, uint8_t* sfb_mx, cudaStream_t stream);
FP8Q_API int fp8_gemm_mx(const uint8_t* qa, const uint8_t* sfa_mx, const uint8_t* qb, const uint8_t* sfb_mx,
                         void* c_bf16, int64_t M, int64_t N, int64_t K, cudaStream_t stream);

/*
 * The two MoE layouts of fp8_gemm_mx, with the arguments and semantics of
 * fp8_grouped_gemm_contiguous / fp8_grouped_gemm_masked: sfa_mx holds the
 * atoms of qa's 128-row blocks (fp8_mx_scales_act of its [M_tot or E*cap,
 * K/128] scales), sfb_mx those of qb [E, N, K] (fp8_mx_scales_w with G = E).
 */
FP8Q_API int fp8_grouped_gemm_mx_contiguous(const uint8_t* qa, const uint8_t* sfa_mx, const uint8_t* qb,
                                            const uint8_t* sfb_mx, const int32_t* m_indices, void* c_bf16,
                                            int64_t M_tot, int64_t N, int64_t K, int64_t E, cudaStream_t stream);
FP8Q_API int fp8_grouped_gemm_mx_masked(const uint8_t* qa, const uint8_t* sfa_mx, const uint8_t* qb,
                                        const uint8_t* sfb_mx, const int32_t* masked_m, void* c_bf16, int64_t E,
                                        int64_t cap, int64_t N, int64_t K, cudaStream_t stream);

/*
 * Accumulation diagnostic ("The Insider Secrets Of Deepseek Discovered": the
 * drift of limited-precision tensor-core accumulation over long K, Figure 7 (b)
 * is its remedy).  Same operands and layouts as fp8_gemm_blockscaled, but the
 * whole K range is accumulated inside the tensor cores with no promotion; the
 * result is scaled once by sa[m,0] * sb[n/128,0].  Only meaningful for
 * per-tensor scales (every sa and sb entry equal); used to measure the
 * tensor cores' own accumulation precision.  Not part of the quantized path.
 */
FP8Q_API int fp8_gemm_unpromoted_diag(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb, void* c_bf16,
                             int64_t M, int64_t N, int64_t K, cudaStream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
FP8Q_API const char* fp8q_status_string(int status);

/*
 * Reads and clears, in one atomic exchange queued on `stream` after the work
 * already on it, the device status word that bounded waits write, then
 * synchronizes `stream`.  Returns FP8Q_OK, FP8Q_ERR_TIMEOUT, or FP8Q_ERR_CUDA
 * if the launch or the synchronization failed.
 * The word is one per device, shared by every stream and every call of the
 * library on that device: a timeout is not attributed to a call or a stream,
 * and a call still running on another stream may record one after the
 * exchange (it is then reported by the next query).  Queries that overlap
 * on different streams each get the value their own exchange took (up to 64
 * queries in flight at once).  A timeout also covers a kernel's final drain
 * running out of its fixed bound (2 s) after an abort.
 */
FP8Q_API int fp8q_get_device_error(cudaStream_t stream);

/* Sets the limit of every later on-device wait, in nanoseconds (0 restores
 * the 4 s default).  Host-side setting; affects launches made after it. */
FP8Q_API int fp8q_set_wait_timeout_ns(uint64_t timeout_ns);

/*
 * Self-test of the bounded-wait path: launches one CTA that waits on an
 * mbarrier nothing will ever complete, with the given limit, so the wait runs
 * out, records FP8Q_ERR_TIMEOUT and the kernel returns normally.  Nothing
 * faults or hangs.  Returns the launch status; read the recorded status with
 * fp8q_get_device_error.
 */
FP8Q_API int fp8q_selftest_wait_timeout(uint64_t timeout_ns, cudaStream_t stream);

/* Number of the library's kernels launched since load (host-side counter),
 * for launch accounting in benchmarks. */
FP8Q_API uint64_t fp8q_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H_ */
