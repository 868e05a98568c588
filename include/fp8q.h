/*
 * fp8q — FP8 W8A8 linear layers for NVIDIA B200 (sm_100a).  C ABI.
 *
 * The method (two web pages on quantized inference for the OneRec-V2
 * generative recommender):
 *   [P1] "Quantized Inference for OneRec-V2：生成式推荐开始直接吃 LLM 量化栈",
 *        section 关键证据: linear weights quantized offline per output
 *        channel; activations quantized per token at run time; the matmul runs
 *        on FP8 tensor cores with FP32 accumulation; the output is cast back to
 *        FP16.  Covered layers: attention QKV/O projections, dense FFN linears
 *        and the sparse-MoE expert grouped GEMM.
 *   [P2] "FP8量化在生成式推荐系统OneRec-V2中的优化实践", §1.2 (FP8 range ±448),
 *        §2.2 (E4M3; per-token dynamic scale = max_code / max(|x|, eps)),
 *        §2.3 (FP8 multiply + FP32 accumulate + FP16 output, Q+GEMM+DQ fused).
 *
 * Numerics, identical in every entry point:
 *   per row:  a' = max(max_k |A[k]|, 1e-12f)
 *             r  = 448 / a'   (IEEE fp32 division, round to nearest)
 *             s  = a' / 448   (IEEE fp32 division, round to nearest; stored)
 *             q[k] = E4M3(fl32(A[k] * r)), round-to-nearest-even, saturating
 *                    to ±448; -0.0 keeps its sign.
 *   linear:   Y[m,n] = fp16_rn( fl32( fl32(acc[m,n] * s_x[m]) * s_w[n] ) ),
 *             acc = FP32 tensor-core accumulation of E4M3 x E4M3 products.
 *
 * Conventions for every entry point:
 *   - Matrices are row-major and dense.  X, W and Y are fp16 ([M,K], [N,K],
 *     [M,N]; K is the contiguous dimension of X and W, like nn.Linear);
 *     E4M3 codes are uint8 with the same layout as their source.
 *   - Every pointer argument is a CUDA device pointer owned by the caller,
 *     allocated on the device that is current when the call is made, and
 *     16-byte aligned.  Outputs must not alias inputs.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work and return; they never synchronize, except
 *     fp8q_device_error().
 *   - Arguments are validated on the host before anything is enqueued; a
 *     rejected call enqueues nothing and returns FP8Q_ERR_INVALID_ARG or
 *     FP8Q_ERR_UNSUPPORTED.  A failed launch returns FP8Q_ERR_CUDA
 *     (fp8q_last_error_message() holds the CUDA error text).
 *   - Shape rules: M, rows >= 0 (0 is a no-op), N > 0, K > 0, K % 16 == 0
 *     (16-byte TMA rows for the FP8 operands), N % 8 == 0 (16-byte fp16
 *     output rows), all sizes < 2^31.
 *   - Kernels bound every wait on the GPU (about 2 s); a wait that runs out
 *     sets a device error word instead of hanging, readable with
 *     fp8q_device_error().
 *   - No call allocates device memory.  Results are bitwise reproducible from
 *     run to run (fixed reduction order everywhere).
 *   - Kernels are chained with programmatic dependent launch: a kernel may
 *     start while the one before it on the stream finishes, and waits for it
 *     before touching its outputs.  The linear kernels treat the quantized
 *     weights (Wq, s_w) as static and begin loading Wq before that wait, so
 *     Wq must not be written by the work enqueued just before the call.  The
 *     weight quantizers of this library (per channel, per tensor, block-wise)
 *     let the next kernel start only once they have finished, so quantizing
 *     the weights and then calling a linear on the same stream is safe.
 */
#ifndef FP8Q_H_
#define FP8Q_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP8Q_OK = 0,
  FP8Q_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment       */
  FP8Q_ERR_UNSUPPORTED = 2,   /* valid request this library cannot serve    */
  FP8Q_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed          */
  FP8Q_ERR_TIMEOUT = 4,       /* a device wait ran out (fp8q_device_error)  */
  FP8Q_ERR_DEVICE_CHECK = 5   /* a device-side input check failed           */
} fp8q_status;

/* Device error-word bits reported by fp8q_device_error(). */
#define FP8Q_DEVERR_TIMEOUT_PRODUCER 0x1u
#define FP8Q_DEVERR_TIMEOUT_MMA      0x2u
#define FP8Q_DEVERR_TIMEOUT_EPILOGUE 0x4u
#define FP8Q_DEVERR_BAD_OFFSETS      0x8u
#define FP8Q_DEVERR_TIMEOUT_CLUSTER  0x10u
#define FP8Q_DEVERR_TIMEOUT_SELFTEST 0x20u

/* Human-readable name of a status code.  Never returns NULL. */
const char* fp8q_status_string(int status);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char* fp8q_last_error_message(void);

/* ABI version of this library (major * 100 + minor). */
int fp8q_version(void);

/*
 * Per-token dynamic activation quantization  [P1 关键证据 step 2; P2 §2.2].
 *   X_f16 [M,K] fp16 in;  Xq [M,K] uint8 E4M3 out;  s_x [M] fp32 out.
 * One scale per row, computed at run time from the row's max |x|.
 * M == 0 is a no-op.
 */
fp8q_status fp8q_quantize_rows_dynamic(const void* X_f16, int64_t M, int64_t K,
                                       uint8_t* Xq, float* s_x, void* stream);

/*
 * Per-output-channel weight quantization, done once offline  [P1 关键证据
 * step 1; P2 §2.1 per-channel for the QKV projection].
 *   W_f16 [N,K] fp16 in;  Wq [N,K] uint8 E4M3 out;  s_w [N] fp32 out.
 * For MoE expert weights [E,N_e,K] pass N = E * N_e (one scale per row of
 * every expert).  Same arithmetic as fp8q_quantize_rows_dynamic.
 */
fp8q_status fp8q_quantize_weight_per_channel(const void* W_f16, int64_t N, int64_t K,
                                             uint8_t* Wq, float* s_w, void* stream);

/*
 * FP8 W8A8 linear with fused dequantization  [P1 关键证据 steps 3-4;
 * P2 §2.3 "FP8 multiply + FP32 accumulate + FP16 output"].
 *   Xq [M,K] uint8, s_x [M] fp32, Wq [N,K] uint8, s_w [N] fp32 in;
 *   Y_f16 [M,N] fp16 out:  Y = fp16(((Xq . Wq^T) * s_x[:,None]) * s_w[None,:]).
 * M == 0 is a no-op.
 */
fp8q_status fp8q_linear(const uint8_t* Xq, const float* s_x,
                        const uint8_t* Wq, const float* s_w,
                        int64_t M, int64_t N, int64_t K,
                        void* Y_f16, void* stream);

/*
 * Quantize + FP8 linear + dequantize from fp16 activations  [P2 §2.3: the
 * QuantizeLinear + GEMM + Dequantize fusion; P1 关键证据 steps 2-4].
 *   X_f16 [M,K] fp16, Wq [N,K] uint8 and s_w [N] fp32 (per-channel
 *   quantized weights) in;  Y_f16 [M,N] fp16 out.  Same results as
 *   fp8q_quantize_rows_dynamic followed by fp8q_linear.
 * With a workspace (Xq_ws [M,K] uint8 and s_x_ws [M] fp32, both non-NULL)
 * the call runs the two steps through it (the workspace then holds the codes
 * and scales).  With Xq_ws = s_x_ws = NULL and up to 64 token rows (K up to
 * 4096 x the split factor) it is one fused kernel: the CTAs of a split-K
 * cluster each take the row maxima over their own K slice, exchange them,
 * and write the E4M3 codes of their slice in shared memory, so no
 * intermediate touches HBM.  NULL workspace with a larger shape returns
 * FP8Q_ERR_INVALID_ARG.
 */
fp8q_status fp8q_quantized_linear(const void* X_f16, const uint8_t* Wq, const float* s_w,
                                  int64_t M, int64_t N, int64_t K, void* Y_f16,
                                  uint8_t* Xq_ws, float* s_x_ws, void* stream);

/*
 * fp8q_quantized_linear as ONE kernel for M > 128 rows  [P2 §2.3: the
 * QuantizeLinear + GEMM + Dequantize fusion]: the CTA-pair GEMM's epilogue
 * warps quantize the fp16 rows (same steps, codes and scales as
 * fp8q_quantize_rows_dynamic) into Xq_ws [M,K] uint8 / s_x_ws [M] fp32 while
 * its tensor cores start on the 128-row blocks already published; Y as
 * fp8q_quantized_linear.  sync_ws: uint32 [fp8q_overlap_sync_words(M)],
 * device, ZERO-FILLED before the first call; every call that completes
 * leaves it zero again.  Calls sharing one sync_ws must not overlap on the
 * GPU; after a device error (fp8q_device_error() != 0) zero it again.  With
 * M <= 128 the call runs the two-step path of fp8q_quantized_linear
 * (sync_ws untouched).  All pointers 16-byte aligned.
 */
fp8q_status fp8q_quantized_linear_overlapped(const void* X_f16, const uint8_t* Wq, const float* s_w,
                                             int64_t M, int64_t N, int64_t K, void* Y_f16,
                                             uint8_t* Xq_ws, float* s_x_ws, uint32_t* sync_ws,
                                             void* stream);

/* Number of uint32 words fp8q_quantized_linear_overlapped needs in sync_ws
 * for M rows: 2 + 2 * ceil(M / 128). */
int64_t fp8q_overlap_sync_words(int64_t M);

/*
 * Allocation-free form of fp8q_quantized_linear (the pages have no
 * counterpart; this is a deployment convenience).  Same inputs, output and
 * numerics as fp8q_quantized_linear with a workspace, but the codes and
 * scales between the quantizer and the GEMM live in a fixed scratch array
 * built into the library, so the caller passes only X, the quantized weights
 * and Y.  It is for callers that cannot call cudaMalloc -- for example code
 * running inside a host framework that owns all device memory through its own
 * pre-sized pool, or a serving loop that must never trigger an allocation
 * (and the device synchronization it can cause) once it is running.
 *   Limits: M*K <= 8388608 and M <= 16384, else FP8Q_ERR_INVALID_ARG with an
 *   explanatory message (fp8q_last_error_message()).  The scratch costs every
 *   GPU that loads the library 8 MiB + 64 KiB of device memory until exit.
 *   The first call on a device looks up the scratch address for that device
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture on the device.  A failed lookup returns
 *   FP8Q_ERR_CUDA and is not remembered: the next call tries again.
 *   All calls on a device share the one scratch array and nothing in it needs
 *   to start at zero (each call overwrites the codes and scales it reads);
 *   two calls whose work overlaps on the GPU (different streams without
 *   ordering) race on it and give wrong results.  No call allocates memory.
 */
fp8q_status fp8q_quantized_linear_noalloc(const void* X_f16, const uint8_t* Wq, const float* s_w,
                                          int64_t M, int64_t N, int64_t K, void* Y_f16, void* stream);

/*
 * MoE expert grouped FP8 linear  [P1 关键证据 item 2: Sparse MoE grouped
 * GEMM; P2 §3.2 MoE acceleration].
 *   Xq [rows,K] uint8 and s_x [rows] fp32: token rows already grouped by
 *       expert (rows offsets[e] .. offsets[e+1]-1 go to expert e);
 *   offsets [E+1] int32, DEVICE memory, non-decreasing, offsets[0] == 0,
 *       offsets[E] == rows (read on the device; the host never syncs on it);
 *   Wq [E,N,K] uint8 and s_w [E,N] fp32: per-expert weights and
 *       per-channel scales;
 *   Y_f16 [rows,N] fp16 out: row i of group e = linear of that row with W_e.
 * Empty groups are legal.  Offsets that break the rules are detected on the
 * device: nothing is written and fp8q_device_error() reports
 * FP8Q_DEVERR_BAD_OFFSETS.  E >= 1 and E <= 1024.
 */
fp8q_status fp8q_moe_grouped_linear(const uint8_t* Xq, const float* s_x,
                                    const int32_t* offsets, int32_t E, int64_t rows,
                                    const uint8_t* Wq, const float* s_w,
                                    int64_t N, int64_t K,
                                    void* Y_f16, void* stream);

/* ---------------------------------------------------------------------------
 * Variants described on the pages [P2]: E5M2 activations (§2.2), a
 * per-tensor weight scale for the FFN linears (§2.1) and 128 x 128
 * block-wise weight scales for the MoE experts (§2.1, §2.2).  Same
 * conventions as above.
 */

/* FP8 code format of the activations: E4M3 (the path's format) or E5M2
 * [P2 §2.2: 5 exponent and 2 mantissa bits; largest finite value 57344]. */
typedef enum {
  FP8Q_FMT_E4M3 = 0,
  FP8Q_FMT_E5M2 = 1
} fp8q_format;

/*
 * fp8q_quantize_rows_dynamic with the code format chosen by fmt.  For
 * FP8Q_FMT_E5M2 the steps use max_code = 57344 instead of 448:
 * r = 57344 / a', s = a' / 57344, q = E5M2(fl32(x * r)), round-to-nearest-
 * even, saturating to ±57344 (never infinity).  Any other fmt value returns
 * FP8Q_ERR_INVALID_ARG.
 */
fp8q_status fp8q_quantize_rows_dynamic_fmt(const void* X_f16, int64_t M, int64_t K, fp8q_format fmt,
                                           uint8_t* Xq, float* s_x, void* stream);

/*
 * Per-tensor weight quantization  [P2 §2.1: the FFN linear transforms use
 * per-tensor quantization].  W_f16 [N,K] fp16 in; Wq [N,K] uint8 E4M3 and
 * s_w [N] fp32 out.  One scale for the whole matrix: a' = max(max |W|,
 * 1e-12), then r, s and the codes as for fp8q_quantize_rows_dynamic; the
 * scale is written to every s_w[n], so the result feeds fp8q_linear as is.
 * N > 0.  s_w[0] serves as the reduction word while the call runs (it is
 * zeroed with cudaMemsetAsync on `stream`, then three kernels follow).
 */
fp8q_status fp8q_quantize_weight_per_tensor(const void* W_f16, int64_t N, int64_t K,
                                            uint8_t* Wq, float* s_w, void* stream);

/*
 * fp8q_linear with the activation codes Xq in format x_fmt (weights E4M3):
 * the tensor cores multiply E5M2 x E4M3 directly (tcgen05 kind::f8f6f4
 * takes the two operand formats separately); everything else is identical.
 */
fp8q_status fp8q_linear_fmt(const uint8_t* Xq, fp8q_format x_fmt, const float* s_x,
                            const uint8_t* Wq, const float* s_w,
                            int64_t M, int64_t N, int64_t K,
                            void* Y_f16, void* stream);

/*
 * Block-wise weight quantization  [P2 §2.1: the MoE expert grouped GEMM is
 * quantized "block-wise 128x128"; §2.2: block-aligned MoE quantization].
 * W_f16 [E,N,K] fp16 (E = 1 for one matrix) in; Wq [E,N,K] uint8 E4M3 and
 * s_wb [E, ceil(N/128), ceil(K/128)] fp32 out.  Each 128 x 128 block of an
 * expert's [N,K] weights (ragged at the edges; blocks never span experts)
 * gets its own a', r, s and codes by the per-row rule.  1 <= E <= 1024.
 */
fp8q_status fp8q_quantize_weight_blockwise(const void* W_f16, int32_t E, int64_t N, int64_t K,
                                           uint8_t* Wq, float* s_wb, void* stream);

/*
 * MoE expert grouped FP8 linear with block-scaled expert weights (from
 * fp8q_quantize_weight_blockwise) and per-token activation scales:
 *   Y[r,n] = fp16( s_x[r] * sum_j s_wb[e, n/128, j] * P_j[r,n] ),
 *   P_j = FP32 tensor-core sum over the 128 inputs of K block j,
 * e the expert of row r (offsets as for fp8q_moe_grouped_linear).  Each K
 * block's partial is scaled and accumulated in FP32 registers (the sum over
 * j runs in K-block order).  1 <= E <= 128.
 */
fp8q_status fp8q_moe_grouped_linear_blockscaled(const uint8_t* Xq, const float* s_x,
                                                const int32_t* offsets, int32_t E, int64_t rows,
                                                const uint8_t* Wq, const float* s_wb,
                                                int64_t N, int64_t K,
                                                void* Y_f16, void* stream);

/*
 * MoE expert grouped linear reading its rows straight from the token matrix
 * [P1 关键证据 item 2 (sparse MoE); P2 §3.2 (expert pipeline)]: the
 * activations are quantized once per token (Xq_tok [tokens,K] uint8, s_x_tok
 * [tokens] fp32, from fp8q_quantize_rows_dynamic), and row r of the grouped
 * product (rows in expert order, offsets as for fp8q_moe_grouped_linear)
 * reads token row_token[r] (int32 [rows], device).  Same result as
 * fp8q_moe_grouped_linear on the gathered rows, without the gathered copy.
 * Y_f16 [rows,N].  A row_token entry outside [0, tokens) sets
 * FP8Q_DEVERR_BAD_OFFSETS and that row reads zeros.
 */
fp8q_status fp8q_moe_grouped_linear_gather(const uint8_t* Xq_tok, const float* s_x_tok, int64_t tokens,
                                           const int32_t* row_token, const int32_t* offsets, int32_t E,
                                           int64_t rows, const uint8_t* Wq, const float* s_w,
                                           int64_t N, int64_t K, void* Y_f16, void* stream);

/*
 * MoE expert grouped linear with the top-k combine in its epilogue (the down
 * projection of the MoE layer) [P1 关键证据 item 2; P2 §3.2]: grouped row r
 * (inputs and offsets as for fp8q_moe_grouped_linear) produces
 * y = (acc * s_x[r]) * s_w[e, n] in fp32 and adds fp16(y * row_weight[r])
 * into row row_token[r] of out_f16 [tokens, N] with an fp16 atomic add
 * (round to nearest).  The call first zeroes out_f16 (cudaMemsetAsync on
 * `stream`).  With at most two rows per token the result does not depend on
 * the order of the additions.  row_token int32 [rows], row_weight fp32
 * [rows] (the router's combine weights), device.  A row_token entry outside
 * [0, tokens) sets FP8Q_DEVERR_BAD_OFFSETS and that row adds nothing.
 */
fp8q_status fp8q_moe_grouped_linear_combine(const uint8_t* Xq, const float* s_x,
                                            const int32_t* offsets, int32_t E, int64_t rows,
                                            const uint8_t* Wq, const float* s_w, int64_t N, int64_t K,
                                            const int32_t* row_token, const float* row_weight,
                                            int64_t tokens, void* out_f16, void* stream);

/*
 * Per-token activation quantization with the MoE dispatch in its store
 * [P2 §2.2 per-token activation scales; §3.2 tokens grouped by expert]:
 * token row t of X_f16 [T, K] is quantized once (the steps of
 * fp8q_quantize_rows_dynamic_fmt, format fmt) and its codes and scale are
 * written to every grouped row token_rows[t * topk + j], j < topk, of Xq
 * [rows, K] and s_x [rows] -- the expert-grouped activation matrix the MoE
 * grouped linear reads.  token_rows int32 [T, topk], device; -1 = no row.
 * A grouped row no entry names is left unwritten.  An entry outside
 * [-1, rows) sets FP8Q_DEVERR_BAD_OFFSETS and is skipped.  topk in [1, 8].
 */
fp8q_status fp8q_quantize_rows_dispatch(const void* X_f16, int64_t T, int64_t K, fp8q_format fmt,
                                        const int32_t* token_rows, int32_t topk, int64_t rows, uint8_t* Xq,
                                        float* s_x, void* stream);

/* fp8q_moe_grouped_linear with the activation codes Xq in format x_fmt. */
fp8q_status fp8q_moe_grouped_linear_fmt(const uint8_t* Xq, fp8q_format x_fmt, const float* s_x,
                                        const int32_t* offsets, int32_t E, int64_t rows,
                                        const uint8_t* Wq, const float* s_w,
                                        int64_t N, int64_t K,
                                        void* Y_f16, void* stream);

/*
 * Diagnostic: the device E4M3 cast on its own, out[i] = E4M3(x[i]) with the
 * same rounding as the quantizers (RNE, saturating to ±448).  n >= 0,
 * x and out need no particular alignment.  Exists so that the cast can be
 * checked against an independent encoder over arbitrary fp32 bit patterns.
 */
fp8q_status fp8q_e4m3_encode_f32(const float* x, int64_t n, uint8_t* out, void* stream);

/*
 * Tuning override for the linear kernels (for measurement and tests; the
 * defaults are chosen per shape).  kernel_family: 0 = automatic, 1 = the
 * single-CTA kernel (128-row tiles), 2 = the CTA-pair kernel (256-row tiles,
 * tcgen05 cta_group::2; also selects it for the MoE grouped linear, whose
 * default is single-CTA), 3 = the swap-AB
 * split-K cluster kernel (M <= 128 only; larger M falls back to automatic).  tile_n: 0 = automatic, else 128,
 * 192, 256 or 512 (pair kernel only).  ksplit: 0 = automatic, else the split-K
 * cluster size 1, 2, 4 or 8 (split-K kernel only).  Process-wide; not thread-safe against
 * concurrent launches.  Environment variables FP8Q_FORCE_KERNEL
 * (auto|single|pair|splitk), FP8Q_BN and FP8Q_KSPLIT (split-K cluster size,
 * 1, 2, 4 or 8) set the initial values.  Two more, read once per process,
 * choose the K bytes a pipeline stage carries (unset: by shape):
 * FP8Q_STAGE_K = 128 or 256 for the CTA-pair kernel, FP8Q_SPLITK_STAGE_K =
 * 128, 256 or 512 for the split-K kernel (512 applies up to 32 rows; above,
 * 256 is used).  Results are the same for every choice up to the order of
 * the FP32 additions across split-K ranks (which K range each rank takes).
 */
fp8q_status fp8q_set_gemm_tuning(int kernel_family, int tile_n, int ksplit);

/*
 * Diagnostic: exercises the bounded-wait path every kernel relies on.  One
 * warp waits on an mbarrier that nothing arrives on, with the same wait
 * routine as the GEMM pipelines but a limit of `limit_us` microseconds
 * (1 .. 2000000), gives up, sets FP8Q_DEVERR_TIMEOUT_SELFTEST and returns.
 * The CUDA context stays usable; fp8q_device_error() then reports
 * FP8Q_ERR_TIMEOUT.
 */
fp8q_status fp8q_selftest_wait_timeout(uint32_t limit_us, void* stream);

/*
 * Synchronizes `stream`, then reads and clears the device error word of the
 * current device (an OR of FP8Q_DEVERR_* bits, 0 if none).  Returns
 * FP8Q_ERR_TIMEOUT if a timeout bit was set, FP8Q_ERR_DEVICE_CHECK if only
 * input-check bits were set, FP8Q_OK otherwise.  `flags` may be NULL.
 */
fp8q_status fp8q_device_error(void* stream, uint32_t* flags);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* FP8Q_H_ */
