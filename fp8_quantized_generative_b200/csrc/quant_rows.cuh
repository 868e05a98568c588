// Per-row dynamic FP8 quantization (per-token activations at run time,
// per-output-channel weights offline).  HBM-bound: 2 bytes read and 1 byte
// written per element plus 4 bytes of scale per row.
//
// Method: "Quantized Inference for OneRec-V2" (关键证据, steps 1-2) and
// "FP8量化在生成式推荐系统OneRec-V2中的优化实践" §2.2 (scale = max_code / max(|x|, eps)),
// with max_code = 448, the E4M3 maximum (§1.2), or 57344 for the E5M2
// activation variant (same page, §2.2).  Per-tensor variant (same page, §2.1,
// FFN weights): one amax over the whole matrix, at the end of this file.
//
// Design: a row is held in registers by TPR threads (TPR in {32..256}), each
// loading VPT 16-byte vectors (8 fp16 values) with coalesced 128-bit loads;
// the row max is reduced with warp shuffles (plus shared memory across the
// warps of one row); the codes are then produced from the registers, so X is
// read from HBM exactly once.  Rows longer than 256 * 8 vectors (K > 16384)
// fall back to a two-pass loop that re-reads the row (from L2).
#pragma once

#include "ptx.cuh"

namespace fp8q {

constexpr float kE4M3Max = 448.0f;
constexpr float kE5M2Max = 57344.0f;
constexpr float kScaleEps = 1e-12f;

template <int F>
__host__ __device__ constexpr float fp8_max() {
  return F == kFmtE4M3 ? kE4M3Max : kE5M2Max;
}

struct RowScale {
  float r;  // max_code / a'   (multiplier that maps the row max onto max_code)
  float s;  // a' / max_code   (stored dequantization scale)
};

template <int F = kFmtE4M3>
__device__ __forceinline__ RowScale row_scale_from_amax(float amax) {
  const float a = fmaxf(amax, kScaleEps);
  RowScale rs;
  rs.r = __fdiv_rn(fp8_max<F>(), a);
  rs.s = __fdiv_rn(a, fp8_max<F>());
  return rs;
}

__device__ __forceinline__ float absmax8(const uint4& v, float m) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
  }
  return m;
}

// 8 fp16 -> 8 FP8 codes (one fp32 multiply by r each, RN), packed little-endian.
template <int F = kFmtE4M3>
__device__ __forceinline__ uint2 encode8(const uint4& v, float r) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    w[i] = cvt_fp8x2<F>(__fmul_rn(f.x, r), __fmul_rn(f.y, r));
  }
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// Output rows of the quantizer.  Plain: input row m writes output row m.
// Dispatch (MoE, a token feeding top-k experts): input row m writes output
// rows rows[m * topk + j] for j < topk, the token's rows in the expert-grouped
// matrix (-1: none), so each token is read and encoded once.  An entry
// outside [-1, out_rows) sets error bit 0x8 and is skipped.
struct RowDispatch {
  const int32_t* rows = nullptr;
  int topk = 0;
  int out_rows = 0;
};

template <int VPT>
__device__ __forceinline__ void store_row_codes(const RowDispatch& d, int row, int t, int tpr, int nvec, int K,
                                                const uint2 (&enc)[VPT], float s, uint8_t* __restrict__ Q,
                                                float* __restrict__ S) {
  const int n = d.rows == nullptr ? 1 : d.topk;
  for (int k = 0; k < n; ++k) {
    int orow = row;
    if (d.rows != nullptr) {
      orow = __ldg(d.rows + static_cast<int64_t>(row) * d.topk + k);
      if (orow < 0 || orow >= d.out_rows) {
        if (orow != -1 && t == 0) raise_error(0x8u);
        continue;
      }
    }
    uint2* dst = reinterpret_cast<uint2*>(Q + static_cast<int64_t>(orow) * K);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int j = t + i * tpr;
      if (j < nvec) dst[j] = enc[i];
    }
    if (t == 0) S[orow] = s;
  }
}

// Grid: ceil(M / (CTA / TPR)) CTAs of CTA threads; TPR threads per row.
// With few rows, small CTAs (two rows of one warp each) spread them over more
// SMs: the grid is a single wave, so its time is that of the most loaded SM.
template <int TPR, int VPT, int F, int CTA = 256>
__global__ void __launch_bounds__(CTA) quant_rows_kernel(const __half* __restrict__ X, int M, int K,
                                                        uint8_t* __restrict__ Q, float* __restrict__ S,
                                                        const RowDispatch d, const bool release_early) {
  static_assert(TPR >= 32 && TPR <= CTA && CTA <= 256 && (TPR & (TPR - 1)) == 0, "TPR");
  // Programmatic dependent launch: let the next kernel start its set-up now
  // (it waits for this grid before touching our outputs), and wait for the
  // previous kernel before reading X or writing Q and S.  Not for weights:
  // the GEMMs request weight tiles before their own wait, so a weight
  // quantization lets the next kernel start only once it has finished.
  if (release_early) pdl_launch_dependents();
  pdl_wait_prior_grid();
  constexpr int kRowsPerCta = CTA / TPR;
  constexpr int kWarpsPerRow = TPR / 32;
  __shared__ float red[8];

  const int t = threadIdx.x % TPR;
  const int slot = threadIdx.x / TPR;
  const int row = blockIdx.x * kRowsPerCta + slot;
  const bool live = row < M;
  const int nvec = K >> 3;

  const uint4* src = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(row) * K);
  uint4 v[VPT];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int j = t + i * TPR;
    if (live && j < nvec) {
      v[i] = __ldg(src + j);
      m = absmax8(v[i], m);
    } else {
      v[i] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (kWarpsPerRow > 1) {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[warp] = m;
    __syncthreads();
    const int w0 = slot * kWarpsPerRow;
#pragma unroll
    for (int w = 0; w < kWarpsPerRow; ++w) m = fmaxf(m, red[w0 + w]);
  }
  if (!live) return;

  const RowScale rs = row_scale_from_amax<F>(m);
  uint2 enc[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) enc[i] = encode8<F>(v[i], rs.r);
  store_row_codes<VPT>(d, row, t, TPR, nvec, K, enc, rs.s, Q, S);
}

// Any K (multiple of 8): one CTA of 256 threads per row, two passes over the row.
template <int F>
__global__ void __launch_bounds__(256) quant_rows_long_kernel(const __half* __restrict__ X, int M, int K,
                                                             uint8_t* __restrict__ Q, float* __restrict__ S,
                                                             const RowDispatch d, const bool release_early) {
  __shared__ float red[8];
  if (release_early) pdl_launch_dependents();
  pdl_wait_prior_grid();
  const int row = blockIdx.x;
  const int nvec = K >> 3;
  const uint4* src = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(row) * K);
  float m = 0.0f;
  for (int j = threadIdx.x; j < nvec; j += 256) m = absmax8(__ldg(src + j), m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w]);
  const RowScale rs = row_scale_from_amax<F>(m);
  const int n = d.rows == nullptr ? 1 : d.topk;
  for (int k = 0; k < n; ++k) {   // (re-encoded per output row: the row does not fit in registers)
    int orow = row;
    if (d.rows != nullptr) {
      orow = __ldg(d.rows + static_cast<int64_t>(row) * d.topk + k);
      if (orow < 0 || orow >= d.out_rows) {
        if (orow != -1 && threadIdx.x == 0) raise_error(0x8u);
        continue;
      }
    }
    uint2* dst = reinterpret_cast<uint2*>(Q + static_cast<int64_t>(orow) * K);
    for (int j = threadIdx.x; j < nvec; j += 256) dst[j] = encode8<F>(__ldg(src + j), rs.r);
    if (threadIdx.x == 0) S[orow] = rs.s;
  }
}

// ------------------------------------------------------------ per-tensor (E4M3)
// One scale for a whole matrix (the FFN weights of "FP8量化在生成式推荐系统
// OneRec-V2中的优化实践" §2.1): the same steps with a = max over all elements.
// Three launches on the stream after S[0] is zeroed:
//   tensor_amax_kernel   every CTA reduces max|x| over its grid-stride share
//                        and raises S[0] with an atomic max on the float bits
//                        (for non-negative floats the unsigned order is the
//                        float order);
//   quant_tensor_kernel  every CTA reads the amax from S[0], derives r and s
//                        (the per-row formulas) and writes its codes, and s
//                        into S[row] for rows >= 1 (S[0] is still being read);
//   quant_tensor_finish  S[0] = s.
// The scale is thus replicated once per row (output channel), the form the
// per-channel GEMM epilogue consumes.  These kernels quantize weights only, so
// none lets the next kernel start early: the GEMMs request weight tiles before
// their programmatic-dependent-launch wait, which is safe only because every
// kernel writing weights has finished before the next kernel starts.
__global__ void __launch_bounds__(256) tensor_amax_kernel(const __half* __restrict__ X, int64_t nvec,
                                                         unsigned int* __restrict__ amax_bits) {
  __shared__ float red[8];
  pdl_wait_prior_grid();
  const uint4* src = reinterpret_cast<const uint4*>(X);
  float m = 0.0f;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; j < nvec;
       j += static_cast<int64_t>(gridDim.x) * 256)
    m = absmax8(__ldg(src + j), m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w]);
    atomicMax(amax_bits, __float_as_uint(m));
  }
}

__global__ void __launch_bounds__(256) quant_tensor_kernel(const __half* __restrict__ X, int M, int64_t nvec,
                                                          uint8_t* __restrict__ Q, float* __restrict__ S) {
  pdl_wait_prior_grid();
  const RowScale rs = row_scale_from_amax<kFmtE4M3>(S[0]);
  const uint4* src = reinterpret_cast<const uint4*>(X);
  uint2* dst = reinterpret_cast<uint2*>(Q);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * 256;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  for (int64_t j = first; j < nvec; j += stride) dst[j] = encode8<kFmtE4M3>(__ldg(src + j), rs.r);
  for (int64_t r = first + 1; r < M; r += stride) S[r] = rs.s;
}

__global__ void quant_tensor_finish_kernel(float* __restrict__ S) {
  pdl_wait_prior_grid();
  if (threadIdx.x == 0 && blockIdx.x == 0) S[0] = row_scale_from_amax<kFmtE4M3>(S[0]).s;
}

// Diagnostic elementwise cast (same device cast as the quantizers).
__global__ void e4m3_encode_kernel(const float* __restrict__ x, int64_t n, uint8_t* __restrict__ out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; 2 * i < n; i += stride) {
    const int64_t k = 2 * i;
    if (k + 1 < n) {
      const uint16_t c = cvt_e4m3x2(x[k], x[k + 1]);
      out[k] = static_cast<uint8_t>(c & 0xFF);
      out[k + 1] = static_cast<uint8_t>(c >> 8);
    } else {
      out[k] = static_cast<uint8_t>(cvt_e4m3x2(x[k], 0.0f) & 0xFF);
    }
  }
}

// Launch on `st` with programmatic stream serialization, so that the launch
// and prologue overlap the previous kernel on the stream.
template <typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Args...), dim3 grid, dim3 block, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Host-side launcher: picks (TPR, VPT) so one row fits in registers.
// release_early = false for weights (see quant_rows_kernel).
template <int F = kFmtE4M3>
inline cudaError_t launch_quant_rows(const __half* X, int M, int K, uint8_t* Q, float* S, cudaStream_t st,
                                     const RowDispatch d = RowDispatch{}, const bool release_early = true) {
  const int nvec = K / 8;
  int tpr = 32;
  while (tpr < 256 && tpr * 8 < nvec) tpr *= 2;
  const int vpt_needed = (nvec + tpr - 1) / tpr;
  if (vpt_needed > 8)
    return launch_pdl(quant_rows_long_kernel<F>, dim3(M), dim3(256), st, X, M, K, Q, S, d, release_early);
  const int vpt = vpt_needed <= 1 ? 1 : vpt_needed <= 2 ? 2 : vpt_needed <= 4 ? 4 : 8;
  // Few rows (fewer than 256 CTAs of 256 threads, i.e. under ~2 per SM):
  // CTAs of 64 threads spread them over more SMs (measured 10% faster at
  // M = 32 and 512); otherwise 256-thread CTAs (2-3% faster at M >= 4096).
  const int big_rows = 256 / tpr;
  const bool small = tpr < 256 && (M + big_rows - 1) / big_rows < 256;
  const int cta = small ? (tpr < 64 ? 64 : tpr) : 256;
  const int rows_per_cta = cta / tpr;
  const dim3 grid((M + rows_per_cta - 1) / rows_per_cta);
#define FP8Q_QR_CASE(T, V)                                                                                      \
  if (tpr == T && vpt == V)                                                                                   \
    return small ? launch_pdl(quant_rows_kernel<T, V, F, (T < 64 ? 64 : T)>, grid, dim3(cta), st, X, M, K, Q, S, d, \
                              release_early)                                                                  \
                 : launch_pdl(quant_rows_kernel<T, V, F, 256>, grid, dim3(cta), st, X, M, K, Q, S, d, release_early);
  FP8Q_QR_CASE(32, 1) FP8Q_QR_CASE(32, 2) FP8Q_QR_CASE(32, 4) FP8Q_QR_CASE(32, 8)
  FP8Q_QR_CASE(64, 8) FP8Q_QR_CASE(128, 8) FP8Q_QR_CASE(256, 8)
#undef FP8Q_QR_CASE
  return cudaErrorInvalidConfiguration;
}

}  // namespace fp8q
