// C ABI of libfp8q: argument validation, TMA descriptor set-up, kernel choice
// and launch.  The operations and their arithmetic are documented in
// include/fp8q.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "fp8q.h"
#include "gemm_fp8.cuh"
#include "quant_rows.cuh"

namespace fp8q {
namespace {

thread_local std::string g_last_error;

fp8q_status cuda_fail(cudaError_t e, const char* what) {
  g_last_error = std::string(what) + ": " + cudaGetErrorName(e) + ": " + cudaGetErrorString(e);
  return FP8Q_ERR_CUDA;
}

fp8q_status invalid(const char* what) {
  g_last_error = what;
  return FP8Q_ERR_INVALID_ARG;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

// ------------------------------------------------------------------ device info
constexpr int kMaxDevices = 64;
struct DeviceInfo {
  std::once_flag once;
  int num_sms = 0;
  cudaError_t err = cudaSuccess;
};
DeviceInfo g_dev[kMaxDevices];

cudaError_t current_device_info(int* dev_out, int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  DeviceInfo& d = g_dev[dev];
  std::call_once(d.once, [&]() { d.err = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev); });
  if (d.err != cudaSuccess) return d.err;
  *dev_out = dev;
  *sms = d.num_sms;
  return cudaSuccess;
}

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, []() {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D K-major uint8 operand [rows, K] read in boxes of box_rows x 128 bytes,
// 128-byte swizzle; out-of-range rows and columns read as zero.
fp8q_status make_operand_map(CUtensorMap* m, const void* base, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) {
    g_last_error = "cuTensorMapEncodeTiled entry point unavailable";
    return FP8Q_ERR_CUDA;
  }
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    std::snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    g_last_error = buf;
    return FP8Q_ERR_CUDA;
  }
  return FP8Q_OK;
}

// ------------------------------------------------------------------ GEMM launch
constexpr int kBN = 256;
constexpr int kStages = 4;

template <bool kGrouped>
fp8q_status launch_gemm(const uint8_t* A, int64_t a_rows, const uint8_t* B, int64_t b_rows, const GemmParams& p,
                        int64_t tiles_upper_bound, cudaStream_t st) {
  using L = GemmLayout<kBN, kStages>;
  int dev = 0, sms = 0;
  cudaError_t e = current_device_info(&dev, &sms);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  CUtensorMap ta, tb;
  fp8q_status s = make_operand_map(&ta, A, a_rows, p.K, kBM);
  if (s != FP8Q_OK) return s;
  s = make_operand_map(&tb, B, b_rows, p.K, kBN);
  if (s != FP8Q_OK) return s;
  auto kernel = fp8_gemm_kernel<kBN, kStages, kGrouped>;
  const size_t smem = L::smem_bytes(kGrouped ? p.E : 0);
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  const int grid = static_cast<int>(tiles_upper_bound < sms ? (tiles_upper_bound < 1 ? 1 : tiles_upper_bound) : sms);
  kernel<<<grid, kGemmThreads, smem, st>>>(ta, tb, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fp8_gemm_kernel launch");
  return FP8Q_OK;
}

fp8q_status check_quant_args(const void* X, int64_t M, int64_t K, const void* Q, const void* S) {
  if (M < 0 || M > kMaxDim) return invalid("M out of range");
  if (K <= 0 || K > kMaxDim) return invalid("K out of range");
  if (K % 16 != 0) return invalid("K must be a multiple of 16");
  if (M * K > (int64_t(1) << 40)) return invalid("M*K too large");
  if (M == 0) return FP8Q_OK;
  if (!aligned16(X) || !aligned16(Q) || !aligned16(S)) return invalid("null or non-16-byte-aligned pointer");
  return FP8Q_OK;
}

fp8q_status quantize(const void* X, int64_t M, int64_t K, uint8_t* Q, float* S, void* stream) {
  fp8q_status s = check_quant_args(X, M, K, Q, S);
  if (s != FP8Q_OK || M == 0) return s;
  const cudaError_t e = launch_quant_rows(static_cast<const __half*>(X), static_cast<int>(M), static_cast<int>(K),
                                          Q, S, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quant_rows launch");
  return FP8Q_OK;
}

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" {

const char* fp8q_status_string(int status) {
  switch (status) {
    case FP8Q_OK: return "FP8Q_OK";
    case FP8Q_ERR_INVALID_ARG: return "FP8Q_ERR_INVALID_ARG";
    case FP8Q_ERR_UNSUPPORTED: return "FP8Q_ERR_UNSUPPORTED";
    case FP8Q_ERR_CUDA: return "FP8Q_ERR_CUDA";
    case FP8Q_ERR_TIMEOUT: return "FP8Q_ERR_TIMEOUT";
    case FP8Q_ERR_DEVICE_CHECK: return "FP8Q_ERR_DEVICE_CHECK";
    default: return "FP8Q_UNKNOWN_STATUS";
  }
}

const char* fp8q_last_error_message(void) { return g_last_error.c_str(); }

int fp8q_version(void) { return 100; }

fp8q_status fp8q_quantize_rows_dynamic(const void* X_f16, int64_t M, int64_t K, uint8_t* Xq, float* s_x,
                                       void* stream) {
  return quantize(X_f16, M, K, Xq, s_x, stream);
}

fp8q_status fp8q_quantize_weight_per_channel(const void* W_f16, int64_t N, int64_t K, uint8_t* Wq, float* s_w,
                                             void* stream) {
  if (N == 0) return invalid("N must be positive");
  return quantize(W_f16, N, K, Wq, s_w, stream);
}

fp8q_status fp8q_linear(const uint8_t* Xq, const float* s_x, const uint8_t* Wq, const float* s_w, int64_t M,
                        int64_t N, int64_t K, void* Y_f16, void* stream) {
  if (M < 0 || M > kMaxDim) return invalid("M out of range");
  if (N <= 0 || N > kMaxDim || N % 8 != 0) return invalid("N must be positive and a multiple of 8");
  if (K <= 0 || K > kMaxDim || K % 16 != 0) return invalid("K must be positive and a multiple of 16");
  if (M == 0) return FP8Q_OK;
  if (!aligned16(Xq) || !aligned16(s_x) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(Y_f16))
    return invalid("null or non-16-byte-aligned pointer");
  GemmParams p;
  p.s_x = s_x;
  p.s_w = s_w;
  p.Y = static_cast<__half*>(Y_f16);
  p.offsets = nullptr;
  p.rows = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.E = 1;
  const int64_t tiles = ((M + kBM - 1) / kBM) * ((N + kBN - 1) / kBN);
  return launch_gemm<false>(Xq, M, Wq, N, p, tiles, static_cast<cudaStream_t>(stream));
}

fp8q_status fp8q_moe_grouped_linear(const uint8_t* Xq, const float* s_x, const int32_t* offsets, int32_t E,
                                    int64_t rows, const uint8_t* Wq, const float* s_w, int64_t N, int64_t K,
                                    void* Y_f16, void* stream) {
  if (E < 1 || E > kMaxExperts) return invalid("E must be in [1, 4096]");
  if (rows < 0 || rows > kMaxDim) return invalid("rows out of range");
  if (N <= 0 || N % 8 != 0 || int64_t(E) * N > kMaxDim) return invalid("N must be positive, a multiple of 8, E*N < 2^31");
  if (K <= 0 || K > kMaxDim || K % 16 != 0) return invalid("K must be positive and a multiple of 16");
  if (offsets == nullptr || (reinterpret_cast<uintptr_t>(offsets) & 3u) != 0) return invalid("offsets pointer");
  if (rows == 0) return FP8Q_OK;
  if (!aligned16(Xq) || !aligned16(s_x) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(Y_f16))
    return invalid("null or non-16-byte-aligned pointer");
  GemmParams p;
  p.s_x = s_x;
  p.s_w = s_w;
  p.Y = static_cast<__half*>(Y_f16);
  p.offsets = offsets;
  p.rows = static_cast<int>(rows);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.E = E;
  const int64_t tiles = ((rows + kBM - 1) / kBM + E) * ((N + kBN - 1) / kBN);
  return launch_gemm<true>(Xq, rows, Wq, int64_t(E) * N, p, tiles, static_cast<cudaStream_t>(stream));
}

fp8q_status fp8q_e4m3_encode_f32(const float* x, int64_t n, uint8_t* out, void* stream) {
  if (n < 0) return invalid("n must be >= 0");
  if (n == 0) return FP8Q_OK;
  if (x == nullptr || out == nullptr || (reinterpret_cast<uintptr_t>(x) & 3u) != 0) return invalid("pointer");
  int dev = 0, sms = 0;
  cudaError_t e = current_device_info(&dev, &sms);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  const int64_t pairs = (n + 1) / 2;
  int64_t blocks = (pairs + 255) / 256;
  if (blocks > int64_t(sms) * 16) blocks = int64_t(sms) * 16;
  e4m3_encode_kernel<<<static_cast<int>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, n, out);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "e4m3_encode launch");
  return FP8Q_OK;
}

fp8q_status fp8q_device_error(void* stream, uint32_t* flags) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  if (flags) *flags = v;
  if (v & (FP8Q_DEVERR_TIMEOUT_PRODUCER | FP8Q_DEVERR_TIMEOUT_MMA | FP8Q_DEVERR_TIMEOUT_EPILOGUE |
           FP8Q_DEVERR_TIMEOUT_CLUSTER))
    return FP8Q_ERR_TIMEOUT;
  if (v) return FP8Q_ERR_DEVICE_CHECK;
  return FP8Q_OK;
}

}  // extern "C"
