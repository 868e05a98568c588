// C ABI of libfp8q: argument validation, TMA descriptor set-up, kernel choice
// and launch.  The operations and their arithmetic are documented in
// include/fp8q.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <climits>
#include <mutex>
#include <string>

#include "fp8q.h"
#include "gemm_fp8.cuh"
#include "gemm_fp8_pair.cuh"
#include "gemm_fp8_splitk.cuh"
#include "gemm_fp8_blockscaled.cuh"
#include "quant_rows.cuh"

namespace fp8q {

// Self-test of the bounded-wait machinery: one warp waits on an mbarrier that
// nothing will ever arrive on, with the same wait routine the GEMMs use, and
// must give up after `limit_ns` and report through the device error word.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0 && !mbar_wait_limit(&bar, 0, nullptr, limit_ns)) raise_error(0x20u);
}

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
  // L2 promotion of operand loads; FP8Q_L2PROMO = 0 / 64 / 128 / 256 (default 256) for sweeps.
  static const CUtensorMapL2promotion promo = [] {
    const char* e = std::getenv("FP8Q_L2PROMO");
    const int v = e ? std::atoi(e) : 256;
    return v == 0 ? CU_TENSOR_MAP_L2_PROMOTION_NONE
         : v == 64 ? CU_TENSOR_MAP_L2_PROMOTION_L2_64B
         : v == 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                    : CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
  }();
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, promo,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    std::snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    g_last_error = buf;
    return FP8Q_ERR_CUDA;
  }
  return FP8Q_OK;
}

// fp16 output [rows, N] written in 32 x 32 boxes through a 64-byte-swizzled
// staging tile; the store clips rows >= rows and columns >= N.
fp8q_status make_output_map(CUtensorMap* m, const void* base, int64_t rows, int64_t N) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) {
    g_last_error = "cuTensorMapEncodeTiled entry point unavailable";
    return FP8Q_ERR_CUDA;
  }
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    std::snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled(output) failed (CUresult %d)", static_cast<int>(r));
    g_last_error = buf;
    return FP8Q_ERR_CUDA;
  }
  return FP8Q_OK;
}

// ------------------------------------------------------------------ GEMM launch
constexpr int kFusedMaxRows = 64;     // fused quantize + GEMM: token rows
constexpr int kBN = 256;        // single-CTA dense tiles (128 x 256)
constexpr int kStages = 4;
constexpr int kBNGrouped = 256; // MoE tiles (128 x 256); 128-wide tiles measured slower on B200
constexpr int kStagesGrouped = 4;

// Tuning knobs read once from the environment (for measurement sweeps):
//   FP8Q_FORCE_KERNEL = auto | single | pair   (dense linear kernel family)
//   FP8Q_BN           = 0 (auto) | 128 | 192 | 256   (pair-kernel tile width)
// fp8q_set_gemm_tuning() overrides both at run time.
struct Knobs {
  int force = 0;  // 0 auto, 1 single, 2 pair, 3 split-K (M <= 128)
  int bn = 0;
  int ksplit = 0; // split-K cluster size, 0 = automatic
  int half_tiles = 1; // FP8Q_HALF_TILES: 0 = CTA-pair grouped kernel uses only M = 256 tiles
  int stage_k = 256;  // FP8Q_STAGE_K: K bytes per stage of the dense pair kernel (128 or 256)
  int splitk_stage_k = 0;    // FP8Q_SPLITK_STAGE_K: the same for the split-K kernel (0 = 512 up to 32 rows, else 256)
};
Knobs& knobs() {
  static Knobs k = []() {
    Knobs r;
    if (const char* f = std::getenv("FP8Q_FORCE_KERNEL")) {
      if (!std::strcmp(f, "single")) r.force = 1;
      if (!std::strcmp(f, "pair")) r.force = 2;
      if (!std::strcmp(f, "splitk")) r.force = 3;
    }
    if (const char* k = std::getenv("FP8Q_KSPLIT")) r.ksplit = std::atoi(k);
    if (const char* b = std::getenv("FP8Q_BN")) r.bn = std::atoi(b);
    if (const char* h = std::getenv("FP8Q_HALF_TILES")) r.half_tiles = h[0] == '0' ? 0 : 1;
    if (const char* v = std::getenv("FP8Q_STAGE_K")) r.stage_k = std::atoi(v) == 128 ? 128 : 256;
    if (const char* v = std::getenv("FP8Q_SPLITK_STAGE_K")) {
      const int k = std::atoi(v);
      r.splitk_stage_k = k == 512 ? 512 : k == 256 ? 256 : k == 128 ? 128 : 0;
    }
    return r;
  }();
  return k;
}

// Raise a kernel's dynamic shared-memory limit once per device (the attribute
// persists; setting it on every call would cost a driver round trip).
template <auto Kernel>
cudaError_t ensure_smem(size_t bytes, int dev) {
  static bool done[kMaxDevices] = {};
  static std::mutex mu;
  std::lock_guard<std::mutex> g(mu);
  if (done[dev]) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

template <typename... Args>
cudaError_t launch_ex(void (*kernel)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
                      bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <bool kGrouped, bool kGather = false>
fp8q_status launch_gemm(const uint8_t* A, int64_t a_rows, const uint8_t* B, int64_t b_rows, const GemmParams& p,
                        int64_t tiles_upper_bound, cudaStream_t st) {
  constexpr int BN = kGrouped ? kBNGrouped : kBN;
  constexpr int STAGES = kGrouped ? kStagesGrouped : kStages;
  using L = GemmLayout<BN, STAGES>;
  int dev = 0, sms = 0;
  cudaError_t e = current_device_info(&dev, &sms);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  CUtensorMap ta, tb;
  fp8q_status s = make_operand_map(&ta, A, a_rows, p.K, kBM);
  if (s != FP8Q_OK) return s;
  s = make_operand_map(&tb, B, b_rows, p.K, BN);
  if (s != FP8Q_OK) return s;
  CUtensorMap ty;   // combine: Y is the [tokens, N] output, written by atomic adds only
  s = make_output_map(&ty, p.Y, p.comb_token != nullptr ? p.tokens : p.rows, p.N);
  if (s != FP8Q_OK) return s;
  auto kernel = fp8_gemm_kernel<BN, STAGES, kGrouped, kGather>;
  const size_t smem = L::smem_bytes(kGrouped ? p.E : 0);
  e = ensure_smem<fp8_gemm_kernel<BN, STAGES, kGrouped, kGather>>(L::smem_bytes(kGrouped ? kMaxExperts : 0), dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  const int grid = static_cast<int>(tiles_upper_bound < sms ? (tiles_upper_bound < 1 ? 1 : tiles_upper_bound) : sms);
  e = launch_ex(kernel, dim3(grid), dim3(kGemmThreads), smem, st, 1, true, ta, tb, ty, p);
  if (e != cudaSuccess) return cuda_fail(e, "fp8_gemm_kernel launch");
  return FP8Q_OK;
}

// Split-K producers prefetch the rest of their weight slice into L2 at the
// start (FP8Q_L2PF = 0 disables it, for sweeps).  Measured: a few percent
// faster for one token row; the same idea slowed the grouped MoE kernel, so
// only the split-K kernel uses it.
int l2_prefetch_enabled() {
  static const int v = [] {
    const char* e = std::getenv("FP8Q_L2PF");
    return (e && e[0] == '0') ? 0 : 1;
  }();
  return v;
}

// Per-device cache of how many 2-CTA clusters of a pair kernel fit at once.
template <int BN, int STAGES, bool kGrouped, int SK = kBK>
int max_pair_clusters(int dev) {
  static int cache[kMaxDevices] = {0};
  static std::mutex mu;
  std::lock_guard<std::mutex> g(mu);
  if (cache[dev] > 0) return cache[dev];
  using L = PairLayout<BN, STAGES, SK>;
  auto kernel = fp8_gemm_pair_kernel<BN, STAGES, kGrouped, false, SK>;
  const size_t smem = L::smem_bytes(kGrouped ? kMaxExperts : 0);
  if (ensure_smem<fp8_gemm_pair_kernel<BN, STAGES, kGrouped, false, SK>>(smem, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    n = 0;
  }
  cache[dev] = n;
  return n;
}

// Tail split of the pair schedule: with F full tiles on C clusters, the
// last F mod C tiles are cut into q in {2, 4} pieces along N when that still
// fits one round (pieces stay multiples of 64 columns); q = 1 otherwise.
struct TailSplit {
  int main_tiles;
  int q;
};
TailSplit tail_split(int64_t full_tiles, int clusters, int bn) {
  // A wide tile (bn = 512) splits only into 256-column halves.
  const int qmax = bn > 256 ? 2 : 4;
  TailSplit r{static_cast<int>(full_tiles), 1};
  static const bool enabled = [] {
    const char* e = std::getenv("FP8Q_TAIL");   // tuning knob: 0 disables the split
    return !(e && e[0] == '0');
  }();
  const int64_t left = full_tiles % clusters;
  if (left == 0 || !enabled) return r;
  for (int q = qmax; q >= 2; q >>= 1) {
    if ((bn / q) % 64 != 0) continue;
    if (left * q <= clusters) {
      r.main_tiles = static_cast<int>(full_tiles - left);
      r.q = q;
      return r;
    }
  }
  return r;
}

// Launch a pair kernel.  Dense: A = Xq [rows, K], B = Wq [N, K].  Grouped:
// B = Wq [E*N, K] and the schedule comes from the device offsets;
// `tiles_upper_bound` caps the grid when the tile count is unknown on the host.
template <int BN, int STAGES, bool kGrouped, bool kQuantA = false, int SK = kBK>
fp8q_status launch_pair(const uint8_t* A, const uint8_t* B, int64_t b_rows, const GemmParams& p0, int dev,
                        cudaStream_t st, int64_t tiles_upper_bound = 0) {
  using L = PairLayout<BN, STAGES, SK>;
  const int clusters = max_pair_clusters<BN, STAGES, kGrouped, SK>(dev);
  if (clusters < 1) {
    g_last_error = "no 2-CTA cluster of the pair GEMM fits on this device";
    return FP8Q_ERR_UNSUPPORTED;
  }
  GemmParams p = p0;
  int64_t tiles;
  TailSplit ts{0, 1};
  if (kGrouped) {
    p.main_tiles = 0;
    p.tail_q = 1;
    tiles = tiles_upper_bound;
  } else {
    const int64_t full = int64_t((p.rows + 2 * kBM - 1) / (2 * kBM)) * ((p.N + BN - 1) / BN);
    ts = tail_split(full, clusters, BN);
    p.main_tiles = ts.main_tiles;
    p.tail_q = ts.q;
    tiles = int64_t(ts.main_tiles) + (full - ts.main_tiles) * ts.q;
  }
  CUtensorMap ta, tah, tb, tbt, ty;
  fp8q_status s = make_operand_map(&ta, A, p.rows, p.K, kBM);
  if (s != FP8Q_OK) return s;
  if (kGrouped) {
    // half tiles: 64 rows of A per CTA
    s = make_operand_map(&tah, A, p.rows, p.K, kBM / 2);
    if (s != FP8Q_OK) return s;
  } else {
    tah = ta;   // unused
  }
  s = make_operand_map(&tb, B, b_rows, p.K, L::kWide ? 128 : L::kBRows);
  if (s != FP8Q_OK) return s;
  s = make_operand_map(&tbt, B, b_rows, p.K, L::kWide ? 128 : L::kBRows / ts.q);
  if (s != FP8Q_OK) return s;
  s = make_output_map(&ty, p.Y, p.rows, p.N);
  if (s != FP8Q_OK) return s;
  auto kernel = fp8_gemm_pair_kernel<BN, STAGES, kGrouped, kQuantA, SK>;
  cudaError_t e = ensure_smem<fp8_gemm_pair_kernel<BN, STAGES, kGrouped, kQuantA, SK>>(
      L::smem_bytes(kGrouped ? kMaxExperts : 0), dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(pair)");
  const int pairs = static_cast<int>(tiles < clusters ? (tiles < 1 ? 1 : tiles) : clusters);
  e = launch_ex(kernel, dim3(2 * pairs), dim3(kGemmThreads), L::smem_bytes(kGrouped ? p.E : 0), st, 2, true, ta, tah,
                tb, tbt, ty, p);
  if (e != cudaSuccess) return cuda_fail(e, "fp8_gemm_pair_kernel launch");
  return FP8Q_OK;
}

// Pair-kernel tile width: the candidate with the least modelled time =
// rounds of tiles x per-tile work / relative efficiency.  Narrower tiles move
// more operand bytes out of L2 per FLOP (256 FLOP/B per SM at BN = 256, 219
// at 192, 171 at 128) and pay the per-tile epilogue more often; the
// efficiency factors are per-FLOP throughputs relative to BN = 256 measured
// on B200 (4096 x 6144 x 2048).  Tail pieces (a full tile cut along N for
// the last round) run at their own width's efficiency, 7% lower still: they
// keep the full tile's stage layout (measured on B200 at 512 x 4096 x 4096:
// 128-wide pieces of 256-wide tiles 13.7 us, native 128-wide tiles 12.8 us).
double pair_tile_efficiency(int width) {
  return width >= 256 ? 1.0 : width >= 192 ? 0.79 : width >= 128 ? 0.60 : 0.40;
}

int choose_pair_bn(int64_t M, int64_t N, int clusters) {
  const int cands[3] = {256, 192, 128};
  constexpr double kPiecePenalty = 0.93;
  int best = 256;
  double best_cost = 1e300;
  for (int i = 0; i < 3; ++i) {
    const int bn = cands[i];
    const int64_t full = ((M + 255) / 256) * ((N + bn - 1) / bn);
    const TailSplit ts = tail_split(full, clusters, bn);
    const int64_t rounds_main = (ts.main_tiles + clusters - 1) / clusters;
    const int64_t pieces = (full - ts.main_tiles) * ts.q;   // after the full rounds
    const int64_t rounds_tail = (pieces + clusters - 1) / clusters;
    double cost = static_cast<double>(rounds_main) * bn / pair_tile_efficiency(bn);
    if (rounds_tail > 0) {
      const int w = bn / ts.q;
      cost += static_cast<double>(rounds_tail) * w / (pair_tile_efficiency(w) * (ts.q > 1 ? kPiecePenalty : 1.0));
    }
    if (cost < best_cost * 0.999) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

// How many clusters of S CTAs of a split-K kernel fit on the device at once.
template <int MPAD, int STAGES, bool kFused, int SK = kBK>
int max_splitk_clusters(int dev, int S) {
  static int cache[kMaxDevices][9] = {};
  static std::mutex mu;
  std::lock_guard<std::mutex> g(mu);
  if (cache[dev][S] != 0) return cache[dev][S];
  using L = SplitKLayout<MPAD, STAGES, kFused, SK>;
  auto kernel = fp8_gemm_splitk_kernel<MPAD, STAGES, kFused, SK>;
  const size_t max_smem = kFused ? L::fused_smem_bytes(L::kFusedMaxKBlocks) : L::kSmemBytes;
  if (ensure_smem<fp8_gemm_splitk_kernel<MPAD, STAGES, kFused, SK>>(max_smem, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return -1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S);
  cfg.blockDim = dim3(kSkThreads);
  // occupancy at the shared memory of a typical launch (8 K blocks per CTA when fused)
  cfg.dynamicSmemBytes = kFused ? L::fused_smem_bytes(8) : L::kSmemBytes;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = S;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    n = -1;
  }
  cache[dev][S] = n;
  return n;
}

// Split factor S in {1, 2, 4, 8} (a divisor of the 128 weight rows of a
// tile, so each CTA of the cluster owns an equal slice of the reduction):
// the largest that keeps every cluster of the grid resident at once (one
// wave; two CTAs share an SM when their shared memory allows) and gives
// each CTA at least one K block.
template <int MPAD, int STAGES, bool kFused, int SK = kBK>
int choose_ksplit(int dev, int n_tiles, int num_kb) {
  int S = 8;
  while (S > 1 && S > num_kb) S >>= 1;
  while (S > 1) {
    const int fit = max_splitk_clusters<MPAD, STAGES, kFused, SK>(dev, S);
    if (fit >= n_tiles) break;
    S >>= 1;
  }
  return S;
}

// Dense linear with at most 128 token rows.  kFused: A is the fp16
// activations (p.x_f16) and the kernel quantizes them itself (<= 64 rows);
// otherwise A is Xq with scales s_x.
template <int MPAD, int STAGES, bool kFused, int SK = kBK>
fp8q_status launch_splitk(const uint8_t* Xq, const uint8_t* Wq, const GemmParams& p, int dev, cudaStream_t st) {
  using L = SplitKLayout<MPAD, STAGES, kFused, SK>;
  CUtensorMap tw, tx;
  fp8q_status s = make_operand_map(&tw, Wq, p.N, p.K, kBM);
  if (s != FP8Q_OK) return s;
  if (kFused) {
    tx = tw;   // unused by the fused kernel
  } else {
    s = make_operand_map(&tx, Xq, p.rows, p.K, MPAD);
    if (s != FP8Q_OK) return s;
  }
  const int n_tiles = (p.N + kBM - 1) / kBM;
  const int num_kb = (p.K + SK - 1) / SK;
  const int S = knobs().ksplit ? knobs().ksplit : choose_ksplit<MPAD, STAGES, kFused, SK>(dev, n_tiles, num_kb);
  const int nkb_max = (num_kb + S - 1) / S;
  if (kFused && nkb_max > L::kFusedMaxKBlocks) {
    g_last_error = "fused path: too many K blocks per CTA";
    return FP8Q_ERR_UNSUPPORTED;
  }
  const size_t smem = kFused ? L::fused_smem_bytes(nkb_max) : L::kSmemBytes;
  auto kernel = fp8_gemm_splitk_kernel<MPAD, STAGES, kFused, SK>;
  cudaError_t e = ensure_smem<fp8_gemm_splitk_kernel<MPAD, STAGES, kFused, SK>>(
      kFused ? L::fused_smem_bytes(L::kFusedMaxKBlocks) : L::kSmemBytes, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(splitk)");
  e = launch_ex(kernel, dim3(n_tiles * S), dim3(kSkThreads), smem, st, S, true, tw, tx, p);
  if (e != cudaSuccess) return cuda_fail(e, "fp8_gemm_splitk_kernel launch");
  return FP8Q_OK;
}

fp8q_status launch_dense(const uint8_t* Xq, const uint8_t* Wq, const GemmParams& p, cudaStream_t st) {
  int dev = 0, sms = 0;
  cudaError_t e = current_device_info(&dev, &sms);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  const Knobs kn = knobs();
  if ((kn.force == 0 && p.rows <= kBM) || kn.force == 3) {
    // Several 128-byte K boxes per stage (more MMAs per barrier wait: four
    // boxes, sixteen MMAs, up to 32 rows; two boxes above, where four would
    // not leave room for two stages), and a ring deep enough to hold all of
    // a CTA's weight slice at a split of 4 up to 64 rows: the whole slice is
    // requested before the dependency wait, so it streams in while the
    // kernel before this one (the activation quantizer) runs.  Measured on
    // B200, quantize + GEMM per step: two-box rings of 4 / 4 / 3 stages took
    // M=1 7.9 -> 7.0 us, M=16 8.1 -> 7.5, M=32 9.0 -> 7.9, M=64 9.8 -> 9.4
    // against two-stage rings, and four-box stages M=1 7.09 -> 6.78 us,
    // M=8 7.40 -> 7.06, M=16 7.43 -> 7.11, M=32 7.94 -> 7.70 against those.
    // At 128 rows the partial exchange buffer leaves room for two stages.
    const int sk = kn.splitk_stage_k ? kn.splitk_stage_k : (p.rows <= 32 ? 512 : 256);
    if (sk == 512 && p.rows <= 32) {
      if (p.rows <= 16) return launch_splitk<16, 2, false, 512>(Xq, Wq, p, dev, st);
      return launch_splitk<32, 2, false, 512>(Xq, Wq, p, dev, st);
    }
    if (sk >= 256) {
      if (p.rows <= 16) return launch_splitk<16, 4, false, 256>(Xq, Wq, p, dev, st);
      if (p.rows <= 32) return launch_splitk<32, 4, false, 256>(Xq, Wq, p, dev, st);
      if (p.rows <= 64) return launch_splitk<64, 3, false, 256>(Xq, Wq, p, dev, st);
      if (p.rows <= 128) return launch_splitk<128, 2, false, 256>(Xq, Wq, p, dev, st);
    }
    // one-box stages (FP8Q_SPLITK_STAGE_K=128)
    if (p.rows <= 16) return launch_splitk<16, 5, false>(Xq, Wq, p, dev, st);
    if (p.rows <= 32) return launch_splitk<32, 4, false>(Xq, Wq, p, dev, st);
    if (p.rows <= 64) return launch_splitk<64, 3, false>(Xq, Wq, p, dev, st);
    if (p.rows <= 128) return launch_splitk<128, 4, false>(Xq, Wq, p, dev, st);
  }
  bool pair = p.rows > kBM;
  // Walk n-blocks first when A is the larger operand: each A block is then
  // reused by every n-block while it is in L2, and the smaller B stays there.
  GemmParams q = p;
  q.n_fastest = int64_t(p.rows) > int64_t(p.N) ? 1 : 0;
  // FP8Q_RASTER = 1 (m-blocks first) / 2 (n-blocks first) overrides the order for sweeps.
  static const int raster = [] {
    const char* e = std::getenv("FP8Q_RASTER");
    return e ? std::atoi(e) : 0;
  }();
  if (raster == 1) q.n_fastest = 0;
  if (raster == 2) q.n_fastest = 1;
  if (kn.force == 1) pair = false;
  if (kn.force == 2) pair = true;
  if (pair) {
    const int clusters = max_pair_clusters<256, 6, false>(dev);
    int bn = kn.bn ? kn.bn : choose_pair_bn(p.rows, p.N, clusters > 0 ? clusters : sms / 2);
    // Two 128-byte K boxes per stage (measured 3-10% faster on B200 than one:
    // the MMA-issuing thread's per-stage work is spread over eight MMAs).
    if (kn.stage_k == 256) {
      switch (bn) {
        case 128: return launch_pair<128, 4, false, false, 256>(Xq, Wq, p.N, q, dev, st);
        case 192: return launch_pair<192, 3, false, false, 256>(Xq, Wq, p.N, q, dev, st);
        case 512: return launch_pair<512, 4, false>(Xq, Wq, p.N, q, dev, st);
        default: return launch_pair<256, 3, false, false, 256>(Xq, Wq, p.N, q, dev, st);
      }
    }
    switch (bn) {
      case 128: return launch_pair<128, 8, false>(Xq, Wq, p.N, q, dev, st);
      case 192: return launch_pair<192, 6, false>(Xq, Wq, p.N, q, dev, st);
      case 512: return launch_pair<512, 4, false>(Xq, Wq, p.N, q, dev, st);
      default: return launch_pair<256, 6, false>(Xq, Wq, p.N, q, dev, st);
    }
  }
  const int64_t tiles = int64_t((p.rows + kBM - 1) / kBM) * ((p.N + kBN - 1) / kBN);
  return launch_gemm<false>(Xq, p.rows, Wq, p.N, q, tiles, st);
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

bool valid_fmt(int fmt) { return fmt == FP8Q_FMT_E4M3 || fmt == FP8Q_FMT_E5M2; }

// weights = true: the kernel lets the next one start only when it has
// finished (the GEMMs read weight tiles before their dependency wait).
fp8q_status quantize(const void* X, int64_t M, int64_t K, uint8_t* Q, float* S, void* stream,
                     int fmt = FP8Q_FMT_E4M3, bool weights = false) {
  fp8q_status s = check_quant_args(X, M, K, Q, S);
  if (s != FP8Q_OK || M == 0) return s;
  const __half* Xh = static_cast<const __half*>(X);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int m = static_cast<int>(M), k = static_cast<int>(K);
  const cudaError_t e = fmt == FP8Q_FMT_E5M2 ? launch_quant_rows<kFmtE5M2>(Xh, m, k, Q, S, st, RowDispatch{}, !weights)
                                             : launch_quant_rows<kFmtE4M3>(Xh, m, k, Q, S, st, RowDispatch{}, !weights);
  if (e != cudaSuccess) return cuda_fail(e, "quant_rows launch");
  return FP8Q_OK;
}

// Dense linear, activations in format x_fmt (weights E4M3).
fp8q_status linear_impl(const uint8_t* Xq, int x_fmt, const float* s_x, const uint8_t* Wq, const float* s_w,
                        int64_t M, int64_t N, int64_t K, void* Y_f16, void* stream) {
  if (!valid_fmt(x_fmt)) return invalid("x_fmt must be FP8Q_FMT_E4M3 or FP8Q_FMT_E5M2");
  if (M < 0 || M > kMaxDim) return invalid("M out of range");
  if (N <= 0 || N > kMaxDim || N % 8 != 0) return invalid("N must be positive and a multiple of 8");
  if (K <= 0 || K > kMaxDim || K % 16 != 0) return invalid("K must be positive and a multiple of 16");
  if (M == 0) return FP8Q_OK;
  if (!aligned16(Xq) || !aligned16(s_x) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(Y_f16))
    return invalid("null or non-16-byte-aligned pointer");
  GemmParams p = {};   // every field set below; zero for the rest
  p.s_x = s_x;
  p.s_w = s_w;
  p.Y = static_cast<__half*>(Y_f16);
  p.offsets = nullptr;
  p.rows = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.E = 1;
  p.n_fastest = 0;
  p.main_tiles = 0;
  p.tail_q = 1;
  p.l2_prefetch = l2_prefetch_enabled();
  p.x_fmt = x_fmt;
  return launch_dense(Xq, Wq, p, static_cast<cudaStream_t>(stream));
}

}  // namespace
// ------------------------------------------------------------------ allocation-free variant
// Scratch for fp8q_quantized_linear_noalloc: the E4M3 codes and per-row
// scales that the two-step path keeps between its quantizer and its GEMM.
// It is part of the library image, so every GPU that loads the library holds
// these 8 MiB + 64 KiB until the process exits.
constexpr size_t kNoAllocCodeBytes = size_t(8) << 20;    // M * K codes
constexpr size_t kNoAllocScaleCount = size_t(16) << 10;  // M scales
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocCodeBytes + kNoAllocScaleCount * 4];

// Device address of the scratch array, looked up with that device current
// (host code cannot use the array's name as a device pointer) and kept once
// the lookup has succeeded; a failed lookup is not kept, so a later call
// tries again.
static fp8q_status noalloc_scratch(uint8_t** out) {
  static uint8_t* slots[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return cuda_fail(cudaErrorInvalidDevice, "device index");
  std::lock_guard<std::mutex> g(mu);
  if (slots[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol, "cudaGetSymbolAddress(scratch)");
    }
    slots[dev] = static_cast<uint8_t*>(p);
  }
  *out = slots[dev];
  return FP8Q_OK;
}

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
  return quantize(W_f16, N, K, Wq, s_w, stream, FP8Q_FMT_E4M3, true);
}

fp8q_status fp8q_quantize_rows_dynamic_fmt(const void* X_f16, int64_t M, int64_t K, fp8q_format fmt, uint8_t* Xq,
                                           float* s_x, void* stream) {
  if (!valid_fmt(fmt)) return invalid("fmt must be FP8Q_FMT_E4M3 or FP8Q_FMT_E5M2");
  return quantize(X_f16, M, K, Xq, s_x, stream, fmt);
}

fp8q_status fp8q_quantize_rows_dispatch(const void* X_f16, int64_t T, int64_t K, fp8q_format fmt,
                                        const int32_t* token_rows, int32_t topk, int64_t rows, uint8_t* Xq,
                                        float* s_x, void* stream) {
  if (!valid_fmt(fmt)) return invalid("fmt must be FP8Q_FMT_E4M3 or FP8Q_FMT_E5M2");
  if (topk < 1 || topk > 8) return invalid("topk must be in [1, 8]");
  if (rows < 0 || rows > kMaxDim || rows * K > (int64_t(1) << 40)) return invalid("rows out of range");
  fp8q_status s = check_quant_args(X_f16, T, K, rows > 0 ? Xq : nullptr, rows > 0 ? s_x : nullptr);
  if (s != FP8Q_OK) return s;
  if (T == 0) return FP8Q_OK;
  if (rows == 0) return invalid("tokens with no grouped rows");
  if (token_rows == nullptr || (reinterpret_cast<uintptr_t>(token_rows) & 3u) != 0)
    return invalid("token_rows pointer");
  RowDispatch d;
  d.rows = token_rows;
  d.topk = topk;
  d.out_rows = static_cast<int>(rows);
  const __half* Xh = static_cast<const __half*>(X_f16);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = fmt == FP8Q_FMT_E5M2
                            ? launch_quant_rows<kFmtE5M2>(Xh, static_cast<int>(T), static_cast<int>(K), Xq, s_x, st, d)
                            : launch_quant_rows<kFmtE4M3>(Xh, static_cast<int>(T), static_cast<int>(K), Xq, s_x, st, d);
  if (e != cudaSuccess) return cuda_fail(e, "quant_rows dispatch launch");
  return FP8Q_OK;
}

fp8q_status fp8q_quantize_weight_per_tensor(const void* W_f16, int64_t N, int64_t K, uint8_t* Wq, float* s_w,
                                            void* stream) {
  if (N == 0) return invalid("N must be positive");
  fp8q_status s = check_quant_args(W_f16, N, K, Wq, s_w);
  if (s != FP8Q_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const __half* W = static_cast<const __half*>(W_f16);
  const int64_t nvec = N * K / 8;
  int dev = 0, sms = 0;
  cudaError_t e = current_device_info(&dev, &sms);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  const int64_t want = (nvec + 255) / 256;
  const int grid = static_cast<int>(want < 4 * sms ? want : 4 * sms);
  e = cudaMemsetAsync(s_w, 0, sizeof(float), st);   // S[0] accumulates the amax bits
  if (e == cudaSuccess)
    e = launch_pdl(tensor_amax_kernel, dim3(grid), dim3(256), st, W, nvec, reinterpret_cast<unsigned int*>(s_w));
  if (e == cudaSuccess)
    e = launch_pdl(quant_tensor_kernel, dim3(grid), dim3(256), st, W, static_cast<int>(N), nvec, Wq, s_w);
  if (e == cudaSuccess) e = launch_pdl(quant_tensor_finish_kernel, dim3(1), dim3(32), st, s_w);
  if (e != cudaSuccess) return cuda_fail(e, "per-tensor quantization launch");
  return FP8Q_OK;
}

fp8q_status fp8q_linear(const uint8_t* Xq, const float* s_x, const uint8_t* Wq, const float* s_w, int64_t M,
                        int64_t N, int64_t K, void* Y_f16, void* stream) {
  return linear_impl(Xq, FP8Q_FMT_E4M3, s_x, Wq, s_w, M, N, K, Y_f16, stream);
}

fp8q_status fp8q_linear_fmt(const uint8_t* Xq, fp8q_format x_fmt, const float* s_x, const uint8_t* Wq,
                            const float* s_w, int64_t M, int64_t N, int64_t K, void* Y_f16, void* stream) {
  return linear_impl(Xq, x_fmt, s_x, Wq, s_w, M, N, K, Y_f16, stream);
}

fp8q_status fp8q_quantized_linear(const void* X_f16, const uint8_t* Wq, const float* s_w, int64_t M, int64_t N,
                                  int64_t K, void* Y_f16, uint8_t* Xq_ws, float* s_x_ws, void* stream) {
  if (M < 0 || M > kMaxDim) return invalid("M out of range");
  if (N <= 0 || N > kMaxDim || N % 8 != 0) return invalid("N must be positive and a multiple of 8");
  if (K <= 0 || K > kMaxDim || K % 16 != 0) return invalid("K must be positive and a multiple of 16");
  if (M == 0) return FP8Q_OK;
  if (!aligned16(X_f16) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(Y_f16))
    return invalid("null or non-16-byte-aligned pointer");
  const bool have_ws = Xq_ws != nullptr || s_x_ws != nullptr;
  if (have_ws && (!aligned16(Xq_ws) || !aligned16(s_x_ws))) return invalid("workspace pointers must both be 16-byte aligned");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // With a workspace: the two launches.  Without one: the fused kernel, up
  // to 64 rows (the CTAs of a split-K cluster share the row maxima of their
  // K slices, so no CTA reads whole fp16 rows).
  if (!have_ws && M <= kFusedMaxRows) {
    int dev = 0, sms = 0;
    const cudaError_t e = current_device_info(&dev, &sms);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    GemmParams p = {};
    p.s_w = s_w;
    p.Y = static_cast<__half*>(Y_f16);
    p.x_f16 = static_cast<const __half*>(X_f16);
    p.rows = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.E = 1;
    p.tail_q = 1;
    p.l2_prefetch = l2_prefetch_enabled();
    const fp8q_status s = M <= 16 ? launch_splitk<16, 5, true>(nullptr, Wq, p, dev, st)
                          : M <= 32 ? launch_splitk<32, 3, true>(nullptr, Wq, p, dev, st)
                                    : launch_splitk<64, 3, true>(nullptr, Wq, p, dev, st);
    if (s != FP8Q_ERR_UNSUPPORTED) return s;   // else: too long a K slice, use the two-step path
  }
  if (!have_ws) return invalid("Xq_ws and s_x_ws are required for this shape (two-step path)");
  fp8q_status s = fp8q_quantize_rows_dynamic(X_f16, M, K, Xq_ws, s_x_ws, stream);
  if (s != FP8Q_OK) return s;
  return fp8q_linear(Xq_ws, s_x_ws, Wq, s_w, M, N, K, Y_f16, stream);
}

fp8q_status fp8q_quantized_linear_overlapped(const void* X_f16, const uint8_t* Wq, const float* s_w, int64_t M,
                                             int64_t N, int64_t K, void* Y_f16, uint8_t* Xq_ws, float* s_x_ws,
                                             uint32_t* sync_ws, void* stream) {
  if (M < 0 || M > kMaxDim) return invalid("M out of range");
  if (N <= 0 || N > kMaxDim || N % 8 != 0) return invalid("N must be positive and a multiple of 8");
  if (K <= 0 || K > kMaxDim || K % 16 != 0) return invalid("K must be positive and a multiple of 16");
  if (M == 0) return FP8Q_OK;
  if (!aligned16(X_f16) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(Y_f16) || !aligned16(Xq_ws) ||
      !aligned16(s_x_ws) || !aligned16(sync_ws))
    return invalid("null or non-16-byte-aligned pointer");
  const Knobs kn = knobs();
  // Up to 128 rows (split-K kernels) or with another kernel family forced:
  // the two launches (the sync words are not touched).
  if (M <= kBM || kn.force == 1 || kn.force == 3)
    return fp8q_quantized_linear(X_f16, Wq, s_w, M, N, K, Y_f16, Xq_ws, s_x_ws, stream);
  int dev = 0, sms = 0;
  const cudaError_t e = current_device_info(&dev, &sms);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  GemmParams p = {};
  p.s_x = s_x_ws;
  p.s_w = s_w;
  p.Y = static_cast<__half*>(Y_f16);
  p.x_f16 = static_cast<const __half*>(X_f16);
  p.q_out = Xq_ws;
  p.s_out = s_x_ws;
  p.sync = sync_ws;
  p.rows = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.E = 1;
  p.tail_q = 1;
  p.x_fmt = FP8Q_FMT_E4M3;
  // n-blocks first: the first round of tiles needs only the first row blocks,
  // which the quantizing warps finish first.  FP8Q_RASTER = 1 overrides.
  static const int raster = [] {
    const char* v = std::getenv("FP8Q_RASTER");
    return v ? std::atoi(v) : 0;
  }();
  p.n_fastest = raster == 1 ? 0 : 1;
  const int clusters = max_pair_clusters<256, 6, false>(dev);
  const int bn = kn.bn ? kn.bn : choose_pair_bn(M, N, clusters > 0 ? clusters : sms / 2);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (kn.stage_k == 256) {
    switch (bn) {
      case 128: return launch_pair<128, 4, false, true, 256>(Xq_ws, Wq, N, p, dev, st);
      case 192: return launch_pair<192, 3, false, true, 256>(Xq_ws, Wq, N, p, dev, st);
      default: return launch_pair<256, 3, false, true, 256>(Xq_ws, Wq, N, p, dev, st);
    }
  }
  switch (bn) {
    case 128: return launch_pair<128, 8, false, true>(Xq_ws, Wq, N, p, dev, st);
    case 192: return launch_pair<192, 6, false, true>(Xq_ws, Wq, N, p, dev, st);
    default: return launch_pair<256, 6, false, true>(Xq_ws, Wq, N, p, dev, st);
  }
}

int64_t fp8q_overlap_sync_words(int64_t M) { return M < 0 ? 0 : qa_sync_words(M); }

fp8q_status fp8q_quantized_linear_noalloc(const void* X_f16, const uint8_t* Wq, const float* s_w, int64_t M,
                                          int64_t N, int64_t K, void* Y_f16, void* stream) {
  if (M < 0 || M > kMaxDim) return invalid("M out of range");
  if (N <= 0 || N > kMaxDim || N % 8 != 0) return invalid("N must be positive and a multiple of 8");
  if (K <= 0 || K > kMaxDim || K % 16 != 0) return invalid("K must be positive and a multiple of 16");
  if (M == 0) return FP8Q_OK;
  if (M * K > int64_t(kNoAllocCodeBytes) || M > int64_t(kNoAllocScaleCount))
    return invalid("fp8q_quantized_linear_noalloc: M*K must be <= 8388608 and M <= 16384 (fixed scratch size)");
  if (!aligned16(X_f16) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(Y_f16))
    return invalid("null or non-16-byte-aligned pointer");
  uint8_t* scratch = nullptr;
  const fp8q_status st = noalloc_scratch(&scratch);
  if (st != FP8Q_OK) return st;
  // codes at the start, scales after them; every call overwrites both in full
  uint8_t* Xq = scratch;
  float* s_x = reinterpret_cast<float*>(scratch + kNoAllocCodeBytes);
  return fp8q_quantized_linear(X_f16, Wq, s_w, M, N, K, Y_f16, Xq, s_x, stream);
}

fp8q_status fp8q_moe_grouped_linear(const uint8_t* Xq, const float* s_x, const int32_t* offsets, int32_t E,
                                    int64_t rows, const uint8_t* Wq, const float* s_w, int64_t N, int64_t K,
                                    void* Y_f16, void* stream) {
  return fp8q_moe_grouped_linear_fmt(Xq, FP8Q_FMT_E4M3, s_x, offsets, E, rows, Wq, s_w, N, K, Y_f16, stream);
}

fp8q_status fp8q_moe_grouped_linear_fmt(const uint8_t* Xq, fp8q_format x_fmt, const float* s_x,
                                        const int32_t* offsets, int32_t E, int64_t rows, const uint8_t* Wq,
                                        const float* s_w, int64_t N, int64_t K, void* Y_f16, void* stream) {
  if (!valid_fmt(x_fmt)) return invalid("x_fmt must be FP8Q_FMT_E4M3 or FP8Q_FMT_E5M2");
  if (E < 1 || E > kMaxExperts) return invalid("E must be in [1, 1024]");
  if (rows < 0 || rows > kMaxDim) return invalid("rows out of range");
  if (N <= 0 || N % 8 != 0 || int64_t(E) * N > kMaxDim) return invalid("N must be positive, a multiple of 8, E*N < 2^31");
  if (K <= 0 || K > kMaxDim || K % 16 != 0) return invalid("K must be positive and a multiple of 16");
  if (offsets == nullptr || (reinterpret_cast<uintptr_t>(offsets) & 3u) != 0) return invalid("offsets pointer");
  if (rows == 0) return FP8Q_OK;
  if (!aligned16(Xq) || !aligned16(s_x) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(Y_f16))
    return invalid("null or non-16-byte-aligned pointer");
  GemmParams p = {};   // every field set below; zero for the rest
  p.s_x = s_x;
  p.s_w = s_w;
  p.Y = static_cast<__half*>(Y_f16);
  p.offsets = offsets;
  p.rows = static_cast<int>(rows);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.E = E;
  p.n_fastest = 0;
  p.main_tiles = 0;
  p.tail_q = 1;
  p.l2_prefetch = l2_prefetch_enabled();
  p.half_tiles = knobs().half_tiles;
  p.x_fmt = x_fmt;
  // Single-CTA 128-row tiles by default; kernel family 2 selects CTA-pair
  // tiles of 256 expert rows (each weight tile read by half as many row
  // blocks), which measured no faster for the up projection and slower for
  // the down projection (8 K blocks per tile) on B200.
  if (knobs().force == 2) {
    int dev = 0, sms = 0;
    const cudaError_t e = current_device_info(&dev, &sms);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    const int64_t tiles = ((rows + 2 * kBM - 1) / (2 * kBM) + E) * ((N + 255) / 256);
    return launch_pair<256, 5, true>(Xq, Wq, int64_t(E) * N, p, dev, static_cast<cudaStream_t>(stream), tiles);
  }
  const int64_t tiles = ((rows + kBM - 1) / kBM + E) * ((N + kBNGrouped - 1) / kBNGrouped);
  return launch_gemm<true>(Xq, rows, Wq, int64_t(E) * N, p, tiles, static_cast<cudaStream_t>(stream));
}

fp8q_status fp8q_moe_grouped_linear_gather(const uint8_t* Xq_tok, const float* s_x_tok, int64_t tokens,
                                           const int32_t* row_token, const int32_t* offsets, int32_t E, int64_t rows,
                                           const uint8_t* Wq, const float* s_w, int64_t N, int64_t K, void* Y_f16,
                                           void* stream) {
  if (E < 1 || E > kMaxExperts) return invalid("E must be in [1, 1024]");
  if (rows < 0 || rows > kMaxDim) return invalid("rows out of range");
  if (tokens <= 0 || tokens > kMaxDim) return invalid("tokens must be positive");
  if (N <= 0 || N % 8 != 0 || int64_t(E) * N > kMaxDim) return invalid("N must be positive, a multiple of 8, E*N < 2^31");
  if (K <= 0 || K > kMaxDim || K % 16 != 0) return invalid("K must be positive and a multiple of 16");
  if (offsets == nullptr || (reinterpret_cast<uintptr_t>(offsets) & 3u) != 0) return invalid("offsets pointer");
  if (row_token == nullptr || (reinterpret_cast<uintptr_t>(row_token) & 3u) != 0) return invalid("row_token pointer");
  if (rows == 0) return FP8Q_OK;
  if (!aligned16(Xq_tok) || !aligned16(s_x_tok) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(Y_f16))
    return invalid("null or non-16-byte-aligned pointer");
  GemmParams p = {};   // every field set below; zero for the rest
  p.s_x = s_x_tok;
  p.s_w = s_w;
  p.Y = static_cast<__half*>(Y_f16);
  p.offsets = offsets;
  p.rows = static_cast<int>(rows);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.E = E;
  p.tail_q = 1;
  p.x_fmt = FP8Q_FMT_E4M3;
  p.xq = Xq_tok;
  p.row_token = row_token;
  p.tokens = static_cast<int>(tokens);
  const int64_t tiles = ((rows + kBM - 1) / kBM + E) * ((N + kBNGrouped - 1) / kBNGrouped);
  // the A tensor map (token matrix) is built but unused: the producer gathers the rows
  return launch_gemm<true, true>(Xq_tok, tokens, Wq, int64_t(E) * N, p, tiles, static_cast<cudaStream_t>(stream));
}

fp8q_status fp8q_moe_grouped_linear_combine(const uint8_t* Xq, const float* s_x, const int32_t* offsets, int32_t E,
                                            int64_t rows, const uint8_t* Wq, const float* s_w, int64_t N, int64_t K,
                                            const int32_t* row_token, const float* row_weight, int64_t tokens,
                                            void* out_f16, void* stream) {
  if (E < 1 || E > kMaxExperts) return invalid("E must be in [1, 1024]");
  if (rows < 0 || rows > kMaxDim) return invalid("rows out of range");
  if (tokens <= 0 || tokens > kMaxDim || tokens * N > (int64_t(1) << 40)) return invalid("tokens out of range");
  if (N <= 0 || N % 8 != 0 || int64_t(E) * N > kMaxDim) return invalid("N must be positive, a multiple of 8, E*N < 2^31");
  if (K <= 0 || K > kMaxDim || K % 16 != 0) return invalid("K must be positive and a multiple of 16");
  if (offsets == nullptr || (reinterpret_cast<uintptr_t>(offsets) & 3u) != 0) return invalid("offsets pointer");
  if (rows > 0 && (row_token == nullptr || (reinterpret_cast<uintptr_t>(row_token) & 3u) != 0))
    return invalid("row_token pointer");
  if (rows > 0 && (row_weight == nullptr || (reinterpret_cast<uintptr_t>(row_weight) & 3u) != 0))
    return invalid("row_weight pointer");
  if (!aligned16(out_f16)) return invalid("null or non-16-byte-aligned output");
  // every check before the output is touched (with no rows, the row-side pointers may be null)
  if (rows > 0 && (!aligned16(Xq) || !aligned16(s_x) || !aligned16(Wq) || !aligned16(s_w)))
    return invalid("null or non-16-byte-aligned pointer");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(out_f16, 0, static_cast<size_t>(tokens * N) * sizeof(__half), st);
  if (e != cudaSuccess) return cuda_fail(e, "combine output clear");
  if (rows == 0) return FP8Q_OK;
  GemmParams p = {};   // every field set below; zero for the rest
  p.s_x = s_x;
  p.s_w = s_w;
  p.Y = static_cast<__half*>(out_f16);
  p.offsets = offsets;
  p.rows = static_cast<int>(rows);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.E = E;
  p.tail_q = 1;
  p.l2_prefetch = l2_prefetch_enabled();
  p.half_tiles = knobs().half_tiles;
  p.x_fmt = FP8Q_FMT_E4M3;
  p.tokens = static_cast<int>(tokens);
  p.comb_token = row_token;
  p.comb_weight = row_weight;
  const int64_t tiles = ((rows + kBM - 1) / kBM + E) * ((N + kBNGrouped - 1) / kBNGrouped);
  return launch_gemm<true>(Xq, rows, Wq, int64_t(E) * N, p, tiles, st);
}

fp8q_status fp8q_quantize_weight_blockwise(const void* W_f16, int32_t E, int64_t N, int64_t K, uint8_t* Wq,
                                           float* s_wb, void* stream) {
  if (E < 1 || E > kMaxExperts) return invalid("E must be in [1, 1024]");
  if (N <= 0 || N > kMaxDim || int64_t(E) * N > kMaxDim) return invalid("N must be positive, E*N < 2^31");
  fp8q_status s = check_quant_args(W_f16, int64_t(E) * N, K, Wq, s_wb);
  if (s != FP8Q_OK) return s;
  const int NB = static_cast<int>((N + kBsBlk - 1) / kBsBlk);
  const int KB = static_cast<int>((K + kBsBlk - 1) / kBsBlk);
  if (KB > 65535) return invalid("K too large for the block grid");
  const cudaError_t e = launch_pdl(quant_blocks_kernel, dim3(E * NB, KB), dim3(256), static_cast<cudaStream_t>(stream),
                                   static_cast<const __half*>(W_f16), static_cast<int>(N), static_cast<int>(K), NB, KB,
                                   Wq, s_wb);
  if (e != cudaSuccess) return cuda_fail(e, "quant_blocks launch");
  return FP8Q_OK;
}

fp8q_status fp8q_moe_grouped_linear_blockscaled(const uint8_t* Xq, const float* s_x, const int32_t* offsets,
                                                int32_t E, int64_t rows, const uint8_t* Wq, const float* s_wb,
                                                int64_t N, int64_t K, void* Y_f16, void* stream) {
  if (E < 1 || E > kBsMaxExperts) return invalid("E must be in [1, 128] for block-scaled weights");
  if (rows < 0 || rows > kMaxDim) return invalid("rows out of range");
  if (N <= 0 || N % 8 != 0 || int64_t(E) * N > kMaxDim) return invalid("N must be positive, a multiple of 8, E*N < 2^31");
  if (K <= 0 || K > kMaxDim || K % 16 != 0) return invalid("K must be positive and a multiple of 16");
  if (offsets == nullptr || (reinterpret_cast<uintptr_t>(offsets) & 3u) != 0) return invalid("offsets pointer");
  if (rows == 0) return FP8Q_OK;
  if (!aligned16(Xq) || !aligned16(s_x) || !aligned16(Wq) || !aligned16(s_wb) || !aligned16(Y_f16))
    return invalid("null or non-16-byte-aligned pointer");
  int dev = 0, sms = 0;
  cudaError_t e = current_device_info(&dev, &sms);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  GemmParams p = {};
  p.s_x = s_x;
  p.s_w = s_wb;   // block scales [E, ceil(N/128), ceil(K/128)]
  p.Y = static_cast<__half*>(Y_f16);
  p.offsets = offsets;
  p.rows = static_cast<int>(rows);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.E = E;
  p.tail_q = 1;
  p.x_fmt = FP8Q_FMT_E4M3;
  constexpr int kStagesBs = 4;
  using L = BsLayout<kStagesBs>;
  CUtensorMap ta, tb, ty;
  fp8q_status s = make_operand_map(&ta, Xq, rows, K, kBM);
  if (s != FP8Q_OK) return s;
  s = make_operand_map(&tb, Wq, int64_t(E) * N, K, kBsBN);
  if (s != FP8Q_OK) return s;
  s = make_output_map(&ty, p.Y, rows, N);
  if (s != FP8Q_OK) return s;
  e = ensure_smem<fp8_gemm_blockscaled_kernel<kStagesBs>>(L::smem_bytes(kBsMaxExperts), dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(blockscaled)");
  const int64_t tiles = ((rows + kBM - 1) / kBM + E) * ((N + kBsBN - 1) / kBsBN);
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  e = launch_ex(fp8_gemm_blockscaled_kernel<kStagesBs>, dim3(grid), dim3(kBsThreads), L::smem_bytes(E),
                static_cast<cudaStream_t>(stream), 1, true, ta, tb, ty, p);
  if (e != cudaSuccess) {
    cudaFuncAttributes fa = {};
    (void)cudaFuncGetAttributes(&fa, fp8_gemm_blockscaled_kernel<kStagesBs>);
    char msg[256];
    std::snprintf(msg, sizeof(msg),
                  "fp8_gemm_blockscaled_kernel launch (%d threads, %zu B dynamic smem; kernel: %d regs, max %d "
                  "threads, %zu B static smem, max dynamic %d)",
                  kBsThreads, L::smem_bytes(E), fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes,
                  fa.maxDynamicSharedSizeBytes);
    return cuda_fail(e, msg);
  }
  return FP8Q_OK;
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

fp8q_status fp8q_set_gemm_tuning(int kernel_family, int tile_n, int ksplit) {
  if (kernel_family < 0 || kernel_family > 3) return invalid("kernel_family must be 0, 1, 2 or 3");
  if (tile_n != 0 && tile_n != 128 && tile_n != 192 && tile_n != 256 && tile_n != 512)
    return invalid("tile_n must be 0, 128, 192, 256 or 512");
  if (ksplit != 0 && ksplit != 1 && ksplit != 2 && ksplit != 4 && ksplit != 8)
    return invalid("ksplit must be 0, 1, 2, 4 or 8");
  knobs().force = kernel_family;
  knobs().bn = tile_n;
  knobs().ksplit = ksplit;
  return FP8Q_OK;
}

fp8q_status fp8q_selftest_wait_timeout(uint32_t limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 2000000u) return invalid("limit_us must be in [1, 2000000]");
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(uint64_t(limit_us) * 1000u);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "wait_timeout_selftest launch");
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
           FP8Q_DEVERR_TIMEOUT_CLUSTER | FP8Q_DEVERR_TIMEOUT_SELFTEST))
    return FP8Q_ERR_TIMEOUT;
  if (v) return FP8Q_ERR_DEVICE_CHECK;
  return FP8Q_OK;
}

}  // extern "C"
