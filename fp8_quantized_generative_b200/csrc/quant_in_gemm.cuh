// Per-token activation quantization inside the CTA-pair GEMM (quantize +
// FP8 GEMM + dequantize as one kernel: "FP8量化在生成式推荐系统OneRec-V2中的
// 优化实践" §2.3, the QuantizeLinear + GEMM + Dequantize fusion; the steps of
// "Quantized Inference for OneRec-V2" 关键证据 steps 2-4).
//
// The row maximum needs the whole fp16 row before the first code, so the
// codes still go through global memory; what the fusion removes is the
// serialization of the two kernels.  The epilogue warps of every CTA, idle
// until their first accumulator is ready, quantize rows round-robin over the
// grid in row order (so the first 128-row blocks finish first), and the TMA
// producer waits only for the row blocks of its own tile:
//   * a warp quantizes one row (same steps and helpers as quant_rows_kernel,
//     so the same codes and scales), fences its stores for the async proxy,
//     and after a warp barrier one lane adds the row to its block's counter
//     with a release add (no return trip);
//   * the producer acquires the counter until the block is complete
//     (bounded wait) and fences the async proxy before its first TMA load of
//     those rows; the epilogue acquires it before reading the rows' scales;
//   * the last CTA to finish clears the counters, so every call starts from
//     zeros (the workspace is zeroed once by its owner).
// All ten warps quantize the first pass of rows (the producer cannot load
// before them anyway); the epilogue warps then quantize the rest.
// Once a waiter has seen every row done (word 1), it needs no further
// acquire or proxy fence in this call.
// Sync words: [0] CTAs finished, [1] rows quantized in all, then per 128-row
// block m [2 + 2m] rows quantized ([3 + 2m] unused).
#pragma once

#include "quant_rows.cuh"

namespace fp8q {

constexpr int kQaRowsPerBlock = 128;   // = the A rows one CTA of a pair loads

__host__ __device__ constexpr int64_t qa_sync_words(int64_t rows) {
  return 2 + 2 * ((rows + kQaRowsPerBlock - 1) / kQaRowsPerBlock);
}
__device__ __forceinline__ uint32_t* qa_count(uint32_t* sync, int blk) { return sync + 2 + 2 * blk; }

__device__ __forceinline__ void red_release_gpu_add(uint32_t* ptr, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}

// One warp: E4M3 codes and scale of row `row` of X [rows, K] (K % 16 == 0).
// Rows up to 2048 elements stay in registers (X read once); longer rows are
// read twice (the second time from L2).
__device__ __forceinline__ void warp_quant_row(const __half* __restrict__ X, int K, int row,
                                               uint8_t* __restrict__ Q, float* __restrict__ S, int lane) {
  const int nvec = K >> 3;
  const uint4* src = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(row) * K);
  uint2* dst = reinterpret_cast<uint2*>(Q + static_cast<int64_t>(row) * K);
  float m = 0.0f;
  RowScale rs;
  if (nvec <= 256) {
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = lane + 32 * i;
      v[i] = j < nvec ? __ldg(src + j) : make_uint4(0, 0, 0, 0);
      m = absmax8(v[i], m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    rs = row_scale_from_amax<kFmtE4M3>(m);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = lane + 32 * i;
      if (j < nvec) dst[j] = encode8<kFmtE4M3>(v[i], rs.r);
    }
  } else {
    for (int j = lane; j < nvec; j += 32) m = absmax8(__ldg(src + j), m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    rs = row_scale_from_amax<kFmtE4M3>(m);
    for (int j = lane; j < nvec; j += 32) dst[j] = encode8<kFmtE4M3>(__ldg(src + j), rs.r);
  }
  if (lane == 0) S[row] = rs.s;
}

// Quantize rows row0, row0 + stride, ... below row_end (one warp) and count
// each in its block.
__device__ __forceinline__ void quantize_rows_strided(const GemmParams& p, int row0, int stride, int row_end,
                                                      int lane) {
  uint32_t done = 0;
  for (int row = row0; row < row_end; row += stride, ++done) {
    warp_quant_row(p.x_f16, p.K, row, p.q_out, p.s_out, lane);
    fence_proxy_async_global();
    __syncwarp();
    if (lane == 0) red_release_gpu_add(qa_count(p.sync, row / kQaRowsPerBlock), 1u);
  }
  if (done > 0 && lane == 0) red_release_gpu_add(p.sync + 1, done);
}

// Rows of the first pass: one per warp of the grid (all warps of every CTA).
__device__ __forceinline__ int qa_first_pass_rows(const GemmParams& p, int ncta, int warps_per_cta) {
  const int n = ncta * warps_per_cta;
  return n < p.rows ? n : p.rows;
}

// Wait (bounded) until the 128-row block holding `row` is complete; rows past
// the matrix need no wait (TMA reads zeros there).  With `for_tma`, fence the
// async proxy so the following TMA loads see the codes.
__device__ __forceinline__ bool wait_rows_ready(const GemmParams& p, int row, bool for_tma) {
  if (row >= p.rows) return true;
  const int blk = row / kQaRowsPerBlock;
  const int left = p.rows - blk * kQaRowsPerBlock;
  const uint32_t need = static_cast<uint32_t>(left < kQaRowsPerBlock ? left : kQaRowsPerBlock);
  const uint32_t* c = qa_count(p.sync, blk);
  if (ld_acquire_gpu_u32(c) < need) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu_u32(c) < need) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
      __nanosleep(64);
    }
  }
  if (for_tma) fence_proxy_async_global();
  return true;
}

// Tracks, for one waiting thread, whether every row is known to be done.
struct RowsReady {
  bool all = false;
  // Wait (bounded) until the rows [row, row + 128) block is complete, or
  // everything is; fence the async proxy for TMA when asked.  false: timeout.
  __device__ __forceinline__ bool wait(const GemmParams& p, int row, bool for_tma) {
    if (all || row >= p.rows) return true;
    if (ld_acquire_gpu_u32(p.sync + 1) >= static_cast<uint32_t>(p.rows)) {
      all = true;
      if (for_tma) fence_proxy_async_global();
      return true;
    }
    return wait_rows_ready(p, row, for_tma);
  }
};

// Called by one thread of every CTA after all of the CTA's reads of the
// counters: the last CTA clears them for the next call.
__device__ __forceinline__ void release_sync(const GemmParams& p) {
  __threadfence();
  if (atomicAdd(p.sync, 1u) + 1u == gridDim.x) {
    const int nblk = (p.rows + kQaRowsPerBlock - 1) / kQaRowsPerBlock;
    for (int b = 0; b < nblk; ++b) atomicExch(qa_count(p.sync, b), 0u);
    atomicExch(p.sync + 1, 0u);
    atomicExch(p.sync, 0u);
    __threadfence();
  }
}

}  // namespace fp8q
