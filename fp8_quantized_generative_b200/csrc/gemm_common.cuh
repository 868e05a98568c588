// Pieces shared by the single-CTA and CTA-pair FP8 GEMM kernels: problem
// parameters, warp roles and the fused dequantization epilogue.
//
// Epilogue arithmetic ("Quantized Inference for OneRec-V2", 关键证据 steps
// 3-4; "FP8量化在生成式推荐系统OneRec-V2中的优化实践" §2.3): the FP32
// accumulator of output (m, n) is scaled by the per-token scale s_x[m] and the
// per-channel scale s_w[n], in that order, each an fp32 multiply rounded to
// nearest, and cast once to fp16 (round to nearest even).
#pragma once

#include <cuda.h>

#include "ptx.cuh"

namespace fp8q {

constexpr int kBM = 128;          // rows of a CTA's output slab (TMEM lanes)
constexpr int kBK = 128;          // K bytes per pipeline stage (one 128-B swizzle row)
constexpr int kUmmaK = 32;        // K per tcgen05.mma for 8-bit operands
constexpr int kEpiWarp0 = 2;      // warps 0, 1: TMA producer, MMA issuer
constexpr int kEpiWarps = 8;      // two epilogue warps per TMEM lane quadrant
constexpr int kGemmThreads = (kEpiWarp0 + kEpiWarps) * 32;
constexpr int kStageTileBytes = 32 * 32 * 2;   // one 32 x 32 fp16 output tile per epilogue warp
constexpr int kEpiSmemBytes = kEpiWarps * kStageTileBytes;
constexpr int kMaxExperts = 1024;

struct GemmParams {
  const float* s_x;         // [rows]
  const float* s_w;         // [E*N]
  __half* Y;                // [rows, N]
  const int32_t* offsets;   // [E+1] device, grouped only
  const __half* x_f16;      // [rows, K] fp16 activations, fused quantize + GEMM only
  int rows;                 // M (dense) or total grouped rows
  int N;
  int K;
  int E;                    // 1 for dense
  int n_fastest;            // dense tile order: 1 = walk n-blocks first
  // CTA-pair kernel tail split: the first main_tiles full tiles run at full
  // width; each remaining full tile is cut along N into tail_q pieces
  // (tail_q in {1, 2, 4}) so that the last round keeps every cluster busy.
  int main_tiles;
  int tail_q;
  int l2_prefetch;          // split-K: 1 = prefetch the rest of the weight slice into L2 at start
};

// One output slab of a CTA: 128 rows starting at row0, BN columns at n0.
struct EpiTile {
  int row0;
  int row_end;   // rows >= row_end are not stored
  int n0;
  int sw0;       // index into s_w of column n0
  bool tma;      // the bulk tensor store may write the whole slab
};

// Staging layout of a 32 x 32 fp16 tile: row r occupies 64 bytes, its four
// 16-byte chunks permuted as chunk c -> c ^ ((r >> 1) & 3).  This is the
// layout a 64-byte-swizzled TMA box of 32 x 32 fp16 expects (chunk bits 4-5
// XOR address bits 7-8), and it makes both the per-row writes and the
// row-group reads of a warp free of bank conflicts.
__device__ __forceinline__ uint32_t stage_off(int r, int c) {
  return static_cast<uint32_t>(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

// The scales one epilogue lane applies to a slab: s_x of its row and, for
// each 32-column chunk of its warp, s_w of column (chunk start + lane).
template <int kMaxChunks>
struct EpiScales {
  float sx;
  float sw[kMaxChunks];
};

template <int kMaxChunks>
__device__ __forceinline__ EpiScales<kMaxChunks> epilogue_scales(const EpiTile& t, const GemmParams& p, int warp,
                                                                 int lane, int bn) {
  EpiScales<kMaxChunks> e;
  const int q = warp & 3;
  const int h = (warp - kEpiWarp0) >> 2;
  const int r = t.row0 + q * 32 + lane;
  e.sx = r < t.row_end ? __ldg(p.s_x + r) : 0.0f;
#pragma unroll
  for (int j = 0; j < kMaxChunks; ++j) {
    const int cl = h * (bn / 2) + j * 32 + lane;
    e.sw[j] = (j < bn / 64 && t.n0 + cl < p.N) ? __ldg(p.s_w + t.sw0 + cl) : 0.0f;
  }
  return e;
}

// One epilogue warp drains its 32 TMEM lanes (rows q*32 .. q*32+31 of the
// slab, q = warp % 4 as tcgen05.ld requires) over its half of the bn columns,
// 32 columns at a time: TMEM -> registers -> scale and cast -> swizzled
// staging tile in shared memory -> one bulk tensor store (or, for a slab cut
// by an expert boundary, coalesced row-masked stores).
// `bn` is the slab width (a multiple of 64, at most 64 * kMaxChunks; each
// warp takes bn/2 columns).
//
// Two paces.  While the MMAs of the next tile run (kDrain = false) each chunk
// fetches its weight scales and waits for its TMEM load before the next one
// starts; a faster epilogue there was measured to slow the concurrent MMAs
// by about 3% (it competes with them for the SM's shared-memory and TMEM
// traffic), more than it saves.  For a CTA's last tile (kDrain = true)
// nothing else runs: the scales `pre` were loaded before the accumulator
// wait, and the TMEM load of chunk j+1 is in flight while chunk j is scaled
// and stored, which shortens the exposed final epilogue by about a third.
template <int kMaxChunks, bool kDrain>
__device__ __forceinline__ void epilogue_slab(const EpiTile& t, const GemmParams& p, const CUtensorMap* tmY,
                                              uint32_t tmem_acc, int warp, int lane, uint8_t* stage, int bn,
                                              const EpiScales<kMaxChunks>& pre) {
  const int q = warp & 3;
  const int h = (warp - kEpiWarp0) >> 2;
  const int nch = bn / 64;
  const int r = t.row0 + q * 32 + lane;
  const float sx = kDrain ? pre.sx : (r < t.row_end ? __ldg(p.s_x + r) : 0.0f);
  const uint32_t sbase = smem_u32(stage);
  const uint32_t taddr0 = tmem_acc + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(h * (bn / 2));
  uint32_t v[2][32];
  if (kDrain) {
    tmem_ld_32x32b_x32(taddr0, v[0]);
    tmem_ld_wait_regs(v[0]);
  }
#pragma unroll
  for (int j = 0; j < kMaxChunks; ++j) {
    if (j >= nch) break;
    const int cl = h * (bn / 2) + j * 32;   // first column of the chunk within the slab
    uint32_t* cur = v[kDrain ? (j & 1) : 0];
    float sw_lane;
    if (kDrain) {
      sw_lane = pre.sw[j];
      if (j + 1 < nch) tmem_ld_32x32b_x32(taddr0 + static_cast<uint32_t>((j + 1) * 32), v[(j + 1) & 1]);
    } else {
      sw_lane = t.n0 + cl + lane < p.N ? __ldg(p.s_w + t.sw0 + cl + lane) : 0.0f;
      tmem_ld_32x32b_x32(taddr0 + static_cast<uint32_t>(j * 32), v[0]);
      tmem_ld_wait_regs(v[0]);
    }
    uint32_t packed[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float w0 = __shfl_sync(0xffffffffu, sw_lane, 2 * i);
      const float w1 = __shfl_sync(0xffffffffu, sw_lane, 2 * i + 1);
      const float y0 = __fmul_rn(__fmul_rn(__uint_as_float(cur[2 * i]), sx), w0);
      const float y1 = __fmul_rn(__fmul_rn(__uint_as_float(cur[2 * i + 1]), sx), w1);
      const __half2 hv = __floats2half2_rn(y0, y1);
      packed[i] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    // The previous bulk store of this warp must have finished reading the tile.
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 4; ++c)
      st_shared_v4(sbase + stage_off(lane, c), packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
    if (t.tma) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(tmY, stage, t.n0 + cl, t.row0 + q * 32);
        bulk_commit_group();
      }
    } else {
      __syncwarp();
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int rr = it * 8 + (lane >> 2);
        const int c = lane & 3;
        const uint4 val = ld_shared_v4(sbase + stage_off(rr, c));
        const int grow = t.row0 + q * 32 + rr;
        const int gcol = t.n0 + cl + c * 8;
        if (grow < t.row_end && gcol < p.N)
          *reinterpret_cast<uint4*>(p.Y + static_cast<int64_t>(grow) * p.N + gcol) = val;
      }
      __syncwarp();
    }
    if (kDrain && j + 1 < nch) tmem_ld_wait_regs(v[(j + 1) & 1]);
  }
}

}  // namespace fp8q
