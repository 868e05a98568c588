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
// Staging for kBufs tiles per epilogue warp: buffer b of warp w at
// (b * kEpiWarps + w) * kStageTileBytes.
__host__ __device__ constexpr int epi_smem_bytes(int bufs) { return bufs * kEpiWarps * kStageTileBytes; }
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
  int half_tiles;           // CTA-pair grouped kernel: an expert's last <= 128 rows as an M = 128 pair tile
  int x_fmt;                // activation code format (Fp8Fmt): E4M3, or E5M2 for the variant
  const uint8_t* xq;        // grouped gather: the token matrix of activation codes [tokens, K]
  const int32_t* row_token; // grouped gather: row r of the product reads token row_token[r] (nullptr: row r)
  int tokens;               // grouped gather / combine: rows of the token matrix
  const int32_t* comb_token; // combine: grouped row r adds into output row comb_token[r] (nullptr: plain store)
  const float* comb_weight;  // combine: the weight of grouped row r
  // CTA-pair dense kernel with the activation quantization inside it: the
  // codes and scales of x_f16 are written to q_out / s_out (= the A operand
  // and s_x); sync holds the per-128-row-block ready flags.
  uint8_t* q_out;
  float* s_out;
  uint32_t* sync;
};

// Row of the activation codes / scales that product row r reads (the row
// itself, or its token in the gathered MoE form; an index out of range reads
// row 0 and is reported by the producer).
__device__ __forceinline__ int act_row(const GemmParams& p, int r) {
  if (p.row_token == nullptr) return r;
  const int t = __ldg(p.row_token + r);
  return (t >= 0 && t < p.tokens) ? t : 0;
}

// One output slab of a CTA: 128 rows starting at row0, BN columns at n0.
struct EpiTile {
  int row0;
  int row_end;   // rows >= row_end are not stored
  int n0;
  int sw0;       // index into s_w of column n0
  bool clip;     // rows >= row_end lie past the output tensor, where a bulk store clips them
};

// Staging layout of a 32 x 32 fp16 tile: row r occupies 64 bytes, its four
// 16-byte chunks permuted as chunk c -> c ^ ((r >> 1) & 3).  This is the
// layout a 64-byte-swizzled TMA box of 32 x 32 fp16 expects (chunk bits 4-5
// XOR address bits 7-8), and it makes both the per-row writes and the
// row-group reads of a warp free of bank conflicts.
__device__ __forceinline__ uint32_t stage_off(int r, int c) {
  return static_cast<uint32_t>(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

// What one epilogue warp drains: 32 output rows from qrow0, nch chunks of
// 32 columns from column col0 of the tile, held in the warp's TMEM lane
// quadrant (q = warp % 4, as tcgen05.ld requires) from TMEM column tcol0.
// Normal tiles: quadrant q holds rows q*32.. of the CTA's 128-row slab and
// the two warps of a quadrant split the bn columns.  Half tiles (a CTA-pair
// MMA with M = 128: 64 rows per CTA) keep the slab's 64 rows twice: lanes
// 0-63 hold columns 0..bn/2-1 and lanes 64-127 columns bn/2..bn-1, both at
// TMEM columns 0..bn/2-1 (measured on B200 with a layout probe).
struct EpiWarpView {
  int qrow0;
  int col0;
  int tcol0;
  int nch;
};

__device__ __forceinline__ EpiWarpView epi_view(const EpiTile& t, int warp, int bn, bool half) {
  const int q = warp & 3;
  const int h = (warp - kEpiWarp0) >> 2;
  EpiWarpView v;
  if (!half) {
    v.qrow0 = t.row0 + q * 32;
    v.col0 = h * (bn / 2);
    v.tcol0 = h * (bn / 2);
    v.nch = bn / 64;
  } else {
    v.qrow0 = t.row0 + (q & 1) * 32;
    v.col0 = (q >> 1) * (bn / 2) + h * (bn / 4);
    v.tcol0 = h * (bn / 4);
    v.nch = bn / 128;
  }
  return v;
}

// The scales one epilogue lane applies: s_x of its row and, for each 32-column
// chunk of its warp, s_w of column (chunk start + lane).  Loaded before the
// wait for the accumulator, so their latency hides behind the tile's MMAs.
template <int kMaxChunks>
struct EpiScales {
  float sx;
  float sw[kMaxChunks];
  float rw;    // combine: weight of this lane's row
  int ctok;    // combine: output (token) row of this lane's row, -1: none
};

template <int kMaxChunks>
__device__ __forceinline__ EpiScales<kMaxChunks> epilogue_scales(const EpiTile& t, const GemmParams& p,
                                                                 const EpiWarpView& w, int lane) {
  EpiScales<kMaxChunks> e;
  const int r = w.qrow0 + lane;
  // With the quantization inside the GEMM (q_out set) s_x is still being
  // written by this kernel: the caller reads it after its block's acquire.
  e.sx = (p.q_out == nullptr && r < t.row_end) ? __ldg(p.s_x + act_row(p, r)) : 0.0f;
  e.rw = 0.0f;
  e.ctok = -1;
  if (p.comb_token != nullptr && r < t.row_end) {
    const int tk = __ldg(p.comb_token + r);
    if (tk >= 0 && tk < p.tokens) {
      e.ctok = tk;
      e.rw = __ldg(p.comb_weight + r);
    } else {
      raise_error(0x8u);
    }
  }
#pragma unroll
  for (int j = 0; j < kMaxChunks; ++j) {
    const int cl = w.col0 + j * 32 + lane;
    e.sw[j] = (j < w.nch && t.n0 + cl < p.N) ? __ldg(p.s_w + t.sw0 + cl) : 0.0f;
  }
  return e;
}

// One epilogue warp drains its view (above), 32 columns at a time:
// TMEM -> registers -> scale and cast -> swizzled staging tile in shared
// memory -> one bulk tensor store.  A warp whose 32 rows all lie past row_end
// does nothing; one whose rows straddle row_end inside the tensor (an MoE
// expert boundary) stores its valid rows with coalesced masked stores
// instead of the bulk store.
// The scales `pre` were loaded before the accumulator wait, the TMEM load of
// chunk j+1 is in flight while chunk j is scaled and stored, and with two
// staging tiles per warp (kBufs = 2) chunk j+1 is written while the bulk
// store of chunk j still reads its tile.  (A slower variant that fetched the
// scales per chunk and waited out every load and store measured no faster
// on the dense shapes and up to 12% slower on the MoE kernels.)
// w.nch <= kMaxChunks.
template <int kMaxChunks, int kBufs>
__device__ __forceinline__ void epilogue_slab(const EpiTile& t, const GemmParams& p, const CUtensorMap* tmY,
                                              uint32_t tmem_acc, const EpiWarpView& w, int warp, int lane,
                                              uint8_t* stage, const EpiScales<kMaxChunks>& pre) {
  static_assert(kBufs == 1 || kBufs == 2, "staging buffers");
  const int q = warp & 3;
  const int nch = w.nch;
  const int qrow0 = w.qrow0;
  const int valid = t.row_end - qrow0;   // rows of this warp that are stored (<= 0: none)
  if (valid <= 0) return;
  // MoE combine: rows go back to their tokens with fp16 atomic adds, read
  // from the staging tile four lanes to a row so that each instruction adds
  // whole 32-byte sectors (half as many L2 atomic operations as one lane per
  // row, 16 bytes at a time).
  const bool combine = p.comb_token != nullptr;
  const bool bulk = !combine && (t.clip || valid >= 32);
  const uint32_t taddr0 = tmem_acc + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(w.tcol0);
  uint32_t v[2][32];
  tmem_ld_32x32b_x32(taddr0, v[0]);
  // Buffer j & 1 below assumes no store of an earlier slab still reads
  // either tile (that slab's last store was issued a whole mainloop ago).
  if (kBufs == 2 && lane == 0) bulk_wait_read_all();
  tmem_ld_wait_regs(v[0]);
#pragma unroll
  for (int j = 0; j < kMaxChunks; ++j) {
    if (j >= nch) break;
    const int cl = w.col0 + j * 32;   // first column of the chunk within the tile
    const uint32_t* cur = v[j & 1];
    if (j + 1 < nch) tmem_ld_32x32b_x32(taddr0 + static_cast<uint32_t>((j + 1) * 32), v[(j + 1) & 1]);
    uint32_t packed[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float w0 = __shfl_sync(0xffffffffu, pre.sw[j], 2 * i);
      const float w1 = __shfl_sync(0xffffffffu, pre.sw[j], 2 * i + 1);
      float y0 = __fmul_rn(__fmul_rn(__uint_as_float(cur[2 * i]), pre.sx), w0);
      float y1 = __fmul_rn(__fmul_rn(__uint_as_float(cur[2 * i + 1]), pre.sx), w1);
      if (combine) {
        y0 = __fmul_rn(y0, pre.rw);
        y1 = __fmul_rn(y1, pre.rw);
      }
      const __half2 hv = __floats2half2_rn(y0, y1);
      packed[i] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    // The staging tile about to be written must have been read by its last
    // bulk store (with two tiles: the store of chunk j-2).
    uint8_t* buf = stage + (kBufs == 2 ? (j & 1) * kEpiWarps * kStageTileBytes : 0);
    if (lane == 0) {
      if (kBufs == 2) bulk_wait_read_1();
      else bulk_wait_read_all();
    }
    __syncwarp();
    const uint32_t sbase = smem_u32(buf);
#pragma unroll
    for (int c = 0; c < 4; ++c)
      st_shared_v4(sbase + stage_off(lane, c), packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
    if (bulk) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(tmY, buf, t.n0 + cl, qrow0);
        bulk_commit_group();
      }
    } else {
      __syncwarp();
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int rr = it * 8 + (lane >> 2);
        const int c = lane & 3;
        const uint4 val = ld_shared_v4(sbase + stage_off(rr, c));
        const int gcol = t.n0 + cl + c * 8;
        if (combine) {
          const int tok = __shfl_sync(0xffffffffu, pre.ctok, rr);   // -1: past the group or rejected
          if (tok >= 0 && gcol < p.N) red_add_f16x8(p.Y + static_cast<int64_t>(tok) * p.N + gcol, val.x, val.y, val.z, val.w);
        } else if (rr < valid && gcol < p.N) {
          *reinterpret_cast<uint4*>(p.Y + static_cast<int64_t>(qrow0 + rr) * p.N + gcol) = val;
        }
      }
      __syncwarp();
    }
    if (j + 1 < nch) tmem_ld_wait_regs(v[(j + 1) & 1]);
  }
}

}  // namespace fp8q
