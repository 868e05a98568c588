// MoE expert grouped FP8 GEMM with 128 x 128 block-scaled expert weights.
//
// Variant of the grouped linear described by "FP8量化在生成式推荐系统OneRec-V2中的
// 优化实践" §2.1 (the MoE expert grouped GEMM is quantized "block-wise
// 128x128") and §2.2 (block-aligned MoE quantization; activations dynamic,
// one scale per token):
//     Y[m,n] = fp16( s_x[m] * sum_j s_w[e, n / 128, j] * P_j[m,n] ),
//     P_j[m,n] = sum over the 128 inputs k of K block j of Xq[m,k] * Wq_e[n,k]
// (E4M3 x E4M3 products, FP32 accumulation).
//
// The weight scale changes every 128 inputs, so one TMEM accumulator cannot
// carry the whole K loop.  Instead each K block's MMAs (M = 128 token rows,
// N = 256 weight rows = two scale blocks, four K = 32 instructions) write a
// fresh FP32 partial into one of two TMEM buffers, and eight promotion warps
// add partial * scale into FP32 accumulators held in registers while the
// tensor core fills the other buffer.  Each promotion warp owns 32 rows (its
// TMEM lane quadrant) x 128 columns -- exactly one weight scale block, so one
// scale per K block -- and reads its partial 16 columns at a time with the
// next load in flight while it multiplies and adds the current one.  After
// the last K block the accumulators are multiplied by s_x and stored as fp16
// through two swizzled staging tiles per warp and bulk tensor stores
// (coalesced masked stores where an expert group ends inside a warp's rows).
//
//   warp 0       TMA producer (A = token rows, B = expert weight rows)
//   warp 1       MMA issuer: K block j -> TMEM partial buffer j % 2
//   warps 2..9   promotion and epilogue
// Tile schedule: the same device-built (expert, n-block, m-block) order as
// the per-channel grouped kernel (gemm_fp8.cuh).  No TMA multicast.
#pragma once

#include "gemm_fp8.cuh"
#include "quant_rows.cuh"

namespace fp8q {

constexpr int kBsBN = 256;                          // tile width (two 128-column scale blocks)
constexpr int kBsBlk = 128;                         // scale block edge
constexpr int kBsWarps = 8;                         // promotion warps: 2 per TMEM lane quadrant
constexpr int kBsThreads = (kEpiWarp0 + kBsWarps) * 32;
constexpr int kBsMaxExperts = 128;

template <int STAGES>
struct BsLayout {
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = kBsBN * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kEpiBytes = 2 * kBsWarps * kStageTileBytes;   // two staging tiles per warp
  static constexpr int kNumBars = 2 * STAGES + 5;   // full, empty, pfull[2], pempty[2], drain
  static constexpr int kTmemCols = 2 * kBsBN;       // two partial buffers
  static constexpr int kFixedBytes = STAGES * kStageBytes + kEpiBytes + kNumBars * 8 + 32;
  static size_t smem_bytes(int E) { return 1024 + kFixedBytes + 2 * static_cast<size_t>(E + 1) * 4 + 16; }
};

// p.s_w holds the block scales [E, NB, KB] (NB = ceil(N/128), KB = ceil(K/128)).
template <int STAGES>
__global__ void __launch_bounds__(kBsThreads, 1)
    fp8_gemm_blockscaled_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
  using L = BsLayout<STAGES>;
  constexpr int BN = kBsBN;
  const uint32_t idesc = idesc_e4m3_f32(kBM, BN) | idesc_a_fmt(p.x_fmt);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::kABytes;
  uint8_t* sEpi = sB + STAGES * L::kBBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + L::kEpiBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* pfull = bars + 2 * STAGES;
  uint64_t* pempty = bars + 2 * STAGES + 2;
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* total_s = reinterpret_cast<int*>(tmem_slot + 2);
  int* tile_prefix = reinterpret_cast<int*>(tmem_slot + 8);
  int* offs = tile_prefix + (p.E + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_n = (p.N + BN - 1) / BN;
  const int num_m = (p.rows + kBM - 1) / kBM;
  const int num_kb = (p.K + kBK - 1) / kBK;
  const int NB = (p.N + kBsBlk - 1) / kBsBlk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&pfull[b], 1);
      mbar_init(&pempty[b], kBsWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  pdl_wait_prior_grid();
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) offs[i] = __ldg(p.offsets + i);
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = offs[0] == 0 && offs[p.E] == p.rows;
    int acc = 0;
    for (int e = 0; e < p.E; ++e) {
      const int cnt = offs[e + 1] - offs[e];
      ok = ok && cnt >= 0;
      tile_prefix[e] = acc;
      acc += (cnt > 0 ? (cnt + kBM - 1) / kBM : 0) * num_n;
    }
    tile_prefix[p.E] = acc;
    *total_s = ok ? acc : 0;
    if (!ok && blockIdx.x == 0) raise_error(0x8u);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = *total_s;
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, armed = 0, armed_ph = 0;
      for (int t = blockIdx.x; t < total; t += gridDim.x) {
        const TileCoord c = decode_tile<true, BN>(t, p, num_m, num_n, tile_prefix, offs);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], L::kStageBytes);
          tma_load_2d(sA + s * L::kABytes, &tmA, &full[s], kb * kBK, c.a_row0);
          tma_load_2d(sB + s * L::kBBytes, &tmB, &full[s], kb * kBK, c.b_row0);
          armed |= 1u << s;
          armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) {
          raise_error(0x1u);
          *abort_flag = 1;
          break;
        }
      }
      for (int i = 0; i < STAGES; ++i)
        if (armed & (1u << i)) mbar_wait(&full[i], (armed_ph >> i) & 1u, nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0, pb = 0;
      uint32_t ph = 0, pb_ph = 0;
      bool issued = false, ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        for (int kb = 0; kb < num_kb; ++kb) {
          // the promotion warps have read this partial buffer's previous K block
          if (!mbar_wait(&pempty[pb], pb_ph ^ 1u, abort_flag) || !mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(pb * BN);
          const uint64_t a0 = sw128_kmajor_desc(smem_u32(sA + s * L::kABytes));
          const uint64_t b0 = sw128_kmajor_desc(smem_u32(sB + s * L::kBBytes));
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k)   // a fresh partial per K block
            mma_f8f6f4(d, a0 + static_cast<uint64_t>(k * kUmmaK / 16), b0 + static_cast<uint64_t>(k * kUmmaK / 16),
                       idesc, k != 0 ? 1u : 0u);
          issued = true;
          mma_commit(&empty[s]);
          mma_commit(&pfull[pb]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
          pb ^= 1;
          if (pb == 0) pb_ph ^= 1u;
        }
      }
      if (!ok) {
        raise_error(0x2u);
        *abort_flag = 1;
      }
      if (issued) {
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ promotion + epilogue
    const int pw = warp - kEpiWarp0;            // 0..7
    const int q = warp & 3;                     // TMEM lane quadrant this warp may read
    const int c128 = pw >> 2;                   // which 128 of the tile's 256 columns (one scale block)
    uint8_t* stage = sEpi + pw * kStageTileBytes;   // buffer b at + b * kBsWarps * kStageTileBytes
    int pb = 0;
    uint32_t pb_ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const TileCoord c = decode_tile<true, BN>(t, p, num_m, num_n, tile_prefix, offs);
      const int e = c.b_row0 / p.N;              // expert of the tile
      const int nbi = c.n0 / kBsBlk + c128;
      const float* srow = p.s_w + (static_cast<int64_t>(e) * NB + (nbi < NB ? nbi : 0)) * num_kb;
      const bool cols_live = nbi < NB;
      const int qrow0 = c.a_row0 + q * 32;
      const int valid = c.row_end - qrow0;      // rows of this warp stored (<= 0: none)
      const float sx = lane < valid ? __ldg(p.s_x + qrow0 + lane) : 0.0f;
      float sc = (cols_live && lane < num_kb) ? __ldg(srow + lane) : 0.0f;   // scales of K blocks 0..31
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (kb > 0 && (kb & 31) == 0) sc = (cols_live && kb + lane < num_kb) ? __ldg(srow + kb + lane) : 0.0f;
        const float s_blk = __shfl_sync(0xffffffffu, sc, kb & 31);
        if (!mbar_wait(&pfull[pb], pb_ph, abort_flag)) {
          raise_error(0x4u);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(pb * BN + c128 * 128);
        // 16 columns at a time, the load of chunk ch+1 in flight during chunk ch
        uint32_t v[2][16];
        tmem_ld_32x32b_x16(taddr, v[0]);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          tmem_ld_wait_regs16(v[ch & 1]);
          if (ch + 1 < 8) tmem_ld_32x32b_x16(taddr + static_cast<uint32_t>((ch + 1) * 16), v[(ch + 1) & 1]);
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[ch * 16 + i] = fmaf(__uint_as_float(v[ch & 1][i]), s_blk, acc[ch * 16 + i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[pb]);
        pb ^= 1;
        if (pb == 0) pb_ph ^= 1u;
      }
      if (!ok || valid <= 0) continue;
      // y = fp16(acc * s_x): four 32 x 32 chunks through two staging tiles
      const bool bulk = valid >= 32;
      // no store of an earlier tile may still read either staging tile
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        const int cl = c128 * 128 + ch * 32;    // first column of the chunk within the tile
        const uint32_t sbase = smem_u32(stage + (ch & 1) * kBsWarps * kStageTileBytes);
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const __half2 hv = __floats2half2_rn(__fmul_rn(acc[ch * 32 + 2 * i], sx), __fmul_rn(acc[ch * 32 + 2 * i + 1], sx));
          packed[i] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        if (lane == 0 && ch >= 2) bulk_wait_read_1();   // the store of chunk ch-2 has read this tile
        __syncwarp();
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)
          st_shared_v4(sbase + stage_off(lane, k4), packed[4 * k4], packed[4 * k4 + 1], packed[4 * k4 + 2],
                       packed[4 * k4 + 3]);
        if (bulk) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, stage + (ch & 1) * kBsWarps * kStageTileBytes, c.n0 + cl, qrow0);
            bulk_commit_group();
          }
        } else {
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int rr = it * 8 + (lane >> 2);
            const int k4 = lane & 3;
            const uint4 val = ld_shared_v4(sbase + stage_off(rr, k4));
            const int gcol = c.n0 + cl + k4 * 8;
            if (rr < valid && gcol < p.N)
              *reinterpret_cast<uint4*>(p.Y + static_cast<int64_t>(qrow0 + rr) * p.N + gcol) = val;
          }
          __syncwarp();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ------------------------------------------------------------ block-wise weight quantization
// One CTA per 128 x 128 block of one expert's [N, K] weights: the block is
// held in registers (256 threads x 8 vectors of 8 fp16), its maximum reduced
// with shuffles and shared memory, then r and s as for per-row scales and
// the codes written back.  Grid (E * NB, KB); S[(e * NB + i) * KB + j].
__global__ void __launch_bounds__(256) quant_blocks_kernel(const __half* __restrict__ W, int N, int K, int NB,
                                                          int KB, uint8_t* __restrict__ Q, float* __restrict__ S) {
  __shared__ float red[8];
  // Weights: the next kernel starts only once this one has finished (the
  // GEMMs request weight tiles before their programmatic-dependent wait).
  pdl_wait_prior_grid();
  const int e = blockIdx.x / NB;
  const int bi = blockIdx.x - e * NB;
  const int bj = blockIdx.y;
  const int r_end = min(kBsBlk, N - bi * kBsBlk);     // rows of this block
  const int c_end = min(kBsBlk, K - bj * kBsBlk);     // columns (a multiple of 16)
  const int64_t base = (static_cast<int64_t>(e) * N + static_cast<int64_t>(bi) * kBsBlk) * K + bj * kBsBlk;
  uint4 v[8];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = threadIdx.x + i * 256;              // 0 .. 2047: row = idx / 16, vector = idx % 16
    const int r = idx >> 4, cv = (idx & 15) * 8;
    if (r < r_end && cv < c_end) {
      v[i] = __ldg(reinterpret_cast<const uint4*>(W + base + static_cast<int64_t>(r) * K + cv));
      m = absmax8(v[i], m);
    } else {
      v[i] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w]);
  const RowScale rs = row_scale_from_amax<kFmtE4M3>(m);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = threadIdx.x + i * 256;
    const int r = idx >> 4, cv = (idx & 15) * 8;
    if (r < r_end && cv < c_end)
      *reinterpret_cast<uint2*>(Q + base + static_cast<int64_t>(r) * K + cv) = encode8<kFmtE4M3>(v[i], rs.r);
  }
  if (threadIdx.x == 0) S[(static_cast<int64_t>(e) * NB + bi) * KB + bj] = rs.s;
}

}  // namespace fp8q
