// FP8 (E4M3 x E4M3) GEMM with FP32 accumulation in tensor memory and a fused
// per-token x per-channel dequantization + FP16 cast epilogue, for sm_100a:
// the single-CTA kernel (128-row tiles), used for the MoE grouped linear and
// for dense problems of at most 128 rows.
//
// Method: "Quantized Inference for OneRec-V2" (关键证据 steps 3-4: FP8 tensor
// cores, FP32 accumulation, FP16 output) and
// "FP8量化在生成式推荐系统OneRec-V2中的优化实践" §2.3 (fused
// Quantize + GEMM + Dequantize; FP8 multiply + FP32 accumulate + FP16 out)
// and §3.2 (MoE expert GEMMs, pipelined across experts).
//
// Each CTA (one per SM, persistent) walks output tiles of 128 x BN:
//   warp 0      TMA producer: 128-byte-swizzled 2-D tile loads of A (token
//               rows, K-major) and B (weight rows, K-major) into a STAGES-deep
//               shared-memory ring, completion tracked by mbarriers;
//   warp 1      MMA issuer: one thread issues tcgen05.mma kind::f8f6f4
//               (M=128, N=BN, K=32 per instruction) into one of two TMEM
//               accumulators; tcgen05.commit frees smem stages and hands a
//               finished accumulator to the epilogue;
//   warps 2..9  epilogue (gemm_common.cuh): TMEM -> scale -> fp16 -> bulk
//               tensor stores, masked at expert-group boundaries.
// Two TMEM accumulators let the epilogue of tile i overlap the MMAs of tile
// i+1.  The MoE tile schedule is built on the device from the expert offsets
// (no host synchronization): tiles are ordered (expert, n-block, m-block), so
// the m-blocks that share one expert weight tile run back to back and reuse
// it from L2.  No TMA multicast is used anywhere.
//
// Gather form (kGather, MoE): product row r reads activation row
// row_token[r] of the token matrix (tokens quantized once; no permuted
// copy).  The whole producer warp then fills a stage's A tile itself: each
// lane copies four rows with 16-byte cp.async (zero-filled past K or past the
// expert group) straight into the 128-byte-swizzled layout the MMA reads,
// and once its copies of a stage have landed (one stage later, keeping
// copies in flight) fences them for the async proxy and arrives on the
// stage's barrier; the weight tile still comes by TMA.
#pragma once

#include "gemm_common.cuh"

namespace fp8q {

template <int BN, int STAGES>
struct GemmLayout {
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = BN * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kNumBars = 2 * STAGES + 5;   // full, empty, tfull[2], tempty[2], drain
  static constexpr int kTmemCols = 2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
  static constexpr int kEpiBufs = 1;   // one staging tile per epilogue warp (shared memory goes to the ring)
  static constexpr int kFixedBytes = STAGES * kStageBytes + epi_smem_bytes(kEpiBufs) + kNumBars * 8 + 32;
  static size_t smem_bytes(int E) { return 1024 + kFixedBytes + 2 * static_cast<size_t>(E + 1) * 4 + 16; }
};

struct TileCoord {
  int a_row0;    // first A (token) row of the tile
  int row_end;   // rows >= row_end are not stored (end of matrix or of the expert group)
  int b_row0;    // first B (weight) row
  int n0;        // first output column
  int sw0;       // index of s_w for column n0
};

template <bool kGrouped, int BN>
__device__ __forceinline__ TileCoord decode_tile(int t, const GemmParams& p, int num_m, int num_n,
                                                 const int* tile_prefix, const int* offs) {
  TileCoord c;
  if (!kGrouped) {
    int m_blk, n_blk;
    if (p.n_fastest) {
      n_blk = t % num_n;
      m_blk = t / num_n;
    } else {
      m_blk = t % num_m;
      n_blk = t / num_m;
    }
    c.a_row0 = m_blk * kBM;
    c.row_end = p.rows;
    c.n0 = n_blk * BN;
    c.b_row0 = c.n0;
    c.sw0 = c.n0;
  } else {
    // expert e with tile_prefix[e] <= t < tile_prefix[e+1]
    int lo = 0, hi = p.E;   // invariant: tile_prefix[lo] <= t < tile_prefix[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tile_prefix[mid] <= t) lo = mid; else hi = mid;
    }
    const int e = lo;
    const int cnt = offs[e + 1] - offs[e];
    const int mt = (cnt + kBM - 1) / kBM;
    const int local = t - tile_prefix[e];
    const int n_blk = local / mt;
    const int m_loc = local - n_blk * mt;
    c.a_row0 = offs[e] + m_loc * kBM;
    c.row_end = offs[e + 1];
    c.n0 = n_blk * BN;
    c.b_row0 = e * p.N + c.n0;
    c.sw0 = e * p.N + c.n0;
  }
  return c;
}

template <int BN, int STAGES, bool kGrouped, bool kGather = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
  using L = GemmLayout<BN, STAGES>;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  static_assert(!kGather || kGrouped, "gathered rows are a grouped (MoE) form");
  constexpr int kGatherLag = 1;   // stages of row copies in flight before a stage is signalled
  static_assert(!kGather || kGatherLag < STAGES, "lag");
  // A = activations: E4M3, or E5M2 for the activation-format variant
  const uint32_t kIdesc = idesc_e4m3_f32(kBM, BN) | idesc_a_fmt(p.x_fmt);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::kABytes;
  uint8_t* sEpi = sB + STAGES * L::kBBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + epi_smem_bytes(L::kEpiBufs));
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = bars + 2 * STAGES + 2;
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], kGather ? 33 : 1);   // gather: + one arrival per producer lane
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
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
  // Inputs (and the expert offsets) may come from the kernel launched just
  // before this one (programmatic dependent launch): wait for it here, after
  // the set-up above has overlapped its tail.
  pdl_wait_prior_grid();
  if (kGrouped) {
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
  } else if (threadIdx.x == 0) {
    *total_s = num_m * num_n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = *total_s;
  // The next kernel on the stream may begin launching (it waits for this
  // grid before touching anything this grid reads or writes).
  pdl_launch_dependents();

  if (kGather && warp == 0) {
    // ------------------------------------------------------------ producer (row gather, whole warp)
    int s = 0, sig = 0, pending = 0;
    uint32_t ph = 0, armed = 0, armed_ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const TileCoord c = decode_tile<kGrouped, BN>(t, p, num_m, num_n, tile_prefix, offs);
      int tok[4];   // tokens of this lane's rows lane, lane+32, lane+64, lane+96 (-1: zero row)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = c.a_row0 + lane + 32 * i;
        tok[i] = row < c.row_end ? __ldg(p.row_token + row) : -1;
        if (tok[i] >= p.tokens || (row < c.row_end && tok[i] < 0)) {
          raise_error(0x8u);
          tok[i] = -1;
        }
      }
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], L::kBBytes);
          tma_load_2d(sB + s * L::kBBytes, &tmB, &full[s], kb * kBK, c.b_row0);
        }
        armed |= 1u << s;
        armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
        const uint32_t dst0 = smem_u32(sA + s * L::kABytes);
        // one instruction copies 4 whole rows: lane l takes 16-byte chunk l % 8
        // of row 4i + l / 8 (coalesced 128-byte lines); the row's token is
        // held by lane (row % 32) in tok[row / 32]
        const int ch = lane & 7;
        const int k = kb * kBK + ch * 16;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int r = 4 * i + (lane >> 3);
          const int tk = __shfl_sync(0xffffffffu, tok[i >> 3], r & 31);
          const bool v = tk >= 0 && k < p.K;
          const uint8_t* src = p.xq + (v ? static_cast<int64_t>(tk) * p.K + k : 0);
          cp_async_16_zfill(dst0 + static_cast<uint32_t>(r * kBK + ((ch ^ (r & 7)) << 4)), src, v ? 16u : 0u);
        }
        cp_async_commit();
        if (++pending > kGatherLag) {
          // the copies of stage `sig` have landed: hand them to the async proxy and signal
          cp_async_wait_group<kGatherLag>();
          fence_proxy_async_smem();
          mbar_arrive(&full[sig]);
          if (++sig == STAGES) sig = 0;
          --pending;
        }
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    cp_async_wait_group<0>();
    fence_proxy_async_smem();
    for (; pending > 0; --pending) {
      mbar_arrive(&full[sig]);
      if (++sig == STAGES) sig = 0;
    }
    if (!ok) {
      raise_error(0x1u);
      *abort_flag = 1;
    }
    // No weight copy may still be in flight when the CTA exits.
    if (lane == 0)
      for (int i = 0; i < STAGES; ++i)
        if (armed & (1u << i)) mbar_wait(&full[i], (armed_ph >> i) & 1u, nullptr);
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, armed = 0, armed_ph = 0;
      for (int t = blockIdx.x; t < total; t += gridDim.x) {
        const TileCoord c = decode_tile<kGrouped, BN>(t, p, num_m, num_n, tile_prefix, offs);
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
      // No copy may still be in flight when the CTA exits.
      for (int i = 0; i < STAGES; ++i)
        if (armed & (1u << i)) mbar_wait(&full[i], (armed_ph >> i) & 1u, nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0, acc = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool issued = false;
      for (int t = blockIdx.x; t < total; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_ph ^ 1u, abort_flag)) {
          raise_error(0x2u);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = sw128_kmajor_desc(smem_u32(sA + s * L::kABytes));
          const uint64_t b0 = sw128_kmajor_desc(smem_u32(sB + s * L::kBBytes));
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k) {
            // advance the start address by k * 32 bytes inside the swizzle row
            mma_f8f6f4(d, a0 + static_cast<uint64_t>(k * kUmmaK / 16), b0 + static_cast<uint64_t>(k * kUmmaK / 16),
                       kIdesc, (kb | k) != 0 ? 1u : 0u);
          }
          issued = true;
          mma_commit(&empty[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) {
          raise_error(0x2u);
          *abort_flag = 1;
          break;
        }
        mma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_ph ^= 1u;
      }
      if (issued) {
        // All issued MMAs must be finished before TMEM is released.
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    uint8_t* stage = sEpi + (warp - kEpiWarp0) * kStageTileBytes;
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const TileCoord c = decode_tile<kGrouped, BN>(t, p, num_m, num_n, tile_prefix, offs);
      EpiTile et;
      et.row0 = c.a_row0;
      et.row_end = c.row_end;
      et.n0 = c.n0;
      et.sw0 = c.sw0;
      et.clip = !kGrouped;   // dense: rows past the end are past the tensor
      const EpiWarpView wv = epi_view(et, warp, BN, false);
      const EpiScales<BN / 64> sc = epilogue_scales<BN / 64>(et, p, wv, lane);
      if (!mbar_wait(&tfull[acc], acc_ph, abort_flag)) {
        raise_error(0x4u);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      epilogue_slab<BN / 64, L::kEpiBufs>(et, p, &tmY, tmem_base + static_cast<uint32_t>(acc * BN), wv, warp, lane,
                                          stage, sc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_ph ^= 1u;
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

}  // namespace fp8q
