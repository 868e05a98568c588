// FP8 GEMM on CTA pairs (tcgen05 cta_group::2) for the dense linear.
//
// Same arithmetic as the single-CTA kernel in gemm_fp8.cuh (E4M3 x E4M3
// products, FP32 accumulation in TMEM, fused y = fp16((acc * s_x) * s_w);
// "Quantized Inference for OneRec-V2" 关键证据 steps 3-4;
// "FP8量化在生成式推荐系统OneRec-V2中的优化实践" §2.3), with the output tile
// of a cluster of two CTAs = 256 rows x BN columns:
//   * each CTA stages its own 128 rows of A and BN/2 rows of B per k-block
//     (32 KB for BN = 256 instead of 48 KB for a 128 x 256 single-CTA tile),
//     so the same shared memory holds a deeper pipeline and every SM pulls
//     a third less operand traffic out of L2;
//   * both CTAs' TMA loads count their bytes on the leader CTA's "full"
//     mbarrier; the leader's single MMA thread issues the M=256 pair MMA,
//     whose commits arrive (multicast) on the same barrier in both CTAs;
//   * each CTA's eight epilogue warps drain their own 128 TMEM lanes
//     (gemm_common.cuh: bulk tensor stores through a swizzled staging tile)
//     and arrive on the leader's "accumulator empty" barrier.
// When the full tiles do not divide evenly over the clusters, the leftover
// tiles are cut along N into 2 or 4 narrower pieces (a runtime MMA N and a
// second B descriptor with a narrower box), so the last round is short
// instead of mostly idle.
// No TMA multicast: every CTA loads only the tiles it stores.
// kQuantA (dense): the kernel also quantizes the fp16 activations
// (quant_in_gemm.cuh): the epilogue warps write the codes and scales, the
// producer waits per 128-row block before loading them.
#pragma once

#include "gemm_fp8.cuh"
#include "quant_in_gemm.cuh"

namespace fp8q {

// SK: K bytes per pipeline stage, kBK (one 128-byte swizzle box per operand)
// or 2 * kBK (two boxes side by side: eight MMAs per barrier round trip
// instead of four, halving the issuing thread's per-MMA bookkeeping).
template <int BN, int STAGES, int SK = kBK>
struct PairLayout {
  static constexpr int kBoxes = SK / kBK;              // 128-byte K boxes per operand per stage
  static constexpr int kABox = kBM * kBK;
  static constexpr int kABytes = kBM * SK;             // own 128 rows of A
  static constexpr int kBRows = BN / 2;                // own half of the B rows
  static constexpr int kBBox = kBRows * kBK;
  static constexpr int kBBytes = kBRows * SK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kNumBars = 2 * STAGES + 5;      // full, empty, tfull[2], tempty[2], drain
  static constexpr int kTmemCols = 512;
  // BN <= 256: two TMEM accumulators (the epilogue of one tile overlaps the
  // MMAs of the next).  BN = 512 ("wide"): one accumulator filling TMEM,
  // computed as two N = 256 halves per k-step; a third less operand traffic
  // per FLOP, but the epilogue no longer overlaps the next tile's MMAs.
  static constexpr bool kWide = BN > 256;
  static constexpr int kNAcc = kWide ? 1 : 2;
  static constexpr int kEpiBufs = 2;                   // two staging tiles per epilogue warp
  static constexpr size_t kSmemBytes =
      1024 + size_t(STAGES) * kStageBytes + epi_smem_bytes(kEpiBufs) + kNumBars * 8 + 32;
  // plus the MoE schedule tables (offsets and tile prefix) when grouped
  static size_t smem_bytes(int E) { return kSmemBytes + 2 * static_cast<size_t>(E + 1) * 4 + 16; }
};

// Tile t of the pair schedule.  Dense: full tiles first, then the tail
// pieces.  Grouped (MoE): tiles ordered (expert, n-block, 256-row block) from
// the device-side tile prefix, so the row blocks sharing an expert's weight
// tile run back to back.
struct PairTile {
  int a_row0;   // first of the pair's 256 token rows
  int row_end;  // rows >= row_end are not stored (end of matrix or expert group)
  int b_row0;   // first weight row of the tile
  int n0;       // first output column
  int sw0;      // s_w index of column n0
  int bn;       // width: BN, or BN / tail_q for a tail piece
  bool tail;
  bool half;    // grouped: M = 128 pair tile (64 rows per CTA) for an expert's last <= 128 rows
};

template <int BN, bool kGrouped>
__device__ __forceinline__ PairTile pair_tile(int t, const GemmParams& p, int num_m, int num_n,
                                              const int* tile_prefix, const int* offs) {
  PairTile r;
  if (kGrouped) {
    int lo = 0, hi = p.E;   // tile_prefix[lo] <= t < tile_prefix[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tile_prefix[mid] <= t) lo = mid; else hi = mid;
    }
    const int e = lo;
    const int cnt = offs[e + 1] - offs[e];
    const int full = cnt / (2 * kBM);
    const int rem = cnt - full * 2 * kBM;
    const int mt = full + (rem > 0 ? 1 : 0);
    const int local = t - tile_prefix[e];
    const int n_blk = local / mt;
    const int m_idx = local - n_blk * mt;
    r.a_row0 = offs[e] + m_idx * 2 * kBM;
    r.row_end = offs[e + 1];
    r.n0 = n_blk * BN;
    r.b_row0 = e * p.N + r.n0;
    r.sw0 = r.b_row0;
    r.bn = BN;
    r.tail = false;
    r.half = p.half_tiles && m_idx == full && rem <= kBM;
    return r;
  }
  int f, piece = 0;
  r.tail = t >= p.main_tiles;
  if (!r.tail) {
    f = t;
  } else {
    const int u = t - p.main_tiles;
    f = p.main_tiles + u / p.tail_q;
    piece = u % p.tail_q;
  }
  const int n_blk = p.n_fastest ? f % num_n : f / num_m;
  const int m_blk = p.n_fastest ? f / num_n : f % num_m;
  r.bn = r.tail ? BN / p.tail_q : BN;
  r.n0 = n_blk * BN + piece * r.bn;
  r.a_row0 = m_blk * 2 * kBM;
  r.row_end = p.rows;
  r.b_row0 = r.n0;
  r.sw0 = r.n0;
  r.half = false;
  return r;
}

template <int BN, int STAGES, bool kGrouped, bool kQuantA = false, int SK = kBK>
__global__ void __launch_bounds__(kGemmThreads, 1)
    fp8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAh,
                         const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmBt,
                         const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
  using L = PairLayout<BN, STAGES, SK>;
  static_assert(SK == kBK || (SK == 2 * kBK && BN <= 256), "stage K: one box, or two for tiles up to 256 wide");
  static_assert(BN % 64 == 0 && BN >= 64 && (BN <= 256 || BN == 512) && (BN / 2) % 8 == 0, "BN");
  static_assert(L::kNAcc * BN <= L::kTmemCols, "accumulators must fit in TMEM");
  static_assert(!(kQuantA && kGrouped), "in-kernel quantization is the dense form");
  constexpr bool kWide = L::kWide;
  // A = activations: E4M3, or E5M2 for the activation-format variant
  const uint32_t kAFmt = idesc_a_fmt(p.x_fmt);
  const uint32_t kIdesc = idesc_e4m3_f32(2 * kBM, kWide ? 256 : BN) | kAFmt;

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
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);
  const int num_m = (p.rows + 2 * kBM - 1) / (2 * kBM);
  const int num_n = (p.N + BN - 1) / BN;
  const int num_kb = (p.K + SK - 1) / SK;   // pipeline stages of SK bytes of K

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);   // one arrival per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    if (kGrouped) prefetch_tmap(&tmAh);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmBt);
    prefetch_tmap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Both CTAs' barriers are initialized before any cross-CTA arrival or copy.
  cluster_arrive();
  cluster_wait();
  const uint32_t tmem_base = *tmem_slot;
  int total;
  if (kGrouped) {
    // The expert offsets may come from the previous kernel: wait for it, then
    // build the tile schedule (and check the offsets) on the device.
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
        acc += (cnt > 0 ? (cnt + 2 * kBM - 1) / (2 * kBM) : 0) * num_n;
      }
      tile_prefix[p.E] = acc;
      *total_s = ok ? acc : 0;
      if (!ok && blockIdx.x == 0) raise_error(0x8u);
    }
    __syncthreads();
    total = *total_s;
  } else {
    total = p.main_tiles + (num_m * num_n - p.main_tiles) * p.tail_q;
  }
  // The next kernel on the stream may begin launching (it waits for this
  // grid before touching anything this grid reads or writes).
  pdl_launch_dependents();
  // In-kernel quantization, first pass: every warp of the grid one row.
  const int qa_first = kQuantA ? qa_first_pass_rows(p, static_cast<int>(gridDim.x), kGemmThreads / 32) : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    // This CTA's share of a tile's weight rows for one k-block.  Normal
    // tiles: rows n0 + rank*bn/2 .. +bn/2.  Wide tiles: for each 256-column
    // half h, rows n0 + 256h + rank*128 .. +128, stored one after the other.
    auto load_b = [&](const PairTile& pt, uint8_t* dst, uint32_t bar, int kx) {
      if (kWide) {
        for (int h = 0; h < pt.bn / 256; ++h)
          tma_load_2d_pair(dst + h * 128 * kBK, &tmB, bar, kx, pt.b_row0 + 256 * h + static_cast<int>(rank) * 128);
      } else {
#pragma unroll
        for (int j = 0; j < L::kBoxes; ++j)
          tma_load_2d_pair(dst + j * L::kBBox, pt.tail ? &tmBt : &tmB, bar, kx + j * kBK,
                           pt.b_row0 + static_cast<int>(rank) * (pt.bn / 2));
      }
    };
    // This CTA's A rows for one stage: kBoxes boxes of 128 bytes of K.
    auto load_a = [&](uint8_t* dst, const CUtensorMap* tm, uint32_t bar, int kx, int row) {
#pragma unroll
      for (int j = 0; j < L::kBoxes; ++j) tma_load_2d_pair(dst + j * L::kABox, tm, bar, kx + j * kBK, row);
    };
    // The weights do not depend on the kernel launched before this one
    // (programmatic dependent launch): request the first ring pass of the
    // first tile's weight tiles before waiting for it; only the activation
    // tiles wait.
    int pre = 0;
    if (lane == 0 && !kGrouped && pair < total) {
      const PairTile pt = pair_tile<BN, kGrouped>(pair, p, num_m, num_n, tile_prefix, offs);
      const uint32_t bytes = 2u * static_cast<uint32_t>(L::kABytes + (pt.bn / 2) * SK);
      pre = num_kb < STAGES ? num_kb : STAGES;
      for (int i = 0; i < pre; ++i) {
        const uint32_t full_leader = mapa_shared(smem_u32(&full[i]), 0);
        if (leader) mbar_arrive_expect_tx(&full[i], bytes);
        load_b(pt, sB + i * L::kBBytes, full_leader, i * SK);
      }
    }
    __syncwarp();
    pdl_wait_prior_grid();
    if (kQuantA)   // while those loads are in flight: this warp's row of the first pass
      quantize_rows_strided(p, static_cast<int>(blockIdx.x) * (kGemmThreads / 32) + warp, 1 << 30, qa_first, lane);
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      RowsReady ready;
      for (int t = pair; t < total && ok; t += npairs) {
        const PairTile pt = pair_tile<BN, kGrouped>(t, p, num_m, num_n, tile_prefix, offs);
        // half tile: 64 rows of A per CTA (box of tmAh) at the start of the stage slot
        const int a_rows = pt.half ? kBM / 2 : kBM;
        const int a_row = pt.a_row0 + static_cast<int>(rank) * a_rows;
        const CUtensorMap* tma_a = pt.half ? &tmAh : &tmA;
        const uint32_t bytes = 2u * static_cast<uint32_t>(a_rows * SK + (pt.bn / 2) * SK);
        if (kQuantA && !ready.wait(p, a_row, true)) {   // this CTA's 128 rows quantized
          ok = false;
          break;
        }
        for (int kb = 0; kb < num_kb; ++kb) {
          if (pre > 0) {
            // stage kb of the first pass: weights already requested
            const uint32_t full_leader = mapa_shared(smem_u32(&full[s]), 0);
            load_a(sA + s * L::kABytes, &tmA, full_leader, kb * SK, a_row);
            --pre;
            if (++s == STAGES) {
              s = 0;
              ph ^= 1u;
            }
            continue;
          }
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t full_leader = mapa_shared(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], bytes);
          load_a(sA + s * L::kABytes, tma_a, full_leader, kb * SK, a_row);
          load_b(pt, sB + s * L::kBBytes, full_leader, kb * SK);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        raise_error(0x1u);
        *abort_flag = 1;
        // Copies already issued complete within microseconds; let them land
        // before this CTA's shared memory can be released.
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 50000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader CTA)
    pdl_wait_prior_grid();
    if (kQuantA)
      quantize_rows_strided(p, static_cast<int>(blockIdx.x) * (kGemmThreads / 32) + warp, 1 << 30, qa_first, lane);
    if (lane == 0 && leader) {
      int s = 0, acc = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool issued = false, ok = true;
      // Addresses and descriptors of stage 0; stage s adds s times the stage
      // size (the descriptor's start-address field counts 16-byte units).
      // Keeping this loop's instruction stream short matters: the issuing
      // thread's scalar work between tensor-core instructions is slow
      // while MMAs are in flight.
      const uint32_t full_a = smem_u32(full), empty_a = smem_u32(empty);
      const uint64_t adesc0 = sw128_kmajor_desc(smem_u32(sA)), bdesc0 = sw128_kmajor_desc(smem_u32(sB));
      for (int t = pair; t < total && ok; t += npairs) {
        if (!mbar_wait(&tempty[acc], acc_ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN);
        uint32_t idesc = (!kWide && t >= p.main_tiles) ? idesc_e4m3_f32(2 * kBM, BN / p.tail_q) | kAFmt : kIdesc;
        // grouped: an M = 128 pair MMA for a half tile (64 rows per CTA)
        if (kGrouped && pair_tile<BN, kGrouped>(t, p, num_m, num_n, tile_prefix, offs).half)
          idesc = idesc_e4m3_f32(kBM, BN) | kAFmt;
        const int halves = kWide ? pair_tile<BN, kGrouped>(t, p, num_m, num_n, tile_prefix, offs).bn / 256 : 1;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_addr(full_a + 8u * s, ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = adesc0 + static_cast<uint64_t>(s * (L::kABytes >> 4));
          const uint64_t b0 = bdesc0 + static_cast<uint64_t>(s * (L::kBBytes >> 4));
#pragma unroll
          for (int k = 0; k < SK / kUmmaK; ++k) {
            // box k / 4 of the stage, 32-byte step k % 4 inside its swizzle row
            const int box = k / (kBK / kUmmaK), kin = k % (kBK / kUmmaK);
            for (int h = 0; h < halves; ++h)   // wide: N = 256 halves at TMEM columns 256h
              mma_f8f6f4_pair(d + static_cast<uint32_t>(256 * h),
                              a0 + static_cast<uint64_t>(box * (L::kABox >> 4) + kin * kUmmaK / 16),
                              b0 + static_cast<uint64_t>(box * (L::kBBox >> 4) + h * 128 * kBK / 16 + kin * kUmmaK / 16),
                              idesc, (kb | k) != 0 ? 1u : 0u);
          }
          issued = true;
          mma_commit_pair_mc_addr(empty_a + 8u * s, 0x3);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair_mc(&tfull[acc], 0x3);
        if (++acc == L::kNAcc) {
          acc = 0;
          acc_ph ^= 1u;
        }
      }
      if (!ok) {
        raise_error(0x2u);
        *abort_flag = 1;
      }
      if (issued) {
        mma_commit_pair_mc(drain, 0x1);
        mbar_wait(drain, 0, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    pdl_wait_prior_grid();   // s_x comes from, and Y may be read by, the neighbouring kernels
    if (kQuantA) {
      // the first pass (one row per warp of the grid), then the rest over the epilogue warps
      quantize_rows_strided(p, static_cast<int>(blockIdx.x) * (kGemmThreads / 32) + warp, 1 << 30, qa_first, lane);
      quantize_rows_strided(p, qa_first + static_cast<int>(blockIdx.x) * kEpiWarps + (warp - kEpiWarp0),
                            static_cast<int>(gridDim.x) * kEpiWarps, p.rows, lane);
    }
    uint8_t* stage = sEpi + (warp - kEpiWarp0) * kStageTileBytes;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int acc = 0;
    uint32_t acc_ph = 0;
    RowsReady ready;
    for (int t = pair; t < total; t += npairs) {
      const PairTile pt = pair_tile<BN, kGrouped>(t, p, num_m, num_n, tile_prefix, offs);
      EpiTile et;
      et.row0 = pt.a_row0 + static_cast<int>(rank) * (pt.half ? kBM / 2 : kBM);
      et.row_end = pt.row_end;
      et.n0 = pt.n0;
      et.sw0 = pt.sw0;
      et.clip = !kGrouped;   // dense: rows past the end are past the tensor
      const EpiWarpView wv = epi_view(et, warp, pt.bn, pt.half);
      EpiScales<BN / 64> sc = epilogue_scales<BN / 64>(et, p, wv, lane);
      if (kQuantA) {
        // the row scales were written in this kernel: read them once the
        // block is complete (it is before its first MMA, so this wait ends)
        if (!ready.wait(p, et.row0, false)) {
          raise_error(0x4u);
          *abort_flag = 1;
          break;
        }
        const int r = wv.qrow0 + lane;
        sc.sx = r < et.row_end ? ld_relaxed_gpu_f32(p.s_x + r) : 0.0f;
      }
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
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
      if (++acc == L::kNAcc) {
        acc = 0;
        acc_ph ^= 1u;
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  __syncthreads();
  if (kQuantA && threadIdx.x == 0) release_sync(p);   // after every read of the flags in this CTA
  // The leader has drained its MMAs (which read both CTAs' shared memory) and
  // all cross-CTA arrivals were issued before this point.
  tc_fence_before();
  cluster_arrive();
  cluster_wait();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}

}  // namespace fp8q
