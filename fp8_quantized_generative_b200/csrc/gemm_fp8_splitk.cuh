// FP8 GEMM for few token rows (M <= 128): swap-AB with split-K reduced in a
// thread-block cluster through distributed shared memory.
//
// Same arithmetic as the other GEMM kernels ("Quantized Inference for
// OneRec-V2" 关键证据 steps 3-4; "FP8量化在生成式推荐系统OneRec-V2中的优化实践"
// §2.3): E4M3 x E4M3 products, FP32 accumulation, y = fp16((acc*s_x)*s_w).
//
// With few rows the linear is bound by streaming the weights once from HBM,
// so the work is spread over (N / 128) x S CTAs:
//   * the weight tile (128 output channels) is the MMA's M operand and the
//     token rows, zero-padded by TMA to MPAD in {16, 32, 64, 128}, are its N
//     operand, so a single token still uses a full-height MMA;
//   * the S CTAs of a cluster (cluster dims (S,1,1)) each take 1/S of the K
//     blocks and accumulate a 128 x MPAD fp32 partial in TMEM;
//   * S is 1, 2, 4 or 8; CTA r owns weight rows [r*128/S, (r+1)*128/S) of
//     the tile.  Each CTA stages its partial in its (now idle) load ring,
//     slice by owner, and ships every other owner's slice with one bulk
//     shared-memory-to-shared-memory copy (cp.async.bulk.shared::cluster)
//     that completes on the owner's mbarrier; the owner then sums the S
//     slices locally in fixed rank order 0..S-1 (reproducible), applies the
//     scales (staged in shared memory beforehand) and writes fp16 -- no
//     global scratch memory;
//   * fused variant (kFused, at most 64 token rows): the kernel takes the
//     fp16 activations; each CTA reads only its K slice of them, the row
//     maxima of the slices are exchanged within the cluster (DSMEM bulk
//     copies), and each CTA derives the per-row scales (the same fp32 steps
//     as quant_rows.cuh) and writes the E4M3 codes of its K slice straight
//     into the 128-byte-swizzled K-major shared-memory layout the MMA reads
//     -- quantize + GEMM + dequantize in one launch
//     ("FP8量化在生成式推荐系统OneRec-V2中的优化实践" §2.3);
//   * the weight tiles do not depend on the kernel launched before this one,
//     so the first STAGES of them are requested before the programmatic-
//     dependent-launch wait: their DRAM latency overlaps that kernel's tail.
#pragma once

#include "gemm_common.cuh"
#include "quant_rows.cuh"

namespace fp8q {

constexpr int kSkThreads = 192;   // producer, MMA, 4 epilogue warps

// kFused: only the weight tiles travel through the ring (the activation
// codes are made in shared memory), so a stage is a weight tile alone and the
// CTA stays small enough for two to share an SM (the next kernel's CTAs can
// then start and stream their weights while this one finishes).
// SK: K bytes per stage, one 128-byte swizzle box (kBK) per operand, or two
// or four side by side (2 * kBK / 4 * kBK: eight / sixteen MMAs per barrier
// wait; each mbarrier test in the issuing thread costs ~100 ns while MMAs
// are in flight).
template <int MPAD, int STAGES, bool kFused = false, int SK = kBK>
struct SplitKLayout {
  static constexpr int kBoxes = SK / kBK;
  static constexpr int kWBox = kBM * kBK;
  static constexpr int kXBox = MPAD * kBK;
  static constexpr int kWBytes = kBM * SK;             // 128 weight rows x SK K bytes
  static constexpr int kXBytes = MPAD * SK;            // MPAD token rows
  static constexpr int kStageBytes = kFused ? kWBytes : kWBytes + kXBytes;
  static constexpr int kRingBytes = STAGES * kStageBytes;
  // Partial rows of MPAD + 4 fp32 words (16-byte aligned rows; the +4 keeps
  // 8 consecutive rows of a 16-byte access on distinct bank groups).
  static constexpr int kPitch = MPAD + 4;
  static constexpr int kPartBytes = kBM * kPitch * 4;  // send buffer (in the ring) and receive buffer
  static_assert(kRingBytes >= kPartBytes, "the send buffer reuses the load ring");
  static constexpr int kScaleFloats = 128 + MPAD;      // owner's s_w slice + the token scales
  static constexpr int kNumBars = 2 * STAGES + 5;      // full, empty, tfull, drain, recv, xready, pmax
  static constexpr int kTmemCols = MPAD < 32 ? 32 : MPAD;
  static constexpr int kBaseBytes = kRingBytes + kPartBytes + kScaleFloats * 4 + kNumBars * 8 + 32;
  static constexpr size_t kSmemBytes = 1024 + size_t(kBaseBytes);
  // Fused variant: 1024-aligned region after the base holding the E4M3 codes
  // of the CTA's K blocks (MPAD x 128 bytes each), then the partial row
  // maxima of every CTA of the cluster (up to 8 x MPAD) and the row scales.
  static constexpr int kFusedOffset = (kBaseBytes + 1023) & ~1023;
  static size_t fused_smem_bytes(int nkb) {
    return 1024 + size_t(kFusedOffset) + size_t(nkb) * kXBytes + (8 + 1) * MPAD * 4;
  }
  // Most K blocks per CTA the fused form takes (its codes stay in shared memory).
  static constexpr int kFusedMaxKBlocks = MPAD <= 32 ? 32 : 16;
};

// The owner's share of the split-K reduction: the S partial slices of its
// kBM / S weight rows (its own slice in the send buffer, the peers' in the
// receive buffer) summed in rank order 0..S-1, scaled and stored as fp16.
// Each of the 128 epilogue threads takes blocks of 4 token rows x 8 weight
// rows: eight 16-byte shared loads per slice, one 16-byte global store per
// token row (the 8 outputs are consecutive columns of Y).
template <int S, typename L>
__device__ __forceinline__ void splitk_reduce_store(const GemmParams& p, const float* send, const float* recv,
                                                    const float* sc_w, const float* sc_x, int n0, int rank, int et) {
  constexpr int SL = kBM / S;
  constexpr int NB = SL / 8;                       // 8-row blocks per owner
  const int m4n = (p.rows + 3) >> 2;
  const int items = m4n * NB;
  for (int idx = et; idx < items; idx += 128) {
    // Token-row blocks vary fastest: the 8 threads of a quarter warp read
    // one partial row at 8 different 16-byte bank groups (weight rows 8
    // apart would all map to the same group: 8 x kPitch is a multiple of 32
    // words).
    const int m = (idx % m4n) * 4;
    const int nl0 = (idx / m4n) * 8;
    const int n = n0 + rank * SL + nl0;
    if (n >= p.N) continue;                        // N % 8 == 0: a block is all in or all out
    float acc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
#pragma unroll
    for (int s2 = 0; s2 < S; ++s2) {
      const float* base =
          (s2 == rank ? send + (rank * SL + nl0) * L::kPitch : recv + (s2 * SL + nl0) * L::kPitch) + m;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 v = *reinterpret_cast<const float4*>(base + j * L::kPitch);
        acc[j][0] = __fadd_rn(acc[j][0], v.x);
        acc[j][1] = __fadd_rn(acc[j][1], v.y);
        acc[j][2] = __fadd_rn(acc[j][2], v.z);
        acc[j][3] = __fadd_rn(acc[j][3], v.w);
      }
    }
    float sw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) sw[j] = sc_w[nl0 + j];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (m + i >= p.rows) break;
      const float sx = sc_x[m + i];
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const __half2 h = __floats2half2_rn(__fmul_rn(__fmul_rn(acc[j][i], sx), sw[j]),
                                            __fmul_rn(__fmul_rn(acc[j + 1][i], sx), sw[j + 1]));
        w[j / 2] = *reinterpret_cast<const uint32_t*>(&h);
      }
      *reinterpret_cast<uint4*>(p.Y + static_cast<int64_t>(m + i) * p.N + n) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

template <int MPAD, int STAGES, bool kFused, int SK = kBK>
__global__ void __launch_bounds__(kSkThreads, 1)
    fp8_gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                           const GemmParams p) {
  using L = SplitKLayout<MPAD, STAGES, kFused, SK>;
  static_assert(SK == kBK || ((SK == 2 * kBK || SK == 4 * kBK) && !kFused),
                "stage K: one box, or two or four for the unfused form");
  static_assert(MPAD % 16 == 0 && MPAD >= 16 && MPAD <= 128, "MPAD");
  // swap-AB: B = activations (E4M3, or E5M2 for the variant; the fused path is E4M3)
  const uint32_t kIdesc = idesc_e4m3_f32(kBM, MPAD) | idesc_b_fmt(kFused ? kFmtE4M3 : p.x_fmt);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sW = smem;
  uint8_t* sX = smem + STAGES * L::kWBytes;
  float* send = reinterpret_cast<float*>(smem);                       // after the mainloop
  float* recv = reinterpret_cast<float*>(smem + L::kRingBytes);
  float* sc_w = reinterpret_cast<float*>(smem + L::kRingBytes + L::kPartBytes);   // 128
  float* sc_x = sc_w + 128;                                                        // MPAD
  uint64_t* bars = reinterpret_cast<uint64_t*>(sc_x + MPAD);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* drain = bars + 2 * STAGES + 1;
  uint64_t* recv_bar = bars + 2 * STAGES + 2;
  uint64_t* xready = bars + 2 * STAGES + 3;   // fused: the CTA's activation codes are in place
  uint64_t* pmax_bar = bars + 2 * STAGES + 4; // fused: the peers' partial row maxima have arrived
  uint8_t* fz_codes = smem + L::kFusedOffset;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = static_cast<int>(cluster_nctarank());
  const int rank = static_cast<int>(cluster_ctarank());
  const int n_tile = static_cast<int>(blockIdx.x) / S;
  const int n0 = n_tile * kBM;
  const int num_kb = (p.K + SK - 1) / SK;   // stages of SK bytes of K
  const int kb0 = static_cast<int>((int64_t(rank) * num_kb) / S);
  const int kb1 = static_cast<int>((int64_t(rank + 1) * num_kb) / S);
  const int nkb = kb1 - kb0;
  const int SL = kBM / S;                          // weight rows owned by each CTA
  const int mcols = (p.rows + 3) & ~3;             // token rows carried, rounded to 4
  const uint32_t slice_bytes = static_cast<uint32_t>(SL * L::kPitch * 4);
  // The partial-maxima table sits at the same offset in every CTA of the
  // cluster (peers copy into it by that offset): after the largest code
  // region any rank has, not after this CTA's own.
  const int nkb_max = (num_kb + S - 1) / S;
  float* fz_pmax = reinterpret_cast<float*>(fz_codes + nkb_max * L::kXBytes);   // [S][MPAD]
  float* fz_r = fz_pmax + 8 * MPAD;
  // Fused: only the weight tiles travel through the ring.
  constexpr uint32_t kLoadBytes = L::kStageBytes;

  // Thread 0 is also the producer: it initializes the barriers and at once
  // requests the weight tiles of the first ring pass.  The weights do not
  // depend on the kernel launched before this one (programmatic dependent
  // launch), so their DRAM latency overlaps that kernel and this set-up.
  const int pre = nkb < STAGES ? nkb : STAGES;
  // One stage's weight / activation boxes (kBoxes of 128 bytes of K each).
  auto load_w = [&](int s, int kb) {
#pragma unroll
    for (int j = 0; j < L::kBoxes; ++j)
      tma_load_2d(sW + s * L::kWBytes + j * L::kWBox, &tmW, &full[s], kb * SK + j * kBK, n0);
  };
  auto load_x = [&](int s, int kb) {
#pragma unroll
    for (int j = 0; j < L::kBoxes; ++j)
      tma_load_2d(sX + s * L::kXBytes + j * L::kXBox, &tmX, &full[s], kb * SK + j * kBK, 0);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    mbar_init(recv_bar, 1);
    mbar_init(xready, 1);
    mbar_init(pmax_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    // The S-1 peers' slices arrive as bulk copies counted on recv_bar (and,
    // fused, their partial row maxima on pmax_bar).
    mbar_arrive_expect_tx(recv_bar, static_cast<uint32_t>(S - 1) * slice_bytes);
    if (kFused) mbar_arrive_expect_tx(pmax_bar, static_cast<uint32_t>(S - 1) * MPAD * 4);
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(&full[i], kLoadBytes);
      load_w(i, kb0 + i);
    }
    // The rest of this CTA's weight slice goes to L2 now, so the whole
    // stream is in flight from the start.
    if (p.l2_prefetch)
      for (int kb = kb0 + pre; kb < kb1; ++kb)
        for (int j = 0; j < L::kBoxes; ++j) tma_prefetch_l2_2d(&tmW, kb * SK + j * kBK, n0);
    prefetch_tmap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The next kernel on the stream may begin launching (it waits for this
  // grid before touching anything this grid reads or writes).
  pdl_launch_dependents();
  // Every CTA of the cluster must be running before any pushes into its
  // shared memory: arrive now, wait just before the first remote access.
  cluster_arrive_relaxed();

  if (warp == 0) {
    if (lane == 0) {
      // The first ring pass of weight tiles is already in flight; the token
      // rows come from the previous kernel.
      if (!kFused) {
        pdl_wait_prior_grid();
        for (int i = 0; i < pre; ++i) load_x(i, kb0 + i);
      }
      int s = pre % STAGES;
      uint32_t ph = pre == STAGES ? 1u : 0u;
      uint32_t armed = pre == STAGES ? (1u << STAGES) - 1u : (1u << pre) - 1u, armed_ph = 0;
      for (int kb = kb0 + pre; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          raise_error(0x1u);
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[s], kLoadBytes);
        load_w(s, kb);
        if (!kFused) load_x(s, kb);
        armed |= 1u << s;
        armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      for (int i = 0; i < STAGES; ++i)
        if (armed & (1u << i)) mbar_wait(&full[i], (armed_ph >> i) & 1u, nullptr);
    }
    __syncwarp();
    cluster_wait();
  } else if (warp == 1) {
    pdl_wait_prior_grid();
    if (lane == 0 && nkb > 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      if (kFused && !mbar_wait(xready, 0, abort_flag)) {
        raise_error(0x2u);
        *abort_flag = 1;
        ok = false;
      }
      for (int kb = 0; kb < nkb && ok; ++kb) {
        if (!mbar_wait(&full[s], ph, abort_flag)) {
          raise_error(0x2u);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t a0 = sw128_kmajor_desc(smem_u32(sW + s * L::kWBytes));
        const uint64_t b0 = sw128_kmajor_desc(smem_u32(kFused ? fz_codes + kb * L::kXBytes : sX + s * L::kXBytes));
#pragma unroll
        for (int k = 0; k < SK / kUmmaK; ++k) {
          // box k / 4 of the stage, 32-byte step k % 4 inside its swizzle row
          const int box = k / (kBK / kUmmaK), kin = k % (kBK / kUmmaK);
          mma_f8f6f4(tmem_base, a0 + static_cast<uint64_t>(box * (L::kWBox >> 4) + kin * kUmmaK / 16),
                     b0 + static_cast<uint64_t>(box * (L::kXBox >> 4) + kin * kUmmaK / 16), kIdesc,
                     (kb | k) != 0 ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (ok) mma_commit(tfull);
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
    __syncwarp();
    cluster_wait();
  } else {
    pdl_wait_prior_grid();
    // Scales the reduction will need, staged while the mainloop runs.
    const int et = threadIdx.x - kEpiWarp0 * 32;   // 0..127
    {
      const int n = n0 + rank * SL + et;
      if (et < SL) sc_w[et] = n < p.N ? __ldg(p.s_w + n) : 0.0f;
      if (!kFused && et < p.rows) sc_x[et] = __ldg(p.s_x + et);
    }
    if (kFused) {
      // Per-token dynamic quantization of the rows this CTA multiplies,
      // shared by the S CTAs of the cluster, each of which reads only its
      // own K slice of the fp16 rows: (1) the maxima of |x| over the slice
      // go to slot [rank] of the partial-maxima
      // table and are copied into the same slot of every peer (bulk
      // shared-memory copies completing on the peer's pmax_bar); (2) each
      // row's maximum is the max of its S partial maxima -- the same value,
      // hence the same fp32 scale, on every CTA -- then r and s by the
      // quantizer's steps; (3) the codes of this CTA's K blocks are written
      // in the swizzled layout of a 128-byte TMA box (row m at m*128,
      // 16-byte chunk c at (c ^ (m & 7)) * 16).  Rows >= M and columns >= K
      // are zero.
      // (1) T = 128 / MPAD consecutive threads per row, each taking every
      // T-th 16-byte vector of the row's slice, eight loads in flight.
      constexpr int T = 128 / MPAD;
      const int v_lo = (kb0 * kBK) >> 3;
      const int v_hi = (kb1 * kBK < p.K ? kb1 * kBK : p.K) >> 3;
      float* own = fz_pmax + rank * MPAD;
      {
        const int m = et / T, sub = et % T;
        float a = 0.0f;
        if (m < p.rows) {
          const uint4* src = reinterpret_cast<const uint4*>(p.x_f16 + static_cast<int64_t>(m) * p.K);
          for (int j0 = v_lo + sub; j0 < v_hi; j0 += 8 * T) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = j0 + u * T < v_hi ? __ldg(src + j0 + u * T) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < 8; ++u) a = absmax8(v[u], a);
          }
        }
#pragma unroll
        for (int o = T / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (sub == 0 && m < p.rows) own[m] = a;
      }
      fence_proxy_async_smem();
      named_barrier(1, 128);
      bool got = true;
      if (S > 1) {
        // Every CTA of the cluster is running (arrived at set-up).  Only with
        // peers: a launch without a cluster (S = 1) treats the cluster barrier
        // as one over the whole CTA, whose MMA warp is waiting for these codes.
        cluster_wait();
        if (et < S && et != rank)
          bulk_copy_to_cluster(mapa_shared(smem_u32(own), static_cast<uint32_t>(et)), own, MPAD * 4,
                               mapa_shared(smem_u32(pmax_bar), static_cast<uint32_t>(et)));
        got = mbar_wait(pmax_bar, 0, abort_flag);
        if (!got) {
          raise_error(0x10u);
          *abort_flag = 1;
        }
      }
      if (et < p.rows) {
        float a = 0.0f;
        for (int s2 = 0; s2 < S; ++s2) a = fmaxf(a, fz_pmax[s2 * MPAD + et]);
        const RowScale rs = row_scale_from_amax(a);
        fz_r[et] = rs.r;
        sc_x[et] = rs.s;
      }
      named_barrier(1, 128);
      // (3) items (k block, row, 16-byte chunk of codes), four per thread
      // per round with all their loads issued first.
      const int items = nkb * MPAD * 8;
      for (int it0 = et; it0 < items; it0 += 4 * 128) {
        uint4 x[4][2];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int it = it0 + u * 128;
          const int m = (it >> 3) % MPAD;
          const int k = (kb0 + (it >> 3) / MPAD) * kBK + (it & 7) * 16;
          x[u][0] = x[u][1] = make_uint4(0, 0, 0, 0);
          if (it < items && m < p.rows && k < p.K) {
            const uint4* src = reinterpret_cast<const uint4*>(p.x_f16 + static_cast<int64_t>(m) * p.K + k);
            x[u][0] = __ldg(src);
            x[u][1] = __ldg(src + 1);
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int it = it0 + u * 128;
          if (it >= items) break;
          const int c = it & 7;
          const int m = (it >> 3) % MPAD;
          const int j = (it >> 3) / MPAD;
          uint4 out = make_uint4(0, 0, 0, 0);
          if (m < p.rows) {
            const float r = fz_r[m];
            const uint2 e0 = encode8(x[u][0], r);
            const uint2 e1 = encode8(x[u][1], r);
            out = make_uint4(e0.x, e0.y, e1.x, e1.y);
          }
          st_shared_v4(smem_u32(fz_codes + j * L::kXBytes + m * kBK) + static_cast<uint32_t>((c ^ (m & 7)) << 4),
                       out.x, out.y, out.z, out.w);
        }
      }
      fence_proxy_async_smem();
      named_barrier(1, 128);
      if (et == 0 && got) mbar_arrive(xready);
    }
    // Partial: TMEM lane = weight row n of the tile, column = token row m.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    bool have = nkb > 0;
    if (have && !mbar_wait(tfull, 0, abort_flag)) {
      raise_error(0x4u);
      *abort_flag = 1;
      have = false;
    }
    tc_fence_after();
    // Stage into the idle ring as [owner][row within owner][pitch].
    float* dst = send + row * L::kPitch;
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    if (MPAD == 16) {
      uint32_t v[16];
      if (have) {
        tmem_ld_32x32b_x16(taddr, v);
        tmem_ld_wait();
      }
#pragma unroll
      for (int i = 0; i < 16; i += 4)
        if (i < mcols)
          *reinterpret_cast<float4*>(dst + i) =
              make_float4(have ? __uint_as_float(v[i]) : 0.f, have ? __uint_as_float(v[i + 1]) : 0.f,
                          have ? __uint_as_float(v[i + 2]) : 0.f, have ? __uint_as_float(v[i + 3]) : 0.f);
    } else {
      // 32 columns at a time, the TMEM load of chunk c+1 in flight while
      // chunk c is written out.
      const int nch = (mcols + 31) / 32;
      uint32_t v[2][32];
      if (have) tmem_ld_32x32b_x32(taddr, v[0]);
#pragma unroll
      for (int c = 0; c < MPAD / 32; ++c) {
        if (c >= nch) break;
        if (have) {
          tmem_ld_wait_regs(v[c & 1]);
          if (c + 1 < nch) tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>((c + 1) * 32), v[(c + 1) & 1]);
        }
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          if (c * 32 + i < mcols)
            *reinterpret_cast<float4*>(dst + c * 32 + i) =
                make_float4(have ? __uint_as_float(v[c & 1][i]) : 0.f, have ? __uint_as_float(v[c & 1][i + 1]) : 0.f,
                            have ? __uint_as_float(v[c & 1][i + 2]) : 0.f,
                            have ? __uint_as_float(v[c & 1][i + 3]) : 0.f);
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    named_barrier(1, 128);   // the four epilogue warps have written the whole send buffer
    if (!kFused || S == 1) cluster_wait();   // every CTA of the cluster is running (fused: waited above)
    if (et < S && et != rank) {
      // ship owner et's rows to its receive slot [rank]
      const uint32_t peer_recv = mapa_shared(smem_u32(recv + rank * SL * L::kPitch), static_cast<uint32_t>(et));
      const uint32_t peer_bar = mapa_shared(smem_u32(recv_bar), static_cast<uint32_t>(et));
      bulk_copy_to_cluster(peer_recv, send + et * SL * L::kPitch, slice_bytes, peer_bar);
    }
    // Own rows: wait for the S-1 peers' slices, sum in rank order, scale, store.
    if (!mbar_wait(recv_bar, 0, abort_flag)) {
      raise_error(0x10u);
      *abort_flag = 1;
    } else {
      switch (S) {
        case 1: splitk_reduce_store<1, L>(p, send, recv, sc_w, sc_x, n0, rank, et); break;
        case 2: splitk_reduce_store<2, L>(p, send, recv, sc_w, sc_x, n0, rank, et); break;
        case 4: splitk_reduce_store<4, L>(p, send, recv, sc_w, sc_x, n0, rank, et); break;
        default: splitk_reduce_store<8, L>(p, send, recv, sc_w, sc_x, n0, rank, et); break;
      }
    }
  }

  // No CTA may leave while a peer's bulk copy still reads its send buffer:
  // every CTA arrives only after all copies into it have landed.
  __syncthreads();
  cluster_arrive();
  cluster_wait();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace fp8q
