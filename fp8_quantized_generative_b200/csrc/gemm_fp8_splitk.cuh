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
//   * every CTA copies its partial into its own shared memory, the cluster
//     synchronizes, and CTA r sums lanes [r*128/S, (r+1)*128/S) of all S
//     partials (ranks in fixed order 0..S-1, so results are reproducible),
//     applies the scales and writes fp16 -- no global scratch memory.
#pragma once

#include "gemm_common.cuh"

namespace fp8q {

constexpr int kSkThreads = 192;   // producer, MMA, 4 epilogue warps

template <int MPAD, int STAGES>
struct SplitKLayout {
  static constexpr int kWBytes = kBM * kBK;            // 128 weight rows x 128 K bytes
  static constexpr int kXBytes = MPAD * kBK;           // MPAD token rows
  static constexpr int kStageBytes = kWBytes + kXBytes;
  static constexpr int kPitch = MPAD + 1;              // fp32 words per partial row (odd: no bank conflicts)
  static constexpr int kPartialBytes = kBM * kPitch * 4;
  static constexpr int kRingBytes = STAGES * kStageBytes;
  static constexpr int kBodyBytes = kRingBytes > kPartialBytes ? kRingBytes : kPartialBytes;
  static constexpr int kNumBars = 2 * STAGES + 2;      // full, empty, tfull, drain
  static constexpr int kTmemCols = MPAD < 32 ? 32 : MPAD;
  static constexpr size_t kSmemBytes = 1024 + size_t(kBodyBytes) + kNumBars * 8 + 32;
};

template <int MPAD, int STAGES>
__global__ void __launch_bounds__(kSkThreads, 1)
    fp8_gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                           const GemmParams p) {
  using L = SplitKLayout<MPAD, STAGES>;
  static_assert(MPAD % 16 == 0 && MPAD >= 16 && MPAD <= 128, "MPAD");
  constexpr uint32_t kIdesc = idesc_e4m3_f32(kBM, MPAD);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sW = smem;
  uint8_t* sX = smem + STAGES * L::kWBytes;
  float* part = reinterpret_cast<float*>(smem);   // reused after the mainloop
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBodyBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* drain = bars + 2 * STAGES + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = static_cast<int>(cluster_nctarank());
  const int rank = static_cast<int>(cluster_ctarank());
  const int n_tile = static_cast<int>(blockIdx.x) / S;
  const int n0 = n_tile * kBM;
  const int num_kb = (p.K + kBK - 1) / kBK;
  const int kb0 = static_cast<int>((int64_t(rank) * num_kb) / S);
  const int kb1 = static_cast<int>((int64_t(rank + 1) * num_kb) / S);
  const int nkb = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
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
  pdl_wait_prior_grid();

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, armed = 0, armed_ph = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          raise_error(0x1u);
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[s], L::kStageBytes);
        tma_load_2d(sW + s * L::kWBytes, &tmW, &full[s], kb * kBK, n0);
        tma_load_2d(sX + s * L::kXBytes, &tmX, &full[s], kb * kBK, 0);
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
  } else if (warp == 1) {
    if (lane == 0 && nkb > 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(&full[s], ph, abort_flag)) {
          raise_error(0x2u);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t a0 = sw128_kmajor_desc(smem_u32(sW + s * L::kWBytes));
        const uint64_t b0 = sw128_kmajor_desc(smem_u32(sX + s * L::kXBytes));
#pragma unroll
        for (int k = 0; k < kBK / kUmmaK; ++k)
          mma_f8f6f4(tmem_base, a0 + static_cast<uint64_t>(k * kUmmaK / 16), b0 + static_cast<uint64_t>(k * kUmmaK / 16),
                     kIdesc, (kb | k) != 0 ? 1u : 0u);
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
  } else {
    // Partial (TMEM lanes = weight rows of the tile, columns = token rows)
    // -> own shared memory, row pitch MPAD + 1 words.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    bool have = nkb > 0;
    if (have && !mbar_wait(tfull, 0, abort_flag)) {
      raise_error(0x4u);
      *abort_flag = 1;
      have = false;
    }
    tc_fence_after();
    float* prow = part + row * L::kPitch;
    if (have) {
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      if (MPAD == 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(taddr, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) prow[i] = __uint_as_float(v[i]);
      } else {
#pragma unroll 1
        for (int c = 0; c < MPAD / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c * 32), v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) prow[c * 32 + i] = __uint_as_float(v[i]);
        }
      }
    } else {
      for (int i = 0; i < MPAD; ++i) prow[i] = 0.0f;
    }
    tc_fence_before();
  }

  __syncthreads();
  cluster_arrive();
  cluster_wait();

  if (warp >= kEpiWarp0) {
    // CTA `rank` reduces weight rows [rank*SL, rank*SL + SL) over all S partials.
    const int SL = kBM / S;
    const int r0 = rank * SL;
    const int t = threadIdx.x - kEpiWarp0 * 32;
    const uint32_t part_local = smem_u32(part);
    uint32_t base[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) base[s] = s < S ? mapa_shared(part_local, static_cast<uint32_t>(s)) : 0u;
    const int total = p.rows * SL;
    for (int idx = t; idx < total; idx += 128) {
      const int nl = idx % SL;
      const int m = idx / SL;
      const int n = n0 + r0 + nl;
      if (n >= p.N) continue;
      const uint32_t off = static_cast<uint32_t>(((r0 + nl) * L::kPitch + m) * 4);
      float acc = 0.0f;
      for (int s = 0; s < S; ++s) acc = __fadd_rn(acc, ld_dsmem_f32(base[s] + off));
      const float y = __fmul_rn(__fmul_rn(acc, __ldg(p.s_x + m)), __ldg(p.s_w + n));
      p.Y[static_cast<int64_t>(m) * p.N + n] = __float2half_rn(y);
    }
  }

  // No CTA may leave while the others still read its shared memory.
  __syncthreads();
  cluster_arrive();
  cluster_wait();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace fp8q
