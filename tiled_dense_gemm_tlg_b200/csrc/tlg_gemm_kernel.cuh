// Persistent, warp-specialised fp16 GEMM for sm_100a.
//
// The tiling is the pages' block decomposition -- one output tile per
// (row block, column block), an fp32 accumulator per tile, operand tiles of
// A[rows, k-block] and B[k-block, cols] staged in shared memory by a
// multi-stage pipeline over the K loop ("tilelang operator-compilation
// walkthrough", lqnn.cn/news/222844, section 2.1) -- mapped onto Blackwell:
//
//   warp 0 (one lane)  producer: TMA loads of the A and B tiles of each
//                      k-block into a STAGES-deep ring, one mbarrier pair per
//                      slot (full: bytes landed; empty: the MMAs read it).
//   warp 1 (one lane)  MMA issuer: tcgen05.mma 128 x BN x 16 into a TMEM
//                      accumulator; two accumulators alternate so the
//                      epilogue of tile i overlaps the main loop of tile i+1.
//                      Warp 1 also owns the TMEM allocation.
//   warps 2-5          epilogue: tcgen05.ld of the accumulator, then bias,
//                      ReLU and the output cast ("domestic-GPU TileLang
//                      adoption", xdnf.cn/news/333523, section 4.2), and a
//                      predicated store of the rows and columns inside M x N.
//
// CTAs are persistent (one per SM) and walk the tile list with a stride of
// gridDim.x; consecutive tiles are grouped by `raster_group` row blocks so
// the CTAs of one wave share A and B tiles in L2.
//
// Ragged M, N and K need no special code in the main loop: the TMA unit fills
// out-of-range elements of a box with zeros, so the last k-block adds 0 for
// k >= K, and rows/columns beyond M/N are simply not stored.
#pragma once

#include "tlg_device.cuh"

namespace tlg {

constexpr int kBM = 128;  // tile rows (TMEM lanes)
constexpr int kBK = 64;   // k-block: 64 fp16 = one 128-byte swizzle row
constexpr int kThreads = 192;

__device__ uint32_t g_device_error;

// Shared-memory plan of one CTA.  CG CTAs (1 or 2) compute one tile of
// 128*CG rows by BN columns; each CTA stages its own 128 rows of A and its own
// BN/CG columns of B per k-block.
template <int CG, int BN, int STAGES>
struct SmemPlan {
  static constexpr int kBNc = BN / CG;  // B columns held by one CTA
  static constexpr uint32_t kABytes = kBM * kBK * 2;
  static constexpr uint32_t kBBytes = kBK * kBNc * 2;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kBarOffset = STAGES * kStageBytes;
  static constexpr uint32_t kNumBars = 2 * STAGES + 4 + 1;  // full, empty, tmem full/empty x2, drain
  static constexpr uint32_t kMiscOffset = kBarOffset + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOffset + 16;
  static constexpr uint32_t kDynamicBytes = kBytes + 1024;  // slack to align the base to 1024
  static constexpr uint32_t kTmemCols = (2 * BN < 32) ? 32 : 2 * BN;
  static_assert(kBNc % 64 == 0, "each CTA's B slice must be whole 64-column swizzle blocks");
  static_assert(kTmemCols <= 512, "two accumulators must fit in TMEM");
  static_assert(kDynamicBytes <= 232448, "shared memory per CTA exceeded");
};

struct GemmParams {
  void *C;
  const __half *bias;
  int64_t ldc;
  int M, N, K;
  int raster_group;
  uint64_t limit_ns;
};

__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int group, int &mb,
                                            int &nb) {
  const int per_group = group * num_n;
  const int g = t / per_group;
  const int first_m = g * group;
  const int gm = min(num_m - first_m, group);
  const int r = t - g * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

template <bool OUT_F16, bool BIAS_RELU>
__device__ __forceinline__ void store_chunk(const GemmParams &p, int row, int col0,
                                            const uint32_t (&r)[32]) {
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
  const bool full = col0 + 32 <= p.N;
  if constexpr (BIAS_RELU) {
    if (full) {
      const uint4 *bp = reinterpret_cast<const uint4 *>(p.bias + col0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 w = __ldg(bp + q);
        const __half2 *h = reinterpret_cast<const __half2 *>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(h[e]);
          v[q * 8 + 2 * e] += f.x;
          v[q * 8 + 2 * e + 1] += f.y;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < p.N) v[j] += __half2float(p.bias[col0 + j]);
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = fmaxf(v[j], 0.0f);
  }
  if constexpr (OUT_F16) {
    __half *crow = reinterpret_cast<__half *>(p.C) + static_cast<int64_t>(row) * p.ldc + col0;
    if (full) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 w;
        __half2 *h = reinterpret_cast<__half2 *>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = __floats2half2_rn(v[q * 8 + 2 * e], v[q * 8 + 2 * e + 1]);
        reinterpret_cast<uint4 *>(crow)[q] = w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < p.N) crow[j] = __float2half_rn(v[j]);
    }
  } else {
    float *crow = reinterpret_cast<float *>(p.C) + static_cast<int64_t>(row) * p.ldc + col0;
    if (full) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4 *>(crow)[q] =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < p.N) crow[j] = v[j];
    }
  }
}

template <int CG, int BN, int STAGES, bool OUT_F16, bool BIAS_RELU>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_sm100_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, const GemmParams p) {
  using Plan = SmemPlan<CG, BN, STAGES>;
  constexpr int kTileM = kBM * CG;
  static_assert(CG == 1 || CG == 2, "one CTA or a CTA pair per tile");
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN must be 64, 128, 192 or 256");

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * Plan::kABytes;
  const uint32_t bar0 = smem_u32(smem + Plan::kBarOffset);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + Plan::kMiscOffset);
  uint32_t *tmem_holder = misc;
  volatile uint32_t *abort_flag = misc + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Work unit = one tile per CTA group: a CTA (CG == 1) or a cluster of two (CG == 2).
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
  const int unit = (CG == 2) ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int num_units = (CG == 2) ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);
  const bool leader = rank == 0;
  const int num_m = (p.M + kTileM - 1) / kTileM;
  const int num_n = (p.N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (p.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4 * CG);  // one arrive per epilogue warp of each CTA
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc<CG>(smem_u32(tmem_holder), Plan::kTmemCols);
    tmem_relinquish<CG>();
  }
  tc_fence_before_sync();
  __syncwarp();
  if constexpr (CG == 2)
    cluster_sync_all();  // both CTAs' barriers exist before either signals the other
  else
    __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tmem_holder);

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer (every CTA)
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_parity = 0;
    bool ok = true;
    for (int t = unit; t < num_tiles && ok; t += num_units) {
      int mb, nb;
      tile_coords(t, num_m, num_n, p.raster_group, mb, nb);
      const int a_row = mb * kTileM + static_cast<int>(rank) * kBM;
      const int b_col = nb * BN + static_cast<int>(rank) * Plan::kBNc;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.limit_ns, kRoleProducer,
                       &g_device_error)) {
          ok = false;
          break;
        }
        const uint32_t a_dst = smem_u32(sA + stage * Plan::kABytes);
        const uint32_t b_dst = smem_u32(sB + stage * Plan::kBBytes);
        if constexpr (CG == 1) {
          mbar_arrive_expect_tx(full_bar(stage), Plan::kStageBytes);
          tma_load_2d(a_dst, &tmA, full_bar(stage), kb * kBK, a_row);
#pragma unroll
          for (int c = 0; c < Plan::kBNc / 64; ++c)
            tma_load_2d(b_dst + c * 8192, &tmB, full_bar(stage), b_col + c * 64, kb * kBK);
        } else {
          // The leader's full barrier counts the bytes of both CTAs' loads.
          if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * Plan::kStageBytes);
          const uint32_t bar = mapa_shared(full_bar(stage), 0);
          tma_load_2d_pair(a_dst, &tmA, bar, kb * kBK, a_row);
#pragma unroll
          for (int c = 0; c < Plan::kBNc / 64; ++c)
            tma_load_2d_pair(b_dst + c * 8192, &tmB, bar, b_col + c * 64, kb * kBK);
        }
        issued_mask |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (ok) {
      // Tail: wait until every slot has been released, so no commit-arrive is
      // still on its way to this CTA's barriers when it exits.
      for (int i = 0; i < STAGES; ++i) {
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.limit_ns, kRoleProducer,
                       &g_device_error)) {
          ok = false;
          break;
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && leader) {
      // Let the copies already issued land before shared memory goes away.
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s))
          mbar_wait(full_bar(s), (issued_parity >> s) & 1u, nullptr, p.limit_ns, kRoleProducer,
                    &g_device_error);
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------------------------------------------------------- MMA issuer (leader CTA)
    constexpr uint32_t idesc = make_idesc_f16(kTileM, BN);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = unit; t < num_tiles && ok; t += num_units) {
      if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.limit_ns, kRoleMma,
                     &g_device_error)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(full_bar(stage), phase, abort_flag, p.limit_ns, kRoleMma,
                       &g_device_error)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t a0 = smem_u32(sA + stage * Plan::kABytes);
        const uint32_t b0 = smem_u32(sB + stage * Plan::kBBytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t adesc = smem_desc_sw128(a0 + kk * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(b0 + kk * 16 * 128, 8192, 1024);
          mma_f16_ss<CG>(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        mma_commit<CG>(empty_bar(stage));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      mma_commit<CG>(tfull_bar(acc));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (!ok) {
      // Wait for the MMAs already in flight before TMEM and shared memory are released.
      mma_commit_local<CG>(drain_bar);
      mbar_wait(drain_bar, 0, nullptr, p.limit_ns, kRoleMma, &g_device_error);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue (every CTA)
    const int quarter = warp & 3;  // TMEM lanes this warp may access: 32*quarter ...
    const int row_in_tile = static_cast<int>(rank) * kBM + quarter * 32 + lane;
    const uint32_t release_bar0 = (CG == 2) ? mapa_shared(tempty_bar(0), 0) : tempty_bar(0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = unit; t < num_tiles; t += num_units) {
      int mb, nb;
      tile_coords(t, num_m, num_n, p.raster_group, mb, nb);
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag, p.limit_ns, kRoleEpilogue,
                     &g_device_error))
        break;
      tc_fence_after_sync();
      const int row = mb * kTileM + row_in_tile;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        __syncwarp();
        tmem_load_32cols(tbase + ch * 32, r);
        const int col0 = nb * BN + ch * 32;
        if (row < p.M && col0 < p.N) store_chunk<OUT_F16, BIAS_RELU>(p, row, col0, r);
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if constexpr (CG == 2)
          mbar_arrive_cluster(release_bar0 + 8u * acc);
        else
          mbar_arrive(release_bar0 + 8u * acc);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before_sync();
  __syncwarp();
  if constexpr (CG == 2)
    cluster_sync_all();  // neither CTA leaves while its peer may still touch its shared memory
  else
    __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc<CG>(tmem_base, Plan::kTmemCols);
  }
}

// C = 0 (or fp16(max(bias[col], 0))) for K == 0, where the sum over k is empty.
template <bool OUT_F16, bool BIAS_RELU>
__global__ void fill_empty_k_kernel(void *C, int64_t ldc, const __half *bias, int M, int N) {
  const int64_t total = static_cast<int64_t>(M) * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / N, c = i % N;
    float v = 0.0f;
    if constexpr (BIAS_RELU) v = fmaxf(__half2float(bias[c]), 0.0f);
    if constexpr (OUT_F16)
      reinterpret_cast<__half *>(C)[r * ldc + c] = __float2half_rn(v);
    else
      reinterpret_cast<float *>(C)[r * ldc + c] = v;
  }
}

// One thread waits on a barrier that nothing signals; the bounded wait gives
// up after limit_ns, records the timeout and the kernel returns normally.
__global__ void selftest_timeout_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_word;
  if (threadIdx.x == 0) {
    abort_word = 0u;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    mbar_wait(smem_u32(&bar), 0, &abort_word, limit_ns, kRoleSelftest, &g_device_error);
  }
}

}  // namespace tlg
