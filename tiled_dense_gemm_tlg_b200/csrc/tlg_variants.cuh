// Launch wrappers for every kernel instantiation, shared by the translation
// units that instantiate them (one per operand layout, compiled in parallel).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tlg.h"
#include "tlg_gemm_kernel.cuh"

namespace tlg {

constexpr int kMaxDevices = 64;

// Per device and instantiation: kernel attributes set, co-resident work units.
struct LaunchState {
  bool ready = false;
  int units = 0;
};

template <int CG, int TN, int STAGES, bool OUT_F16, int EK, bool AT, bool BT, bool LSU, int KS = 1>
struct Variant {
  static constexpr int NH = TN > 256 ? 2 : 1;  // MMA halves per tile
  static constexpr int BN = TN / NH;           // the MMA's N
  static constexpr int kClusterCtas = CG * KS;  // CTAs of one work unit (a cluster when > 1)
  using Plan = SmemPlan<CG, BN, STAGES, NH, KS>;
  static_assert(Plan::kDynamicBytes <= 232448, "shared memory per CTA exceeded");

  // attr must hold 2 entries.  With overlap_prev the kernel may start while
  // the previous kernel in the stream finishes (programmatic stream
  // serialization); it waits for that kernel before touching global memory.
  static void fill_launch(cudaLaunchConfig_t *cfg, cudaLaunchAttribute *attr, cudaStream_t s,
                          bool overlap_prev = false) {
    *cfg = {};
    cfg->blockDim = dim3(LSU ? kThreadsLsu : kThreads, 1, 1);
    cfg->dynamicSmemBytes = Plan::kDynamicBytes;
    cfg->stream = s;
    int n = 0;
    if (overlap_prev) {
      attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[n].val.programmaticStreamSerializationAllowed = 1;
      ++n;
    }
    if (kClusterCtas > 1) {
      attr[n].id = cudaLaunchAttributeClusterDimension;
      attr[n].val.clusterDim.x = kClusterCtas;
      attr[n].val.clusterDim.y = 1;
      attr[n].val.clusterDim.z = 1;
      ++n;
    }
    cfg->attrs = attr;
    cfg->numAttrs = n;
  }

  // Work units (CTAs, or clusters of CTAs) that can be resident at once: one per SM,
  // or the number of clusters the occupancy calculator admits.
  static tlg_status units(int dev, int sms, int *out) {
    static LaunchState state[kMaxDevices];
    auto kernel = gemm_sm100_kernel<CG, BN, STAGES, OUT_F16, EK, NH, AT, BT, LSU, KS>;
    static std::mutex mutex;
    std::lock_guard<std::mutex> lock(mutex);
    LaunchState &st = state[dev];
    if (!st.ready) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Plan::kDynamicBytes) != cudaSuccess) {
        cudaGetLastError();
        return TLG_ERR_CUDA;
      }
      int n = sms;
      if (kClusterCtas > 1) {
        cudaLaunchConfig_t cfg;
        cudaLaunchAttribute attr[2];
        fill_launch(&cfg, attr, nullptr);
        cfg.gridDim = dim3(kClusterCtas * (sms / kClusterCtas), 1, 1);
        if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n < 1) {
          cudaGetLastError();
          return TLG_ERR_CUDA;
        }
      }
      st.units = n;
      st.ready = true;
    }
    *out = st.units;
    return TLG_OK;
  }

  static tlg_status launch(int units, const CUtensorMap &tmA, const CUtensorMap &tmB,
                           const CUtensorMap &tmC, const CUtensorMap &tmR, const GemmParams &p,
                           bool overlap_prev, cudaStream_t s) {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[2];
    fill_launch(&cfg, attr, s, overlap_prev);
    cfg.gridDim = dim3(static_cast<unsigned>(units * kClusterCtas), 1, 1);
    const cudaError_t e = cudaLaunchKernelEx(
        &cfg, gemm_sm100_kernel<CG, BN, STAGES, OUT_F16, EK, NH, AT, BT, LSU, KS>, tmA, tmB, tmC,
        tmR, p);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return TLG_ERR_CUDA;
    }
    return TLG_OK;
  }
};

struct VariantFns {
  tlg_status (*units)(int, int, int *);
  tlg_status (*launch)(int, const CUtensorMap &, const CUtensorMap &, const CUtensorMap &,
                       const CUtensorMap &, const GemmParams &, bool, cudaStream_t);
};


constexpr int kNumVariants = 9;

#define TLG_FNS(CG, TN, ST, F16, BR, AT, BT, L, KS)                  \
  VariantFns {                                                       \
    Variant<CG, TN, ST, F16, BR, AT, BT, L, KS>::units,              \
        Variant<CG, TN, ST, F16, BR, AT, BT, L, KS>::launch          \
  }
#define TLG_VARIANT_KS(CG, TN, ST, AT, BT, L, KS)                                       \
  {                                                                                     \
    TLG_FNS(CG, TN, ST, false, kEpiNone, AT, BT, L, KS),                                \
        TLG_FNS(CG, TN, ST, true, kEpiNone, AT, BT, L, KS),                             \
        TLG_FNS(CG, TN, ST, true, kEpiFused, AT, BT, L, KS),                            \
        TLG_FNS(CG, TN, ST, false, kEpiFused, AT, BT, L, KS),                           \
        TLG_FNS(CG, TN, ST, true, kEpiBiasRelu, AT, BT, L, KS)                          \
  }
#define TLG_VARIANT(CG, TN, ST, AT, BT, L) TLG_VARIANT_KS(CG, TN, ST, AT, BT, L, 1)
#define TLG_NONE                                                                          \
  {                                                                                       \
    VariantFns{nullptr, nullptr}, VariantFns{nullptr, nullptr}, VariantFns{nullptr, nullptr}, \
        VariantFns{nullptr, nullptr}, VariantFns{nullptr, nullptr}                        \
  }
// The TMA variants of one layout, in kBuilt's order.  The cluster k-split tiles
// (the last three) are built for untransposed operands only (TLG_LAYOUT_NN).
#define TLG_LAYOUT_COMMON(AT, BT)                                                            \
    TLG_VARIANT(1, 64, 8, AT, BT, false), TLG_VARIANT(1, 128, 6, AT, BT, false),             \
        TLG_VARIANT(1, 256, 4, AT, BT, false), TLG_VARIANT(2, 128, 8, AT, BT, false),        \
        TLG_VARIANT(2, 256, 6, AT, BT, false), TLG_VARIANT(2, 512, 4, AT, BT, false)
#define TLG_LAYOUT(AT, BT) \
  { TLG_LAYOUT_COMMON(AT, BT), TLG_NONE, TLG_NONE, TLG_NONE }
#define TLG_LAYOUT_NN                                                                       \
  {                                                                                         \
    TLG_LAYOUT_COMMON(false, false), TLG_VARIANT_KS(1, 128, 5, false, false, false, 2),     \
        TLG_VARIANT_KS(1, 256, 2, false, false, false, 2),                                  \
        TLG_VARIANT_KS(1, 256, 2, false, false, false, 4)                                   \
  }
// The same with plain loads, for the variants marked plain_loads in kBuilt.
#define TLG_LAYOUT_PLAIN(AT, BT)                                                       \
  {                                                                                    \
    TLG_VARIANT(1, 64, 8, AT, BT, true), TLG_NONE, TLG_NONE, TLG_NONE,                 \
        TLG_VARIANT(2, 256, 6, AT, BT, true), TLG_NONE, TLG_NONE, TLG_NONE, TLG_NONE   \
  }


// Output kinds of the launcher tables: plain fp32, plain fp16, the general
// fused epilogue (bias / activation / residual) with an fp16 or an fp32 C, and
// the bias + ReLU build with an fp16 C.
constexpr int kKindF32 = 0, kKindF16 = 1, kKindF16Epi = 2, kKindF32Epi = 3, kKindF16BiasRelu = 4,
              kNumKinds = 5;

// Tables of one operand layout: [variant, same order as the host's table][output kind]
struct LayoutTables {
  VariantFns tma[kNumVariants][kNumKinds];
  VariantFns plain[kNumVariants][kNumKinds];
};

// Defined by tlg_layout_{nn,nt,tn,tt}.cu.
extern const LayoutTables kLayoutNN, kLayoutNT, kLayoutTN, kLayoutTT;

// Device error word of each translation unit (every unit has its own copy).
tlg_status error_word_nn(bool clear, uint32_t *out);
tlg_status error_word_nt(bool clear, uint32_t *out);
tlg_status error_word_tn(bool clear, uint32_t *out);
tlg_status error_word_tt(bool clear, uint32_t *out);

#define TLG_DEFINE_ERROR_WORD_READER(NAME)                                            \
  tlg_status NAME(bool clear, uint32_t *out) {                                        \
    uint32_t v = 0;                                                                   \
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) {         \
      cudaGetLastError();                                                             \
      return TLG_ERR_CUDA;                                                            \
    }                                                                                 \
    if (clear && v != 0) {                                                            \
      const uint32_t zero = 0;                                                        \
      if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) {   \
        cudaGetLastError();                                                           \
        return TLG_ERR_CUDA;                                                          \
      }                                                                               \
    }                                                                                 \
    *out = v;                                                                         \
    return TLG_OK;                                                                    \
  }

}  // namespace tlg
