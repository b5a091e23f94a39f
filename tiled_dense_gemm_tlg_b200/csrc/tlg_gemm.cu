// Host side of libtlg: argument checks, TMA descriptor encoding, the per-shape
// configuration table and the launches behind the C interface in tlg.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "tlg.h"
#include "tlg_gemm_kernel.cuh"

namespace {

using namespace tlg;

constexpr int kMaxDevices = 64;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per pipeline wait

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

tlg_status current_device(int *dev, DeviceInfo *info) {
  if (cudaGetDevice(dev) != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  if (*dev < 0 || *dev >= kMaxDevices) return TLG_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo &d = g_devices[*dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess) {
      cudaGetLastError();
      return TLG_ERR_CUDA;
    }
    d.supported = (major == 10 && minor == 0);
    d.sm_count = sms;
    d.probed = true;
  }
  if (g_encode == nullptr) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
      cudaGetLastError();
      return TLG_ERR_CUDA;
    }
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *info = d;
  return d.supported ? TLG_OK : TLG_ERR_UNSUPPORTED;
}

// A pointer the kernels may read or write: device memory of `dev`, or managed memory.
bool device_accessible(const void *p, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (a.type == cudaMemoryTypeManaged) return true;
  return a.type == cudaMemoryTypeDevice && a.device == dev;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte range [lo, hi) touched by a rows x cols matrix with row stride ld.
void extent(const void *p, int64_t rows, int64_t cols, int64_t ld, int64_t esz, uintptr_t *lo,
            uintptr_t *hi) {
  *lo = reinterpret_cast<uintptr_t>(p);
  *hi = *lo + static_cast<uintptr_t>(((rows - 1) * ld + cols) * esz);
}

bool overlaps(uintptr_t a0, uintptr_t a1, uintptr_t b0, uintptr_t b1) { return a0 < b1 && b0 < a1; }

// --------------------------------------------------------------------------- configurations

struct KernelCfg {
  int cta_group;
  int block_n;
  int stages;
  double eff;  // fraction of the MMA peak one tile sustains (used to rank tile shapes)
};

// Tile shapes the library is built with.  A tile is 128*cta_group rows by
// block_n columns; `stages` is the deepest operand ring that fits in 227 KB of
// shared memory next to the barriers.  Per-CTA ring slot: 16 KB of A plus
// 128*block_n/cta_group bytes of B.
// `eff` is measured: TFLOP/s of each shape on a B200 at M = N = K = 4096 and
// 8192 after dividing out the wave count, relative to the 2 x 256 pair tile.
constexpr KernelCfg kBuilt[] = {
    {1, 64, 8, 0.35}, {1, 128, 6, 0.60}, {1, 256, 4, 0.90}, {2, 128, 8, 0.60}, {2, 256, 6, 1.00}};

const KernelCfg *find_built(int cta_group, int block_n) {
  for (const KernelCfg &k : kBuilt)
    if (k.cta_group == cta_group && k.block_n == block_n) return &k;
  return nullptr;
}

// Pick the tile shape with the fewest estimated SM-time units: whole waves of
// tiles over the available CTAs (pairs), times the tile's work over its
// sustained fraction of the MMA peak.  Narrow and single-SM tiles sustain less
// because each 128-row MMA reads all of its A tile from shared memory for
// every block_n columns it produces.
void choose(int64_t M, int64_t N, int sms, tlg_config *c) {
  double best = 0;
  const KernelCfg *pick = &kBuilt[0];
  for (const KernelCfg &k : kBuilt) {
    const int64_t tile_m = 128 * k.cta_group;
    const int64_t tiles = ((M + tile_m - 1) / tile_m) * ((N + k.block_n - 1) / k.block_n);
    const int64_t units = sms / k.cta_group;
    const int64_t waves = (tiles + units - 1) / units;
    const double cost = static_cast<double>(waves) * tile_m * k.block_n / (k.cta_group * k.eff);
    if (&k == &kBuilt[0] || cost < best * 0.999) {
      best = cost;
      pick = &k;
    }
  }
  c->block_n = pick->block_n;
  c->stages = pick->stages;
  c->cta_group = pick->cta_group;
  c->raster_group = 8;
  c->max_ctas = 0;
}

tlg_status resolve_config(int64_t M, int64_t N, int sms, const tlg_config *req, tlg_config *out) {
  choose(M, N, sms, out);
  if (req == nullptr) return TLG_OK;
  int cg = req->cta_group != 0 ? req->cta_group : out->cta_group;
  int bn = req->block_n != 0 ? req->block_n : out->block_n;
  const KernelCfg *k = find_built(cg, bn);
  if (k == nullptr) {
    // a width given alone may exist only for the other CTA-group size
    if (req->cta_group == 0 && req->block_n != 0) {
      cg = 3 - cg;
      k = find_built(cg, bn);
    }
    if (k == nullptr) return TLG_ERR_UNSUPPORTED;
  }
  out->cta_group = cg;
  out->block_n = bn;
  out->stages = k->stages;
  if (req->stages != 0 && req->stages != k->stages) return TLG_ERR_UNSUPPORTED;
  if (req->raster_group != 0) {
    if (req->raster_group < 1 || req->raster_group > 64) return TLG_ERR_UNSUPPORTED;
    out->raster_group = req->raster_group;
  }
  if (req->max_ctas < 0) return TLG_ERR_UNSUPPORTED;
  out->max_ctas = req->max_ctas;
  return TLG_OK;
}

// --------------------------------------------------------------------------- launch

bool encode_2d(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims,
                              strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct LaunchState {
  bool attr_set = false;
  int max_clusters = 0;  // co-resident clusters of this kernel (cta_group 2)
};

// Launch one kernel instantiation: persistent grid of one CTA per SM (or one
// cluster per SM pair, limited to the clusters that fit at once), capped by
// the tile count and max_ctas.
template <int CG, int BN, int STAGES, bool OUT_F16, bool BIAS_RELU>
tlg_status launch_gemm(int dev, int sms, const CUtensorMap &tmA, const CUtensorMap &tmB,
                       const GemmParams &p, int64_t tiles, int max_ctas, cudaStream_t stream) {
  using Plan = SmemPlan<CG, BN, STAGES>;
  auto kernel = gemm_sm100_kernel<CG, BN, STAGES, OUT_F16, BIAS_RELU>;
  static LaunchState state[kMaxDevices];
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Plan::kDynamicBytes;
  cfg.stream = stream;
  if (CG == 2) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    LaunchState &st = state[dev];
    if (!st.attr_set) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Plan::kDynamicBytes) != cudaSuccess) {
        cudaGetLastError();
        return TLG_ERR_CUDA;
      }
      if (CG == 2) {
        cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n < 1) {
          cudaGetLastError();
          return TLG_ERR_CUDA;
        }
        st.max_clusters = n;
      }
      st.attr_set = true;
    }
  }
  int64_t units = CG == 2 ? state[dev].max_clusters : sms;
  if (max_ctas > 0) units = std::min<int64_t>(units, std::max(1, max_ctas / CG));
  units = std::min<int64_t>(units, tiles);
  cfg.gridDim = dim3(static_cast<unsigned>(units * CG), 1, 1);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  return TLG_OK;
}

template <bool OUT_F16, bool BIAS_RELU>
tlg_status dispatch(int dev, int sms, const tlg_config &c, const CUtensorMap &tmA,
                    const CUtensorMap &tmB, const GemmParams &p, cudaStream_t s) {
  const int64_t tile_m = 128 * c.cta_group;
  const int64_t tiles = ((p.M + tile_m - 1) / tile_m) * ((p.N + c.block_n - 1) / c.block_n);
  const int mc = c.max_ctas;
  if (c.cta_group == 1) {
    switch (c.block_n) {
      case 256: return launch_gemm<1, 256, 4, OUT_F16, BIAS_RELU>(dev, sms, tmA, tmB, p, tiles, mc, s);
      case 128: return launch_gemm<1, 128, 6, OUT_F16, BIAS_RELU>(dev, sms, tmA, tmB, p, tiles, mc, s);
      case 64: return launch_gemm<1, 64, 8, OUT_F16, BIAS_RELU>(dev, sms, tmA, tmB, p, tiles, mc, s);
      default: return TLG_ERR_UNSUPPORTED;
    }
  }
  switch (c.block_n) {
    case 256: return launch_gemm<2, 256, 6, OUT_F16, BIAS_RELU>(dev, sms, tmA, tmB, p, tiles, mc, s);
    case 128: return launch_gemm<2, 128, 8, OUT_F16, BIAS_RELU>(dev, sms, tmA, tmB, p, tiles, mc, s);
    default: return TLG_ERR_UNSUPPORTED;
  }
}

template <bool OUT_F16, bool BIAS_RELU>
tlg_status launch_fill(void *C, int64_t ldc, const void *bias, int M, int N, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(M) * N;
  const int threads = 256;
  const int blocks = static_cast<int>(total / threads + 1 > 4096 ? 4096 : total / threads + 1);
  fill_empty_k_kernel<OUT_F16, BIAS_RELU><<<blocks, threads, 0, s>>>(
      C, ldc, static_cast<const __half *>(bias), M, N);
  const cudaError_t e = cudaPeekAtLastError();
  if (e != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  return TLG_OK;
}

tlg_status gemm_impl(int64_t M, int64_t N, int64_t K, const void *A, int64_t lda, const void *B,
                     int64_t ldb, const void *bias, void *C, int64_t ldc, tlg_out out,
                     tlg_epilogue epi, const tlg_config *req, void *stream) {
  // ---- host-only checks first: nothing below touches the GPU until they pass
  if (out != TLG_OUT_F32 && out != TLG_OUT_F16) return TLG_ERR_INVALID_ARG;
  if (epi != TLG_EPI_NONE && epi != TLG_EPI_BIAS_RELU) return TLG_ERR_INVALID_ARG;
  if (epi == TLG_EPI_BIAS_RELU && out != TLG_OUT_F16) return TLG_ERR_UNSUPPORTED;
  if ((epi == TLG_EPI_BIAS_RELU) != (bias != nullptr)) return TLG_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0) return TLG_ERR_INVALID_ARG;
  // TMA coordinates and tile indices are 32-bit: keep every extent (plus one tile) below 2^31.
  const int64_t kMax = 0x7fffffff - 256;
  if (M > kMax || N > kMax || K > kMax) return TLG_ERR_UNSUPPORTED;
  if (((M + kBM - 1) / kBM) * ((N + 63) / 64) > kMax) return TLG_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return TLG_OK;
  const int64_t osz = out == TLG_OUT_F32 ? 4 : 2;
  if (C == nullptr || ldc < N) return TLG_ERR_INVALID_ARG;
  if (K > 0 && (A == nullptr || B == nullptr || lda < K || ldb < N)) return TLG_ERR_INVALID_ARG;
  if (!aligned16(C) || (ldc * osz) % 16 != 0) return TLG_ERR_ALIGNMENT;
  if (bias != nullptr && !aligned16(bias)) return TLG_ERR_ALIGNMENT;
  if (K > 0 && (!aligned16(A) || !aligned16(B) || (lda * 2) % 16 != 0 || (ldb * 2) % 16 != 0))
    return TLG_ERR_ALIGNMENT;
  if (ldc > (int64_t(1) << 36) || lda > (int64_t(1) << 36) || ldb > (int64_t(1) << 36))
    return TLG_ERR_UNSUPPORTED;
  uintptr_t c0, c1;
  extent(C, M, N, ldc, osz, &c0, &c1);
  if (K > 0) {
    uintptr_t a0, a1, b0, b1;
    extent(A, M, K, lda, 2, &a0, &a1);
    extent(B, K, N, ldb, 2, &b0, &b1);
    if (overlaps(c0, c1, a0, a1) || overlaps(c0, c1, b0, b1)) return TLG_ERR_INVALID_ARG;
  }
  if (bias != nullptr) {
    const uintptr_t s0 = reinterpret_cast<uintptr_t>(bias);
    if (overlaps(c0, c1, s0, s0 + static_cast<uintptr_t>(2 * N))) return TLG_ERR_INVALID_ARG;
  }

  // ---- device checks
  int dev = 0;
  DeviceInfo info;
  const tlg_status ds = current_device(&dev, &info);
  if (ds != TLG_OK) return ds;
  if (!device_accessible(C, dev)) return TLG_ERR_INVALID_ARG;
  if (K > 0 && (!device_accessible(A, dev) || !device_accessible(B, dev)))
    return TLG_ERR_INVALID_ARG;
  if (bias != nullptr && !device_accessible(bias, dev)) return TLG_ERR_INVALID_ARG;

  tlg_config cfg;
  const tlg_status cs = resolve_config(M, N, info.sm_count, req, &cfg);
  if (cs != TLG_OK) return cs;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool f16 = out == TLG_OUT_F16;
  const bool br = epi == TLG_EPI_BIAS_RELU;
  if (K == 0) {
    if (!f16) return launch_fill<false, false>(C, ldc, bias, int(M), int(N), s);
    if (br) return launch_fill<true, true>(C, ldc, bias, int(M), int(N), s);
    return launch_fill<true, false>(C, ldc, bias, int(M), int(N), s);
  }

  CUtensorMap tmA, tmB;
  if (!encode_2d(&tmA, A, uint64_t(K), uint64_t(M), uint64_t(lda) * 2, kBK, kBM) ||
      !encode_2d(&tmB, B, uint64_t(N), uint64_t(K), uint64_t(ldb) * 2, 64, kBK))
    return TLG_ERR_CUDA;

  GemmParams p;
  p.C = C;
  p.bias = static_cast<const __half *>(bias);
  p.ldc = ldc;
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.raster_group = cfg.raster_group;
  p.limit_ns = kWaitLimitNs;
  if (!f16) return dispatch<false, false>(dev, info.sm_count, cfg, tmA, tmB, p, s);
  if (br) return dispatch<true, true>(dev, info.sm_count, cfg, tmA, tmB, p, s);
  return dispatch<true, false>(dev, info.sm_count, cfg, tmA, tmB, p, s);
}

}  // namespace

extern "C" {

tlg_status tlg_gemm_f16f32(int64_t M, int64_t N, int64_t K, const void *A, int64_t lda,
                           const void *B, int64_t ldb, float *C, int64_t ldc, void *stream) {
  return gemm_impl(M, N, K, A, lda, B, ldb, nullptr, C, ldc, TLG_OUT_F32, TLG_EPI_NONE, nullptr,
                   stream);
}

tlg_status tlg_gemm_f16f16(int64_t M, int64_t N, int64_t K, const void *A, int64_t lda,
                           const void *B, int64_t ldb, void *C, int64_t ldc, void *stream) {
  return gemm_impl(M, N, K, A, lda, B, ldb, nullptr, C, ldc, TLG_OUT_F16, TLG_EPI_NONE, nullptr,
                   stream);
}

tlg_status tlg_gemm_bias_relu_f16(int64_t M, int64_t N, int64_t K, const void *A, int64_t lda,
                                  const void *B, int64_t ldb, const void *bias, void *C,
                                  int64_t ldc, void *stream) {
  if (bias == nullptr && M > 0 && N > 0) return TLG_ERR_INVALID_ARG;
  return gemm_impl(M, N, K, A, lda, B, ldb, bias, C, ldc, TLG_OUT_F16, TLG_EPI_BIAS_RELU, nullptr,
                   stream);
}

tlg_status tlg_gemm_ex(int64_t M, int64_t N, int64_t K, const void *A, int64_t lda, const void *B,
                       int64_t ldb, const void *bias, void *C, int64_t ldc, tlg_out out,
                       tlg_epilogue epilogue, const tlg_config *config, void *stream) {
  return gemm_impl(M, N, K, A, lda, B, ldb, bias, C, ldc, out, epilogue, config, stream);
}

tlg_status tlg_choose_config(int64_t M, int64_t N, int64_t K, tlg_out out, tlg_epilogue epilogue,
                             tlg_config *config) {
  (void)out;
  (void)epilogue;
  if (config == nullptr || M < 0 || N < 0 || K < 0) return TLG_ERR_INVALID_ARG;
  int dev = 0;
  DeviceInfo info;
  const tlg_status ds = current_device(&dev, &info);
  if (ds != TLG_OK) return ds;
  const tlg_config req = *config;
  return resolve_config(M, N, info.sm_count, &req, config);
}

tlg_status tlg_device_error(int clear, uint32_t *code_out) {
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, tlg::g_device_error, sizeof(v)) != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  if (clear && v != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(tlg::g_device_error, &zero, sizeof(zero)) != cudaSuccess) {
      cudaGetLastError();
      return TLG_ERR_CUDA;
    }
  }
  if (code_out) *code_out = v;
  return v ? TLG_ERR_TIMEOUT : TLG_OK;
}

tlg_status tlg_selftest_timeout(uint32_t limit_us, void *stream) {
  if (limit_us < 1 || limit_us > 1000000) return TLG_ERR_INVALID_ARG;
  int dev = 0;
  DeviceInfo info;
  const tlg_status ds = current_device(&dev, &info);
  if (ds != TLG_OK) return ds;
  tlg::selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      uint64_t(limit_us) * 1000ull);
  if (cudaPeekAtLastError() != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  return TLG_OK;
}

const char *tlg_status_string(tlg_status status) {
  switch (status) {
    case TLG_OK: return "TLG_OK";
    case TLG_ERR_INVALID_ARG: return "TLG_ERR_INVALID_ARG: bad size, null or host pointer, ld too small, or overlapping output";
    case TLG_ERR_ALIGNMENT: return "TLG_ERR_ALIGNMENT: pointers must be 16-byte aligned and row strides multiples of 16 bytes";
    case TLG_ERR_UNSUPPORTED: return "TLG_ERR_UNSUPPORTED: device is not sm_100, size too large, or configuration not provided";
    case TLG_ERR_CUDA: return "TLG_ERR_CUDA: a CUDA call failed";
    case TLG_ERR_TIMEOUT: return "TLG_ERR_TIMEOUT: a kernel pipeline wait exceeded its time limit";
  }
  return "unknown tlg_status";
}

int32_t tlg_version(void) { return 100; }

}  // extern "C"
