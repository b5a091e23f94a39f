// Host side of libtlg: argument checks, TMA descriptor encoding, the per-shape
// configuration table, the work schedule and the launches behind the C
// interface in tlg.h; also the small kernels around the GEMM (the K = 0 fill,
// the aligned copies of operands TMA cannot describe, the timeout self-test).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "tlg.h"
#include "tlg_variants.cuh"

namespace {

using namespace tlg;

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per pipeline wait
constexpr size_t kCounterBytes = 4096;            // slice counters at the start of a workspace
constexpr size_t kWorkspaceAlign = 256;

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

// --------------------------------------------------------------------------- kernel variants

struct KernelCfg {
  int cta_group;
  int block_n;  // tile width; 512 = two 256-column MMA halves filling TMEM
  int stages;
  double eff;         // sustained fraction of the MMA peak, relative (ranks tile shapes)
  double exposed_kb;  // k-blocks per tile the main loop waits for the epilogue
  bool plain_loads;   // also built with the plain-load path (operands TMA cannot describe)
  int ks;             // CTAs of a cluster sharing each tile's K range (1: none)
  double reduce_kb;   // k-split: the reduction through distributed shared memory, in k-blocks
};

// Kernel variants the library is built with.  A tile is 128*cta_group rows by
// block_n columns; `stages` is the depth of the operand ring (per-CTA slot:
// 16 KB of A plus 128*block_n/cta_group bytes of B), as deep as fits in
// 227 KB of shared memory next to 32 KB of output staging.
// `eff` is measured: TFLOP/s of each shape on a B200 at M = N = K = 4096 and
// 8192 after dividing out the wave count, relative to the 2 x 256 pair tile.
// The 512-wide tile moves 25 % fewer operand bytes per FLOP, which under the
// 1000 W cap buys a higher clock (sustained at 8192^3: 1297 vs 1170 MHz), but
// its single accumulator leaves part of each epilogue exposed (exposed_kb).
// Its two numbers fit both measured points at equal wave fill: 0.93x the pair
// 256 tile at 4096^3 (64 k-blocks) and 1.05x at 8192^3 (128 k-blocks).
// The last three split each tile's K range over a cluster of 2 or 4 CTAs and
// reduce the partial sums through distributed shared memory (their receive
// buffers leave room for fewer ring stages); they are built for untransposed
// TMA operands.  A CTA of such a cluster streams only its share of the
// k-blocks, so a shape with few tiles keeps more SMs busy, and the wider tile
// reads fewer operand bytes per FLOP than the 128 x 64 tile that would
// otherwise spread it.  Their reduce_kb is the cost of the exchange in k-blocks
// of their tile (B200, one tile per cluster, fp32 C: about 1.3 us for 32 KB per
// CTA each way, 2-5 us for 64-96 KB), fitted to forced runs of every tile on ten
// long-K shapes from 256 x 256 x 4096 to 1536 x 1536 x 4096: the 128 x 256
// clusters lost to the 128 x 128 tile, split or not, on all of them (512 x 768 x
// 4096: 27.0 and 34.4 us against 22.0), so their exchange is charged 24 k-blocks.
// So they pay off only where K is long next to M x N, not at 256^3 or 1024^3.
constexpr KernelCfg kBuilt[] = {{1, 64, 8, 0.35, 0, true, 1, 0},   {1, 128, 6, 0.60, 0, false, 1, 0},
                                {1, 256, 4, 0.90, 0, false, 1, 0},  {2, 128, 8, 0.60, 0, false, 1, 0},
                                {2, 256, 6, 1.00, 0, true, 1, 0},   {2, 512, 4, 1.20, 19, false, 1, 0},
                                {1, 128, 5, 0.60, 0, false, 2, 6.0}, {1, 256, 2, 0.90, 0, false, 2, 24.0},
                                {1, 256, 2, 0.90, 0, false, 4, 24.0}};
constexpr int kNumBuilt = sizeof(kBuilt) / sizeof(kBuilt[0]);
static_assert(kNumBuilt == kNumVariants, "one launcher table entry per built variant");

// ek: the epilogue kind (kEpiNone, kEpiFused, kEpiBiasRelu; the last is built
// for an fp16 C only).
const VariantFns &fns_for(int idx, bool f16, int ek, bool at = false, bool bt = false,
                          bool plain = false) {
  static const LayoutTables *const layouts[4] = {&kLayoutNN, &kLayoutNT, &kLayoutTN, &kLayoutTT};
  const LayoutTables &t = *layouts[(at ? 2 : 0) + (bt ? 1 : 0)];
  int kind = f16 ? kKindF16 : kKindF32;
  if (ek == kEpiFused) kind = f16 ? kKindF16Epi : kKindF32Epi;
  if (ek == kEpiBiasRelu) kind = f16 ? kKindF16BiasRelu : kKindF32Epi;
  return plain ? t.plain[idx][kind] : t.tma[idx][kind];
}

// --------------------------------------------------------------------------- schedule

// How one launch spreads the tiles over its work units.
struct Schedule {
  int64_t tiles = 0;
  int units = 0;  // grid size in work units
  int dp_tiles = 0;
  int split = 1;
  int tail_items = 0;
  size_t workspace = 0;  // bytes needed (0 without a split tail)
  double cost = 0;       // k-blocks on the longest unit's path
};

size_t split_workspace_bytes(int tail_items, int cta_group, int block_n) {
  return kCounterBytes +
         static_cast<size_t>(tail_items) * cta_group * 4 * 32 * block_n * sizeof(float);
}

// Plan for `split` k-slices per tail tile (1 = every tile whole, one after the
// other on `resident` units).  A split keeps ceil(T/U)-1 whole waves and cuts
// the remaining tiles so that the last wave is as short as a slice.
bool plan(int64_t tiles, int resident, int num_kb, int split, int cta_group, int block_n,
          Schedule *s) {
  s->tiles = tiles;
  if (split <= 1) {
    s->units = static_cast<int>(std::min<int64_t>(resident, tiles));
    s->dp_tiles = static_cast<int>(tiles);
    s->split = 1;
    s->tail_items = 0;
    s->workspace = 0;
    // A partial last wave costs less than a full one: under the power cap
    // the SMs it leaves idle let the busy ones clock higher.  Measured at
    // 8192^3 on a device holding fewer than 74 pairs, where both tiles end in
    // a nearly empty wave: the wide tile ran 5 % faster than the pair 256
    // tile, which whole-wave counting ranks the other way.
    const int64_t full = tiles / s->units;
    const double frac = static_cast<double>(tiles - full * s->units) / s->units;
    s->cost = (static_cast<double>(full) + (frac > 0 ? 0.35 + 0.65 * frac : 0.0)) * num_kb;
    return true;
  }
  if (split > num_kb) return false;
  const int64_t full = tiles / resident;
  const int64_t rem = full > 0 ? tiles % resident : tiles;
  if (rem == 0 || rem * split > resident) return false;
  s->units = full > 0 ? resident : static_cast<int>(rem * split);
  s->dp_tiles = static_cast<int>(full * resident);
  s->split = split;
  s->tail_items = static_cast<int>(rem * split);
  s->workspace = split_workspace_bytes(s->tail_items, cta_group, block_n);
  // A whole tile follows the slice (see work_item), so its partial-sum traffic
  // hides behind that tile's main loop unless there is none, and then it costs
  // about 2 + split k-blocks.  The
  // hiding fails for short tiles: with 16 k-blocks a split tail lost 4-11 %
  // (8192 x 2048 x 1024, 12288 x 4096 x 1024, pair 256 tile) while at 64 it gains
  // 4.5 %.  So each slice's fp32 partial, counted in k-blocks of operand bytes
  // (the CTA's partial over its stage), is charged 0.3 of it, scaled by
  // (16 / k-blocks)^2 up to 1.
  const double slice = static_cast<double>((num_kb + split - 1) / split);
  double fixup = 2.0 + split;
  if (full > 0) {
    const double partial_kb = (128.0 * block_n * 4.0) / (128.0 * kBK * 2.0 + kBK * (block_n / cta_group) * 2.0);
    const double r = std::min(1.0, 16.0 / num_kb);
    fixup = 0.5 + 0.3 * split * partial_kb * r * r;
  }
  s->cost = static_cast<double>(full) * num_kb + slice + fixup;
  return true;
}

struct Resolved {
  tlg_config cfg;
  int idx;
  Schedule sched;
};

// Choose (or check) the kernel variant and the schedule.  Shapes are ranked by
// k-blocks on the critical path times the per-k-block time of the tile (tile
// area over its sustained fraction of the MMA peak, per SM).
// at / bt select the operand-layout instantiation whose launch attributes are
// prepared (the schedule itself does not depend on the layout).
tlg_status resolve(int dev, int sms, int64_t M, int64_t N, int64_t K, bool f16, int ek,
                   bool at, bool bt, bool plain, const tlg_config *req, size_t ws_bytes,
                   Resolved *out) {
  const int num_kb = static_cast<int>((K + kBK - 1) / kBK);
  tlg_config r = {};
  if (req != nullptr) r = *req;
  if (r.raster_group < 0 || r.raster_group > 64 || r.max_ctas < 0 || r.split_k < 0 ||
      r.split_k > 16 || r.stages < 0 || r.block_n < 0 || r.cta_group < 0 ||
      (r.overlap_prev != 0 && r.overlap_prev != 1) || r.k_split < 0 || r.k_split > 16)
    return TLG_ERR_UNSUPPORTED;
  double best_cost = 0;
  bool found = false;
  bool shape_exists = false;
  for (int i = 0; i < kNumBuilt; ++i) {
    const KernelCfg &k = kBuilt[i];
    if (r.cta_group != 0 && r.cta_group != k.cta_group) continue;
    if (r.block_n != 0 && r.block_n != k.block_n) continue;
    if (r.stages != 0 && r.stages != k.stages) continue;
    if (plain && !k.plain_loads) continue;
    if (r.k_split != 0 && r.k_split != k.ks) continue;
    // a k-split: untransposed TMA operands, at least one k-block per CTA, no split tail
    if (k.ks > 1 && (at || bt || plain || num_kb < k.ks || r.split_k >= 2)) continue;
    shape_exists = true;
    int resident = 0;
    const tlg_status us = fns_for(i, f16, ek, at, bt, plain).units(dev, sms, &resident);
    if (us != TLG_OK) return us;
    if (r.max_ctas > 0) resident = std::max(1, std::min(resident, r.max_ctas / (k.cta_group * k.ks)));
    const int64_t tile_m = 128 * k.cta_group;
    const int64_t tiles = ((M + tile_m - 1) / tile_m) * ((N + k.block_n - 1) / k.block_n);
    // Automatic choice (split_k == 0): every tile whole, or, when the caller's
    // workspace can hold it, a split tail of 2..4 k-slices if the model ranks
    // it faster.  A split is only chosen behind at least one whole wave, whose
    // tiles hide the partial sums' traffic: measured on a B200, split 2 at
    // 4096^3 (3.46 waves) ran 4.5 % faster, while a split with no whole wave
    // before it lost at 1024^3, where the fix-up is exposed.
    const int split_lo = r.split_k == 0 ? 1 : r.split_k;
    const int split_hi = r.split_k == 0 && k.ks == 1 ? (ws_bytes > 0 ? 4 : 1) : split_lo;
    // k-blocks one CTA of the tile's group sums (its slice, with a k-split)
    const int kb_unit = (num_kb + k.ks - 1) / k.ks;
    for (int split = split_lo; split <= split_hi; ++split) {
      Schedule sch;
      if (!plan(tiles, resident, kb_unit, split, k.cta_group, k.block_n, &sch)) continue;
      if (r.split_k == 0 && split > 1 && (sch.dp_tiles == 0 || sch.workspace > ws_bytes)) continue;
      // the busiest unit's tile count, each tile paying the exposed part of its epilogue
      const double per_unit_tiles = static_cast<double>((tiles + sch.units - 1) / sch.units);
      const double cost = (sch.cost + per_unit_tiles * (k.exposed_kb + k.reduce_kb)) *
                          static_cast<double>(tile_m * k.block_n) / (k.cta_group * k.eff);
      if (!found || cost < best_cost * 0.999) {
        found = true;
        best_cost = cost;
        out->idx = i;
        out->sched = sch;
        out->cfg.cta_group = k.cta_group;
        out->cfg.block_n = k.block_n;
        out->cfg.stages = k.stages;
        out->cfg.k_split = k.ks;
      }
    }
  }
  if (!shape_exists || !found) return TLG_ERR_UNSUPPORTED;
  // Tile rows walked together: 8, or 16 for the 256 x 512 tile, whose wave then covers
  // a squarer block (ncu at 8192^3: 870 MB of DRAM reads against 912 MB with 8).
  out->cfg.raster_group = r.raster_group != 0 ? r.raster_group : (out->cfg.block_n > 256 ? 16 : 8);
  out->cfg.max_ctas = out->sched.units * out->cfg.cta_group * out->cfg.k_split;  // CTAs launched
  out->cfg.split_k = out->sched.split;
  out->cfg.overlap_prev = r.overlap_prev;
  return TLG_OK;
}

// --------------------------------------------------------------------------- launch

bool encode_2d(CUtensorMap *tm, CUtensorMapDataType dtype, const void *base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = g_encode(tm, dtype, 2, const_cast<void *>(base), dims, strides, box, estride,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static_assert(kActNone == TLG_ACT_NONE && kActRelu == TLG_ACT_RELU && kActGelu == TLG_ACT_GELU &&
                  kActSilu == TLG_ACT_SILU && kActGeluTanh == TLG_ACT_GELU_TANH,
              "the kernels' activation codes are tlg_activation's values");

// The epilogue of one call, from either interface: bias, activation and
// residual, and whether the fused-epilogue kernels run at all.
struct Epi {
  bool fused = false;
  const void *bias = nullptr;
  int act = kActNone;
  const void *R = nullptr;
  int64_t ldr = 0;
};

// tlg_gemm_ex's selector: TLG_EPI_BIAS_RELU is the bias, then the ReLU, fp16 C only.
tlg_status legacy_epilogue(tlg_out out, tlg_epilogue epi, const void *bias, Epi *e) {
  if (out != TLG_OUT_F32 && out != TLG_OUT_F16) return TLG_ERR_INVALID_ARG;
  if (epi != TLG_EPI_NONE && epi != TLG_EPI_BIAS_RELU) return TLG_ERR_INVALID_ARG;
  if (epi == TLG_EPI_BIAS_RELU && out != TLG_OUT_F16) return TLG_ERR_UNSUPPORTED;
  if ((epi == TLG_EPI_BIAS_RELU) != (bias != nullptr)) return TLG_ERR_INVALID_ARG;
  *e = Epi{};
  if (epi == TLG_EPI_BIAS_RELU) {
    e->fused = true;
    e->bias = bias;
    e->act = kActRelu;
  }
  return TLG_OK;
}

// tlg_gemm_fused's descriptor.  An empty one (or NULL) runs the plain kernels.
tlg_status fused_epilogue(tlg_out out, const tlg_fused_epilogue *d, Epi *e) {
  if (out != TLG_OUT_F32 && out != TLG_OUT_F16) return TLG_ERR_INVALID_ARG;
  *e = Epi{};
  if (d == nullptr) return TLG_OK;
  if (d->activation != TLG_ACT_NONE && d->activation != TLG_ACT_RELU &&
      d->activation != TLG_ACT_GELU && d->activation != TLG_ACT_SILU &&
      d->activation != TLG_ACT_GELU_TANH)
    return TLG_ERR_INVALID_ARG;
  e->bias = d->bias;
  e->act = d->activation;
  e->R = d->residual;
  e->ldr = d->ldr;
  e->fused = e->bias != nullptr || e->act != kActNone || e->R != nullptr;
  return TLG_OK;
}

template <bool OUT_F16, bool EPI>
tlg_status launch_fill(void *C, int64_t ldc, const Epi &e, int M, int N, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(M) * N;
  const int threads = 256;
  const int blocks = static_cast<int>(total / threads + 1 > 4096 ? 4096 : total / threads + 1);
  fill_empty_k_kernel<OUT_F16, EPI><<<blocks, threads, 0, s>>>(
      C, ldc, static_cast<const __half *>(e.bias), e.act, e.R, e.ldr, M, N);
  if (cudaPeekAtLastError() != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  return TLG_OK;
}

// ---------------------------------------------------------------- aligned copies
//
// Operands the TMA unit cannot describe (a base or row stride off 16 bytes) are
// copied, when the call's workspace has room, into an aligned layout in the
// workspace; the GEMM then runs its TMA path on the copies.  A C that TMA cannot
// store is produced in the workspace and copied out.  Both copies are
// memory-bound and move each byte once.

constexpr size_t kCopyAlign = 256;

size_t round_up_sz(size_t x, size_t a) { return (x + a - 1) / a * a; }

// An aligned copy of a rows x cols matrix of esz-byte elements: rows of
// round_up(cols * esz, 16) bytes.
size_t aligned_copy_bytes(int64_t rows, int64_t cols, int64_t esz) {
  return round_up_sz(static_cast<size_t>(rows) * round_up_sz(static_cast<size_t>(cols * esz), 16),
                     kCopyAlign);
}

// Realigning copies.  One side of every copy is the workspace layout (16-byte
// base and row stride); the other is the caller's matrix at any element-aligned
// address.  A warp moves one 512-byte piece of a row per step: 32 lanes, one
// aligned 16-byte block each, on both sides.  On the caller's side the blocks
// are the aligned blocks that hold the row's bytes; each lane rebuilds its
// output block from its own block and a neighbour's (a shuffle) with funnel
// shifts.  Only the partial blocks at the two ends of a caller's row are
// stored element by element.  Every aligned block loaded from the caller's
// matrix holds at least one byte of it, so it lies inside the allocation.
// Measured on a B200 against an element-wise copy (a call of 8192 x 64 x 8192
// whose 128 MB A is copied in: 105 vs 132 us; of 8192 x 8192 x 64 whose fp16 C
// is copied out: 111 vs 132 us).
constexpr int kCopyThreads = 256;
constexpr int kCopyWarps = kCopyThreads / 32;
constexpr int kCopyUnroll = 4;  // pieces per warp in flight: 64 bytes per lane
constexpr int kCopyBlocksPerSm = 4;  // 32 warps: 64 KB in flight per SM

// Bytes [Q*4 + sh/8, +16) of the 32-byte concatenation lo:hi, Q fixed.
template <int Q>
__device__ __forceinline__ uint4 bytes_from_q(const uint4 &lo, const uint4 &hi, uint32_t sh) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  return make_uint4(__funnelshift_r(w[Q], w[Q + 1], sh), __funnelshift_r(w[Q + 1], w[Q + 2], sh),
                    __funnelshift_r(w[Q + 2], w[Q + 3], sh), __funnelshift_r(w[Q + 3], w[Q + 4], sh));
}

// Bytes [s, s + 16) of lo:hi, 0 <= s < 16 (the same s across the warp).
__device__ __forceinline__ uint4 bytes_from(const uint4 &lo, const uint4 &hi, int s) {
  const uint32_t sh = 8u * static_cast<uint32_t>(s & 3);
  switch (s >> 2) {
    case 0: return bytes_from_q<0>(lo, hi, sh);
    case 1: return bytes_from_q<1>(lo, hi, sh);
    case 2: return bytes_from_q<2>(lo, hi, sh);
    default: return bytes_from_q<3>(lo, hi, sh);
  }
}

__device__ __forceinline__ uint4 shfl_v4(const uint4 &v, int delta, bool down) {
  uint4 r;
  if (down) {
    r.x = __shfl_down_sync(0xffffffffu, v.x, delta);
    r.y = __shfl_down_sync(0xffffffffu, v.y, delta);
    r.z = __shfl_down_sync(0xffffffffu, v.z, delta);
    r.w = __shfl_down_sync(0xffffffffu, v.w, delta);
  } else {
    r.x = __shfl_up_sync(0xffffffffu, v.x, delta);
    r.y = __shfl_up_sync(0xffffffffu, v.y, delta);
    r.z = __shfl_up_sync(0xffffffffu, v.z, delta);
    r.w = __shfl_up_sync(0xffffffffu, v.w, delta);
  }
  return r;
}

// The (row, piece) items of a copy, one warp each, warps striding by the
// grid's warp count; advanced without a division per item.
struct PieceIter {
  int64_t r, g, pieces, dq, dr;
  __device__ PieceIter(int64_t item, int64_t stride, int64_t pieces_per_row) : pieces(pieces_per_row) {
    r = item / pieces;
    g = item - r * pieces;
    dq = stride / pieces;
    dr = stride - dq * pieces;
  }
  __device__ void advance() {
    g += dr;
    r += dq;
    if (g >= pieces) {
      g -= pieces;
      ++r;
    }
  }
};

// One matrix of a copy: `rows` rows of `row_bytes` bytes, strides in bytes.
struct CopyJob {
  const char *src;
  int64_t src_ld;
  char *dst;
  int64_t dst_ld;
  int64_t rows;
  int64_t row_bytes;
};

// Into the workspace: dst (16-byte base and row stride) <- src (any address).
// Row r's output block b is src bytes [16b, 16b + 16) of the row, which sit in
// the aligned source blocks b and b + 1 counted from the row's first byte
// rounded down to 16.  The last output block of a row may run past row_bytes
// into the row's padding (the layout rounds rows up to 16 bytes).
// One launch copies A and B: blocks [0, j1_first) take j0, the rest j1.  The
// GEMM that reads the copies may be launched as a programmatic dependent: it
// is let in at once and waits for this grid before it touches global memory.
__global__ void __launch_bounds__(kCopyThreads, kCopyBlocksPerSm)
    copy_in_kernel(CopyJob j0, CopyJob j1, unsigned j1_first) {
  grid_launch_dependents();
  const bool second = blockIdx.x >= j1_first;
  const char *const src = second ? j1.src : j0.src;
  char *const dst = second ? j1.dst : j0.dst;
  const int64_t src_ld_bytes = second ? j1.src_ld : j0.src_ld;
  const int64_t dst_ld_bytes = second ? j1.dst_ld : j0.dst_ld;
  const int64_t rows = second ? j1.rows : j0.rows;
  const int64_t row_bytes = second ? j1.row_bytes : j0.row_bytes;
  const unsigned block = second ? blockIdx.x - j1_first : blockIdx.x;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(second ? gridDim.x - j1_first : j1_first) * kCopyWarps;
  PieceIter it(static_cast<int64_t>(block) * kCopyWarps + (threadIdx.x >> 5), nwarps,
               (row_bytes + 511) / 512);
  while (it.r < rows) {
    uint4 lo[kCopyUnroll], next[kCopyUnroll];
    int ru[kCopyUnroll], gu[kCopyUnroll];  // rows and pieces per row are below 2^31
    unsigned live = 0;
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      ru[u] = static_cast<int>(it.r);
      gu[u] = static_cast<int>(it.g);
      lo[u] = make_uint4(0u, 0u, 0u, 0u);
      next[u] = make_uint4(0u, 0u, 0u, 0u);
      if (it.r < rows) {
        live |= 1u << u;
        const uintptr_t sb = reinterpret_cast<uintptr_t>(src) + static_cast<uintptr_t>(it.r * src_ld_bytes);
        const uintptr_t se = sb + static_cast<uintptr_t>(row_bytes);
        const uintptr_t a = (sb & ~uintptr_t(15)) + static_cast<uintptr_t>(it.g * 512 + 16 * lane);
        if (a < se) lo[u] = __ldg(reinterpret_cast<const uint4 *>(a));
        if (lane == 31 && (sb & 15) != 0 && a + 16 < se)
          next[u] = __ldg(reinterpret_cast<const uint4 *>(a + 16));
      }
      it.advance();
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      if (!(live >> u & 1u)) break;  // the same for the whole warp
      const uintptr_t sb = reinterpret_cast<uintptr_t>(src) + static_cast<uintptr_t>(ru[u] * src_ld_bytes);
      uint4 hi = shfl_v4(lo[u], 1, true);
      if (lane == 31) hi = next[u];
      const int64_t b = static_cast<int64_t>(gu[u]) * 32 + lane;
      if (b * 16 < row_bytes)
        reinterpret_cast<uint4 *>(dst + ru[u] * dst_ld_bytes)[b] = bytes_from(lo[u], hi, static_cast<int>(sb & 15));
    }
  }
}

// Out of the workspace: dst (any ESZ-aligned address) <- src (16-byte base
// and row stride).  Row r's destination bytes sit in the aligned blocks from
// its first byte rounded down to 16; block b there holds row bytes
// [16b - t, 16b - t + 16), t the row's offset in its first block, which are
// bytes [16 - t, 32 - t) of source blocks b - 1 and b.  Blocks wholly inside
// the row are stored whole; the row's first and last blocks element by element.
// Launched as a programmatic dependent of the GEMM that writes src: it waits
// for that grid before touching global memory.
template <int ESZ>
__global__ void __launch_bounds__(kCopyThreads, kCopyBlocksPerSm)
    copy_out_kernel(CopyJob j) {
  grid_dependency_wait();
  const char *const src = j.src;
  char *const dst = j.dst;
  const int64_t src_ld_bytes = j.src_ld, dst_ld_bytes = j.dst_ld;
  const int64_t rows = j.rows, row_bytes = j.row_bytes;
  const int lane = threadIdx.x & 31;
  const int64_t src_blocks = (row_bytes + 15) / 16;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kCopyWarps;
  // dst blocks of a row: at most ceil((t + row_bytes) / 16) with t <= 14
  PieceIter it(static_cast<int64_t>(blockIdx.x) * kCopyWarps + (threadIdx.x >> 5), nwarps,
               ((row_bytes + 29) / 16 + 31) / 32);
  while (it.r < rows) {
    uint4 cur[kCopyUnroll], prev0[kCopyUnroll];
    int ru[kCopyUnroll], gu[kCopyUnroll];  // rows and pieces per row are below 2^31
    unsigned live = 0;
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      ru[u] = static_cast<int>(it.r);
      gu[u] = static_cast<int>(it.g);
      cur[u] = make_uint4(0u, 0u, 0u, 0u);
      prev0[u] = make_uint4(0u, 0u, 0u, 0u);
      if (it.r < rows) {
        live |= 1u << u;
        const uint4 *srow = reinterpret_cast<const uint4 *>(src + it.r * src_ld_bytes);
        const uintptr_t db = reinterpret_cast<uintptr_t>(dst) + static_cast<uintptr_t>(it.r * dst_ld_bytes);
        const int64_t b = it.g * 32 + lane;
        if (b < src_blocks) cur[u] = __ldg(srow + b);
        if (lane == 0 && (db & 15) != 0 && b >= 1 && b - 1 < src_blocks) prev0[u] = __ldg(srow + b - 1);
      }
      it.advance();
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      if (!(live >> u & 1u)) break;  // the same for the whole warp
      const uintptr_t db = reinterpret_cast<uintptr_t>(dst) + static_cast<uintptr_t>(ru[u] * dst_ld_bytes);
      const uintptr_t de = db + static_cast<uintptr_t>(row_bytes);
      const int t = static_cast<int>(db & 15);
      uint4 prev = shfl_v4(cur[u], 1, false);
      if (lane == 0) prev = prev0[u];
      const uint4 out = t == 0 ? cur[u] : bytes_from(prev, cur[u], 16 - t);
      const int64_t b = static_cast<int64_t>(gu[u]) * 32 + lane;
      const uintptr_t a = (db & ~uintptr_t(15)) + static_cast<uintptr_t>(16 * b);
      if (a >= db && a + 16 <= de) {
        *reinterpret_cast<uint4 *>(a) = out;
      } else if (a < de && a + 16 > db) {
        const uint32_t w[4] = {out.x, out.y, out.z, out.w};
#pragma unroll
        for (int k = 0; k < 16 / ESZ; ++k) {
          const uintptr_t e = a + static_cast<uintptr_t>(k * ESZ);
          if (e < db || e >= de) continue;
          if (ESZ == 4)
            *reinterpret_cast<uint32_t *>(e) = w[k];
          else
            *reinterpret_cast<uint16_t *>(e) = static_cast<uint16_t>(w[k / 2] >> (16 * (k % 2)));
        }
      }
    }
  }
}

// Aligned row stride, in elements, of a copy of a matrix with `cols` columns.
int64_t aligned_ld(int64_t cols, int64_t esz) {
  return static_cast<int64_t>(round_up_sz(static_cast<size_t>(cols * esz), 16)) / esz;
}

bool aligned_rows(const void *q, int64_t ld_bytes) { return aligned16(q) && ld_bytes % 16 == 0; }

// Blocks for `items` warp-sized pieces, at most `cap`.
int64_t copy_blocks(int64_t items, int64_t cap) {
  return std::max<int64_t>(1, std::min<int64_t>(cap, (items + kCopyWarps - 1) / kCopyWarps));
}

// Copies of A and/or B into the workspace (dst rows 16-byte aligned), one
// launch; b may be null.  The blocks (one wave at most) are shared in
// proportion to the two matrices' sizes.
tlg_status launch_copy_in(const CopyJob &a, const CopyJob *b, int sms, cudaStream_t s) {
  // the workspace side must be 16-byte aligned (never otherwise: it is planned so)
  if (!aligned_rows(a.dst, a.dst_ld) || (b != nullptr && !aligned_rows(b->dst, b->dst_ld)))
    return TLG_ERR_INVALID_ARG;
  const int64_t cap = static_cast<int64_t>(std::max(sms, 1)) * kCopyBlocksPerSm;
  const int64_t ia = a.rows * ((a.row_bytes + 511) / 512);
  const int64_t ib = b != nullptr ? b->rows * ((b->row_bytes + 511) / 512) : 0;
  int64_t na = copy_blocks(ia, cap), nb = b != nullptr ? copy_blocks(ib, cap) : 0;
  if (b != nullptr && na + nb > cap) {
    na = std::max<int64_t>(1, std::min<int64_t>(na, (cap * ia) / (ia + ib)));
    nb = std::max<int64_t>(1, std::min<int64_t>(nb, cap - na));
  }
  copy_in_kernel<<<static_cast<unsigned>(na + nb), kCopyThreads, 0, s>>>(a, b != nullptr ? *b : a,
                                                                        static_cast<unsigned>(na));
  if (cudaPeekAtLastError() != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  return TLG_OK;
}

// The copy of C out of the workspace (src rows 16-byte aligned), launched as
// a programmatic dependent of the GEMM before it.
tlg_status launch_copy_out(const CopyJob &c, int64_t esz, int sms, cudaStream_t s) {
  if (!aligned_rows(c.src, c.src_ld)) return TLG_ERR_INVALID_ARG;  // the workspace side, as planned
  const int64_t cap = static_cast<int64_t>(std::max(sms, 1)) * kCopyBlocksPerSm;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(copy_blocks(c.rows * (((c.row_bytes + 29) / 16 + 31) / 32), cap)));
  cfg.blockDim = dim3(kCopyThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = esz == 4 ? cudaLaunchKernelEx(&cfg, copy_out_kernel<4>, c)
                                 : cudaLaunchKernelEx(&cfg, copy_out_kernel<2>, c);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  return TLG_OK;
}

// Which of the call's matrices TMA cannot describe, and the workspace their
// aligned copies take.
struct CopyPlan {
  bool a = false, b = false, c = false;
  size_t a_bytes = 0, b_bytes = 0, c_bytes = 0;
  size_t ab_bytes() const { return a_bytes + b_bytes; }
};

CopyPlan copy_plan(int64_t M, int64_t N, int64_t K, bool at, const void *A, int64_t lda, bool bt,
                   const void *B, int64_t ldb, const void *C, int64_t ldc, int64_t osz) {
  CopyPlan cp;
  auto tma_ok = [](const void *q, int64_t ld, int64_t esz) {
    return (reinterpret_cast<uintptr_t>(q) & 15u) == 0 && (ld * esz) % 16 == 0;
  };
  if (K > 0) {
    cp.a = !tma_ok(A, lda, 2);
    cp.b = !tma_ok(B, ldb, 2);
    if (cp.a) cp.a_bytes = aligned_copy_bytes(at ? K : M, at ? M : K, 2);
    if (cp.b) cp.b_bytes = aligned_copy_bytes(bt ? N : K, bt ? K : N, 2);
  }
  cp.c = !tma_ok(C, ldc, osz);
  if (cp.c) cp.c_bytes = aligned_copy_bytes(M, N, osz);
  return cp;
}

// Host-only argument checks shared by every entry point; nothing here touches the GPU.
// at / bt: A stored K x M (lda >= M), B stored N x K (ldb >= K), the product
// using their transposes.
tlg_status check_args(int64_t M, int64_t N, int64_t K, bool at, const void *A, int64_t lda,
                      bool bt, const void *B, int64_t ldb, const Epi &e, const void *C,
                      int64_t ldc, tlg_out out) {
  if (out != TLG_OUT_F32 && out != TLG_OUT_F16) return TLG_ERR_INVALID_ARG;
  const void *bias = e.bias;
  if (M < 0 || N < 0 || K < 0) return TLG_ERR_INVALID_ARG;
  // TMA coordinates and tile indices are 32-bit: keep every extent (plus one tile) below 2^31.
  const int64_t kMax = 0x7fffffff - 256;
  if (M > kMax || N > kMax || K > kMax) return TLG_ERR_UNSUPPORTED;
  if (((M + kBM - 1) / kBM) * ((N + 63) / 64) > kMax) return TLG_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return TLG_OK;
  const int64_t osz = out == TLG_OUT_F32 ? 4 : 2;
  if (C == nullptr || ldc < N) return TLG_ERR_INVALID_ARG;
  if (K > 0 && (A == nullptr || B == nullptr || lda < (at ? M : K) || ldb < (bt ? K : N)))
    return TLG_ERR_INVALID_ARG;
  // Only element alignment is required; strides and bases TMA cannot describe
  // take the plain-load / plain-store paths.
  auto misaligned = [](const void *q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) % a) != 0; };
  if (misaligned(C, static_cast<uintptr_t>(osz))) return TLG_ERR_ALIGNMENT;
  if (bias != nullptr && misaligned(bias, 2)) return TLG_ERR_ALIGNMENT;
  if (K > 0 && (misaligned(A, 2) || misaligned(B, 2))) return TLG_ERR_ALIGNMENT;
  if (ldc > (int64_t(1) << 36) || lda > (int64_t(1) << 36) || ldb > (int64_t(1) << 36))
    return TLG_ERR_UNSUPPORTED;
  // Every matrix must span less than 2^60 bytes, so the extent arithmetic below
  // cannot overflow (rows < 2^31 and ld <= 2^36 alone would allow 2^67).
  auto spans = [](int64_t rows, int64_t ld, int64_t esz) {
    return rows <= 1 || (rows - 1) <= ((int64_t(1) << 60) / esz) / ld;
  };
  if (!spans(M, ldc, osz) || (K > 0 && (!spans(at ? K : M, lda, 2) || !spans(bt ? N : K, ldb, 2))))
    return TLG_ERR_UNSUPPORTED;
  uintptr_t c0, c1;
  extent(C, M, N, ldc, osz, &c0, &c1);
  if (K > 0) {
    uintptr_t a0, a1, b0, b1;
    if (at)
      extent(A, K, M, lda, 2, &a0, &a1);
    else
      extent(A, M, K, lda, 2, &a0, &a1);
    if (bt)
      extent(B, N, K, ldb, 2, &b0, &b1);
    else
      extent(B, K, N, ldb, 2, &b0, &b1);
    if (overlaps(c0, c1, a0, a1) || overlaps(c0, c1, b0, b1)) return TLG_ERR_INVALID_ARG;
  }
  if (bias != nullptr) {
    const uintptr_t s0 = reinterpret_cast<uintptr_t>(bias);
    if (overlaps(c0, c1, s0, s0 + static_cast<uintptr_t>(2 * N))) return TLG_ERR_INVALID_ARG;
  }
  if (e.R != nullptr) {
    // The residual has C's type.  It may be C itself (same base and row
    // stride: each element is read before the one thread that owns it writes
    // it); any other overlap with C would race.
    if (misaligned(e.R, static_cast<uintptr_t>(osz))) return TLG_ERR_ALIGNMENT;
    if (e.ldr < N) return TLG_ERR_INVALID_ARG;
    if (e.ldr > (int64_t(1) << 36) || !spans(M, e.ldr, osz)) return TLG_ERR_UNSUPPORTED;
    if (!(e.R == C && e.ldr == ldc)) {
      uintptr_t r0, r1;
      extent(e.R, M, N, e.ldr, osz, &r0, &r1);
      if (overlaps(c0, c1, r0, r1)) return TLG_ERR_INVALID_ARG;
    }
  }
  return TLG_OK;
}

// ws/ws_bytes: scratch for the split-K tail (nullptr/0: none).  static_ws: ws is the
// library's own static scratch (tlg_gemm_ex_noalloc), whose split-K counters hold whatever
// the last call left: they are cleared on the stream just before this call's first launch,
// and a schedule that needs more scratch than it has is TLG_ERR_UNSUPPORTED.
tlg_status gemm_impl(int64_t M, int64_t N, int64_t K, bool at, const void *A, int64_t lda,
                     bool bt, const void *B, int64_t ldb, const Epi &e, void *C, int64_t ldc,
                     tlg_out out, const tlg_config *req, void *ws, size_t ws_bytes, void *stream,
                     bool static_ws = false) {
  const tlg_status hs = check_args(M, N, K, at, A, lda, bt, B, ldb, e, C, ldc, out);
  const void *bias = e.bias;
  if (hs != TLG_OK || M == 0 || N == 0) return hs;
  const int64_t osz = out == TLG_OUT_F32 ? 4 : 2;
  if (ws == nullptr) ws_bytes = 0;
  if (ws != nullptr) {
    if ((reinterpret_cast<uintptr_t>(ws) % kWorkspaceAlign) != 0) return TLG_ERR_ALIGNMENT;
    uintptr_t c0, c1;
    extent(C, M, N, ldc, osz, &c0, &c1);
    const uintptr_t w0 = reinterpret_cast<uintptr_t>(ws);
    if (overlaps(c0, c1, w0, w0 + ws_bytes)) return TLG_ERR_INVALID_ARG;
    if (K > 0) {
      uintptr_t a0, a1, b0, b1;
      extent(A, at ? K : M, at ? M : K, lda, 2, &a0, &a1);
      extent(B, bt ? N : K, bt ? K : N, ldb, 2, &b0, &b1);
      if (overlaps(w0, w0 + ws_bytes, a0, a1) || overlaps(w0, w0 + ws_bytes, b0, b1))
        return TLG_ERR_INVALID_ARG;
    }
    if (e.R != nullptr) {
      uintptr_t r0, r1;
      extent(e.R, M, N, e.ldr, osz, &r0, &r1);
      if (overlaps(w0, w0 + ws_bytes, r0, r1)) return TLG_ERR_INVALID_ARG;
    }
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
  if (e.R != nullptr && !device_accessible(e.R, dev)) return TLG_ERR_INVALID_ARG;
  if (ws != nullptr && !device_accessible(ws, dev)) return TLG_ERR_INVALID_ARG;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool f16 = out == TLG_OUT_F16;
  const bool fused = e.fused;
  if (K == 0) {
    if (f16)
      return fused ? launch_fill<true, true>(C, ldc, e, int(M), int(N), s)
                   : launch_fill<true, false>(C, ldc, e, int(M), int(N), s);
    return fused ? launch_fill<false, true>(C, ldc, e, int(M), int(N), s)
                 : launch_fill<false, false>(C, ldc, e, int(M), int(N), s);
  }
  // Bias + ReLU alone (an fp16 C, no residual) runs the kernels built for it.
  const int ek = !fused ? kEpiNone
                        : (f16 && e.bias != nullptr && e.act == kActRelu && e.R == nullptr)
                              ? kEpiBiasRelu
                              : kEpiFused;

  // TMA needs 16-byte aligned bases and row strides.  Operands that break
  // that rule are copied into an aligned layout in the workspace when it has
  // room (after the split-K scratch, never over its counters); otherwise A and
  // B go through the plain-load warps and C through plain stores.
  const CopyPlan cp = copy_plan(M, N, K, at, A, lda, bt, B, ldb, C, ldc, osz);
  bool copy_ab = false, copy_c = false;
  Resolved rv;
  tlg_status rs = TLG_ERR_UNSUPPORTED;
  size_t copy_base = 0;
  if ((cp.a || cp.b) && ws_bytes >= kCounterBytes + cp.ab_bytes()) {
    // The TMA path with copies of A and/or B.  The split scratch (counters
    // included) starts the workspace and the copies follow it, 256-byte
    // aligned, so the scratch may take what the copies leave, rounded down.
    const size_t split_room = (ws_bytes - cp.ab_bytes()) / kCopyAlign * kCopyAlign;
    rs = resolve(dev, info.sm_count, M, N, K, f16, ek, at, bt, false, req, split_room, &rv);
    if (rs == TLG_OK) {
      copy_ab = true;
      copy_base = round_up_sz(std::max<size_t>(rv.sched.workspace, kCounterBytes), kCopyAlign);
      if (copy_base + cp.ab_bytes() > ws_bytes) copy_ab = false;
    }
  }
  const bool plain = (cp.a || cp.b) && !copy_ab;
  if (!copy_ab) {
    rs = resolve(dev, info.sm_count, M, N, K, f16, ek, at, bt, plain, req, ws_bytes, &rv);
    copy_base = round_up_sz(std::max<size_t>(rv.sched.workspace, kCounterBytes), kCopyAlign);
  }
  if (rs != TLG_OK) return rs;
  if (rv.sched.workspace > ws_bytes)  // a forced split needs scratch
    return static_ws ? TLG_ERR_UNSUPPORTED : TLG_ERR_INVALID_ARG;
  const size_t c_off = copy_base + (copy_ab ? cp.ab_bytes() : 0);
  if (cp.c && ws != nullptr && c_off + cp.c_bytes <= ws_bytes) copy_c = true;
  const bool c_plain = cp.c && !copy_c;
  char *wsb = static_cast<char *>(ws);
  const void *A_use = A, *B_use = B;
  int64_t lda_use = lda, ldb_use = ldb;
  if (static_ws && rv.sched.split > 1 &&
      cudaMemsetAsync(ws, 0, kCounterBytes, s) != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  if (copy_ab) {
    size_t off = copy_base;
    CopyJob jobs[2];
    int n = 0;
    if (cp.a) {
      const int64_t rows = at ? K : M, cols = at ? M : K;
      lda_use = aligned_ld(cols, 2);
      jobs[n++] = {static_cast<const char *>(A), lda * 2, wsb + off, lda_use * 2, rows, cols * 2};
      A_use = wsb + off;
      off += cp.a_bytes;
    }
    if (cp.b) {
      const int64_t rows = bt ? N : K, cols = bt ? K : N;
      ldb_use = aligned_ld(cols, 2);
      jobs[n++] = {static_cast<const char *>(B), ldb * 2, wsb + off, ldb_use * 2, rows, cols * 2};
      B_use = wsb + off;
    }
    const tlg_status cs = launch_copy_in(jobs[0], n > 1 ? &jobs[1] : nullptr, info.sm_count, s);
    if (cs != TLG_OK) return cs;
  }
  void *C_use = copy_c ? static_cast<void *>(wsb + c_off) : C;
  const int64_t ldc_use = copy_c ? aligned_ld(N, osz) : ldc;

  // Boxes (inner x outer, elements): A 64 k x 128 rows, or 64 m x 64 k when
  // stored transposed; B 64 n x 64 k, or 64 k x (columns per CTA) when stored
  // transposed; C 128 bytes x 32 rows.
  // (Maps a path does not use stay zeroed and are never read by the kernel.)
  CUtensorMap tmA = {}, tmB = {}, tmC = {}, tmR = {};
  const CUtensorMapDataType h16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const CUtensorMapDataType c_type = f16 ? h16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const uint32_t b_rows_per_cta =
      static_cast<uint32_t>((rv.cfg.block_n > 256 ? 256 : rv.cfg.block_n) / rv.cfg.cta_group);
  if (!plain) {
    const bool a_ok = at ? encode_2d(&tmA, h16, A_use, uint64_t(M), uint64_t(K), uint64_t(lda_use) * 2, 64, kBK)
                         : encode_2d(&tmA, h16, A_use, uint64_t(K), uint64_t(M), uint64_t(lda_use) * 2, kBK, kBM);
    const bool b_ok = bt ? encode_2d(&tmB, h16, B_use, uint64_t(K), uint64_t(N), uint64_t(ldb_use) * 2, kBK,
                                     b_rows_per_cta)
                         : encode_2d(&tmB, h16, B_use, uint64_t(N), uint64_t(K), uint64_t(ldb_use) * 2, 64, kBK);
    if (!a_ok || !b_ok) return TLG_ERR_CUDA;
  }
  if (!c_plain && !encode_2d(&tmC, c_type, C_use, uint64_t(N), uint64_t(M), uint64_t(ldc_use) * osz,
                             uint32_t(128 / osz), 32))
    return TLG_ERR_CUDA;

  GemmParams p;
  p.bias = static_cast<const __half *>(bias);
  p.C = C_use;
  p.ldc = ldc_use;
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.raster_group = rv.cfg.raster_group;
  p.n_aligned = (N * osz) % 16 == 0 ? 1 : 0;
  p.limit_ns = kWaitLimitNs;
  p.dp_tiles = rv.sched.dp_tiles;
  p.split = rv.sched.split;
  p.tail_items = rv.sched.tail_items;
  p.counters = static_cast<uint32_t *>(ws);
  p.ws = ws != nullptr ? reinterpret_cast<float *>(static_cast<char *>(ws) + kCounterBytes)
                       : nullptr;
  p.A = static_cast<const __half *>(A_use);
  p.B = static_cast<const __half *>(B_use);
  p.lda = lda_use;
  p.ldb = ldb_use;
  p.c_plain = c_plain ? 1 : 0;
  p.bias_aligned = (bias != nullptr && aligned16(bias)) ? 1 : 0;
  p.act = e.act;
  p.R = e.R;
  p.ldr = e.ldr;
  p.r_vec = (e.R != nullptr && aligned16(e.R) && (e.ldr * osz) % 16 == 0) ? 1 : 0;
  // An fp16 residual TMA can describe: the last tile of each unit stages it in the ring
  // (32 x 64 boxes, the epilogue warps' pieces).
  p.r_tma = 0;
  if (ek == kEpiFused && f16 && !plain && p.r_vec != 0 &&
      encode_2d(&tmR, h16, e.R, uint64_t(N), uint64_t(M), uint64_t(e.ldr) * 2, 64, 32))
    p.r_tma = 1;
  // After this call's own copy kernel the GEMM starts as its programmatic
  // dependent: its set-up overlaps the copy's tail.
  const tlg_status ls = fns_for(rv.idx, f16, ek, at, bt, plain)
                             .launch(rv.sched.units, tmA, tmB, tmC, tmR, p,
                                     rv.cfg.overlap_prev != 0 || copy_ab, s);
  if (ls != TLG_OK || !copy_c) return ls;
  const CopyJob jc = {static_cast<const char *>(C_use), aligned_ld(N, osz) * osz, static_cast<char *>(C),
                      ldc * osz, M, N * osz};
  return launch_copy_out(jc, osz, info.sm_count, s);
}

// ---------------------------------------------------------------- allocation-free scratch
//
// Scratch for tlg_gemm_ex_noalloc: the split-K tail's partial sums and
// counters live in this array instead of a caller workspace.  It is part of
// the library's device image, so every GPU that loads the library holds its
// 16 MiB until the process exits; no call allocates anything.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

struct StaticScratch {
  bool ready = false;
  void *ptr = nullptr;
};
StaticScratch g_static_scratch_of[kMaxDevices];

// Device address of g_static_scratch on the current device.  The host-side
// name is only a stand-in for the symbol; the address a kernel may use comes
// from cudaGetSymbolAddress, asked once per device with that device current.
tlg_status static_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return TLG_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  StaticScratch &s = g_static_scratch_of[dev];
  if (!s.ready) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return TLG_ERR_CUDA;
    }
    s.ptr = p;
    s.ready = true;
  }
  *out = s.ptr;
  return TLG_OK;
}

tlg_status resolve_public(int64_t M, int64_t N, int64_t K, tlg_out out, tlg_epilogue epilogue,
                          const tlg_config *req, size_t ws_bytes, Resolved *rv) {
  if (out != TLG_OUT_F32 && out != TLG_OUT_F16) return TLG_ERR_INVALID_ARG;
  if (epilogue != TLG_EPI_NONE && epilogue != TLG_EPI_BIAS_RELU) return TLG_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0) return TLG_ERR_INVALID_ARG;
  int dev = 0;
  DeviceInfo info;
  const tlg_status ds = current_device(&dev, &info);
  if (ds != TLG_OK) return ds;
  return resolve(dev, info.sm_count, std::max<int64_t>(M, 1), std::max<int64_t>(N, 1),
                 std::max<int64_t>(K, 1), out == TLG_OUT_F16,
                 epilogue != TLG_EPI_BIAS_RELU ? kEpiNone
                                               : (out == TLG_OUT_F16 ? kEpiBiasRelu : kEpiFused),
                 false,
                 false, false, req, ws_bytes, rv);
}

}  // namespace

namespace tlg {

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


TLG_DEFINE_ERROR_WORD_READER(error_word_host)

}  // namespace tlg

extern "C" {

tlg_status tlg_gemm_f16f32(int64_t M, int64_t N, int64_t K, const void *A, int64_t lda,
                           const void *B, int64_t ldb, float *C, int64_t ldc, void *stream) {
  return gemm_impl(M, N, K, false, A, lda, false, B, ldb, Epi{}, C, ldc, TLG_OUT_F32, nullptr,
                   nullptr, 0, stream);
}

tlg_status tlg_gemm_f16f16(int64_t M, int64_t N, int64_t K, const void *A, int64_t lda,
                           const void *B, int64_t ldb, void *C, int64_t ldc, void *stream) {
  return gemm_impl(M, N, K, false, A, lda, false, B, ldb, Epi{}, C, ldc, TLG_OUT_F16, nullptr,
                   nullptr, 0, stream);
}

tlg_status tlg_gemm_bias_relu_f16(int64_t M, int64_t N, int64_t K, const void *A, int64_t lda,
                                  const void *B, int64_t ldb, const void *bias, void *C,
                                  int64_t ldc, void *stream) {
  if (bias == nullptr && M > 0 && N > 0) return TLG_ERR_INVALID_ARG;
  Epi e;
  const tlg_status es = legacy_epilogue(TLG_OUT_F16, TLG_EPI_BIAS_RELU, bias, &e);
  if (es != TLG_OK) return es;
  return gemm_impl(M, N, K, false, A, lda, false, B, ldb, e, C, ldc, TLG_OUT_F16, nullptr, nullptr,
                   0, stream);
}

tlg_status tlg_gemm_ex(int64_t M, int64_t N, int64_t K, const void *A, int64_t lda, const void *B,
                       int64_t ldb, const void *bias, void *C, int64_t ldc, tlg_out out,
                       tlg_epilogue epilogue, const tlg_config *config, void *workspace,
                       size_t workspace_bytes, void *stream) {
  Epi e;
  const tlg_status es = legacy_epilogue(out, epilogue, bias, &e);
  if (es != TLG_OK) return es;
  return gemm_impl(M, N, K, false, A, lda, false, B, ldb, e, C, ldc, out, config, workspace,
                   workspace_bytes, stream);
}

tlg_status tlg_gemm_op(int64_t M, int64_t N, int64_t K, tlg_op op_a, const void *A, int64_t lda,
                       tlg_op op_b, const void *B, int64_t ldb, const void *bias, void *C,
                       int64_t ldc, tlg_out out, tlg_epilogue epilogue, const tlg_config *config,
                       void *workspace, size_t workspace_bytes, void *stream) {
  Epi e;
  const tlg_status es = legacy_epilogue(out, epilogue, bias, &e);
  if (es != TLG_OK) return es;
  if ((op_a != TLG_OP_N && op_a != TLG_OP_T) || (op_b != TLG_OP_N && op_b != TLG_OP_T))
    return TLG_ERR_INVALID_ARG;
  return gemm_impl(M, N, K, op_a == TLG_OP_T, A, lda, op_b == TLG_OP_T, B, ldb, e, C, ldc, out,
                   config, workspace, workspace_bytes, stream);
}

tlg_status tlg_gemm_fused(int64_t M, int64_t N, int64_t K, tlg_op op_a, const void *A,
                          int64_t lda, tlg_op op_b, const void *B, int64_t ldb,
                          const tlg_fused_epilogue *epilogue, void *C, int64_t ldc, tlg_out out,
                          const tlg_config *config, void *workspace, size_t workspace_bytes,
                          void *stream) {
  Epi e;
  const tlg_status es = fused_epilogue(out, epilogue, &e);
  if (es != TLG_OK) return es;
  if ((op_a != TLG_OP_N && op_a != TLG_OP_T) || (op_b != TLG_OP_N && op_b != TLG_OP_T))
    return TLG_ERR_INVALID_ARG;
  return gemm_impl(M, N, K, op_a == TLG_OP_T, A, lda, op_b == TLG_OP_T, B, ldb, e, C, ldc, out,
                   config, workspace, workspace_bytes, stream);
}

tlg_status tlg_gemm_ex_noalloc(int64_t M, int64_t N, int64_t K, const void *A, int64_t lda,
                               const void *B, int64_t ldb, const void *bias, void *C, int64_t ldc,
                               tlg_out out, tlg_epilogue epilogue, const tlg_config *config,
                               void *stream) {
  Epi e;
  const tlg_status es = legacy_epilogue(out, epilogue, bias, &e);
  if (es != TLG_OK) return es;
  // Looked up on every call, split or not, so that a device's first call does it.
  void *scratch = nullptr;
  const tlg_status ss = static_scratch(&scratch);
  if (ss != TLG_OK) return ss;
  const bool split = config != nullptr && config->split_k >= 2;
  if (!split)  // no scratch needed: exactly tlg_gemm_ex without a workspace
    return gemm_impl(M, N, K, false, A, lda, false, B, ldb, e, C, ldc, out, config, nullptr, 0,
                     stream);
  // gemm_impl rejects a schedule that needs more scratch than the array holds before it
  // launches anything, and clears the counters just before its first launch.
  return gemm_impl(M, N, K, false, A, lda, false, B, ldb, e, C, ldc, out, config, scratch,
                   kStaticScratchBytes, stream, true);
}

tlg_status tlg_gemm_workspace_size(int64_t M, int64_t N, int64_t K, tlg_out out,
                                   tlg_epilogue epilogue, const tlg_config *config, size_t *bytes) {
  if (bytes == nullptr) return TLG_ERR_INVALID_ARG;
  *bytes = 0;
  if (M < 0 || N < 0 || K < 0) return TLG_ERR_INVALID_ARG;
  if (M == 0 || N == 0 || K == 0) return TLG_OK;
  Resolved rv;
  const tlg_status rs = resolve_public(M, N, K, out, epilogue, config, SIZE_MAX, &rv);
  if (rs != TLG_OK) return rs;
  *bytes = rv.sched.workspace;
  return TLG_OK;
}

tlg_status tlg_gemm_workspace_size_op(int64_t M, int64_t N, int64_t K, tlg_op op_a,
                                      const void *A, int64_t lda, tlg_op op_b, const void *B,
                                      int64_t ldb, const void *C, int64_t ldc, tlg_out out,
                                      const tlg_config *config, size_t *bytes) {
  if (bytes == nullptr) return TLG_ERR_INVALID_ARG;
  *bytes = 0;
  if ((op_a != TLG_OP_N && op_a != TLG_OP_T) || (op_b != TLG_OP_N && op_b != TLG_OP_T))
    return TLG_ERR_INVALID_ARG;
  const bool at = op_a == TLG_OP_T, bt = op_b == TLG_OP_T;
  const tlg_status hs = check_args(M, N, K, at, A, lda, bt, B, ldb, Epi{}, C, ldc, out);
  if (hs != TLG_OK || M == 0 || N == 0 || K == 0) return hs;
  const int64_t osz = out == TLG_OUT_F32 ? 4 : 2;
  const CopyPlan cp = copy_plan(M, N, K, at, A, lda, bt, B, ldb, C, ldc, osz);
  int dev = 0;
  DeviceInfo info;
  const tlg_status ds = current_device(&dev, &info);
  if (ds != TLG_OK) return ds;
  Resolved rv;
  const tlg_status rs = resolve(dev, info.sm_count, M, N, K, out == TLG_OUT_F16, kEpiNone, at, bt,
                                false, config, SIZE_MAX, &rv);
  if (rs != TLG_OK) return rs;
  if (!cp.a && !cp.b && !cp.c) {
    *bytes = rv.sched.workspace;
    return TLG_OK;
  }
  *bytes = round_up_sz(std::max<size_t>(rv.sched.workspace, kCounterBytes), kCopyAlign) +
           cp.ab_bytes() + cp.c_bytes;
  return TLG_OK;
}

tlg_status tlg_choose_config(int64_t M, int64_t N, int64_t K, tlg_out out, tlg_epilogue epilogue,
                             tlg_config *config) {
  if (config == nullptr) return TLG_ERR_INVALID_ARG;
  Resolved rv;
  const tlg_config req = *config;
  const tlg_status rs = resolve_public(M, N, K, out, epilogue, &req, SIZE_MAX, &rv);
  if (rs != TLG_OK) return rs;
  *config = rv.cfg;
  return TLG_OK;
}

tlg_status tlg_device_error(int clear, uint32_t *code_out) {
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return TLG_ERR_CUDA;
  }
  // Every translation unit's kernels report into that unit's own word.
  tlg_status (*const readers[])(bool, uint32_t *) = {tlg::error_word_host, tlg::error_word_nn,
                                                     tlg::error_word_nt, tlg::error_word_tn,
                                                     tlg::error_word_tt};
  uint32_t v = 0;
  for (auto read : readers) {
    uint32_t w = 0;
    const tlg_status rs = read(clear != 0, &w);
    if (rs != TLG_OK) return rs;
    v |= w;
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
    case TLG_ERR_INVALID_ARG:
      return "TLG_ERR_INVALID_ARG: bad size, null or host pointer, ld too small, overlapping "
             "buffers, or a workspace too small for the requested split";
    case TLG_ERR_ALIGNMENT:
      return "TLG_ERR_ALIGNMENT: a matrix or bias pointer not aligned to its element (2 bytes for "
             "fp16, 4 for fp32), or a workspace not 256-byte aligned";
    case TLG_ERR_UNSUPPORTED:
      return "TLG_ERR_UNSUPPORTED: device is not sm_100, size too large, or configuration not "
             "provided";
    case TLG_ERR_CUDA: return "TLG_ERR_CUDA: a CUDA call failed";
    case TLG_ERR_TIMEOUT: return "TLG_ERR_TIMEOUT: a kernel pipeline wait exceeded its time limit";
  }
  return "unknown tlg_status";
}

int32_t tlg_version(void) { return 200; }

}  // extern "C"
