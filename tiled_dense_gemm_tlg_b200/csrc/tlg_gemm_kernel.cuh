// Persistent, warp-specialised fp16 GEMM for sm_100a.
//
// The tiling is the pages' block decomposition -- one output tile per
// (row block, column block), an fp32 accumulator per tile, operand tiles of
// A[rows, k-block] and B[k-block, cols] staged in shared memory by a
// multi-stage pipeline over the K loop ("tilelang operator-compilation
// walkthrough", lqnn.cn/news/222844, section 2.1) -- mapped onto Blackwell.
// A tile is 128*CG rows (CG = 1 CTA, or a 2-CTA cluster issuing
// tcgen05.mma.cta_group::2) by BN*NH columns (NH = 2: two MMA halves that fill
// TMEM):
//
//   warp 0 (one lane)  producer: TMA loads of the A and B tiles of each
//                      k-block into a STAGES-deep ring, one mbarrier pair per
//                      slot (full: bytes landed; empty: the MMAs read it).
//   warp 1 (one lane)  MMA issuer (the pair's leader CTA): tcgen05.mma into a
//                      TMEM accumulator; with NH == 1 two accumulators
//                      alternate, so the epilogue of tile i overlaps the main
//                      loop of tile i+1.  Warp 1 also owns the TMEM allocation.
//   warps 2-5          epilogue: tcgen05.ld of the accumulator, the fused
//                      epilogue of the build (none; bias + ReLU, "domestic-GPU
//                      TileLang adoption", xdnf.cn/news/333523, section 4.2;
//                      or bias, activation and residual chosen per call,
//                      section 4.1) and the output cast, staged in shared
//                      memory and written by TMA bulk-tensor stores, which clip
//                      the rows and columns outside M x N.
//   warps 6-9          plain-load builds only: loader warps that fill the ring
//                      with ordinary loads for operands TMA cannot describe
//                      (warp 0 then idles).
//
// Work units (CTAs, or CTA pairs) are persistent and walk the tile list with a
// stride of the unit count; consecutive tiles are grouped by `raster_group`
// row blocks so the units of one wave share A and B tiles in L2.  An optional
// split-K tail cuts the tiles left after the last whole wave into k-slices
// whose fp32 partials the last-arriving slice sums in a fixed order.
//
// Ragged M, N and K need no special code in the main loop: the TMA unit fills
// out-of-range elements of a box with zeros, so the last k-block adds 0 for
// k >= K, and the TMA store skips the rows/columns beyond M/N.
#pragma once

#include "tlg_device.cuh"

namespace tlg {

constexpr int kBM = 128;  // tile rows per CTA (TMEM lanes)
constexpr int kBK = 64;   // k-block: 64 fp16 = one 128-byte swizzle row
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kEpiWarps);  // producer warp, MMA warp, epilogue warps
// Operands TMA cannot describe (a row stride or base not 16-byte aligned) are
// loaded by kLoaderWarps extra warps with plain loads instead.
constexpr int kLoaderWarps = 4;
constexpr int kThreadsLsu = kThreads + 32 * kLoaderWarps;
constexpr uint32_t kStageOutBytes = 32 * 128;   // one TMA store box: 32 rows x 128 bytes
constexpr uint64_t kWaitPerKBlockNs = 20000;     // the epilogue's wait budget per k-block of a tile

// Device error word (see tlg_device_error in tlg.h); internal linkage, so
// every translation unit that includes this header has its own copy, and the
// host side reads them all.
static __device__ uint32_t g_device_error;

// Shared-memory plan of one CTA.  CG CTAs (1 or 2) compute one tile of
// 128*CG rows by NH*BN columns (BN = the MMA's N; NH = 1, or 2 for a tile of
// two MMA halves that fills TMEM); each CTA stages its own 128 rows of A and
// its own BN/CG columns of each half of B per k-block, plus two 4 KB output
// boxes per epilogue warp.  With a cluster k-split (KS > 1 CTAs share one
// tile's K range) each CTA also receives, for the BN/KS columns it finishes,
// the fp32 partial sums of its KS - 1 peers.  Where it still fits, the tile's
// bias is kept there too, converted to fp32 once per tile (with two barriers
// that pass it between the epilogue warps).
template <int CG, int BN, int STAGES, int NH = 1, int KS = 1>
struct SmemPlan {
  static constexpr int kBNc = BN / CG;  // B columns of one MMA half held by one CTA
  static constexpr uint32_t kABytes = kBM * kBK * 2;
  static constexpr uint32_t kHalfBBytes = kBK * kBNc * 2;
  static constexpr uint32_t kBBytes = kHalfBBytes * NH;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kOutOffset = STAGES * kStageBytes;
  static constexpr uint32_t kOutBytes = kEpiWarps * 2 * kStageOutBytes;
  static constexpr int kOwnCols = BN / KS;  // columns of a tile one CTA of a k-split finishes
  static constexpr uint32_t kRecvSlotBytes = kBM * kOwnCols * 4;  // one peer's fp32 partial of them
  static constexpr uint32_t kRecvOffset = kOutOffset + kOutBytes;
  static constexpr uint32_t kRecvBytes = (KS - 1) * kRecvSlotBytes;
  static constexpr uint32_t kBiasOffset = kRecvOffset + kRecvBytes;
  // full, empty, tmem full/empty x2, drain; with a k-split also recv-full and send-free
  static constexpr uint32_t kNumBarsBase = 2 * STAGES + 4 + 1 + (KS > 1 ? 2 : 0);
  static constexpr uint32_t kBiasWant = BN * NH * 4;  // the tile's bias in fp32
  static constexpr bool kBiasSmem =
      kBiasOffset + kBiasWant + (kNumBarsBase + 3) * 8 + 16 + 1024 <= 232448;
  static constexpr uint32_t kBiasBytes = kBiasSmem ? kBiasWant : 0;
  static constexpr uint32_t kBarOffset = kBiasOffset + kBiasBytes;
  // with the bias in shared memory also bias-full and bias-free; last, residual-full
  static constexpr uint32_t kNumBars = kNumBarsBase + (kBiasSmem ? 2 : 0) + 1;
  static constexpr uint32_t kMiscOffset = kBarOffset + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOffset + 16;
  static constexpr uint32_t kDynamicBytes = kBytes + 1024;  // slack to align the base to 1024
  static constexpr uint32_t kTmemCols = (2 * BN < 32) ? 32 : 2 * BN;
  static_assert(kBNc % 64 == 0, "each CTA's B slice must be whole 64-column swizzle blocks");
  static_assert(kTmemCols <= 512, "two accumulators must fit in TMEM");
  static_assert(KS == 1 || (CG == 1 && NH == 1 && kOwnCols % 64 == 0),
                "a k-split is built for one-CTA tiles whose CTAs each finish whole 64-column pieces");
  static_assert(kDynamicBytes <= 232448, "shared memory per CTA exceeded");
};

struct GemmParams {
  const __half *bias;
  void *C;       // used only for the ragged last column box when N is not 16-byte aligned
  int64_t ldc;
  int M, N, K;
  int raster_group;
  int n_aligned;  // N * sizeof(out) is a multiple of 16: every box may go through TMA
  uint64_t limit_ns;
  // Split-K tail (split > 1): tiles [dp_tiles, num_tiles) are each cut into
  // `split` k-slices, tail_items = (num_tiles - dp_tiles) * split <= work units.
  int dp_tiles;
  int split;
  int tail_items;
  float *ws;           // fp32 partial sums of the tail slices
  uint32_t *counters;  // per (tail tile, CTA of the group, epilogue warp): slices written so far
  // Plain-load path (kernels built with LSU): the stored operands.
  const __half *A;
  const __half *B;
  int64_t lda, ldb;
  int c_plain;       // C cannot be written by TMA (base or row stride not 16-byte aligned)
  int bias_aligned;  // the bias may be read 16 bytes at a time
  // Fused epilogue (kernels built with kEpiFused): C = act(acc + bias[col]) + R[row, col].
  int act;           // kActNone, kActRelu, kActGelu, kActSilu or kActGeluTanh
  const void *R;     // residual in C's type, or nullptr; may be C itself (same ldc)
  int64_t ldr;
  int r_vec;         // R's base and row stride are 16-byte aligned
  int r_tma;         // tmR describes R (fp16 C, TMA path): the last tile's residual is staged
};

// One unit of work: a tile, or one k-slice of a tail tile.
struct WorkItem {
  int mb, nb;    // tile coordinates (in tiles)
  int kb0, kb1;  // k-blocks [kb0, kb1)
  int tail;      // index among the tail tiles, or -1 for a whole tile
  int slice;
};

// Work list of one unit (a CTA, or a CTA pair): the whole tiles unit,
// unit + num_units, ... below dp_tiles, with its tail slice, if it has one,
// second when at least two whole tiles follow it and first otherwise.  A whole
// tile after the slice lets its partial-sum traffic run in the epilogue while
// that tile's main loop already runs; starting on a whole tile spreads the
// first wave's loads over more tiles than the few tail tiles the slices share
// (B200, 4096^3 with the split tail: 1419 -> 1435 TFLOP/s).
__device__ __forceinline__ int work_count(const GemmParams &p, int unit, int num_units) {
  const int whole = p.dp_tiles > unit ? (p.dp_tiles - unit + num_units - 1) / num_units : 0;
  return whole + (unit < p.tail_items ? 1 : 0);
}

__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int group, int &mb,
                                            int &nb);

__device__ __forceinline__ WorkItem work_item(const GemmParams &p, int k, int unit, int num_units,
                                              int num_m, int num_n, int num_kb) {
  WorkItem w;
  const bool has_tail = unit < p.tail_items;
  const int whole = p.dp_tiles > unit ? (p.dp_tiles - unit + num_units - 1) / num_units : 0;
  const int slice_at = whole >= 2 ? 1 : 0;
  int t;
  if (has_tail && k == slice_at) {
    w.tail = unit / p.split;
    w.slice = unit - w.tail * p.split;
    t = p.dp_tiles + w.tail;
    w.kb0 = static_cast<int>(static_cast<int64_t>(w.slice) * num_kb / p.split);
    w.kb1 = static_cast<int>(static_cast<int64_t>(w.slice + 1) * num_kb / p.split);
  } else {
    w.tail = -1;
    w.slice = 0;
    t = unit + (has_tail && k > slice_at ? k - 1 : k) * num_units;
    w.kb0 = 0;
    w.kb1 = num_kb;
  }
  tile_coords(t, num_m, num_n, p.raster_group, w.mb, w.nb);
  return w;
}

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

// Epilogue kinds a kernel is built with: the plain product; the general fused
// epilogue (bias, activation and residual chosen at run time); and bias +
// ReLU alone, whose code is a small part of the general one.  The epilogue
// warps share each SM sub-partition's instruction cache with the producer and
// MMA warps, and the general epilogue's larger code measurably slows the main
// loop even where it does the same work, so the common bias + ReLU case gets
// its own build.
constexpr int kEpiNone = 0;
constexpr int kEpiFused = 1;
constexpr int kEpiBiasRelu = 2;

// Activation codes of the fused epilogue (the values of tlg_activation).
constexpr int kActNone = 0;
constexpr int kActRelu = 1;
constexpr int kActGelu = 2;
constexpr int kActSilu = 3;
constexpr int kActGeluTanh = 4;

// Hardware approximations (PTX rcp.approx / ex2.approx, flushing subnormals).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Packed fp32 pairs.  sm_100's add/mul/fma .f32x2 do two fp32 operations
// in one instruction, each rounded exactly as its scalar form, so a pair of
// columns costs the issue slot of one (the epilogue warps share each SM
// sub-partition's issue slots with the producer and MMA warps).  The pair
// sits in one 64-bit register (the even column in the low word).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t f2_splat(float c) { return f2_pack(c, c); }

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// x0 += b0, x1 += b1 as one packed add.
__device__ __forceinline__ void f2_add_to(float &x0, float &x1, float b0, float b1) {
  f2_unpack(f2_add(f2_pack(x0, x1), f2_pack(b0, b1)), x0, x1);
}

// x0 += the low fp16 half of w, x1 += its high half: sm_100's mixed-precision
// add takes the fp16 operand as it is (no conversion instruction) and rounds
// the fp32 sum once, exactly as a conversion followed by an fp32 add.
__device__ __forceinline__ void add_half2_to(float &x0, float &x1, uint32_t w) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.f16 %0, lo, %0;\n\tadd.rn.f32.f16 %1, hi, %1;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "r"(w));
}

// GELU in its exact form x * Phi(x), Phi the standard normal CDF, in fp32.
// With a = min(|x|, 6) and q = Phi(-a), the standard normal tail,
//   x Phi(x) = max(x, 0) - a q
// (x (1 - q) for x >= 0, -|x| q for x < 0; beyond |x| = 6, q < 1e-9 and a q
// < 6e-9): one fused multiply-add, no select, and q is computed directly, so
// the negative tail has no cancellation.  q = 2^g(a) with g a polynomial
// fitted to log2 Phi(-a) on [0, 6] and made near-minimax by Lawson's
// reweighted least squares (fit_gelu_tail.py beside this file prints the
// coefficients and the errors).  Two fits, by the type of C:
//  - fp32 C: degree 6, the error weighted by what it costs in GELU
//    (a Phi(-a) ln 2): GELU error below 3e-7 on [-8, 8];
//  - fp16 C: degree 5, the error weighted in fp16 units in the last place
//    of a Phi(-a): at most 0.14 of a unit before the rounding to fp16, so
//    every fp16 result lies within 0.64 units of the exact GELU.
// One exp2 and no reciprocal.  The epilogue's instruction count is what the
// main loop running beside it feels, so the form is written for the fewest:
// the polynomial runs in na = -a = max.NaN(-|x|, -6) with the odd
// coefficients negated (sum c_k a^k = sum (-1)^k c_k na^k).  Each Horner step
// then yields exactly the negation of the step in a (round to nearest is
// symmetric), so g has the same bits, and -a q + max(x, 0) is one packed
// fused multiply-add for two values.  max.NaN keeps a NaN input NaN.
template <bool F16>
__device__ __forceinline__ constexpr float gelu_tail_coef(int k) {  // c_k, lowest degree first
  if constexpr (F16) {
    constexpr float c[6] = {-1.00010169f, -1.14941466f, -0.463673383f, -0.0485566817f,
                            0.00592234265f, -0.000330398412f};
    return c[k];
  } else {
    constexpr float c[7] = {-0.999993086f,  -1.15120173f,     -0.458770931f, -0.0534121692f,
                            0.00808076002f, -0.000769232807f, 3.30943076e-05f};
    return c[k];
  }
}

template <bool F16>
constexpr int kGeluTailDegree = F16 ? 5 : 6;

// The coefficient of na^k.
template <bool F16>
__device__ __forceinline__ constexpr float gelu_tail_coef_neg(int k) {
  return (k & 1) ? -gelu_tail_coef<F16>(k) : gelu_tail_coef<F16>(k);
}

__device__ __forceinline__ float gelu_tail_narg(float x) {  // -min(|x|, 6), NaN stays NaN
  float na;
  asm("{\n\t.reg .f32 t;\n\tabs.f32 t, %1;\n\tneg.f32 t, t;\n\tmax.NaN.f32 %0, t, %2;\n\t}"
      : "=f"(na)
      : "f"(x), "f"(-6.0f));
  return na;
}

template <bool F16>
__device__ __forceinline__ float gelu_erf(float x) {
  constexpr int D = kGeluTailDegree<F16>;
  const float na = gelu_tail_narg(x);
  float g = gelu_tail_coef_neg<F16>(D);
#pragma unroll
  for (int k = D - 1; k >= 0; --k) g = fmaf(g, na, gelu_tail_coef_neg<F16>(k));
  return fmaf(na, ex2_approx(g), fmaxf(x, 0.0f));  // 2^g = q = Phi(-a)
}

// gelu_erf on two values with the packed instructions: the same operations in
// the same order, so the same bits.
template <bool F16>
__device__ __forceinline__ void gelu_erf_2(float &x0, float &x1) {
  constexpr int D = kGeluTailDegree<F16>;
  const uint64_t na = f2_pack(gelu_tail_narg(x0), gelu_tail_narg(x1));
  uint64_t g = f2_splat(gelu_tail_coef_neg<F16>(D));
#pragma unroll
  for (int k = D - 1; k >= 0; --k) g = f2_fma(g, na, f2_splat(gelu_tail_coef_neg<F16>(k)));
  float g0, g1;
  f2_unpack(g, g0, g1);
  const uint64_t m = f2_pack(fmaxf(x0, 0.0f), fmaxf(x1, 0.0f));
  f2_unpack(f2_fma(na, f2_pack(ex2_approx(g0), ex2_approx(g1)), m), x0, x1);
}

// SiLU and the tanh form of GELU are both x * sigmoid(c1 x + c3 x^3):
//   SiLU:      c1 = 1,                 c3 = 0;
//   tanh GELU: x/2 (1 + tanh(y)) = x sigmoid(2y) with y = sqrt(2/pi) (x + 0.044715 x^3),
//              so c1 = 2 sqrt(2/pi),  c3 = 0.044715 c1.
// sigmoid(z) = 1 / (1 + 2^(-z log2 e)); one code path for both, with the
// coefficients chosen per call.
struct SigmoidForm {
  float c1, c3;  // already multiplied by -log2(e)
};

__device__ __forceinline__ SigmoidForm sigmoid_form(int act) {
  constexpr float kNegLog2e = -1.4426950408889634f;
  constexpr float kTanhC1 = 1.5957691216057308f;  // 2 sqrt(2/pi)
  if (act == kActSilu) return {kNegLog2e, 0.0f};
  return {kNegLog2e * kTanhC1, kNegLog2e * kTanhC1 * 0.044715f};
}

__device__ __forceinline__ float sigmoid_form_apply(SigmoidForm f, float x) {
  const float z = x * fmaf(f.c3, x * x, f.c1);  // -(c1 x + c3 x^3) log2(e)
  return x * rcp_approx(1.0f + ex2_approx(z));
}

// sigmoid_form_apply on two values with the packed instructions (same bits).
__device__ __forceinline__ void sigmoid_form_apply_2(SigmoidForm f, float &x0, float &x1) {
  const uint64_t x = f2_pack(x0, x1);
  float z0, z1;
  f2_unpack(f2_mul(x, f2_fma(f2_splat(f.c3), f2_mul(x, x), f2_splat(f.c1))), z0, z1);
  float d0, d1;
  f2_unpack(f2_add(f2_splat(1.0f), f2_pack(ex2_approx(z0), ex2_approx(z1))), d0, d1);
  f2_unpack(f2_mul(x, f2_pack(rcp_approx(d0), rcp_approx(d1))), x0, x1);
}

template <bool F16>
__device__ __forceinline__ float activate(int act, float x) {
  if (act == kActRelu) return fmaxf(x, 0.0f);
  if (act == kActGelu) return gelu_erf<F16>(x);
  if (act == kActSilu || act == kActGeluTanh) return sigmoid_form_apply(sigmoid_form(act), x);
  return x;
}

// The activation over 32 values; `act` is the same for every thread, so the
// branch does not diverge.  F16: the result is rounded to fp16 (GELU's fit).
template <bool F16>
__device__ __forceinline__ void activate_32(int act, float (&v)[32]) {
  if (act == kActRelu) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = fmaxf(v[j], 0.0f);
  } else if (act == kActGelu) {
#pragma unroll
    for (int j = 0; j < 32; j += 2) gelu_erf_2<F16>(v[j], v[j + 1]);
  } else if (act == kActSilu || act == kActGeluTanh) {
    const SigmoidForm f = sigmoid_form(act);
#pragma unroll
    for (int j = 0; j < 32; j += 2) sigmoid_form_apply_2(f, v[j], v[j + 1]);
  }
}

// Adds the residual R[row, col0 + j] (j < 32), read in C's type.  Rows >= M
// and columns >= N are not read.  R may be C itself: every element is read
// here, by the one thread that later writes it, before that write, and no
// other thread touches it.  The loads are ordinary (not the read-only path)
// for that reason.
template <bool OUT_F16>
__device__ __forceinline__ void add_residual_32(const GemmParams &p, int row, int col0,
                                                float (&v)[32]) {
  if (row >= p.M) return;
  if constexpr (OUT_F16) {
    const __half *r = static_cast<const __half *>(p.R) + static_cast<int64_t>(row) * p.ldr + col0;
    if (p.r_vec && col0 + 32 <= p.N) {
      const uint4 *q = reinterpret_cast<const uint4 *>(r);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 w = q[c];
        add_half2_to(v[c * 8], v[c * 8 + 1], w.x);
        add_half2_to(v[c * 8 + 2], v[c * 8 + 3], w.y);
        add_half2_to(v[c * 8 + 4], v[c * 8 + 5], w.z);
        add_half2_to(v[c * 8 + 6], v[c * 8 + 7], w.w);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < p.N) v[j] += __half2float(r[j]);
    }
  } else {
    const float *r = static_cast<const float *>(p.R) + static_cast<int64_t>(row) * p.ldr + col0;
    if (p.r_vec && col0 + 32 <= p.N) {
      const float4 *q = reinterpret_cast<const float4 *>(r);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 w = q[c];
        f2_add_to(v[4 * c], v[4 * c + 1], w.x, w.y);
        f2_add_to(v[4 * c + 2], v[4 * c + 3], w.z, w.w);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < p.N) v[j] += r[j];
    }
  }
}

// Epilogue input of one 64-column piece of this lane's row loaded ahead of
// its use: the fp16 residual row piece (128 bytes, 16 at a time), whose DRAM
// latency would otherwise stall every piece.  The bias (a few KB, reused by
// every row) and an fp32 residual are read in epi_apply: holding them too
// would push the epilogue past the register file.  Pieces the vector loads
// cannot serve (ragged or unaligned) are also read in epi_apply.  ON = false
// (an fp32 C, or the plain-load kernels, whose extra loader warps leave each
// thread fewer registers) keeps nothing and reads the residual at its use.
template <bool ON>
struct EpiIn {
  uint4 r[ON ? 8 : 1];  // R[row, col0 .. col0+63], fp16
  bool has_r;
};

template <bool ON>
__device__ __forceinline__ void epi_prefetch(const GemmParams &p, int row, int col0,
                                             EpiIn<ON> &in) {
  in.has_r = ON && p.R != nullptr && p.r_vec != 0 && col0 + 64 <= p.N && row < p.M;
  if constexpr (ON) {
    if (in.has_r) {
      // Ordinary loads, not the read-only path: R may be C itself.
      const uint4 *q = reinterpret_cast<const uint4 *>(static_cast<const __half *>(p.R) +
                                                       static_cast<int64_t>(row) * p.ldr + col0);
#pragma unroll
      for (int c = 0; c < 8; ++c) in.r[c] = q[c];
    }
  }
}

// The bias of one tile's columns, spread over the warp: lane l holds columns
// [l * CPL, (l + 1) * CPL) of the tile (CPL = tile width / 32) as packed fp16
// pairs.  Loaded once per tile, before the accumulator is ready, so no piece
// of the epilogue waits on a bias load; a piece gets its columns with warp
// shuffles.
template <int CPL>
struct BiasSlice {
  static_assert(CPL >= 2 && CPL % 2 == 0, "whole fp16 pairs per lane");
  uint32_t w[CPL / 2];
};

template <int CPL>
__device__ __forceinline__ void load_bias_slice(const GemmParams &p, int tile_col0, int lane,
                                                BiasSlice<CPL> &s) {
  const int c = tile_col0 + lane * CPL;
  if (p.bias_aligned != 0 && c + CPL <= p.N) {
    // c * 2 bytes is a multiple of CPL * 2 >= 4 and the bias base is 16-byte aligned.
    if constexpr (CPL == 2) {
      s.w[0] = __ldg(reinterpret_cast<const unsigned int *>(p.bias + c));
    } else if constexpr (CPL == 4) {
      const uint2 x = __ldg(reinterpret_cast<const uint2 *>(p.bias + c));
      s.w[0] = x.x;
      s.w[1] = x.y;
    } else {
#pragma unroll
      for (int q = 0; q < CPL / 8; ++q) {
        const uint4 x = __ldg(reinterpret_cast<const uint4 *>(p.bias + c) + q);
        s.w[4 * q] = x.x;
        s.w[4 * q + 1] = x.y;
        s.w[4 * q + 2] = x.z;
        s.w[4 * q + 3] = x.w;
      }
    }
  } else {
    const unsigned short *b = reinterpret_cast<const unsigned short *>(p.bias);
#pragma unroll
    for (int i = 0; i < CPL / 2; ++i) {
      const uint32_t lo = c + 2 * i < p.N ? b[c + 2 * i] : 0u;
      const uint32_t hi = c + 2 * i + 1 < p.N ? b[c + 2 * i + 1] : 0u;
      s.w[i] = lo | (hi << 16);
    }
  }
}

// v[j] += bias[tile column t0 + j], j < 32, t0 a multiple of 32, from the slice.
template <int CPL>
__device__ __forceinline__ void add_bias_slice_32(const BiasSlice<CPL> &s, int t0,
                                                  float (&v)[32]) {
#pragma unroll
  for (int jj = 0; jj < 16; ++jj) {
    // columns t0 + 2jj and t0 + 2jj + 1 sit in one word of lane (t0 + 2jj) / CPL
    const uint32_t w = __shfl_sync(0xffffffffu, s.w[((2 * jj) % CPL) / 2], (t0 + 2 * jj) / CPL);
    add_half2_to(v[2 * jj], v[2 * jj + 1], w);
  }
}

// v[j] += bias[tile column t0 + j], j < 32, from the tile's fp32 bias in
// shared memory at sbias: every lane reads the same 16 bytes at a time (a
// broadcast), two packed adds each.
__device__ __forceinline__ void add_bias_smem_32(uint32_t sbias, int t0, float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint4 b = ld_shared_v4(sbias + static_cast<uint32_t>(t0 + 4 * q) * 4u);
    f2_add_to(v[4 * q], v[4 * q + 1], __uint_as_float(b.x), __uint_as_float(b.y));
    f2_add_to(v[4 * q + 2], v[4 * q + 3], __uint_as_float(b.z), __uint_as_float(b.w));
  }
}

// The fused epilogue on half `half` (columns col0 + 32*half ..) of a
// 64-column piece at tile column tcol: + bias, activation, + residual.  Done
// one half at a time so that the first half is packed for the store (and its
// registers freed) before the second half's activation runs.
template <bool OUT_F16, bool ON, bool SBIAS, int CPL>
__device__ __forceinline__ void epi_apply_32(const GemmParams &p, const EpiIn<ON> &in,
                                             const BiasSlice<CPL> &bias, uint32_t sbias, int row,
                                             int col0, int tcol, int half, float (&v)[32]) {
  const int c0 = col0 + 32 * half;
  if (p.bias != nullptr) {
    if constexpr (SBIAS)
      add_bias_smem_32(sbias, tcol + 32 * half, v);
    else
      add_bias_slice_32<CPL>(bias, tcol + 32 * half, v);
  }
  activate_32<OUT_F16>(p.act, v);
  if (p.R != nullptr) {
    if (ON && in.has_r) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 w = in.r[4 * half + c];
        add_half2_to(v[c * 8], v[c * 8 + 1], w.x);
        add_half2_to(v[c * 8 + 2], v[c * 8 + 3], w.y);
        add_half2_to(v[c * 8 + 4], v[c * 8 + 5], w.z);
        add_half2_to(v[c * 8 + 6], v[c * 8 + 7], w.w);
      }
    } else {
      add_residual_32<OUT_F16>(p, row, c0, v);
    }
  }
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

// pack_half2 followed by max(., 0) on both halves.  Rounding is monotonic and
// 0 is exact, so this equals rounding max(x, 0); like fmaxf, max.f16x2 returns
// the other operand for a NaN, so ReLU(NaN) = 0 as in the fp32 form.
__device__ __forceinline__ uint32_t pack_half2_relu(float lo, float hi) {
  uint32_t r;
  asm("max.f16x2 %0, %1, %2;" : "=r"(r) : "r"(pack_half2(lo, hi)), "r"(0u));
  return r;
}

// Writes one 128-byte row piece (eight 16-byte pieces) of a 32-row output box
// in the TMA 128-byte swizzle: piece c of row r sits at (c ^ (r % 8)) * 16.
__device__ __forceinline__ void st_box_row(uint32_t box, int r, const uint32_t (&w)[32],
                                           int first_word) {
  const uint32_t row = box + static_cast<uint32_t>(r) * 128u;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t addr = row + static_cast<uint32_t>((c ^ (r & 7)) * 16);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                 "r"(w[first_word + 4 * c]), "r"(w[first_word + 4 * c + 1]),
                 "r"(w[first_word + 4 * c + 2]), "r"(w[first_word + 4 * c + 3])
                 : "memory");
  }
}

// Plain predicated stores of one thread's row piece of 128 bytes (`w`, in
// the output format: 32 fp32 words, or 64 fp16 values packed in pairs)
// starting at column col0, only the columns below N.  Used for
// the last column box when N * sizeof(out) is not a multiple of 16 bytes: the
// TMA store's clipping would then write whole 16-byte pieces past column N.
template <bool OUT_F16>
__device__ __forceinline__ void store_row_tail(const GemmParams &p, int row, int col0,
                                               const uint32_t (&w)[32]) {
  if (row >= p.M) return;
  if constexpr (OUT_F16) {
    __half *c = reinterpret_cast<__half *>(p.C) + static_cast<int64_t>(row) * p.ldc + col0;
#pragma unroll
    for (int j = 0; j < 64; ++j)
      if (col0 + j < p.N)
        c[j] = __ushort_as_half(static_cast<unsigned short>(w[j / 2] >> (16 * (j & 1))));
  } else {
    float *c = reinterpret_cast<float *>(p.C) + static_cast<int64_t>(row) * p.ldc + col0;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j < p.N) c[j] = __uint_as_float(w[j]);
  }
}

// ------------------------------------------------------------------ plain-load path

// Elements (row, col) and (row, col + 1) of a row-major fp16 matrix with
// `rows` x `cols` valid elements and row stride ld, packed low/high; elements
// outside the matrix read as 0 (as the TMA path's out-of-range fill).  Any
// 2-byte alignment is fine.
// Predicated read-only global load of one 16-bit element (0 when !pred).
// Volatile, like the shared-memory stores, so a batch's loads stay in program
// order ahead of its stores and are all in flight together.
__device__ __forceinline__ uint32_t ld_u16_pred(const void *ptr, bool pred) {
  uint16_t x;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %2, 0;\n\t"
      "mov.u16 %0, 0;\n\t"
      "@p ld.global.nc.u16 %0, [%1];\n\t}"
      : "=h"(x)
      : "l"(ptr), "r"(static_cast<uint32_t>(pred)));
  return x;
}

__device__ __forceinline__ uint32_t load_pair(const __half *base, int row, int col, int64_t ld,
                                              int rows, int cols) {
  const unsigned short *q = reinterpret_cast<const unsigned short *>(base) +
                            static_cast<int64_t>(row < rows ? row : 0) * ld + col;
  const uint32_t lo = ld_u16_pred(q, row < rows && col < cols);
  const uint32_t hi = ld_u16_pred(q + 1, row < rows && col + 1 < cols);
  return lo | (hi << 16);
}

// No memory clobber: the loads of a batch may be issued ahead of its stores;
// the async-proxy fence that follows a stage (volatile, with a clobber) keeps
// every store before the barrier arrive.
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v));
}

// Byte offsets in the 128-byte-swizzled operand layouts the tensor core reads
// (the same layouts the TMA path writes).  K-major: one 128-byte row of 64 k
// per M/N index.  MN-major: 64-element blocks of 64 rows (one per k), 8 KB apart.
__device__ __forceinline__ uint32_t kmajor_offset(int mn, int k) {
  return static_cast<uint32_t>(mn * 128 + ((((k >> 3) ^ (mn & 7))) << 4) + (k & 7) * 2);
}

__device__ __forceinline__ uint32_t mnmajor_offset(int mn, int k) {
  return static_cast<uint32_t>((mn >> 6) * 8192 + k * 128 + (((((mn & 63) >> 3) ^ (k & 7))) << 4) +
                               (mn & 7) * 2);
}

// NH == 1: each tile is one BN-wide accumulator and two accumulators
// alternate in TMEM, so the epilogue of one tile overlaps the next tile's
// main loop.  NH == 2: each tile is 2*BN wide and fills TMEM with two
// BN-column halves; the epilogue hands half 0 back before draining half 1, so
// the next tile's MMAs into half 0 start while half 1 is still being stored.
//
// AT / BT select how the operands are stored.  AT == false: A is M x K
// row-major (K contiguous, a K-major operand); AT == true: the stored matrix
// is K x M row-major and the product uses its transpose (an MN-major
// operand).  BT == false: B is K x N row-major (MN-major operand); BT == true:
// the stored matrix is N x K row-major, transposed (K-major operand).
//
// LSU: the operands are loaded by kLoaderWarps extra warps with 2-byte global
// loads into the same swizzled shared-memory layouts, for strides and bases
// the TMA unit cannot describe; the tensor-core pipeline is unchanged.
//
// KS > 1 (one-CTA tiles only): a cluster of KS CTAs shares every tile, CTA s
// summing k-blocks [s*kb/KS, (s+1)*kb/KS).  The partial sums are reduced
// through distributed shared memory: each CTA finishes BN/KS of the tile's
// columns, receiving the other CTAs' fp32 partials of them into its own shared
// memory, and adds all KS slices in slice order before the epilogue.  No
// global scratch is needed, and the result does not depend on timing.
template <int CG, int BN, int STAGES, bool OUT_F16, int EK, int NH = 1, bool AT = false,
          bool BT = false, bool LSU = false, int KS = 1>
__global__ void __launch_bounds__(LSU ? kThreadsLsu : kThreads, 1)
    gemm_sm100_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmC,
                      const __grid_constant__ CUtensorMap tmR, const GemmParams p) {
  using Plan = SmemPlan<CG, BN, STAGES, NH, KS>;
  constexpr int kTileM = kBM * CG;
  constexpr int kTileN = BN * NH;
  static_assert(CG == 1 || CG == 2, "one CTA or a CTA pair per tile");
  static_assert(NH == 1 || NH == 2, "one accumulator per tile, or two halves");
  static_assert(!LSU || NH == 1, "the plain-load path is built for one-accumulator tiles");
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN must be 64, 128, 192 or 256");
  static_assert(KS == 1 || (CG == 1 && NH == 1 && !LSU), "the k-split is built for one-CTA TMA tiles");
  constexpr bool kCluster = CG == 2 || KS > 1;  // CTAs of a work unit form a cluster

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
  // k-split: this CTA's receive buffer is full (every peer wrote and arrived) / every
  // peer has consumed this CTA's partials from its own receive buffer.
  const uint32_t recv_full_bar = bar0 + 8u * (2 * STAGES + 5);
  const uint32_t send_free_bar = bar0 + 8u * (2 * STAGES + 6);
  // Bias in shared memory: every epilogue warp has written its share of the tile's
  // bias / has done reading it.
  const uint32_t bias_full_bar = bar0 + 8u * Plan::kNumBarsBase;
  const uint32_t bias_free_bar = bar0 + 8u * (Plan::kNumBarsBase + 1);
  // The last item's residual boxes have landed in the ring (see the producer).
  const uint32_t res_bar = bar0 + 8u * (Plan::kNumBars - 1);
  // Staging of the last tile's fp16 residual (fused epilogue, TMA path, whole tiles of one
  // accumulator): kResBoxes boxes of 32 rows x 64 columns (4 KB, 128-byte swizzle), box
  // j = quarter * kResPieces + piece, kResPerStage to a ring slot (its A part, then its B
  // part), starting at the first slot the producer would fill next.
  constexpr bool kResSmem = EK == kEpiFused && OUT_F16 && KS == 1 && NH == 1 && !LSU;
  constexpr int kResPieces = kTileN / 64;
  constexpr int kResBoxes = (kBM / 32) * kResPieces;
  constexpr int kResPerA = static_cast<int>(Plan::kABytes / 4096);
  constexpr int kResPerStage = kResPerA + static_cast<int>(Plan::kBBytes / 4096);
  constexpr int kResStages = (kResBoxes + kResPerStage - 1) / kResPerStage;
  static_assert(!kResSmem || kResStages <= STAGES, "the residual of a tile fits the ring");
  auto res_box = [&](int first_stage, int j) -> uint32_t {
    const int st = (first_stage + j / kResPerStage) % STAGES;
    const int b = j % kResPerStage;
    return b < kResPerA ? smem_u32(sA + st * Plan::kABytes) + static_cast<uint32_t>(b) * 4096u
                        : smem_u32(sB + st * Plan::kBBytes) + static_cast<uint32_t>(b - kResPerA) * 4096u;
  };
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + Plan::kMiscOffset);
  uint32_t *tmem_holder = misc;
  volatile uint32_t *abort_flag = misc + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Work unit = one tile per CTA group: a CTA (CG == 1), a cluster of two (CG == 2), or a
  // cluster of KS CTAs that split each tile's K range.
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
  const int kslice = (KS > 1) ? static_cast<int>(cluster_ctarank()) : 0;
  const int unit = kCluster ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int num_units = kCluster ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);
  const bool leader = rank == 0;
  const int num_m = (p.M + kTileM - 1) / kTileM;
  const int num_n = (p.N + kTileN - 1) / kTileN;
  const int num_kb = (p.K + kBK - 1) / kBK;
  const int n_work = work_count(p, unit, num_units);
  // The k-th work item of this unit; with a k-split, this CTA's slice of its k-blocks
  // (the host guarantees at least KS k-blocks, so no slice is empty).
  auto item = [&](int k) {
    WorkItem w = work_item(p, k, unit, num_units, num_m, num_n, num_kb);
    if constexpr (KS > 1) {
      w.kb0 = static_cast<int>(static_cast<int64_t>(kslice) * num_kb / KS);
      w.kb1 = static_cast<int>(static_cast<int64_t>(kslice + 1) * num_kb / KS);
    }
    return w;
  };

  // The k-blocks of a unit's item k in processing order: whole tiles walk K
  // ascending on even k and descending on odd k, so a tile starts on the k-blocks
  // the unit's previous tile (and its wave's) read last, which L2 still holds.
  // Tail slices, k-split slices and the plain-load path keep ascending order.
  auto kb_at = [&](const WorkItem &w, int k, int i) {
    const bool down = !LSU && KS == 1 && w.tail < 0 && (k & 1) != 0;
    return down ? w.kb1 - 1 - i : w.kb0 + i;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), LSU ? kLoaderWarps * CG : 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), kEpiWarps * CG);  // one arrive per epilogue warp of each CTA
    }
    mbar_init(drain_bar, 1);
    if constexpr (KS > 1) {
      mbar_init(recv_full_bar, (KS - 1) * 32 * kEpiWarps);  // every epilogue thread of each peer
      mbar_init(send_free_bar, (KS - 1) * 32 * kEpiWarps);
    }
    if constexpr (Plan::kBiasSmem) {
      mbar_init(bias_full_bar, kEpiWarps);  // lane 0 of each epilogue warp
      mbar_init(bias_free_bar, kEpiWarps);
    }
    mbar_init(res_bar, 1);  // the producer's one arrive, plus the boxes' bytes
    *abort_flag = 0u;
    fence_mbar_init();
    if constexpr (!LSU) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
    }
    if (!p.c_plain) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc<CG>(smem_u32(tmem_holder), Plan::kTmemCols);
    tmem_relinquish<CG>();
  }
  tc_fence_before_sync();
  __syncwarp();
  if constexpr (kCluster)
    cluster_sync_all();  // every CTA's barriers exist before any other signals them
  else
    __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tmem_holder);
  // Everything above touched only this CTA's shared memory and TMEM, so it may
  // overlap the previous kernel in the stream; global memory (A, B, bias, C,
  // the workspace) is touched only after that kernel has completed.
  grid_dependency_wait();
  grid_launch_dependents();

  if (!LSU && warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer (every CTA)
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_parity = 0;
    bool ok = true;
    for (int k = 0; k < n_work && ok; ++k) {
      const WorkItem w = item(k);
      const int a_row = w.mb * kTileM + static_cast<int>(rank) * kBM;
      const int b_col = w.nb * kTileN + static_cast<int>(rank) * Plan::kBNc;
      for (int i = 0; i < w.kb1 - w.kb0; ++i) {
        const int kb = kb_at(w, k, i);
        if (!mbar_wait_spin(empty_bar(stage), phase ^ 1u, abort_flag, p.limit_ns, kRoleProducer,
                       &g_device_error, 4096)) {
          ok = false;
          break;
        }
        const uint32_t a_dst = smem_u32(sA + stage * Plan::kABytes);
        const uint32_t b_dst = smem_u32(sB + stage * Plan::kBBytes);
        uint32_t bar;
        if constexpr (CG == 1) {
          bar = full_bar(stage);
          mbar_arrive_expect_tx(bar, Plan::kStageBytes);
        } else {
          // The leader's full barrier counts the bytes of both CTAs' loads.
          if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * Plan::kStageBytes);
          bar = mapa_shared(full_bar(stage), 0);
        }
        auto load = [&](uint32_t dst, const CUtensorMap *tm, int32_t x, int32_t y) {
          if constexpr (CG == 1)
            tma_load_2d(dst, tm, bar, x, y);
          else
            tma_load_2d_pair(dst, tm, bar, x, y);
        };
        // A tile: 128 rows x 64 k.  K-major: one box; MN-major: two 64-row boxes.
        if constexpr (!AT) {
          load(a_dst, &tmA, kb * kBK, a_row);
        } else {
          load(a_dst, &tmA, a_row, kb * kBK);
          load(a_dst + 8192, &tmA, a_row + 64, kb * kBK);
        }
        // B slice of each half: kBNc columns x 64 k.  MN-major: 64-column boxes;
        // K-major: one box of kBNc rows.
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if constexpr (!BT) {
#pragma unroll
            for (int c = 0; c < Plan::kBNc / 64; ++c)
              load(b_dst + h * Plan::kHalfBBytes + c * 8192, &tmB, b_col + h * BN + c * 64,
                   kb * kBK);
          } else {
            load(b_dst + h * Plan::kHalfBBytes, &tmB, kb * kBK, b_col + h * BN);
          }
        }
        issued_mask |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // The last item's fp16 residual: once the final k-blocks no longer need the ring
    // slots after them (their MMAs are done), those slots take the tile's residual rows,
    // loaded while the last MMAs run.  The epilogue of the last tile, which nothing
    // overlaps, then reads them from shared memory instead of waiting on DRAM.
    int res_stages = 0;
    if constexpr (kResSmem) {
      const WorkItem wl = item(n_work > 0 ? n_work - 1 : 0);
      if (ok && p.r_tma != 0 && n_work > 0 && wl.tail < 0) {
        const int first = stage;
        misc[2] = static_cast<uint32_t>(first);
        const int y0 = wl.mb * kTileM + static_cast<int>(rank) * kBM;
        for (int j = 0; j < kResBoxes && ok;) {
          if (!mbar_wait_spin(empty_bar(stage), phase ^ 1u, abort_flag, p.limit_ns, kRoleProducer,
                              &g_device_error, 4096)) {
            ok = false;
            break;
          }
          const int nbox = kResBoxes - j < kResPerStage ? kResBoxes - j : kResPerStage;
          mbar_expect_tx(res_bar, static_cast<uint32_t>(nbox) * 4096u);
          for (int b = 0; b < nbox; ++b, ++j)
            tma_load_2d(res_box(first, j), &tmR, res_bar,
                        wl.nb * kTileN + (j % kResPieces) * 64, y0 + (j / kResPieces) * 32);
          ++res_stages;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        mbar_arrive(res_bar);
        // Every box issued has landed before this CTA's shared memory goes away, whatever
        // the other roles do (no abort flag: the wait ends on the bytes or the limit).
        mbar_wait(res_bar, 0, nullptr, p.limit_ns, kRoleProducer, &g_device_error);
      }
    }
    if (ok) {
      // Tail: wait until every slot has been released, so no commit-arrive is
      // still on its way to this CTA's barriers when it exits (the slots that took
      // the residual were released before it went in).
      for (int i = 0; i < STAGES - res_stages; ++i) {
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
    constexpr uint32_t idesc = make_idesc_f16(kTileM, BN, AT, !BT);
    int stage = 0;
    uint32_t phase = 0;
    // Accumulator slots are the two BN-column halves of TMEM.  NH == 1: tiles
    // alternate between them (acc); NH == 2: every tile uses both.
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    // The MMAs of accumulator half h (h = 0 with NH == 1) for the k-block in ring slot st.
    // Descriptors of ring slot 0; another slot, half or 16-k step only moves the start
    // address, whose field (bits 0-13, in 16-byte units) never carries: shared-memory
    // offsets stay below 256 KB.  K-major: 16 k = 32 bytes along the swizzled row;
    // MN-major: 16 k = 16 rows of 128 bytes, 64-element blocks 8192 bytes apart.
    const uint64_t adesc0 = !AT ? smem_desc_sw128(smem_u32(sA), 16, 1024)
                                : smem_desc_sw128(smem_u32(sA), 8192, 1024);
    const uint64_t bdesc0 = !BT ? smem_desc_sw128(smem_u32(sB), 8192, 1024)
                                : smem_desc_sw128(smem_u32(sB), 16, 1024);
    constexpr uint32_t kAStep = !AT ? 32 / 16 : 16 * 128 / 16;  // per 16 k, in 16-byte units
    constexpr uint32_t kBStep = !BT ? 16 * 128 / 16 : 32 / 16;
    auto issue_half = [&](int st, int h, bool first_kb) {
      const uint64_t ad = adesc0 + static_cast<uint32_t>(st * Plan::kABytes / 16);
      const uint64_t bd =
          bdesc0 + static_cast<uint32_t>((st * Plan::kBBytes + h * Plan::kHalfBBytes) / 16);
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>((NH == 1 ? acc : h) * BN);
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk)
        mma_f16_ss<CG>(d_tmem, ad + kk * kAStep, bd + kk * kBStep, idesc,
                       (!first_kb || kk > 0) ? 1u : 0u);
    };
    for (int k = 0; k < n_work && ok; ++k) {
      const WorkItem w = item(k);
      if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.limit_ns, kRoleMma,
                     &g_device_error)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      // NH == 2: when this tile's first k-blocks land, the epilogue may still be draining
      // half 1 of the previous tile.  Their half-0 MMAs then run ahead (up to the ring's
      // depth, the slots held), and their half-1 MMAs follow in k order as soon as half 1
      // is handed back; only then are the slots released.  Each half still sums its
      // k-blocks in ascending order.
      bool half1_free = NH == 1;
      int pend = 0;        // k-blocks w.kb0 .. w.kb0 + pend - 1: half 0 issued, half 1 not yet
      int pend_stage = 0;  // the ring slot of the first of them
      auto half1_ready = [&]() {
        tc_fence_after_sync();
        half1_free = true;
        int st = pend_stage;
        for (int i = 0; i < pend; ++i) {
          issue_half(st, 1, i == 0);
          mma_commit<CG>(empty_bar(st));
          if (++st == STAGES) st = 0;
        }
        pend = 0;
      };
      for (int i = 0; i < w.kb1 - w.kb0; ++i) {
        if (NH == 2 && !half1_free && pend == STAGES) {
          // every slot holds a run-ahead k-block: nothing more can land before half 1 is free
          if (!mbar_wait(tempty_bar(1), acc_phase ^ 1u, abort_flag, p.limit_ns, kRoleMma,
                         &g_device_error)) {
            ok = false;
            break;
          }
          half1_ready();
        }
        if (!mbar_wait_spin(full_bar(stage), phase, abort_flag, p.limit_ns, kRoleMma,
                       &g_device_error, 4096)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        if (NH == 2 && !half1_free && mbar_test_wait(tempty_bar(1), acc_phase ^ 1u)) half1_ready();
        if (NH == 2 && !half1_free) {
          if (pend == 0) pend_stage = stage;
          issue_half(stage, 0, i == 0);
          ++pend;
        } else {
#pragma unroll
          for (int h = 0; h < NH; ++h) issue_half(stage, h, i == 0);
          mma_commit<CG>(empty_bar(stage));
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && NH == 2 && !half1_free) {
        // a tile shorter than the epilogue's half 1: finish its half-1 MMAs now
        if (!mbar_wait(tempty_bar(1), acc_phase ^ 1u, abort_flag, p.limit_ns, kRoleMma,
                       &g_device_error))
          ok = false;
        else
          half1_ready();
      }
      if (!ok) break;
      mma_commit<CG>(tfull_bar(acc));
      if (NH == 1) {
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      } else {
        acc_phase ^= 1u;  // both halves' barriers complete once per tile
      }
    }
    if (!ok) {
      // Wait for the MMAs already in flight before TMEM and shared memory are released.
      mma_commit_local<CG>(drain_bar);
      mbar_wait(drain_bar, 0, nullptr, p.limit_ns, kRoleMma, &g_device_error);
    }
  } else if (LSU && warp >= 2 + kEpiWarps) {
    // ---------------------------------------------------------------- plain loaders (every CTA)
    // Each loader warp fills a quarter of every A and B stage, two elements
    // per lane along the stored matrix's contiguous dimension (coalesced),
    // then makes its shared-memory writes visible to the tensor core and
    // arrives on the slot's full barrier (the pair leader's, with CG == 2).
    const int lw = warp - (2 + kEpiWarps);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int k = 0; k < n_work && ok; ++k) {
      const WorkItem w = item(k);
      const int a_row = w.mb * kTileM + static_cast<int>(rank) * kBM;
      const int b_col = w.nb * kTileN + static_cast<int>(rank) * Plan::kBNc;
      for (int kb = w.kb0; kb < w.kb1; ++kb) {
        int got = 1;
        if (lane == 0)
          got = mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.limit_ns, kRoleProducer,
                          &g_device_error);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        const uint32_t a_dst = smem_u32(sA + stage * Plan::kABytes);
        const uint32_t b_dst = smem_u32(sB + stage * Plan::kBBytes);
        const int k0 = kb * kBK;
        const int kk2 = 2 * lane;  // this lane's pair along a 64-element row
        // This warp's share of the stage: NA values of A and NB of B (two
        // elements each).  All loads are issued before any store, so one
        // memory latency covers the whole stage.
        constexpr int NA = 32;                                       // A: 32 rows, or 16 k rows x 2
        constexpr int NB = !BT ? 16 * (Plan::kBNc / 64) : Plan::kBNc / kLoaderWarps;
        uint32_t va[NA], vb[NB];
#pragma unroll
        for (int j = 0; j < NA; ++j) {
          if constexpr (!AT)  // A stored M x K: rows lw*32 .. +31, 64 k each
            va[j] = load_pair(p.A, a_row + lw * 32 + j, k0 + kk2, p.lda, p.M, p.K);
          else  // A stored K x M: k rows lw*16 .. +15, 128 m each in two passes
            va[j] = load_pair(p.A, k0 + lw * 16 + (j & 15), a_row + (j >> 4) * 64 + kk2, p.lda,
                              p.K, p.M);
        }
#pragma unroll
        for (int j = 0; j < NB; ++j) {
          if constexpr (!BT)  // B stored K x N: k rows lw*16 .. +15, kBNc columns in 64s
            vb[j] = load_pair(p.B, k0 + lw * 16 + (j & 15), b_col + (j >> 4) * 64 + kk2, p.ldb,
                              p.K, p.N);
          else  // B stored N x K: n rows j*4 + lw, 64 k each
            vb[j] = load_pair(p.B, b_col + j * kLoaderWarps + lw, k0 + kk2, p.ldb, p.N, p.K);
        }
#pragma unroll
        for (int j = 0; j < NA; ++j) {
          if constexpr (!AT)
            st_shared_u32(a_dst + kmajor_offset(lw * 32 + j, kk2), va[j]);
          else
            st_shared_u32(a_dst + mnmajor_offset((j >> 4) * 64 + kk2, lw * 16 + (j & 15)), va[j]);
        }
#pragma unroll
        for (int j = 0; j < NB; ++j) {
          if constexpr (!BT)
            st_shared_u32(b_dst + mnmajor_offset((j >> 4) * 64 + kk2, lw * 16 + (j & 15)), vb[j]);
          else
            st_shared_u32(b_dst + kmajor_offset(j * kLoaderWarps + lw, kk2), vb[j]);
        }
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          if constexpr (CG == 1)
            mbar_arrive(full_bar(stage));
          else
            mbar_arrive_cluster(mapa_shared(full_bar(stage), 0));
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // Tail: every slot released, so no commit-arrive is still on its way.
    if (ok && lane == 0) {
      for (int i = 0; i < STAGES; ++i) {
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.limit_ns, kRoleProducer,
                       &g_device_error))
          break;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    __syncwarp();
  } else if (warp >= 2 && warp < 2 + kEpiWarps) {
    // ---------------------------------------------------------------- epilogue (every CTA)
    // Warp w drains TMEM lanes 32*(w%4) .. +31 (the lanes a warp may access),
    // 64 accumulator columns at a time, into two 4 KB boxes it owns in turn.
    const int quarter = warp & 3;
    const int box_row0_in_tile = static_cast<int>(rank) * kBM + quarter * 32;
    const uint32_t box0 = smem_u32(smem + Plan::kOutOffset) +
                          static_cast<uint32_t>((warp - 2) * 2) * kStageOutBytes;
    const uint32_t release_bar0 = (CG == 2) ? mapa_shared(tempty_bar(0), 0) : tempty_bar(0);
    constexpr int kOutEsz = OUT_F16 ? 2 : 4;
    constexpr int kBoxCols = 128 / kOutEsz;  // 64 fp16 or 32 fp32 columns per box
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t boxes_used = 0;

    // Fused epilogue (bias, activation, residual: inputs prefetched in `in`),
    // output rounding and the store of one 32-row x 64-column piece (this
    // lane's row, columns col0 .. col0+63).  next_col0 >= 0: once `in` is
    // used, load the epilogue inputs of the piece at next_col0 into it, so
    // their latency passes while this piece is stored.
    constexpr int kCPL = kTileN / 32;  // bias columns per lane
    constexpr bool kPrefR = EK == kEpiFused && OUT_F16 && !LSU;  // residual pieces loaded ahead
    // The tile's bias in fp32 in shared memory (where the plan has room for it), else
    // spread over the lanes as fp16 and fetched by shuffles.
    constexpr bool kSBias = EK != kEpiNone && Plan::kBiasSmem;
    const uint32_t sbias = smem_u32(smem + Plan::kBiasOffset);
    // The epilogue of one 32-column half of a piece (tile columns tcol + 32*half ..).
    // bias + ReLU (fp16 C only) leaves the ReLU to the packing.
    static_assert(EK != kEpiBiasRelu || OUT_F16, "the bias + ReLU build writes fp16");
    auto epi32 = [&](const EpiIn<kPrefR> &in, const BiasSlice<kCPL> &bias, int row, int col0,
                     int tcol, int half, float(&v)[32]) {
      if constexpr (EK == kEpiFused) {
        epi_apply_32<OUT_F16, kPrefR, kSBias, kCPL>(p, in, bias, sbias, row, col0, tcol, half, v);
      } else if constexpr (EK == kEpiBiasRelu) {
        if constexpr (kSBias)
          add_bias_smem_32(sbias, tcol + 32 * half, v);
        else
          add_bias_slice_32<kCPL>(bias, tcol + 32 * half, v);
      }
    };
    // The residual pieces of the unit's last tile come from the ring (kResSmem, staged
    // by the producer); every other piece is loaded from R by epi_prefetch.
    bool r_smem = false;
    uint32_t res_first = 0;
    auto fetch_r = [&](int row, int col0, EpiIn<kPrefR> &in) {
      if constexpr (kResSmem) {
        if (r_smem) {
          in.has_r = p.R != nullptr && col0 + 64 <= p.N && row < p.M;
          if (in.has_r) {
            const uint32_t box = res_box(static_cast<int>(res_first),
                                         quarter * kResPieces + (col0 % kTileN) / 64) +
                                 static_cast<uint32_t>(lane) * 128u;
#pragma unroll
            for (int c = 0; c < 8; ++c) in.r[c] = ld_shared_v4(box + static_cast<uint32_t>((c ^ (lane & 7)) * 16));
          }
          return;
        }
      }
      epi_prefetch<kPrefR>(p, row, col0, in);
    };
    auto pack = [&](float lo, float hi) {
      if constexpr (EK == kEpiBiasRelu)
        return pack_half2_relu(lo, hi);
      else
        return pack_half2(lo, hi);
    };
    auto emit64 = [&](float (&va)[32], float (&vb)[32], int box_row0, int col0, int tcol,
                      const BiasSlice<kCPL> &bias, EpiIn<kPrefR> &in, int next_col0) {
      if constexpr (OUT_F16) {
        uint32_t h[32];  // 64 fp16 values, round to nearest even
        epi32(in, bias, box_row0 + lane, col0, tcol, 0, va);
#pragma unroll
        for (int j = 0; j < 16; ++j) h[j] = pack(va[2 * j], va[2 * j + 1]);
        epi32(in, bias, box_row0 + lane, col0, tcol, 1, vb);
#pragma unroll
        for (int j = 0; j < 16; ++j) h[16 + j] = pack(vb[2 * j], vb[2 * j + 1]);
        if constexpr (kPrefR) {
          if (next_col0 >= 0) fetch_r(box_row0 + lane, next_col0, in);
        }
        if (p.c_plain || (!p.n_aligned && col0 + kBoxCols > p.N)) {
          store_row_tail<true>(p, box_row0 + lane, col0, h);
          return;
        }
        const uint32_t box = box0 + (boxes_used & 1u) * kStageOutBytes;
        if (lane == 0) bulk_wait_group_read<1>();  // this box's previous store has read it
        __syncwarp();
        st_box_row(box, lane, h, 0);
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmC, box, col0, box_row0);
          bulk_commit_group();
        }
        ++boxes_used;
      } else {
        epi32(in, bias, box_row0 + lane, col0, tcol, 0, va);
        epi32(in, bias, box_row0 + lane, col0, tcol, 1, vb);
        if constexpr (kPrefR) {
          if (next_col0 >= 0) fetch_r(box_row0 + lane, next_col0, in);
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (col0 + half * kBoxCols >= p.N) break;
          uint32_t w[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(half == 0 ? va[j] : vb[j]);
          if (p.c_plain || (!p.n_aligned && col0 + half * kBoxCols + kBoxCols > p.N)) {
            store_row_tail<false>(p, box_row0 + lane, col0 + half * kBoxCols, w);
            continue;
          }
          const uint32_t box = box0 + (boxes_used & 1u) * kStageOutBytes;
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          st_box_row(box, lane, w, 0);
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmC, box, col0 + half * kBoxCols, box_row0);
            bulk_commit_group();
          }
          ++boxes_used;
        }
      }
    };

    // k-split (KS > 1): the reduction of one tile through distributed shared memory.
    // Receive buffer of a CTA: one slot per peer (in rank order, skipping itself); in a
    // slot, for epilogue warp w, 32-column chunk c and 4-column group g, lane l's 16
    // bytes sit at ((w * kOwn / 32 + c) * 8 + g) * 512 + l * 16, so each warp-wide
    // 16-byte store or load covers 512 contiguous bytes.
    uint32_t recv_parity = 0, free_parity = 0;
    auto ks_tile = [&](const WorkItem &w, int box_row0, const BiasSlice<kCPL> &bias,
                       EpiIn<kPrefR> &in) -> bool {
      constexpr int kOwn = Plan::kOwnCols;
      const uint32_t recv0 = smem_u32(smem + Plan::kRecvOffset);
      const uint32_t tmem_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                static_cast<uint32_t>(acc * BN);
      const uint32_t warp_off = static_cast<uint32_t>(quarter * (kOwn / 32)) * 4096u +
                                static_cast<uint32_t>(lane) * 16u;
      // 1. This CTA's partial of every peer's columns, into that peer's receive buffer,
      //    once every peer has consumed the previous tile's.
      if (!mbar_wait_cluster(send_free_bar, free_parity ^ 1u, abort_flag, p.limit_ns,
                             kRoleEpilogue, &g_device_error))
        return false;
      free_parity ^= 1u;
#pragma unroll 1
      for (int q = 0; q < KS; ++q) {
        if (q == kslice) continue;
        const uint32_t dst = mapa_shared(recv0, static_cast<uint32_t>(q)) +
                             static_cast<uint32_t>(kslice < q ? kslice : kslice - 1) *
                                 Plan::kRecvSlotBytes +
                             warp_off;
#pragma unroll 1
        for (int c = 0; c < kOwn; c += 32) {
          uint32_t r[32];
          __syncwarp();
          tmem_load_32cols(tmem_row + static_cast<uint32_t>(q * kOwn + c), r);
#pragma unroll
          for (int g = 0; g < 8; ++g)
            st_cluster_v4(dst + static_cast<uint32_t>(c / 32) * 4096u + g * 512u, r[4 * g],
                          r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]);
        }
        mbar_arrive_cluster(mapa_shared(recv_full_bar, static_cast<uint32_t>(q)));
      }
      // 2. This CTA's own columns: wait for the peers' partials, add the KS slices in
      //    slice order, then the epilogue and the store of each 64-column piece.
      if (!mbar_wait_cluster(recv_full_bar, recv_parity, abort_flag, p.limit_ns, kRoleEpilogue,
                             &g_device_error))
        return false;
      recv_parity ^= 1u;
#pragma unroll 1
      for (int tc = 0; tc < kOwn; tc += 64) {
        const int tcol = kslice * kOwn + tc;  // column within the tile
        const int col0 = w.nb * kTileN + tcol;
        uint32_t ra[32], rb[32];
        __syncwarp();
        tmem_load_2x32cols(tmem_row + static_cast<uint32_t>(tcol), ra, rb);
        if (tc + 64 >= kOwn) {
          // last read of this accumulator: hand it back to the MMA warp
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty_bar(acc));
        }
        if (box_row0 >= p.M || col0 >= p.N) continue;  // the whole 32 x 64 piece is clipped
        float va[32], vb[32];
#pragma unroll 1
        for (int sl = 0; sl < KS; ++sl) {
          if (sl == kslice) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              va[j] = sl == 0 ? __uint_as_float(ra[j]) : va[j] + __uint_as_float(ra[j]);
              vb[j] = sl == 0 ? __uint_as_float(rb[j]) : vb[j] + __uint_as_float(rb[j]);
            }
          } else {
            const uint32_t src = recv0 +
                                 static_cast<uint32_t>(sl < kslice ? sl : sl - 1) * Plan::kRecvSlotBytes +
                                 warp_off + static_cast<uint32_t>(tc / 32) * 4096u;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              const uint4 xa = ld_shared_v4(src + g * 512u);
              const uint4 xb = ld_shared_v4(src + 4096u + g * 512u);
              const float fa[4] = {__uint_as_float(xa.x), __uint_as_float(xa.y), __uint_as_float(xa.z),
                                   __uint_as_float(xa.w)};
              const float fb[4] = {__uint_as_float(xb.x), __uint_as_float(xb.y), __uint_as_float(xb.z),
                                   __uint_as_float(xb.w)};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                va[4 * g + e] = sl == 0 ? fa[e] : va[4 * g + e] + fa[e];
                vb[4 * g + e] = sl == 0 ? fb[e] : vb[4 * g + e] + fb[e];
              }
            }
          }
        }
        const int next_col0 = (tc + 64 < kOwn && col0 + 64 < p.N) ? col0 + 64 : -1;
        emit64(va, vb, box_row0, col0, tcol, bias, in, next_col0);
      }
      // Every read of the receive buffer is done: the peers may write it again.
#pragma unroll 1
      for (int q = 0; q < KS; ++q)
        if (q != kslice) mbar_arrive_cluster(mapa_shared(send_free_bar, static_cast<uint32_t>(q)));
      return true;
    };

    for (int k = 0; k < n_work; ++k) {
      const WorkItem w = item(k);
      const int box_row0 = w.mb * kTileM + box_row0_in_tile;
      // The tile's bias and the first piece's residual load while the main
      // loop still runs.
      EpiIn<kPrefR> in;
      BiasSlice<kCPL> bias;
      if constexpr (kSBias) {
        if (p.bias != nullptr) {
          // The shared bias buffer holds one tile's bias: once every epilogue warp is
          // done with the previous tile's, each writes its share of this tile's.
          if (k > 0 && !mbar_wait(bias_free_bar, (k - 1) & 1, abort_flag, p.limit_ns,
                                  kRoleEpilogue, &g_device_error))
            break;
          float *sb = reinterpret_cast<float *>(smem + Plan::kBiasOffset);
          for (int c = (warp - 2) * 32 + lane; c < kTileN; c += 32 * kEpiWarps) {
            const int col = w.nb * kTileN + c;
            sb[c] = col < p.N ? __half2float(p.bias[col]) : 0.0f;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bias_full_bar);
          if (!mbar_wait(bias_full_bar, k & 1, abort_flag, p.limit_ns, kRoleEpilogue,
                         &g_device_error))
            break;
        }
      } else if constexpr (EK != kEpiNone) {
        if (p.bias != nullptr && w.nb * kTileN < p.N) load_bias_slice<kCPL>(p, w.nb * kTileN, lane, bias);
      }
      r_smem = kResSmem && p.r_tma != 0 && k + 1 == n_work && w.tail < 0;
      const int first_col = w.nb * kTileN + (KS > 1 ? kslice * Plan::kOwnCols : 0);
      if constexpr (kPrefR) {
        if (!r_smem && w.tail < 0 && box_row0 < p.M && first_col < p.N)
          epi_prefetch<kPrefR>(p, box_row0 + lane, first_col, in);
      }
      // This wait spans the tile's whole main loop, so its limit grows with the
      // tile's k-blocks (20 us each, far above a k-block's time on any built
      // tile, the plain-load path included): a long K is not a stalled pipeline.
      const uint64_t tile_limit_ns =
          p.limit_ns + static_cast<uint64_t>(w.kb1 - w.kb0) * kWaitPerKBlockNs;
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag, tile_limit_ns, kRoleEpilogue,
                     &g_device_error))
        break;
      tc_fence_after_sync();
      if constexpr (kResSmem) {
        if (r_smem) {
          if (!mbar_wait(res_bar, 0, abort_flag, p.limit_ns, kRoleEpilogue, &g_device_error)) break;
          res_first = *reinterpret_cast<volatile uint32_t *>(misc + 2);
          if (box_row0 < p.M && first_col < p.N) fetch_r(box_row0 + lane, first_col, in);
        }
      }
      if constexpr (KS > 1) {
        if (!ks_tile(w, box_row0, bias, in)) break;
      } else {
      // A k-slice of a tail tile writes its fp32 partial (this warp's 32 rows x
      // kTileN columns, column by column so each store is 128 contiguous bytes).
      float *part = nullptr;
      if (w.tail >= 0)
        part = p.ws + static_cast<int64_t>(((w.tail * p.split + w.slice) * CG + static_cast<int>(rank)) * 4 +
                                           quarter) * (32 * kTileN);
      // Pass 0 drains the accumulator: it stores the tile, or writes a tail
      // slice's partial.  Pass 1 runs only in the warp that completes a tail
      // tile's count: it sums every slice's partial in slice order (a fixed
      // order: the result does not depend on which slice finished last) and
      // stores the tile piece.  Both passes share one copy of the epilogue.
      uint32_t *counter = nullptr;
      const float *part0 = nullptr;
      const int64_t slice_stride = static_cast<int64_t>(CG) * 4 * 32 * kTileN;
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        if (pass == 1) {
          if (part == nullptr) break;
          counter = p.counters + (w.tail * CG + static_cast<int>(rank)) * 4 + quarter;
          __syncwarp();
          uint32_t before = 0;
          if (lane == 0) {
            __threadfence();
            before = atomicAdd(counter, 1u);
          }
          before = __shfl_sync(0xffffffffu, before, 0);
          if (before != static_cast<uint32_t>(p.split - 1)) break;
          __threadfence();
          part0 = p.ws + static_cast<int64_t>(((w.tail * p.split) * CG + static_cast<int>(rank)) * 4 +
                                              quarter) * (32 * kTileN);
          if constexpr (kPrefR) {
            if (box_row0 < p.M && w.nb * kTileN < p.N)
              epi_prefetch<kPrefR>(p, box_row0 + lane, w.nb * kTileN, in);
          }
        }
#pragma unroll 1
        for (int tc = 0; tc < kTileN; tc += 64) {
          const int col0 = w.nb * kTileN + tc;
          float va[32], vb[32];
          if (pass == 0) {
            const int slot = NH == 1 ? acc : tc / BN;  // TMEM half holding these columns
            const int ch = tc % BN;
            uint32_t ra[32], rb[32];
            __syncwarp();
            tmem_load_2x32cols(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(slot * BN + ch),
                               ra, rb);
            if (ch + 64 >= BN) {
              // Last read of this accumulator half: hand it back to the MMA warp
              // now, before the stores, so the next tile's main loop can start.
              tc_fence_before_sync();
              __syncwarp();
              if (lane == 0) {
                if constexpr (CG == 2)
                  mbar_arrive_cluster(release_bar0 + 8u * slot);
                else
                  mbar_arrive(release_bar0 + 8u * slot);
              }
            }
            if (part != nullptr) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                st_global_cg(part + (tc + j) * 32 + lane, __uint_as_float(ra[j]));
                st_global_cg(part + (tc + 32 + j) * 32 + lane, __uint_as_float(rb[j]));
              }
              continue;
            }
            if (box_row0 >= p.M || col0 >= p.N) continue;  // the whole 32 x 64 piece is clipped
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              va[j] = __uint_as_float(ra[j]);
              vb[j] = __uint_as_float(rb[j]);
            }
          } else {
            if (box_row0 >= p.M || col0 >= p.N) continue;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              va[j] = ld_global_cg(part0 + (tc + j) * 32 + lane);
              vb[j] = ld_global_cg(part0 + (tc + 32 + j) * 32 + lane);
            }
            for (int sl = 1; sl < p.split; ++sl) {
              const float *ps = part0 + sl * slice_stride;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                va[j] += ld_global_cg(ps + (tc + j) * 32 + lane);
                vb[j] += ld_global_cg(ps + (tc + 32 + j) * 32 + lane);
              }
            }
          }
          const int next_col0 = (tc + 64 < kTileN && col0 + 64 < p.N) ? col0 + 64 : -1;
          emit64(va, vb, box_row0, col0, tc, bias, in, next_col0);
        }
        if (pass == 1) {
          __syncwarp();
          if (lane == 0) atomicExch(counter, 0u);  // ready for the next call
        }
      }
      }  // KS == 1
      if constexpr (kSBias) {
        if (p.bias != nullptr) {
          __syncwarp();
          if (lane == 0) mbar_arrive(bias_free_bar);  // this warp is done with the tile's bias
        }
      }
      if (NH == 1) {
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      } else {
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait_group<0>();  // every store of this warp has completed
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncwarp();
  if constexpr (kCluster)
    cluster_sync_all();  // no CTA leaves while a peer may still touch its shared memory
  else
    __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc<CG>(tmem_base, Plan::kTmemCols);
  }
}

// K == 0, where the sum over k is empty: C = 0, or with the fused epilogue
// C = act(bias[col]) + R[row, col] (each element read and written by one thread).
template <bool OUT_F16, bool EPI>
__global__ void fill_empty_k_kernel(void *C, int64_t ldc, const __half *bias, int act,
                                    const void *R, int64_t ldr, int M, int N) {
  const int64_t total = static_cast<int64_t>(M) * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / N, c = i % N;
    float v = 0.0f;
    if constexpr (EPI) {
      if (bias != nullptr) v = __half2float(bias[c]);
      v = activate<OUT_F16>(act, v);
      if (R != nullptr)
        v += OUT_F16 ? __half2float(static_cast<const __half *>(R)[r * ldr + c])
                     : static_cast<const float *>(R)[r * ldr + c];
    }
    if constexpr (OUT_F16)
      reinterpret_cast<__half *>(C)[r * ldc + c] = __float2half_rn(v);
    else
      reinterpret_cast<float *>(C)[r * ldc + c] = v;
  }
}

}  // namespace tlg
