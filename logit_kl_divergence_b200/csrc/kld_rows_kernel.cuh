// kld_rows_kernel.cuh -- fused single-pass row kernel for sm_100a (device code,
// instantiated by kld_rows.cu and, with the top-k scan, by kld_rows_scan.cu).
//
// For every row i it reads base b[i, :] and quant q[i, :] from HBM exactly
// once and produces KL(P_base || P_quant) over the full vocabulary, the
// lowest-index argmax of both rows and, with token ids, the quantized row's
// NLL of the given token ("Qwen3.6 27B Quantization Benchmark", sections
// "Measurement method" and "Understand KLD and Same Top P"; direction and
// full vocabulary from "Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S GGUF", "How it
// was made", step 5).
//
// Streaming form of the statistic. With p = softmax(b), r = softmax(q) and
// the exact per-element log-ratio x_j = (q_j - b_j) + K (K: any constant),
//   KL = sum_j p_j (log p_j - log r_j) = -E_p[x] + ln E_p[e^x]
//      = -A/S + log1p(B/S),   S = sum e_j,  A = sum e_j x_j,
//                             B = sum e_j (e^x_j - 1) = sum (h_j - e_j),
// where e_j = 2^(b_j*L - R_b) are base weights in a frame R_b near the row
// maximum and h_j = e_j e^x_j the matching quant weights. When the two rows
// are close, A/S and log1p(B/S) are both O(sigma) and cancel to O(sigma^2),
// so B is split as B = A + C with C = sum e_j phi(x_j), phi(y) = e^y - 1 - y
// evaluated by a fitted polynomial (see phi_poly_fit.py): every term keeps
// ~1e-7 relative accuracy and rounding errors of the exponentials enter only
// at second order; each chunk uses the cheapest of three polynomial tiers
// whose range holds all its |x|. Chunks where some |x| > 2.5 (or x is not
// finite: masked or infinite entries) take a direct path that sums
// h_j = 2^(q_j*L - R_q) with its own exponential instead. K follows (b - q)
// at the element that last moved the frame (per warp: the frame moves when a
// chunk's maximum of b passes the previous one by more than four nats), so x
// is ~0 where the base mass sits and the split keeps its accuracy for peaked
// rows; moving K by d is an exact rebase in fp64:
// A += d*S, C -> e^{ld} C + (e^{ld} - 1) l A + (e^{ld} - 1 - l d) S. L = log2(e)
// rounded to fp32; all exponentials are of lambda*y with lambda = L*ln2
// = 1 + 1.4e-8, i.e. the statistic of softmax(lambda*b) and softmax(lambda*q),
// within 3e-8 relative of the exact one.
//
// Structure (whole rows: one CTA per SM, persistent over rows
// r = blockIdx.x + k*grid; split rows, for the last partial wave or a few
// rows: a CTA takes a contiguous run of a row's 512-element chunks, and the
// parts merge through global memory or in shared memory of a cluster):
//   - warp 16 (producer): one lane streams the 16-byte-aligned body of each
//     row pair in 32 KB tiles per operand into a 3-stage shared-memory ring
//     with cp.async.bulk (no multicast) completing on mbarriers, running
//     ahead across row boundaries.
//   - warps 0..15 (consumers): 512-element chunks (16 elements per lane,
//     conflict-free 16-byte shared loads): lane maxima, a vote on whether
//     the frame must move (then the warp maximum and a warp-uniform rebase),
//     then the fp32 terms of the chunk folded into per-lane fp64
//     accumulators. Each lane also remembers the first chunk in which its
//     own maxima appeared. At the end of a row each warp reduces its
//     accumulators and exact maxima and publishes them in a 4-slot shared
//     ring, then goes on with the next row.
//   - warp 17 (epilogue): per row, the unaligned head/tail (< 16 bytes each)
//     and the token gather, the exact lowest-index argmax (re-reading only
//     the chunks of lanes whose maximum equals the row maximum), the fp64
//     combine of the 17 partials and the 40-byte record.
//   All waits are mbarrier waits bounded by wall time; a wait that gives up
//   sets an error bit that the reduction reports, and the CTA leaves only
//   after its bulk copies have landed.
// 16-bit quant rows stay packed in the consumers (see Packed). The top-k
// scan form (kld_rows_kernel<DT, true>, see TopkScan; instantiated in
// kld_rows_scan.cu) also copies out the lanes holding candidates and sums
// the rest masses of the others.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <climits>

#include "kld_finish.cuh"
#include "kld_internal.h"

namespace kld {
namespace {

constexpr float kLog2e = 1.4426950408889634f;  // log2(e) rounded to fp32
constexpr double kLog2eD = static_cast<double>(kLog2e);
constexpr double kLn2 = 0.6931471805599453;  // ln(2)
constexpr double kLambda = kLog2eD * kLn2;   // 1 + 1.4e-8
constexpr float kBig = 1.0e30f;
constexpr float kTau = 2.5f;                 // |x| bound of the polynomial path
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// phi(y) = y^2 * P(y), P fitted by phi_poly_fit.py in three tiers, the
// cheapest whose range holds every |x| of a chunk being used (max relative
// error of phi in fp32 evaluation):
//   tier A: degree 5 on [-1, 1]     (1.7e-6)
//   tier B: degree 6 on [-1.5, 1.5] (1.6e-6)
//   tier C: degree 8 on [-2.5, 2.5] (9.0e-7)
// The kernel evaluates phi(lambda*x) = x^2 * Q(x), Q_k = P_k * lambda^(k+2).
constexpr float kTauA = 1.0f, kTauB = 1.5f;
constexpr double kPA[6] = {0.5000007367, 0.1666656843, 0.0416529078,
                           0.008336109943, 0.001426139768, 0.0001990834212};
constexpr double kPB[7] = {0.5000002972, 0.1666698525, 0.0416645243, 0.008321388792,
                           0.001390665576, 0.0002093027501, 2.499857965e-05};
constexpr double kP0 = 0.4999997655, kP1 = 0.1666656346, kP2 = 0.0416678794,
                 kP3 = 0.008335872564, kP4 = 0.00138800956, kP5 = 0.0001968192101,
                 kP6 = 2.495779646e-05, kP7 = 3.111933302e-06, kP8 = 2.814820757e-07;
constexpr double lam_pow(int n) { return n == 0 ? 1.0 : kLambda * lam_pow(n - 1); }
constexpr float kQ0 = static_cast<float>(kP0 * lam_pow(2));
constexpr float kQ1 = static_cast<float>(kP1 * lam_pow(3));
constexpr float kQ2 = static_cast<float>(kP2 * lam_pow(4));
constexpr float kQ3 = static_cast<float>(kP3 * lam_pow(5));
constexpr float kQ4 = static_cast<float>(kP4 * lam_pow(6));
constexpr float kQ5 = static_cast<float>(kP5 * lam_pow(7));
constexpr float kQ6 = static_cast<float>(kP6 * lam_pow(8));
constexpr float kQ7 = static_cast<float>(kP7 * lam_pow(9));
constexpr float kQ8 = static_cast<float>(kP8 * lam_pow(10));

constexpr int kProducerWarp = kConsumerWarps;

// ------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `parity` to complete; gives up after kWaitLimitNs or
// as soon as another thread of the CTA has raised *abort.
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort,
                                            uint64_t limit_ns = kWaitLimitNs) {
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort) return false;
      if (globaltimer() - t0 > limit_ns) return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  return mbar_try_wait(bar, parity) || mbar_wait_slow(bar, parity, abort);
}
// For the producer and epilogue warps, which spend most of their time
// waiting: each probe suspends the thread for up to kIdleSuspendNs (it wakes
// as soon as the phase completes), so the waiting warp does not take issue
// slots from the consumer warps on its scheduler.
constexpr uint32_t kIdleSuspendNs = 2000;
__device__ __forceinline__ bool mbar_try_wait_idle(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kIdleSuspendNs)
      : "memory");
  return ok != 0;
}
__device__ __noinline__ bool mbar_wait_idle(uint32_t bar, uint32_t parity, volatile int* abort) {
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_idle(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > kWaitLimitNs) return false;
  }
}
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float warp_max(float x) {
  float y;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}
// Packed pairs of fp32 (sm_100 f32x2 arithmetic: one issue slot for two
// lanes of FMA-pipe work).
struct f2 {
  unsigned long long v;
};
__device__ __forceinline__ f2 pk(float a, float b) {
  f2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk(f2 x, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(x.v));
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
  f2 r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}
__device__ __forceinline__ f2 sub2(f2 a, f2 b) {
  f2 r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
  f2 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
  f2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r.v) : "l"(a.v), "l"(b.v), "l"(c.v));
  return r;
}
__device__ __forceinline__ f2 splat(float a) { return pk(a, a); }

// phi(lambda*x) / x^2 by Horner (scalar and packed).
__device__ __forceinline__ float phi_q(float x) {
  float q = fmaf(kQ8, x, kQ7);
  q = fmaf(q, x, kQ6);
  q = fmaf(q, x, kQ5);
  q = fmaf(q, x, kQ4);
  q = fmaf(q, x, kQ3);
  q = fmaf(q, x, kQ2);
  q = fmaf(q, x, kQ1);
  return fmaf(q, x, kQ0);
}
// The coefficients Q_k as (c, c) pairs in constant memory (packed FMAs take
// no immediates): 6 for tier A, 7 for tier B, 9 for tier C.
constexpr float qa(int k) { return static_cast<float>(kPA[k] * lam_pow(k + 2)); }
constexpr float qb(int k) { return static_cast<float>(kPB[k] * lam_pow(k + 2)); }
__constant__ __align__(8) float kQpair[44] = {
    qa(0), qa(0), qa(1), qa(1), qa(2), qa(2), qa(3), qa(3), qa(4), qa(4), qa(5), qa(5),
    qb(0), qb(0), qb(1), qb(1), qb(2), qb(2), qb(3), qb(3), qb(4), qb(4), qb(5), qb(5),
    qb(6), qb(6),
    kQ0, kQ0, kQ1, kQ1, kQ2, kQ2, kQ3, kQ3, kQ4, kQ4, kQ5, kQ5, kQ6, kQ6, kQ7, kQ7, kQ8, kQ8};
__device__ __forceinline__ f2 qc(int k) {
  f2 r;
  r.v = reinterpret_cast<const unsigned long long*>(kQpair)[k];
  return r;
}
// Horner for tier T (0: A, 1: B, 2: C) on a packed pair.
template <int T>
__device__ __forceinline__ f2 phi_q2(f2 x) {
  constexpr int o = T == 0 ? 0 : (T == 1 ? 6 : 13);
  constexpr int nc = T == 0 ? 6 : (T == 1 ? 7 : 9);
  f2 q = fma2(qc(o + nc - 1), x, qc(o + nc - 2));
#pragma unroll
  for (int k = nc - 3; k >= 0; --k) q = fma2(q, x, qc(o + k));
  return q;
}

// Maximum that propagates NaN (so a NaN anywhere fails a "<= bound" test).
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float y;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}
// Maxima of N values as a tree of 3-input maxima (depth ~log3 N instead of
// a chain of N/2); plain (NaN-ignoring) and NaN-propagating.
template <int N, bool kNan>
__device__ __forceinline__ float tree_max(const float* v) {
  if constexpr (N == 1) {
    return v[0];
  } else if constexpr (N == 2) {
    return kNan ? max3_nan(v[0], v[1], v[1]) : fmaxf(v[0], v[1]);
  } else {
    constexpr int M = N / 3 + (N % 3 != 0 ? 1 : 0);
    float w[M];
#pragma unroll
    for (int i = 0; i < N / 3; ++i)
      w[i] = kNan ? max3_nan(v[3 * i], v[3 * i + 1], v[3 * i + 2])
                  : max3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
    if constexpr (N % 3 == 1) w[M - 1] = v[N - 1];
    if constexpr (N % 3 == 2)
      w[M - 1] = kNan ? max3_nan(v[N - 2], v[N - 1], v[N - 1]) : fmaxf(v[N - 2], v[N - 1]);
    return tree_max<M, kNan>(w);
  }
}

__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// ------------------------------------------------------------ element types

template <int DT>
struct Elem;

template <>
struct Elem<KLD_F32> {
  static constexpr int kBytes = 4;
  static constexpr int kPerVec = 4;
  __device__ static float load(const void* row, int64_t j) {
    return __ldg(static_cast<const float*>(row) + j);
  }
  __device__ static void unpack(const uint4& v, float* o) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
};

template <>
struct Elem<KLD_BF16> {
  static constexpr int kBytes = 2;
  static constexpr int kPerVec = 8;
  __device__ static float load(const void* row, int64_t j) {
    const unsigned short h = __ldg(static_cast<const unsigned short*>(row) + j);
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
  }
  // bf16 is the top half of an fp32: widening is a shift / mask.
  __device__ static void unpack(const uint4& v, float* o) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      o[2 * k] = __uint_as_float(w[k] << 16);
      o[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
};

template <>
struct Elem<KLD_F16> {
  static constexpr int kBytes = 2;
  static constexpr int kPerVec = 8;
  __device__ static float load(const void* row, int64_t j) {
    const unsigned short h = __ldg(static_cast<const unsigned short*>(row) + j);
    return __half2float(__ushort_as_half(h));
  }
  __device__ static void unpack(const uint4& v, float* o) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
      o[2 * k] = f.x;
      o[2 * k + 1] = f.y;
    }
  }
};

// ------------------------------------------------------------- per-row state

// Warp-uniform frames of one row operand pair.
// The base frame and centre move only when a chunk's maximum exceeds the
// one they were set at by more than kRaiseMargin nats (a few moves per row
// instead of one per new maximum; e stays below 2^(4L+1) ~ 2^6.8). Measured
// on rows with one dominant element at gaps of 0.1..14 nats and quant noise
// 0.001..0.1, the error against the oracle is the same as with a margin of
// 1 (<= 5e-9 absolute), while a margin of 8 raised it fourfold. The exact
// maximum of b is tracked per lane in Best and reduced when the warp
// publishes its partial.
constexpr float kRaiseMargin = 4.0f;
struct Ref {
  float Mb;   // maximum of b when the frame was last set (-inf before any)
  float Mqf;  // maximum of q over this warp's direct-path chunks (-inf before)
  float Rb, Rq;  // integer frames floor(M*L) once M is finite, 0 before
  float K;       // log-ratio centre: (b - q) at the element that set Mb
  float T;       // Mb + kRaiseMargin: a chunk maximum above it moves the frame
  int mode;      // order of the log-ratio's two roundings (see log_ratios)
};

// Order in which x = q - b + K is formed in fp32. For 16-bit inputs q - b is
// exact, so (q - b) + K rounds once. For fp32 inputs q - b rounds to half an
// ulp of |q - b|: rows whose logits are offset by a large constant (|K| >=
// kShiftForm) would lose ~1e-5 there, so the operand as large as K is paired
// with K first, which is then exact: (q + K) - b when |q| >= |b| at the
// element that set K, q - (b - K) otherwise.
__device__ __forceinline__ int ratio_form(float Mb, float K) {
  if (!(fabsf(K) >= kShiftForm)) return 0;
  return fabsf(Mb - K) >= fabsf(Mb) ? 1 : 2;
}

// Per-lane fp64 accumulators (see the file comment): S_b over all chunks;
// Ap = sum e*x and C = sum e*phi over polynomial-path chunks; Ad = sum e*x,
// Se = sum e and Sh = sum h over direct-path chunks. A = Ap + Ad.
struct Acc {
  double Sb, Ap, C, Ad, Se, Sh;
};

// Top-k scan state (TopkScan), in shared memory after the control block of
// scan launches, so that it costs the consumers' hot loop few registers: per
// consumer warp the region of its current row; per lane its rest sums of
// base weights (rest[0]) and quant weights (rest[1]) in the lane's frame and
// centre (kept in registers, they made the scan kernel spill in its hot loop).
struct ScanArea {
  uint4* region[kConsumerWarps];
  double rest[2][kConsumerWarps][32];
};
constexpr int kScanSmemBytes = static_cast<int>((sizeof(ScanArea) + 127) / 128 * 128);
// The warp-uniform part of the scan state that every chunk touches, kept in
// registers: the row's threshold and the lanes copied so far.
struct ScanRegs {
  int ncopy;
  float tf;
};
static_assert(kRowSmemBytes + kScanSmemBytes <= 227 * 1024, "row kernel shared memory");
__device__ __forceinline__ ScanArea& scan_area() {
  extern __shared__ __align__(128) unsigned char smem[];
  return *reinterpret_cast<ScanArea*>(smem + kRowSmemBytes);
}

struct Best {
  float b, q;  // lane maxima so far
  int lb, lq;  // chunk in which each first appeared
};

// Per-warp partial handed to the epilogue warp.
struct WarpPart {
  float Mb, Mq, Rb, Rq, K;
  int pad;
  double Sb, Ap, C, Ad, Se, Sh;
  unsigned cand_b, cand_q;  // lanes whose own maximum equals the warp maximum
};

struct Slot {
  WarpPart part[kConsumerWarps];
  int loc_b[kConsumerWarps][32];
  int loc_q[kConsumerWarps][32];
  double rest[kConsumerWarps][2];  // top-k scan: the warps' Sr, Qr
};

// Merged partial of a contiguous part of a row (a warp, a CTA, a cluster):
// maxima, base frame Cb (integer log2), centre K, and in that frame / centre
// S = sum e, A = sum e x, B = sum e (e^{lx} - 1); exact lowest argmax indices
// of the part (INT_MAX if none); flags (kPartNonfinite, kPartInfKl).
struct __align__(16) MPart {
  float Mb, Mq, Cb, K;
  double Sb, A, B;
  int amax_b, amax_q;
  unsigned flags, pad;
  unsigned long long pad2;  // 64 bytes: four 16-byte words
};
constexpr unsigned kPartNonfinite = 1u, kPartInfKl = 2u;
constexpr unsigned kPartFailed = 4u;  // a bounded wait gave up on this part
constexpr unsigned kPartHasTok = 8u;  // vocabulary slice holding the token: pad2 = (q, b) at it
static_assert(sizeof(MPart) == kSplitPartBytes && sizeof(MPart) == kPartialBytes, "MPart layout");

struct Ctrl {
  unsigned long long full[kStages];
  unsigned long long empty[kStages];
  unsigned long long slot_full[kSlots];
  unsigned long long slot_empty[kSlots];
  unsigned long long cl_full;  // split mode: cluster peers' partials arrived (leader)
  int abort;
  int pad;
  MPart cl_part[kMaxClusterCtas];  // split mode: partials pushed by the cluster peers
  Slot slot[kSlots];
};
static_assert(sizeof(Ctrl) <= kRowCtrlBytes, "control block too large");

// Exact 2^k for an integer-valued difference of frames (0 on underflow).
__device__ __forceinline__ double pow2i(float k) {
  return ldexp(1.0, static_cast<int>(fmaxf(k, -2000.f)));
}

// Polynomial path of one step: every x finite with |x| within tier T's range.
// S += e, Ap += e*x, C += e*x^2*Q_T(x), e = 2^(b*L - R_b).
// kScan: a lane left unflagged by the top-k scan (keep) also adds its
// weights to the rest sums: base e, quant e e^{lambda x} = e (1 + lambda x +
// phi), formed in fp32 with lambda rounded to 1.
template <int PE, int T, bool kScan>
__device__ __forceinline__ void poly_accumulate(const float* b, const f2* X, const Ref& r,
                                                Acc& a, bool keep) {
  constexpr int NP = (PE + 1) / 2;
  const f2 L2 = splat(kLog2e), nR2 = splat(-r.Rb);
  // Two accumulator sets (even / odd pairs) halve the dependent-add chains.
  f2 SB[2] = {splat(0.f), splat(0.f)}, SA[2] = {splat(0.f), splat(0.f)};
  f2 SC[2] = {splat(0.f), splat(0.f)};
#pragma unroll
  for (int j = 0; j < NP; ++j) {
    const int i0 = 2 * j, i1 = (2 * j + 1 < PE) ? 2 * j + 1 : 2 * j;
    float u0, u1;
    upk(fma2(pk(b[i0], b[i1]), L2, nR2), u0, u1);
    const f2 E = pk(ex2(u0), i1 == i0 ? 0.f : ex2(u1));
    const f2 T2 = mul2(E, X[j]);
    SB[j & 1] = add2(SB[j & 1], E);
    SA[j & 1] = add2(SA[j & 1], T2);
    SC[j & 1] = fma2(mul2(T2, X[j]), phi_q2<T>(X[j]), SC[j & 1]);
  }
  float sb0, sb1, sa0, sa1, sc0, sc1;
  upk(add2(SB[0], SB[1]), sb0, sb1);
  upk(add2(SA[0], SA[1]), sa0, sa1);
  upk(add2(SC[0], SC[1]), sc0, sc1);
  const float sb = sb0 + sb1, sa = sa0 + sa1, sc = sc0 + sc1;
  a.Sb += static_cast<double>(sb);
  a.Ap += static_cast<double>(sa);
  a.C += static_cast<double>(sc);
  if constexpr (kScan) {
    if (keep) {
      const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
      ScanArea& s = scan_area();
      s.rest[0][w][lane] += static_cast<double>(sb);
      s.rest[1][w][lane] += static_cast<double>((sb + sa) + sc);
    }
  }
}

// 16-bit quant rows stay packed in the hot loop (two elements per 32-bit
// word: element 2w in the low half, 2w + 1 in the high half): their maximum
// is taken on packed pairs and q - b by a mixed-precision subtract of the
// 16-bit operand from the fp32 base, so the quant row is never widened
// (measured for bf16: row pass 0.943 -> 0.906 ms at 8192 x 151936). Results
// are bit-identical: q - b of two bf16 or two f16 values is exact in fp32,
// and the maximum of 16-bit values is one of them.
template <int DT>
struct Packed;
template <>
struct Packed<KLD_BF16> {
  static constexpr uint32_t kNegInfPair = 0xff80ff80u;
  __device__ __forceinline__ static float lo(uint32_t w) { return __uint_as_float(w << 16); }
  __device__ __forceinline__ static float hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
  __device__ __forceinline__ static uint32_t max2(uint32_t a, uint32_t c) {
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(c));
    return d;
  }
  __device__ __forceinline__ static void sub(uint32_t w, float b0, float b1, float& x0, float& x1) {
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tsub.f32.bf16 %0, lo, %3;\n\t"
        "sub.f32.bf16 %1, hi, %4;\n\t}"
        : "=f"(x0), "=f"(x1) : "r"(w), "f"(b0), "f"(b1));
  }
};
template <>
struct Packed<KLD_F16> {
  static constexpr uint32_t kNegInfPair = 0xfc00fc00u;
  __device__ __forceinline__ static float lo(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xffffu)));
  }
  __device__ __forceinline__ static float hi(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
  }
  __device__ __forceinline__ static uint32_t max2(uint32_t a, uint32_t c) {
    uint32_t d;
    asm("max.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(c));
    return d;
  }
  __device__ __forceinline__ static void sub(uint32_t w, float b0, float b1, float& x0, float& x1) {
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tsub.f32.f16 %0, lo, %3;\n\t"
        "sub.f32.f16 %1, hi, %4;\n\t}"
        : "=f"(x0), "=f"(x1) : "r"(w), "f"(b0), "f"(b1));
  }
};
// Quant element i of a step: from the packed words (kPk = the row's 16-bit
// type) or the widened array (kPk = 0).
template <int kPk>
__device__ __forceinline__ float q_el(const float* q, const uint32_t* qw, int i) {
  if constexpr (kPk != 0)
    return (i & 1) ? Packed<kPk>::hi(qw[i >> 1]) : Packed<kPk>::lo(qw[i >> 1]);
  else
    return q[i];
}

// Log-ratios x = q - b + K of one step, in packed pairs (x = 0 for absent
// elements), and the largest |x| of the lane (NaN if any x is NaN). kForm
// picks the order of the roundings (ratio_form): 0 (q - b) + K, 1
// (q + K) - b, 2 q - (b - K).
template <int PE, int kForm, int kPk = 0>
__device__ __forceinline__ float log_ratios(const float* b, const float* q, unsigned valid,
                                            float K, f2* X, const uint32_t* qw = nullptr) {
  constexpr int NP = (PE + 1) / 2;
  float ax0 = 0.f, ax1 = 0.f;
  const f2 K2 = splat(K);
#pragma unroll
  for (int j = 0; j < NP; ++j) {
    const int i0 = 2 * j, i1 = (2 * j + 1 < PE) ? 2 * j + 1 : 2 * j;
    if constexpr (kPk != 0) {
      float d0, d1;
      Packed<kPk>::sub(qw[j], b[i0], b[i1], d0, d1);
      X[j] = add2(pk(d0, d1), K2);
    } else {
      const f2 Q = pk(q[i0], q[i1]), B = pk(b[i0], b[i1]);
      if (kForm == 1)
        X[j] = sub2(add2(Q, K2), B);
      else if (kForm == 2)
        X[j] = sub2(Q, sub2(B, K2));
      else
        X[j] = add2(sub2(Q, B), K2);
    }
    float x0, x1;
    upk(X[j], x0, x1);
    if (((valid >> i0) & 1u) == 0u) x0 = 0.f;
    if (((valid >> i1) & 1u) == 0u || i1 == i0) x1 = 0.f;
    X[j] = pk(x0, x1);
    if (j & 1)
      ax1 = max3_nan(ax1, fabsf(x0), fabsf(x1));
    else
      ax0 = max3_nan(ax0, fabsf(x0), fabsf(x1));
  }
  return max3_nan(ax0, ax1, 0.f);
}

// One step of PE element pairs per lane (a 16-element consumer chunk, or the
// head/tail elements one per lane). Elements whose bit in `valid` is clear
// are absent (b = q = -inf, x = 0: they contribute nothing).
// kWide: fp32 inputs (the log-ratio's rounding order follows the centre,
// ratio_form); 16-bit inputs always form q - b first, which is exact.
// kScan: the top-k scan (TopkScan): returns true for a lane holding a base
// logit >= the row's threshold, and for every lane of a direct-path step:
// those lanes are copied (see process_chunk); the other lanes add their
// weights to the rest sums in poly_accumulate.
template <int PE, bool kWide, bool kScan = false, int kPk = 0>
__device__ __forceinline__ bool chunk_step(const float* b, const float* q, unsigned valid,
                                           Ref& r, Acc& a, Best& best, int chunk_id,
                                           const uint32_t* qw = nullptr, float scan_tf = 0.f) {
  constexpr int NP = (PE + 1) / 2;
  const float mb = tree_max<PE, false>(b);
  float mq;
  if constexpr (kPk != 0) {
    uint32_t m2 = qw[0];
#pragma unroll
    for (int w = 1; w < NP; ++w) m2 = Packed<kPk>::max2(m2, qw[w]);
    mq = fmaxf(Packed<kPk>::lo(m2), Packed<kPk>::hi(m2));
  } else {
    mq = tree_max<PE, false>(q);
  }
  f2 X[NP];  // log-ratios, formed once the centre K of this step is settled
  // The warp maximum is needed only when some lane's maximum passes the
  // threshold (a few chunks per row): a vote first, then the shuffle tree.
  if (__any_sync(0xffffffffu, mb > r.T)) {
    // raise the base frame and move the centre (warp-uniform)
    const float wmb = warp_max(mb);
    // New centre: (b - q) at the lowest lane's first element holding wmb.
    float dl = 0.f;
    bool has = false;
#pragma unroll
    for (int i = 0; i < PE; ++i) {
      if (!has && b[i] == wmb) {
        dl = b[i] - q_el<kPk>(q, qw, i);
        has = true;
      }
    }
    const unsigned who = __ballot_sync(0xffffffffu, has);
    const float Kn = __shfl_sync(0xffffffffu, dl, __ffs(who) - 1);
    const float nR = floorf(wmb * kLog2e);
    if (isfinite(Kn)) {
      const double d = static_cast<double>(Kn) - static_cast<double>(r.K);
      if (r.Mb != -INFINITY) {
        // e^{ld} - 1 = l d + phi(l d); phi from the same polynomial when
        // |d| is in its range, so the (e^{ld} - 1 - l d) term stays exact.
        double ph;
        if (fabs(d) <= static_cast<double>(kTau)) {
          const float df = static_cast<float>(d);
          ph = static_cast<double>(df * df * phi_q(df));
        } else {
          ph = expm1(kLambda * d) - kLambda * d;
        }
        const double em = kLambda * d + ph;
        if (isfinite(em)) {
          const double Sp = a.Sb - a.Se;
          a.C = (em + 1.0) * a.C + em * kLambda * a.Ap + ph * Sp;
          a.Ap += d * Sp;
          a.Ad += d * a.Se;
          if constexpr (kScan)  // quant weights follow the centre
            scan_area().rest[1][threadIdx.x >> 5][threadIdx.x & 31] *= em + 1.0;
          r.K = Kn;
          if (kWide) r.mode = ratio_form(wmb, Kn);
        }
      } else {
        // First finite maximum: only direct-path terms of masked base
        // entries (e = 0) can have been accumulated.
        a.Ad += d * a.Se;
        r.K = Kn;
        if (kWide) r.mode = ratio_form(wmb, Kn);
      }
    }
    if (r.Mb != -INFINITY) {
      const double sc = pow2i(r.Rb - nR);  // exact power of two
      a.Sb *= sc;
      a.Ap *= sc;
      a.C *= sc;
      a.Ad *= sc;
      a.Se *= sc;
      if constexpr (kScan) {
        ScanArea& s = scan_area();
        s.rest[0][threadIdx.x >> 5][threadIdx.x & 31] *= sc;
        s.rest[1][threadIdx.x >> 5][threadIdx.x & 31] *= sc;
      }
    }
    r.Rb = nR;
    r.Mb = wmb;
    r.T = wmb + kRaiseMargin;
  }
  float axl;
  if (!kWide || r.mode == 0)
    axl = log_ratios<PE, 0, kPk>(b, q, valid, r.K, X, qw);
  else if (r.mode == 1)
    axl = log_ratios<PE, 1>(b, q, valid, r.K, X);
  else
    axl = log_ratios<PE, 2>(b, q, valid, r.K, X);

  // The cheapest polynomial tier whose range holds every |x| of the warp's
  // step (a NaN fails every test and takes the direct path).
  bool flag = false;
  if constexpr (kScan) {
    // the vote first, in every lane (a short-circuit would leave lanes out)
    const bool direct = !__all_sync(0xffffffffu, axl <= kTau);  // the direct path follows
    flag = direct || mb >= scan_tf;
  }
  if (__all_sync(0xffffffffu, axl <= kTauA)) {
    poly_accumulate<PE, 0, kScan>(b, X, r, a, !flag);
  } else if (__all_sync(0xffffffffu, axl <= kTauB)) {
    poly_accumulate<PE, 1, kScan>(b, X, r, a, !flag);
  } else if (__all_sync(0xffffffffu, axl <= kTau)) {
    poly_accumulate<PE, 2, kScan>(b, X, r, a, !flag);
  } else {
    // Direct path: quant weights in their own frame. x -> +BIG keeps 0*x = 0
    // for masked base entries; x = -inf (quant masked, base finite) makes A
    // -inf, i.e. KL = +inf.
    const float wmq = warp_max(mq);
    if (wmq > r.Mqf) {  // raise the quant frame (direct-path sums only)
      const float nR = floorf(wmq * kLog2e);
      if (r.Mqf != -INFINITY) a.Sh *= pow2i(r.Rq - nR);
      r.Rq = nR;
      r.Mqf = wmq;
    }
    const float nRb = -r.Rb, nRq = -r.Rq;
    float sb = 0.f, sa = 0.f, sh = 0.f;
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      float x0, x1;
      upk(X[j], x0, x1);
      const float xs[2] = {x0, x1};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = 2 * j + h;
        if (i < PE) {
          const float e = ex2(fmaf(b[i], kLog2e, nRb));
          sb += e;
          sa = fmaf(e, fminf(xs[h], kBig), sa);
          sh += ex2(fmaf(q_el<kPk>(q, qw, i), kLog2e, nRq));
        }
      }
    }
    a.Sb += static_cast<double>(sb);
    a.Se += static_cast<double>(sb);
    a.Ad += static_cast<double>(sa);
    a.Sh += static_cast<double>(sh);
  }
  if (mb > best.b) {
    best.b = mb;
    best.lb = chunk_id;
  }
  if (mq > best.q) {
    best.q = mq;
    best.lq = chunk_id;
  }
  return flag;
}

// One 512-element chunk of the current tile (16 elements per lane).
template <int DT, bool kMasked, bool kScan>
__device__ __forceinline__ void process_chunk(const uint4* cb, const uint4* cq, int lane,
                                              int valid_vecs, Ref& r, Acc& a, Best& best,
                                              int chunk_id, ScanRegs* sr) {
  constexpr int E = Elem<DT>::kPerVec;
  constexpr int VPC = kLaneElems / E;
  constexpr int kPk = DT == KLD_F32 ? 0 : DT;  // 16-bit quant rows stay packed
  float xb[kLaneElems], xq[kPk ? 1 : kLaneElems];
  uint32_t qw[kLaneElems / 2];
  unsigned valid = (1u << kLaneElems) - 1u;
#pragma unroll
  for (int k = 0; k < VPC; ++k) {
    const int vi = k * 32 + lane;
    const uint4 vb = cb[vi];
    const uint4 vq = cq[vi];
    Elem<DT>::unpack(vb, &xb[k * E]);
    if constexpr (kPk != 0) {
      qw[4 * k] = vq.x;
      qw[4 * k + 1] = vq.y;
      qw[4 * k + 2] = vq.z;
      qw[4 * k + 3] = vq.w;
    } else {
      Elem<DT>::unpack(vq, &xq[k * E]);
    }
    if (kMasked && vi >= valid_vecs) {
      valid &= ~(((1u << E) - 1u) << (k * E));
#pragma unroll
      for (int i = 0; i < E; ++i) {
        xb[k * E + i] = -INFINITY;
        if constexpr (kPk == 0) xq[k * E + i] = -INFINITY;
      }
      if constexpr (kPk != 0) {
#pragma unroll
        for (int u = 0; u < 4; ++u) qw[4 * k + u] = Packed<kPk>::kNegInfPair;
      }
    }
  }
  const bool cp = chunk_step<kLaneElems, DT == KLD_F32, kScan, kPk>(
      xb, xq, valid, r, a, best, chunk_id, qw, kScan ? sr->tf : 0.f);
  if constexpr (kScan) {
    // copy the marked lanes' vectors from the stage into their records
    // (past the body's end of a last chunk they hold stale data; the top-k
    // pass bounds every element by the body)
    const unsigned fm = __ballot_sync(0xffffffffu, cp);
    if (fm != 0u) {
      ScanArea& s = scan_area();
      const int w = threadIdx.x >> 5;
      const int n0 = sr->ncopy;
      if (cp) {
        const int pos = n0 + __popc(fm & ((1u << lane) - 1u));
        if (pos < kCopyCap) {
          uint4* dst = s.region[w] + pos * kCopyVecs;
#pragma unroll
          for (int k = 0; k < VPC; ++k) {
            dst[k] = cb[k * 32 + lane];
            dst[VPC + k] = cq[k * 32 + lane];
          }
          reinterpret_cast<uint32_t*>(s.region[w] + kCopyCap * kCopyVecs)[pos] =
              static_cast<uint32_t>(chunk_id) * 32u + static_cast<uint32_t>(lane);
        }
      }
      sr->ncopy = n0 + __popc(fm);
    }
  }
}

__device__ __forceinline__ void fail(Ctrl* ctrl, uint32_t* derr) {
  atomicOr(derr, kErrWaitTimeout);
  *reinterpret_cast<volatile int*>(&ctrl->abort) = 1;
}

// Row geometry: the unaligned head and tail (< 16 bytes each) are read
// directly; the 16-byte-aligned body is streamed in tiles.
struct RowGeom {
  int64_t head, body_len, tail, nch;  // nch: 512-element chunks of the body
};

template <int DT>
__device__ __forceinline__ RowGeom row_geom(const void* rowb, int64_t V) {
  const RowSpan sp = row_span(rowb, V, Elem<DT>::kBytes);
  RowGeom g;
  g.head = sp.head;
  g.body_len = sp.body;
  g.tail = sp.tail;
  g.nch = (g.body_len + kChunkElems - 1) / kChunkElems;
  return g;
}

// Offset (within the body) of element i of lane `lane` in chunk `chunk_id`.
template <int DT>
__device__ __forceinline__ int64_t chunk_elem_offset(int chunk_id, int lane, int i) {
  constexpr int E = Elem<DT>::kPerVec;
  return static_cast<int64_t>(chunk_id) * kChunkElems +
         static_cast<int64_t>((i / E) * 32 + lane) * E + (i % E);
}

// Element i of a tile staged in shared memory.
template <int DT>
__device__ __forceinline__ float load_staged(const unsigned char* stage, int i) {
  if constexpr (DT == KLD_F32) {
    return reinterpret_cast<const float*>(stage)[i];
  } else if constexpr (DT == KLD_BF16) {
    return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const unsigned short*>(stage)[i]) << 16);
  } else {
    return __half2float(__ushort_as_half(reinterpret_cast<const unsigned short*>(stage)[i]));
  }
}

// Lowest index holding `m` among the candidate lanes (mask) of one warp's
// published partial (chunk ids counted from body element s0); lanes 0..15 of
// the calling warp each test one element. staged (nullable): the item's
// tiles are still in the shared-memory ring (tile t in stage t; a split part
// of at most kStages tiles), so the elements are read there instead of from
// global memory; n = the item's element count.
template <int DT>
__device__ int rescan_candidates(const void* row, const RowGeom& g, int64_t s0, unsigned mask,
                                 const int* locs, float m, int lane,
                                 const unsigned char* staged = nullptr, int64_t n = 0) {
  constexpr int kStageElems = kStageBytes / Elem<DT>::kBytes;
  int best = INT_MAX;
  while (mask) {
    const int cl = __ffs(mask) - 1;
    mask &= mask - 1u;
    const int loc = locs[cl];
    int idx = INT_MAX;
    if (lane < kLaneElems && loc >= 0) {
      const int64_t io = chunk_elem_offset<DT>(loc, cl, lane);  // within the item
      const int64_t off = s0 + io;
      if (off < g.body_len) {
        const float x = staged != nullptr && io < n
                            ? load_staged<DT>(staged + (io / kStageElems) * kStageBytes,
                                              static_cast<int>(io % kStageElems))
                            : Elem<DT>::load(row, g.head + off);
        if (x == m) idx = static_cast<int>(g.head + off);
      }
    }
    idx = __reduce_min_sync(0xffffffffu, idx);
    if (idx < best) best = idx;
  }
  return best;
}

// Launch schedule (computed on the host, see plan_rows):
//   P > 1: cluster split, one item per CTA: part blockIdx % P of row
//          blockIdx / P (each row's chunks divided evenly over P CTAs);
//   else:  W rounds of whole rows (CTA b takes rows b + j*gridDim, j < W,
//          r < N), then the R remaining rows [W*gridDim, N) as a tail that
//          the first Gt CTAs share by balanced ranges of the tail's
//          Tc = R * nchv virtual chunks (nchv = chunks of a full row): CTA b
//          takes [Tc*b/Gt, Tc*(b+1)/Gt), which touches at most two rows;
//          a row is split among the at most 32 CTAs whose ranges touch it.
//   A > 0: no whole rounds and the tail's ranges fall on row boundaries
//          (Gt = R * A): CTA b is part b % A of row b / A, found in 32-bit
//          arithmetic (the general case needs 64-bit divisions).
struct Sched {
  int P, W, R, Gt, nchv, A;
  int64_t Tc;
};

// One work item: body elements [s0, s1) of row r; part k of the row's np
// parts (np == 1: the item is the whole row). rt: the row's index among the
// split rows (its ticket and partial slots). whole: a whole-row round.
struct Item {
  int64_t r, s0, s1, rt;
  int k, np;
  bool whole;
};

// CTA holding virtual chunk c of the tail (ranges [Tc*b/Gt, Tc*(b+1)/Gt)).
__device__ __forceinline__ int64_t tail_cta(int64_t c, const Sched& sc) {
  return ((c + 1) * sc.Gt - 1) / sc.Tc;
}

template <int DT>
__device__ __forceinline__ bool item_at(int j, const Sched& sc, const char* B, int64_t N, int64_t V,
                                        Item& it, RowGeom& g) {
  constexpr int EB = Elem<DT>::kBytes;
  const int64_t b = blockIdx.x;
  if (sc.P > 1) {
    if (j > 0) return false;
    it.r = b / sc.P;
    it.rt = it.r;
    it.k = static_cast<int>(b % sc.P);
    it.np = sc.P;
    it.whole = false;
    g = row_geom<DT>(B + it.r * V * EB, V);
    const int64_t c0 = g.nch * it.k / sc.P, c1 = g.nch * (it.k + 1) / sc.P;
    it.s0 = c0 * kChunkElems;
    it.s1 = c1 * kChunkElems < g.body_len ? c1 * kChunkElems : g.body_len;
    if (it.s1 < it.s0) it.s1 = it.s0;
    return true;
  }
  if (sc.A > 0) {
    if (j > 0) return false;
    const int bi = static_cast<int>(blockIdx.x);
    it.r = bi / sc.A;
    it.rt = it.r;
    it.k = bi % sc.A;
    it.np = sc.A;
    it.whole = false;
    g = row_geom<DT>(B + it.r * V * EB, V);
    const int64_t lo = static_cast<int64_t>(static_cast<unsigned>(sc.nchv) * static_cast<unsigned>(it.k) /
                                            static_cast<unsigned>(sc.A));
    const int64_t hi = static_cast<int64_t>(static_cast<unsigned>(sc.nchv) * static_cast<unsigned>(it.k + 1) /
                                            static_cast<unsigned>(sc.A));
    it.s0 = lo * kChunkElems < g.body_len ? lo * kChunkElems : g.body_len;
    it.s1 = hi * kChunkElems < g.body_len ? hi * kChunkElems : g.body_len;
    return true;
  }
  if (j < sc.W) {
    it.r = b + static_cast<int64_t>(j) * gridDim.x;
    if (it.r >= N) return false;
    g = row_geom<DT>(B + it.r * V * EB, V);
    it.s0 = 0;
    it.s1 = g.body_len;
    it.rt = -1;
    it.k = 0;
    it.np = 1;
    it.whole = true;
    return true;
  }
  const int t = j - sc.W;
  if (t > 1 || b >= sc.Gt) return false;
  const int64_t c0 = sc.Tc * b / sc.Gt, c1 = sc.Tc * (b + 1) / sc.Gt;
  const int64_t rt = c0 / sc.nchv + t;
  if (rt > (c1 - 1) / sc.nchv) return false;
  it.rt = rt;
  it.r = static_cast<int64_t>(sc.W) * gridDim.x + rt;
  g = row_geom<DT>(B + it.r * V * EB, V);
  const int64_t rc0 = rt * sc.nchv;
  const int64_t lo = (c0 > rc0 ? c0 : rc0) - rc0;
  const int64_t hi = (c1 < rc0 + sc.nchv ? c1 : rc0 + sc.nchv) - rc0;
  it.s0 = lo * kChunkElems < g.body_len ? lo * kChunkElems : g.body_len;
  it.s1 = hi * kChunkElems < g.body_len ? hi * kChunkElems : g.body_len;
  const int64_t first = tail_cta(rc0, sc);
  it.k = static_cast<int>(b - first);
  it.np = static_cast<int>(tail_cta(rc0 + sc.nchv - 1, sc) - first + 1);
  it.whole = false;
  return true;
}

// MPart as eight 64-bit words and back (explicit, so no copy goes through
// local memory).
__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  return static_cast<unsigned long long>(__float_as_uint(lo)) |
         (static_cast<unsigned long long>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ unsigned long long pack2(unsigned lo, unsigned hi) {
  return static_cast<unsigned long long>(lo) | (static_cast<unsigned long long>(hi) << 32);
}
__device__ __forceinline__ void part_words(const MPart& m, unsigned long long (&w)[8]) {
  w[0] = pack2(m.Mb, m.Mq);
  w[1] = pack2(m.Cb, m.K);
  w[2] = static_cast<unsigned long long>(__double_as_longlong(m.Sb));
  w[3] = static_cast<unsigned long long>(__double_as_longlong(m.A));
  w[4] = static_cast<unsigned long long>(__double_as_longlong(m.B));
  w[5] = pack2(static_cast<unsigned>(m.amax_b), static_cast<unsigned>(m.amax_q));
  w[6] = pack2(m.flags, 0u);
  w[7] = m.pad2;  // a vocabulary slice's token logits (kPartHasTok)
}
__device__ __forceinline__ MPart part_from_words(const unsigned long long (&w)[8]) {
  MPart m;
  m.Mb = __uint_as_float(static_cast<unsigned>(w[0]));
  m.Mq = __uint_as_float(static_cast<unsigned>(w[0] >> 32));
  m.Cb = __uint_as_float(static_cast<unsigned>(w[1]));
  m.K = __uint_as_float(static_cast<unsigned>(w[1] >> 32));
  m.Sb = __longlong_as_double(static_cast<long long>(w[2]));
  m.A = __longlong_as_double(static_cast<long long>(w[3]));
  m.B = __longlong_as_double(static_cast<long long>(w[4]));
  m.amax_b = static_cast<int>(static_cast<unsigned>(w[5]));
  m.amax_q = static_cast<int>(static_cast<unsigned>(w[5] >> 32));
  m.flags = static_cast<unsigned>(w[6]);
  m.pad = 0u;
  m.pad2 = w[7];
  return m;
}

__device__ __forceinline__ MPart empty_part() {
  MPart m;
  m.Mb = m.Mq = -INFINITY;
  m.Cb = m.K = 0.f;
  m.Sb = m.A = m.B = 0.0;
  m.amax_b = m.amax_q = INT_MAX;
  m.flags = m.pad = 0u;
  m.pad2 = 0ull;
  return m;
}

// Warp-collective merge of the partials held by the lanes. Every lane gets
// the merged partial: its frame is the largest base frame among parts with
// base mass, its centre that of the part holding the maximum of b. Moving a
// part by dK = K' - K and fb = 2^(Cb - Cb'): S' = S fb, A' = (A + dK S) fb,
// B' = (B + (e^{l dK} - 1)(B + S)) fb. A part without base mass (every b is
// -inf) carries only quant weight B, moved by one power of two.
__device__ MPart warp_merge(const MPart& p) {
  const bool has_b = p.Sb != 0.0;
  const bool used = has_b || p.B != 0.0;
  MPart m;
  m.Mb = warp_max(p.Mb);
  m.Mq = warp_max(p.Mq);
  m.flags = __reduce_or_sync(0xffffffffu, p.flags);
  m.amax_b = __reduce_min_sync(0xffffffffu, p.Mb == m.Mb ? p.amax_b : INT_MAX);
  m.amax_q = __reduce_min_sync(0xffffffffu, p.Mq == m.Mq ? p.amax_q : INT_MAX);
  m.pad = 0u;
  m.pad2 = 0ull;
  if (__any_sync(0xffffffffu, has_b)) {
    m.Cb = warp_max(has_b ? p.Cb : -INFINITY);
    const unsigned kmask = __ballot_sync(0xffffffffu, has_b && p.Mb == m.Mb);
    m.K = __shfl_sync(0xffffffffu, p.K, kmask ? __ffs(kmask) - 1 : 0);
  } else {
    m.Cb = __any_sync(0xffffffffu, used) ? warp_max(used ? p.Cb : -INFINITY) : 0.f;
    m.K = 0.f;
  }
  double sb = 0.0, sa = 0.0, sB = 0.0;
  const double dK = static_cast<double>(m.K) - static_cast<double>(p.K);
  if (has_b) {
    const double fb = pow2i(p.Cb - m.Cb);
    const double em = expm1(kLambda * dK);
    sb = p.Sb * fb;
    sa = (m.flags & kPartInfKl) ? 0.0 : (p.A + dK * p.Sb) * fb;
    sB = (p.B + em * (p.B + p.Sb)) * fb;
  } else if (used) {
    sB = p.B * exp2(static_cast<double>(p.Cb) - static_cast<double>(m.Cb) + dK * kLog2eD);
  }
  m.Sb = warp_sum(sb);
  m.A = warp_sum(sa);
  m.B = warp_sum(sB);
  return m;
}

// The record of a whole row from its merged partial.
// Called by a full warp with warp-uniform arguments: the record's three
// logarithms run at once on lanes 0-2 (all as log1p, so the warp does not
// diverge) and its two exponentials on lanes 1-2.
__device__ kld_row_t finalize_row(const MPart& m, bool has_tok, bool tok_ok, float q_tok,
                                  float b_tok) {
  const int lane = threadIdx.x & 31;
  // lane 0: log1p(B/S); lane 1: log(B + S); lane 2 and up: log(S). S >= 1
  // (the frame's maximum weight is at least 1), and B + S >= 0.5 but for
  // rows whose quant row misses the base maximum (taken apart below).
  const double bs = m.B + m.Sb;
  const double lg = log1p(lane == 0 ? m.B / m.Sb : (lane == 1 ? bs - 1.0 : m.Sb - 1.0));
  const double log1p_bs = __shfl_sync(0xffffffffu, lg, 0);
  double log_bs = __shfl_sync(0xffffffffu, lg, 1);
  const double log_s = __shfl_sync(0xffffffffu, lg, 2);
  if (!(bs >= 0.5)) log_bs = log(bs);
  kld_row_t rec;
  uint32_t flags = 0;
  if (has_tok && !tok_ok) flags |= KLD_ROW_BAD_TOKEN;
  const double nan = __longlong_as_double(0x7ff8000000000000ll);
  rec.kld = nan;
  rec.nll = nan;
  rec.nll_base = nan;
  rec.argmax_base = -1;
  rec.argmax_quant = -1;
  const bool nonfinite = (m.flags & (kPartNonfinite | kPartFailed)) || isnan(m.Sb) || isnan(m.B) ||
                         !(m.Mb < INFINITY) || !(m.Mq < INFINITY);
  if (nonfinite) {
    flags |= KLD_ROW_NONFINITE;
  } else if (m.Mb == -INFINITY || m.Mq == -INFINITY) {
    flags |= KLD_ROW_EMPTY;
  } else {
    if (m.flags & kPartInfKl) {
      rec.kld = INFINITY;
      flags |= KLD_ROW_INF_KL;
    } else {
      rec.kld = -kLambda * (m.A / m.Sb) + log1p_bs;
    }
    if (tok_ok) {
      if (q_tok == -INFINITY) {
        rec.nll = INFINITY;
        flags |= KLD_ROW_INF_NLL;
      } else {
        // B + S is the sum of all quant weights in frame Cb - K*L.
        rec.nll = log_bs +
                  kLn2 * (static_cast<double>(m.Cb) -
                          (static_cast<double>(m.K) + static_cast<double>(q_tok)) * kLog2eD);
      }
      if (b_tok == -INFINITY) {
        rec.nll_base = INFINITY;
        flags |= KLD_ROW_INF_NLL_BASE;
      } else {
        // S is the sum of all base weights in frame Cb.
        rec.nll_base = log_s + kLn2 * (static_cast<double>(m.Cb) -
                                           static_cast<double>(b_tok) * kLog2eD);
      }
    }
    rec.argmax_base = m.amax_b;
    rec.argmax_quant = m.amax_q;
  }
  rec.flags = flags;
  // P(tok) = exp(-NLL) for each model (exp(-inf) = 0), differenced in fp64
  const double ex = exp(-(lane == 1 ? rec.nll : rec.nll_base));
  rec.dp = static_cast<float>(__shfl_sync(0xffffffffu, ex, 1) - __shfl_sync(0xffffffffu, ex, 2));
  return rec;
}

// Per-row normalisers for the gradient and top-k passes, from the merged
// partial: softmax(lambda*b)_j = 2^(b_j*L - Fb) * mb and softmax(lambda*q)_j
// = 2^(q_j*L - Fq) * mq, with integer frames Fb = floor(log2 of the base
// sum), Fq likewise, and mb, mq in (0.5, 1] (so the exponents stay small
// near the row maximum and every value keeps fp32 accuracy); the base
// log-normaliser and log1p(B/S) in fp64 for the top-k KL. A NaN Fb marks a
// row excluded from the statistics.
__device__ RowAux row_aux(const MPart& m, const kld_row_t& rec) {
  RowAux a;
  a.flags = rec.flags;
  a.pad = 0ull;
  a.rest_b = 0.0;
  a.rest_q = 0.0;
  a.K = m.K;
  if (rec.flags & (KLD_ROW_NONFINITE | KLD_ROW_EMPTY)) {
    const float nan = __int_as_float(0x7fc00000);
    a.Fb = a.Fq = nan;
    a.mb = a.mq = 0.f;
    a.lse_b = a.lr = __longlong_as_double(0x7ff8000000000000ll);
    return a;
  }
  const double cb = log2(m.Sb) + static_cast<double>(m.Cb);
  const double cq = log2(m.B + m.Sb) + static_cast<double>(m.Cb) -
                    static_cast<double>(m.K) * kLog2eD;
  const double fb = floor(cb), fq = floor(cq);
  a.Fb = static_cast<float>(fb);
  a.mb = static_cast<float>(exp2(fb - cb));
  a.Fq = static_cast<float>(fq);
  a.mq = static_cast<float>(exp2(fq - cq));
  a.lse_b = cb * kLn2;
  a.lr = log1p(m.B / m.Sb);
  return a;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

// Arguments of the row kernel (passed by value, __grid_constant__).
struct RowParams {
  const void* base;
  const void* quant;
  const int32_t* tok;
  int64_t N, V;
  kld_row_t* rows;
  uint32_t* derr;
  Sched sc;
  MPart* gparts;       // split rows: partials, kPartSlots per split row
  unsigned* tickets;   // split rows: one arrival counter per split row
  RowAux* aux;         // nullable: per-row normalisers
  MPart* part_out;     // nullable: vocabulary-slice partials instead of records
  int64_t col0;
  // Few split rows (nullable): the launch also reduces its records into
  // *out, counting finished rows on *counter (see count_row).
  kld_result_t* out;
  unsigned* counter;
  TopkScan scan;  // top-k scan (kld_rows_kernel<DT, true> only)
};

// Slots of partials per split row in the split scratch (one per part; a
// row has at most 32 parts, merged by one warp).
constexpr int kPartSlots = kPartSlotsPerRow;

// Few split rows (RowParams.out set): every row's finaliser counts its
// record on the launch's counter; the warp that counts the last record
// reduces all N records on the spot, so the statistic needs no second
// kernel. The counter goes back to zero for the next launch.
__device__ __forceinline__ void count_row(unsigned* counter, const kld_row_t* rows, int64_t N,
                                          int has_nll, uint32_t* derr, kld_result_t* out,
                                          int lane) {
  unsigned t = 0u;
  if (lane == 0)  // release: this warp's record; acquire: every other record
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(t) : "l"(counter) : "memory");
  t = __shfl_sync(0xffffffffu, t, 0);
  if (t != static_cast<unsigned>(N - 1)) return;
  __syncwarp();  // lane 0's acquire orders the other lanes' loads
  if (lane == 0) *counter = 0u;
  fin::reduce_few_rows(rows, static_cast<int>(N), has_nll, derr, out, lane);
}

// A finished row, written by lane 0 of the warp that finalised it: the
// record and the row's normalisers.
__device__ __forceinline__ void write_row(const RowParams& p, int64_t r, const kld_row_t& rec,
                                          const MPart& m, double rest_b = 0.0,
                                          double rest_q = 0.0) {
  p.rows[r] = rec;
  if (p.aux != nullptr) {
    RowAux a = row_aux(m, rec);
    a.rest_b = rest_b;
    a.rest_q = rest_q;
    p.aux[r] = a;
  }
}

// kScan: the top-k scan (prm.scan; whole-row launches only).
template <int DT, bool kScan>
__global__ void __launch_bounds__(kRowThreads, 1) kld_rows_kernel(const __grid_constant__ RowParams prm) {
  const void* __restrict__ base = prm.base;
  const void* __restrict__ quant = prm.quant;
  const int32_t* __restrict__ tok = prm.tok;
  const int64_t N = prm.N, V = prm.V;
  kld_row_t* __restrict__ rows = prm.rows;
  uint32_t* __restrict__ derr = prm.derr;
  const Sched& sc = prm.sc;  // read from parameter space where used
  MPart* __restrict__ gparts = prm.gparts;
  unsigned* __restrict__ tickets = prm.tickets;
  MPart* __restrict__ part_out = prm.part_out;
  const int64_t col0 = prm.col0;
  constexpr int EB = Elem<DT>::kBytes;
  constexpr int E = Elem<DT>::kPerVec;
  constexpr int kStageElems = kStageBytes / EB;
  constexpr int kChunksPerTile = kStageElems / kChunkElems;

  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stage_b = smem;
  unsigned char* stage_q = smem + kStages * kStageBytes;
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + 2 * kStages * kStageBytes);
  volatile int* abort = &ctrl->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t G = sc.P > 1 ? cluster_nctarank() : 1u;  // CTAs per cluster

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&ctrl->full[s]), 1);
      mbar_init(smem_u32(&ctrl->empty[s]), kConsumerWarps);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(smem_u32(&ctrl->slot_full[s]), kConsumerWarps);
      mbar_init(smem_u32(&ctrl->slot_empty[s]), 1);
    }
    mbar_init(smem_u32(&ctrl->cl_full), G > 1 ? G - 1 : 1);
    ctrl->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // Cluster barrier, first phase: every thread arrives now (the barrier
  // initialisation above is released with it) and waits only where it next
  // touches a peer's shared memory, so no CTA stalls here at start-up.
  bool cl_waited = false;
  if (G > 1) asm volatile("barrier.cluster.arrive.release;" ::: "memory");
  // The reduction launched after this pass may be scheduled now; it waits
  // for this grid's completion before reading anything.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const char* B = static_cast<const char*>(base);
  const char* Q = static_cast<const char*>(quant);

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = evict_first_policy();
      int s = 0;
      uint32_t ph = 0u;
      uint32_t issued = 0;
      bool ok = true;
      Item it;
      RowGeom g;
      for (int j = 0; ok && item_at<DT>(j, sc, B, N, V, it, g); ++j) {
        const char* rb = B + it.r * V * EB;
        const char* rq = Q + it.r * V * EB;
        const int64_t n = it.s1 - it.s0;
        const int64_t ntiles = (n + kStageElems - 1) / kStageElems;
        for (int64_t t = 0; t < ntiles; ++t) {
          if (!mbar_try_wait(smem_u32(&ctrl->empty[s]), ph ^ 1u) &&
              !mbar_wait_idle(smem_u32(&ctrl->empty[s]), ph ^ 1u, abort)) {
            fail(ctrl, derr);
            ok = false;
            break;
          }
          const int64_t off = g.head + it.s0 + t * kStageElems;
          int64_t len = n - t * kStageElems;
          if (len > kStageElems) len = kStageElems;
          const uint32_t bytes = static_cast<uint32_t>(len * EB);
          const uint32_t fb = smem_u32(&ctrl->full[s]);
          mbar_arrive_expect_tx(fb, 2u * bytes);
          bulk_load(smem_u32(stage_b + s * kStageBytes), rb + off * EB, bytes, fb, pol);
          bulk_load(smem_u32(stage_q + s * kStageBytes), rq + off * EB, bytes, fb, pol);
          ++issued;
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // Never leave with copies in flight: wait (bounded) for the last
      // stages issued. In a normal run they have long completed.
      const uint32_t last = issued < kStages ? issued : kStages;
      for (uint32_t k = 0; k < last; ++k) {
        if (--s < 0) {
          s = kStages - 1;
          ph ^= 1u;
        }
        const uint32_t fb = smem_u32(&ctrl->full[s]);
        if (!mbar_try_wait(fb, ph)) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(fb, ph)) {
            if (globaltimer() - t0 > kWaitLimitNs) {
              atomicOr(derr, kErrWaitTimeout);
              break;
            }
          }
        }
      }
    }
  } else if (warp < kConsumerWarps) {
    // ----------------------------------------------------------- consumers
    constexpr int kChunksPerWarp = kChunksPerTile / kConsumerWarps;
    static_assert(kChunksPerTile % kConsumerWarps == 0, "chunks must split evenly");
    int s = 0;         // stage of the next tile
    uint32_t ph = 0u;  // its phase parity
    // One item of n body elements of row r (chunk ids count from its
    // start): stream its tiles, then publish the warp partial in slot
    // j % kSlots. The whole-row and split-row loops below each inline their
    // own copy, so the split bookkeeping costs the whole-row loop no
    // registers.
    auto consume = [&](int n, int j, int64_t r) -> bool {
      Ref ref{-INFINITY, -INFINITY, 0.f, 0.f, 0.f, -INFINITY, 0};
      Acc acc{0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
      Best best{-INFINITY, -INFINITY, -1, -1};
      ScanRegs sr{0, 0.f};
      if constexpr (kScan) {
        ScanArea& s = scan_area();
        sr.tf = __ldg(prm.scan.tf + r);
        if (lane == 0) s.region[warp] = prm.scan.regions + (r * kConsumerWarps + warp) * kRegionVecs;
        s.rest[0][warp][lane] = 0.0;
        s.rest[1][warp][lane] = 0.0;
        __syncwarp();
      }
      const int ntiles = (n + kStageElems - 1) / kStageElems;
      for (int t = 0; t < ntiles; ++t) {
        if (!mbar_wait(smem_u32(&ctrl->full[s]), ph, abort)) {
          fail(ctrl, derr);
          return false;
        }
        const uint4* tb = reinterpret_cast<const uint4*>(stage_b + s * kStageBytes);
        const uint4* tq = reinterpret_cast<const uint4*>(stage_q + s * kStageBytes);
        const int rem = n - t * kStageElems;
        if (rem >= kStageElems) {
          // Full tile: this warp's chunks, no masking. Not unrolled: one
          // copy of the chunk code keeps the hot loop small for the
          // instruction cache (measured faster than two copies).
#pragma unroll 1
          for (int k = 0; k < kChunksPerWarp; ++k) {
            const int c = warp + k * kConsumerWarps;
            process_chunk<DT, false, kScan>(tb + c * (kChunkElems / E), tq + c * (kChunkElems / E),
                                            lane, 0, ref, acc, best, t * kChunksPerTile + c, &sr);
          }
        } else {
          const int len = rem;
#pragma unroll 1
          for (int k = 0; k < kChunksPerWarp; ++k) {
            const int c = warp + k * kConsumerWarps;
            const int cstart = c * kChunkElems;
            if (cstart >= len) break;
            process_chunk<DT, true, kScan>(tb + cstart / E, tq + cstart / E, lane,
                                           (len - cstart) / E, ref, acc, best,
                                           t * kChunksPerTile + c, &sr);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctrl->empty[s]));
        if (++s == kStages) {
          s = 0;
          ph ^= 1u;
        }
      }

      // Publish the warp partial into the slot ring.
      const int slot = j % kSlots;
      const uint32_t sph = (j / kSlots) & 1u;
      const double Sb = warp_sum(acc.Sb), Ap = warp_sum(acc.Ap), C = warp_sum(acc.C);
      // Direct-path sums are zero unless some chunk of the row took that path
      // (a NaN compares unequal to zero and keeps them).
      double Ad = 0.0, Se = 0.0, Sh = 0.0;
      if (__any_sync(0xffffffffu, acc.Ad != 0.0 || acc.Se != 0.0 || acc.Sh != 0.0)) {
        Ad = warp_sum(acc.Ad);
        Se = warp_sum(acc.Se);
        Sh = warp_sum(acc.Sh);
      }
      double Sr = 0.0, Qr = 0.0;
      if constexpr (kScan) {
        const ScanArea& s = scan_area();
        Sr = warp_sum(s.rest[0][warp][lane]);
        Qr = warp_sum(s.rest[1][warp][lane]);
        if (lane == 0) prm.scan.counts[r * kConsumerWarps + warp] = sr.ncopy;
      }
      const float wb = warp_max(best.b);  // the warp's exact maxima of b and q
      const float wq = warp_max(best.q);
      const unsigned cb_mask = __ballot_sync(0xffffffffu, wb > -INFINITY && best.b == wb);
      const unsigned cq_mask = __ballot_sync(0xffffffffu, wq > -INFINITY && best.q == wq);
      if (!mbar_wait(smem_u32(&ctrl->slot_empty[slot]), sph ^ 1u, abort)) {
        fail(ctrl, derr);
        return false;
      }
      Slot& sl = ctrl->slot[slot];
      if ((cb_mask >> lane) & 1u) sl.loc_b[warp][lane] = best.lb;
      if ((cq_mask >> lane) & 1u) sl.loc_q[warp][lane] = best.lq;
      if (lane == 0) {
        WarpPart p;
        p.Mb = wb;
        p.Mq = wq;
        p.Rb = ref.Rb;
        p.Rq = ref.Rq;
        p.K = ref.K;
        p.pad = 0;
        p.Sb = Sb;
        p.Ap = Ap;
        p.C = C;
        p.Ad = Ad;
        p.Se = Se;
        p.Sh = Sh;
        p.cand_b = cb_mask;
        p.cand_q = cq_mask;
        sl.part[warp] = p;
        if constexpr (kScan) {
          sl.rest[warp][0] = Sr;
          sl.rest[warp][1] = Qr;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctrl->slot_full[slot]));
      return true;
    };
    if (sc.P <= 1 && sc.Gt == 0) {
      // Whole rows only (the common launch): a loop of its own, with
      // nothing else live across it (measured 2 % faster for 16-bit
      // inputs than the general loops below).
      for (int j = 0;; ++j) {
        const int64_t r = blockIdx.x + static_cast<int64_t>(j) * gridDim.x;
        if (r >= N) break;
        const RowGeom g = row_geom<DT>(B + r * V * EB, V);
        if (!consume(static_cast<int>(g.body_len), j, r)) break;
      }
    } else {
      bool ok = true;
      int j = 0;
      if (sc.P <= 1) {
        for (; j < sc.W; ++j) {  // whole rows
          const int64_t r = blockIdx.x + static_cast<int64_t>(j) * gridDim.x;
          if (r >= N) break;
          const RowGeom g = row_geom<DT>(B + r * V * EB, V);
          if (!(ok = consume(static_cast<int>(g.body_len), j, r))) break;
        }
      }
      if (ok) {  // parts of split rows
        Item it;
        RowGeom g;
        for (j = sc.P > 1 ? 0 : sc.W; item_at<DT>(j, sc, B, N, V, it, g); ++j)
          if (!consume(static_cast<int>(it.s1 - it.s0), j, it.r)) break;
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    Item it;
    RowGeom g;
    for (int j = 0; item_at<DT>(j, sc, B, N, V, it, g); ++j) {
      const int64_t r = it.r;
      const char* rb = B + r * V * EB;
      const char* rq = Q + r * V * EB;
      // Head/tail elements (one per lane; part 0 of a row only), issued
      // before waiting for the consumers' partials.
      const int n_extra = it.k == 0 ? static_cast<int>(g.head + g.tail) : 0;
      float xe_b = -INFINITY, xe_q = -INFINITY;
      int idx_e = INT_MAX;
      if (lane < n_extra) {
        const int64_t jj = lane < g.head ? lane : g.head + g.body_len + (lane - g.head);
        idx_e = static_cast<int>(jj);
        xe_b = Elem<DT>::load(rb, jj);
        xe_q = Elem<DT>::load(rq, jj);
      }
      // Next-token gather, issued now so that its latency hides behind the
      // consumers' work (the CTA that finalises the row needs it).
      int32_t tk = 0;
      bool tok_ok = false;
      float q_tok = 0.f, b_tok = 0.f;
      if (tok != nullptr && part_out == nullptr) {
        tk = __ldg(tok + r);
        tok_ok = tk >= 0 && static_cast<int64_t>(tk) < V;
        if (tok_ok) {
          q_tok = Elem<DT>::load(rq, tk);
          b_tok = Elem<DT>::load(rb, tk);
        }
      }
      Ref eref{-INFINITY, -INFINITY, 0.f, 0.f, 0.f, -INFINITY, 0};
      Acc eacc{0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
      Best ebest{-INFINITY, -INFINITY, -1, -1};
      if (n_extra > 0)
        chunk_step<1, DT == KLD_F32>(&xe_b, &xe_q, lane < n_extra ? 1u : 0u, eref, eacc, ebest, 0);
      const float eMb = warp_max(xe_b), eMq = warp_max(xe_q);
      const double eSb = warp_sum(eacc.Sb), eAp = warp_sum(eacc.Ap), eC = warp_sum(eacc.C);
      const double eAd = warp_sum(eacc.Ad), eSe = warp_sum(eacc.Se), eSh = warp_sum(eacc.Sh);

      const int slot = j % kSlots;
      const uint32_t sph = (j / kSlots) & 1u;
      const bool got = mbar_try_wait(smem_u32(&ctrl->slot_full[slot]), sph) ||
                       mbar_wait_idle(smem_u32(&ctrl->slot_full[slot]), sph, abort);
      MPart m = empty_part();
      double rest_b = 0.0, rest_q = 0.0;  // top-k scan: shares of the unflagged lanes
      if (!got) {
        // Whole rows: nothing is written for this or later rows. Split rows:
        // the part still travels, flagged, so the row's combine completes.
        fail(ctrl, derr);
        if (it.np == 1) break;
        m.flags = kPartFailed;
      } else {
      const Slot& sl = ctrl->slot[slot];

      // Lane w < 16 holds warp w's partial, lane 16 the head/tail partial,
      // each as a merged partial in its own frame and centre.
      MPart mp = empty_part();
      unsigned cand_b = 0u, cand_q = 0u;
      double lSr = 0.0, lQr = 0.0;  // top-k scan: this lane's warp, its frame and centre
      float lRb = 0.f, lK = 0.f;
      if (lane <= kConsumerWarps) {
        WarpPart p;
        if (lane < kConsumerWarps) {
          p = sl.part[lane];
          cand_b = p.cand_b;
          cand_q = p.cand_q;
          if constexpr (kScan) {
            if (p.Mb > -INFINITY) {
              lSr = sl.rest[lane][0];
              lQr = sl.rest[lane][1];
              lRb = p.Rb;
              lK = p.K;
            }
          }
        } else {
          p.Mb = eMb;
          p.Mq = eMq;
          p.Rb = eref.Rb;
          p.Rq = eref.Rq;
          p.K = eref.K;
          p.Sb = eSb;
          p.Ap = eAp;
          p.C = eC;
          p.Ad = eAd;
          p.Se = eSe;
          p.Sh = eSh;
        }
        mp.Mb = p.Mb;
        mp.Mq = p.Mq;
        if (p.Mb > -INFINITY) {
          mp.Cb = p.Rb;
          mp.K = p.K;
          mp.Sb = p.Sb;
          mp.A = p.Ap + p.Ad;
          // direct-path quant weights from their own frame to Rb - K*L
          const double Bh = p.Sh != 0.0 ? p.Sh * exp2(static_cast<double>(p.Rq) -
                                                       static_cast<double>(p.Rb) +
                                                       static_cast<double>(p.K) * kLog2eD)
                                        : 0.0;
          mp.B = kLambda * p.Ap + p.C + Bh - p.Se;
        } else {
          // no finite b: only quant weights, in their own frame (K = 0)
          mp.Cb = p.Rq;
          mp.B = p.Sh;
        }
        if (isnan(p.Sb) || isnan(p.Sh) || isnan(p.C)) mp.flags |= kPartNonfinite;
        if (!isfinite(p.Ad)) mp.flags |= kPartInfKl;
      }
      m = warp_merge(mp);
      if constexpr (kScan) {
        // the unflagged lanes' weights in the row's frame and centre (as
        // warp_merge moves S and S + B), as shares of S and S + B
        double sr = 0.0, qr = 0.0;
        if (lSr != 0.0 || lQr != 0.0) {
          const double fb = pow2i(lRb - m.Cb);
          sr = lSr * fb;
          qr = lQr * fb * (1.0 + expm1(kLambda * (static_cast<double>(m.K) - static_cast<double>(lK))));
        }
        rest_b = warp_sum(sr) / m.Sb;
        rest_q = warp_sum(qr) / (m.B + m.Sb);
      }

      // Exact lowest index of this part's maxima: re-read only the chunks
      // of lanes whose maximum equals it.
      if (!(m.flags & kPartNonfinite)) {
        const bool fin_b = m.Mb > -INFINITY && m.Mb < INFINITY;
        const bool fin_q = m.Mq > -INFINITY && m.Mq < INFINITY;
        int amb = (fin_b && xe_b == m.Mb) ? idx_e : INT_MAX;
        int amq = (fin_q && xe_q == m.Mq) ? idx_e : INT_MAX;
        amb = __reduce_min_sync(0xffffffffu, amb);
        amq = __reduce_min_sync(0xffffffffu, amq);
        unsigned wb = __ballot_sync(0xffffffffu, fin_b && lane < kConsumerWarps && mp.Mb == m.Mb);
        unsigned wq = __ballot_sync(0xffffffffu, fin_q && lane < kConsumerWarps && mp.Mq == m.Mq);
        // A split part of at most kStages tiles (the CTA's only item) is
        // still whole in the ring: rescan it there.
        const int64_t n_item = it.s1 - it.s0;
        Item nx;
        RowGeom ng;
        const bool in_ring = !it.whole && j == 0 &&
                             n_item <= static_cast<int64_t>(kStages) * (kStageBytes / EB) &&
                             !item_at<DT>(1, sc, B, N, V, nx, ng);
        while (wb) {
          const int w = __ffs(wb) - 1;
          wb &= wb - 1u;
          const unsigned cm = __shfl_sync(0xffffffffu, cand_b, w);
          const int i = rescan_candidates<DT>(rb, g, it.s0, cm, sl.loc_b[w], m.Mb, lane,
                                              in_ring ? stage_b : nullptr, n_item);
          if (i < amb) amb = i;
        }
        while (wq) {
          const int w = __ffs(wq) - 1;
          wq &= wq - 1u;
          const unsigned cm = __shfl_sync(0xffffffffu, cand_q, w);
          const int i = rescan_candidates<DT>(rq, g, it.s0, cm, sl.loc_q[w], m.Mq, lane,
                                              in_ring ? stage_q : nullptr, n_item);
          if (i < amq) amq = i;
        }
        m.amax_b = amb;
        m.amax_q = amq;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctrl->slot_empty[slot]));
      }


      if (part_out != nullptr) {
        // Vocabulary slice [col0, col0 + V) of a wider row: publish the
        // merged partial with global argmax indices, and the token's logits
        // when the token falls in this slice; the rows' slices meet in
        // kld_merge_kernel.
        MPart o = m;
        if (o.amax_b != INT_MAX) o.amax_b += static_cast<int>(col0);
        if (o.amax_q != INT_MAX) o.amax_q += static_cast<int>(col0);
        if (tok != nullptr) {
          const int64_t local = static_cast<int64_t>(__ldg(tok + r)) - col0;
          if (local >= 0 && local < V) {
            o.flags |= kPartHasTok;
            o.pad2 = pack2(Elem<DT>::load(rq, local), Elem<DT>::load(rb, local));
          }
        }
        if (lane == 0) {
          unsigned long long wds[8];
          part_words(o, wds);
          ulonglong2* dst = reinterpret_cast<ulonglong2*>(part_out + r);
#pragma unroll
          for (int w = 0; w < 4; ++w) dst[w] = make_ulonglong2(wds[2 * w], wds[2 * w + 1]);
        }
        continue;
      }
      if (it.np == 1) {  // the whole row is this item
        const kld_row_t rec = finalize_row(m, tok != nullptr, tok_ok, q_tok, b_tok);
        if (lane == 0) {
          if constexpr (kScan)
            write_row(prm, r, rec, m, rest_b, rest_q);
          else
            write_row(prm, r, rec, m);
        }
        if (prm.out != nullptr) count_row(prm.counter, rows, N, tok != nullptr, derr, prm.out, lane);
        continue;
      }

      // ---------------- split row: cluster combine through DSMEM, then across
      // the row's clusters (or the CTAs sharing a tail row) through global
      // memory and a ticket.
      MPart cm = m;
      int nparts = it.np, part = it.k;
      int64_t tix = it.rt;  // the row's ticket and partial slots
      if (sc.P > 1) {
        const uint32_t rank = G > 1 ? cluster_ctarank() : 0u;
        if (G > 1 && rank != 0) {
          // Push this CTA's partial into the leader's shared memory (its
          // barrier is initialised once the first cluster phase completes),
          // then arrive on the leader's barrier (release at cluster scope).
          asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
          cl_waited = true;
          if (lane == 0) {
            const uint32_t dst = map_to_rank(smem_u32(&ctrl->cl_part[rank]), 0u);
            unsigned long long wds[8];
            part_words(m, wds);
#pragma unroll
            for (int w = 0; w < 8; ++w)
              asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(dst + 8 * w), "l"(wds[w])
                           : "memory");
            const uint32_t bar = map_to_rank(smem_u32(&ctrl->cl_full), 0u);
            asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar)
                         : "memory");
          }
          continue;
        }
        if (G > 1) {
          // Wait (bounded) for the peers' partials; every lane acquires them.
          const uint32_t bar = smem_u32(&ctrl->cl_full);
          uint32_t okw = 0;
          const uint64_t t0 = globaltimer();
          for (uint32_t i = 0;; ++i) {
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(okw)
                : "r"(bar)
                : "memory");
            if (okw) break;
            if ((i & 63u) == 63u && globaltimer() - t0 > kWaitLimitNs) break;
          }
          MPart q = empty_part();
          if (__all_sync(0xffffffffu, okw != 0)) {
            if (lane == 0) q = m;
            if (lane >= 1 && lane < static_cast<int>(G)) {
              const ulonglong2* src = reinterpret_cast<const ulonglong2*>(&ctrl->cl_part[lane]);
              unsigned long long wds[8];
#pragma unroll
              for (int w = 0; w < 4; ++w) {
                const ulonglong2 v = src[w];
                wds[2 * w] = v.x;
                wds[2 * w + 1] = v.y;
              }
              q = part_from_words(wds);
            }
          } else {
            fail(ctrl, derr);
            if (lane == 0) {
              q = m;
              q.flags |= kPartFailed;
            }
          }
          cm = warp_merge(q);
        }
        nparts = sc.P / static_cast<int>(G);  // clusters per row
        part = it.k / static_cast<int>(G);
        tix = r;
        if (nparts == 1) {
          const kld_row_t rec = finalize_row(cm, tok != nullptr, tok_ok, q_tok, b_tok);
          if (lane == 0) write_row(prm, r, rec, cm);
          if (prm.out != nullptr) count_row(prm.counter, rows, N, tok != nullptr, derr, prm.out, lane);
          continue;
        }
      }
      MPart* slots = gparts + tix * kPartSlots;
      unsigned ticket = 0u;
      if (lane == 0) {
        unsigned long long wds[8];
        part_words(cm, wds);
        ulonglong2* dst = reinterpret_cast<ulonglong2*>(&slots[part]);
#pragma unroll
        for (int w = 0; w < 4; ++w) dst[w] = make_ulonglong2(wds[2 * w], wds[2 * w + 1]);
        // release: the partial above is visible to whoever sees the count;
        // acquire: the last arriver sees every other part's partial
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                     : "=r"(ticket)
                     : "l"(&tickets[tix])
                     : "memory");
      }
      ticket = __shfl_sync(0xffffffffu, ticket, 0);
      if (ticket != static_cast<unsigned>(nparts - 1)) continue;  // not the last part
      __syncwarp();  // lane 0's acquire orders the other lanes' loads below
      MPart q = empty_part();
      if (lane < nparts) {
        const ulonglong2* src = reinterpret_cast<const ulonglong2*>(&slots[lane]);
        unsigned long long wds[8];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const ulonglong2 v = __ldcg(src + w);
          wds[2 * w] = v.x;
          wds[2 * w + 1] = v.y;
        }
        q = part_from_words(wds);
      }
      const MPart fm = warp_merge(q);
      const kld_row_t rec = finalize_row(fm, tok != nullptr, tok_ok, q_tok, b_tok);
      if (lane == 0) {
        write_row(prm, r, rec, fm);
        tickets[tix] = 0u;  // ready for the next launch
      }
      if (prm.out != nullptr) count_row(prm.counter, rows, N, tok != nullptr, derr, prm.out, lane);
    }
  }

  if (G > 1) {
    // Second phase: no CTA leaves while a peer may still store into its
    // shared memory.
    if (!cl_waited) asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
  }

}

}  // namespace
}  // namespace kld
