// kld_rows.cu -- fused single-pass row kernel for sm_100a.
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
// at second order. Chunks where some |x| > 1.25 (or x is not finite: masked
// or infinite entries) take a direct path that sums h_j = 2^(q_j*L - R_q)
// with its own exponential instead. K follows (b - q) at the running maximum
// of b (per warp), so x is ~0 where the base mass sits and the split keeps
// its accuracy for peaked rows; moving K by d is an exact rebase in fp64:
// A += d*S, C -> e^{ld} C + (e^{ld} - 1) l A + (e^{ld} - 1 - l d) S. L = log2(e)
// rounded to fp32; all exponentials are of lambda*y with lambda = L*ln2
// = 1 + 1.4e-8, i.e. the statistic of softmax(lambda*b) and softmax(lambda*q),
// within 3e-8 relative of the exact one.
//
// Structure (one CTA per SM, persistent over rows r = blockIdx.x + k*grid):
//   - warp 16 (producer): one lane streams the 16-byte-aligned body of each
//     row pair in 32 KB tiles per operand into a 3-stage shared-memory ring
//     with cp.async.bulk (no multicast) completing on mbarriers, running
//     ahead across row boundaries.
//   - warps 0..15 (consumers): 512-element chunks (16 elements per lane,
//     conflict-free 16-byte shared loads): lane and warp maxima (redux.sync),
//     a warp-uniform frame raise when the maximum grew, then the fp32 terms
//     of the chunk folded into per-lane fp64 accumulators. Each lane also
//     remembers the first chunk in which its own maxima appeared. At the end
//     of a row each warp reduces its accumulators and publishes them in a
//     4-slot shared ring, then goes on with the next row.
//   - warp 17 (epilogue): per row, the unaligned head/tail (< 16 bytes each)
//     and the token gather, the exact lowest-index argmax (re-reading only
//     the chunks of lanes whose maximum equals the row maximum), the fp64
//     combine of the 17 partials and the 32-byte record.
//   All waits are mbarrier waits bounded by wall time; a wait that gives up
//   sets an error bit that the reduction reports, and the CTA leaves only
//   after its bulk copies have landed.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <climits>

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

// phi(y) = y^2 * P(y), P of degree 8 fitted on [-2.5, 2.5]
// (phi_poly_fit.py, max relative error of phi in fp32 9e-7); the kernel
// evaluates phi(lambda*x) = x^2 * Q(x), Q_k = P_k * lambda^(k+2).
// Narrower ranges need fewer terms; each chunk takes the cheapest
// polynomial whose range holds all of its |x| (same accuracy, ~5e-7):
// degree 5 on [-0.75, 0.75], degree 6 on [-1.25, 1.25], degree 8 on [-2.5, 2.5].
constexpr float kTauA = 0.75f, kTauB = 1.25f;
constexpr double kPA[6] = {0.5000001341, 0.1666664912, 0.0416622865,
                           0.00833420901, 0.001409831012, 0.0001987944535};
constexpr double kPB[7] = {0.5000000702, 0.1666677589, 0.04166594746, 0.008327533423,
                           0.001389740978, 0.0002059674399, 2.494043224e-05};
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
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort) {
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort) return false;
      if (globaltimer() - t0 > kWaitLimitNs) return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  return mbar_try_wait(bar, parity) || mbar_wait_slow(bar, parity, abort);
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
// The coefficients, scaled by lambda^(k+2), as (c, c) pairs in constant
// memory (packed FMAs take no immediates): 6 for tier A, 7 for tier B, 9 for
// tier C.
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
// Horner for tier T (0, 1, 2) with NC coefficients.
template <int T, int NC>
__device__ __forceinline__ f2 phi_q2(f2 x) {
  constexpr int o = T == 0 ? 0 : (T == 1 ? 6 : 13);
  f2 q = fma2(qc(o + NC - 1), x, qc(o + NC - 2));
#pragma unroll
  for (int k = NC - 3; k >= 0; --k) q = fma2(q, x, qc(o + k));
  return q;
}

// Maximum that propagates NaN (so a NaN anywhere fails a "<= bound" test).
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float y;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
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
struct Ref {
  float Mb;   // running maximum of b seen by this warp (-inf before any)
  float Mqf;  // maximum of q over this warp's direct-path chunks (-inf before)
  float Rb, Rq;  // integer frames floor(M*L) once M is finite, 0 before
  float K;       // log-ratio centre: (b - q) at the running maximum of b
};

// Per-lane fp64 accumulators (see the file comment): S_b over all chunks;
// Ap = sum e*x and C = sum e*phi over polynomial-path chunks; Ad = sum e*x,
// Se = sum e and Sh = sum h over direct-path chunks. A = Ap + Ad.
struct Acc {
  double Sb, Ap, C, Ad, Se, Sh;
};

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
};

struct Ctrl {
  unsigned long long full[kStages];
  unsigned long long empty[kStages];
  unsigned long long slot_full[kSlots];
  unsigned long long slot_empty[kSlots];
  int abort;
  int pad;
  Slot slot[kSlots];
};
static_assert(sizeof(Ctrl) <= kRowCtrlBytes, "control block too large");

// Exact 2^k for an integer-valued difference of frames (0 on underflow).
__device__ __forceinline__ double pow2i(float k) {
  return ldexp(1.0, static_cast<int>(fmaxf(k, -2000.f)));
}

// Polynomial path of one step: every x finite with |x| within tier T's range.
// S += e, Ap += e*x, C += e*x^2*Q_T(x), e = 2^(b*L - R_b).
template <int PE, int T, int NC>
__device__ __forceinline__ void poly_accumulate(const float* b, const f2* X, const Ref& r,
                                                Acc& a) {
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
    SC[j & 1] = fma2(mul2(T2, X[j]), phi_q2<T, NC>(X[j]), SC[j & 1]);
  }
  float sb0, sb1, sa0, sa1, sc0, sc1;
  upk(add2(SB[0], SB[1]), sb0, sb1);
  upk(add2(SA[0], SA[1]), sa0, sa1);
  upk(add2(SC[0], SC[1]), sc0, sc1);
  a.Sb += static_cast<double>(sb0 + sb1);
  a.Ap += static_cast<double>(sa0 + sa1);
  a.C += static_cast<double>(sc0 + sc1);
}

// One step of PE element pairs per lane (a 16-element consumer chunk, or the
// head/tail elements one per lane). Elements whose bit in `valid` is clear
// are absent (b = q = -inf, x = 0: they contribute nothing).
template <int PE>
__device__ __forceinline__ void chunk_step(const float* b, const float* q, unsigned valid,
                                           Ref& r, Acc& a, Best& best, int chunk_id) {
  float mb = b[0], mq = q[0];
#pragma unroll
  for (int i = 1; i + 1 < PE; i += 2) {
    mb = max3(mb, b[i], b[i + 1]);
    mq = max3(mq, q[i], q[i + 1]);
  }
  if (PE % 2 == 0) {
    mb = fmaxf(mb, b[PE - 1]);
    mq = fmaxf(mq, q[PE - 1]);
  }
  const float wmb = warp_max(mb);
  if (wmb > r.Mb) {  // raise the base frame and move the centre (warp-uniform)
    // New centre: (b - q) at the lowest lane's first element holding wmb.
    float dl = 0.f;
    bool has = false;
#pragma unroll
    for (int i = 0; i < PE; ++i) {
      if (!has && b[i] == wmb) {
        dl = b[i] - q[i];
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
          r.K = Kn;
        }
      } else {
        // First finite maximum: only direct-path terms of masked base
        // entries (e = 0) can have been accumulated.
        a.Ad += d * a.Se;
        r.K = Kn;
      }
    }
    if (r.Mb != -INFINITY) {
      const double sc = pow2i(r.Rb - nR);  // exact power of two
      a.Sb *= sc;
      a.Ap *= sc;
      a.C *= sc;
      a.Ad *= sc;
      a.Se *= sc;
    }
    r.Rb = nR;
    r.Mb = wmb;
  }

  // Log-ratios x = (q - b) + K, in packed pairs.
  constexpr int NP = (PE + 1) / 2;
  f2 X[NP];
  float ax0 = 0.f, ax1 = 0.f;  // max |x| of the lane (two chains), NaN if any x is NaN
  const f2 K2 = splat(r.K);
#pragma unroll
  for (int j = 0; j < NP; ++j) {
    const int i0 = 2 * j, i1 = (2 * j + 1 < PE) ? 2 * j + 1 : 2 * j;
    X[j] = add2(sub2(pk(q[i0], q[i1]), pk(b[i0], b[i1])), K2);
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
  // Warp max of |x| (NaN if any x is NaN: every comparison below fails).
  float wax;
  asm volatile("redux.sync.max.NaN.f32 %0, %1, 0xffffffff;" : "=f"(wax) : "f"(max3_nan(ax0, ax1, 0.f)));
  if (wax <= kTau) {
    poly_accumulate<PE, 2, 9>(b, X, r, a);
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
          sh += ex2(fmaf(q[i], kLog2e, nRq));
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
}

// One 512-element chunk of the current tile (16 elements per lane).
template <int DT, bool kMasked>
__device__ __forceinline__ void process_chunk(const uint4* cb, const uint4* cq, int lane,
                                              int valid_vecs, Ref& r, Acc& a, Best& best,
                                              int chunk_id) {
  constexpr int E = Elem<DT>::kPerVec;
  constexpr int VPC = kLaneElems / E;
  float xb[kLaneElems], xq[kLaneElems];
  unsigned valid = (1u << kLaneElems) - 1u;
#pragma unroll
  for (int k = 0; k < VPC; ++k) {
    const int vi = k * 32 + lane;
    const uint4 vb = cb[vi];
    const uint4 vq = cq[vi];
    Elem<DT>::unpack(vb, &xb[k * E]);
    Elem<DT>::unpack(vq, &xq[k * E]);
    if (kMasked && vi >= valid_vecs) {
      valid &= ~(((1u << E) - 1u) << (k * E));
#pragma unroll
      for (int i = 0; i < E; ++i) {
        xb[k * E + i] = -INFINITY;
        xq[k * E + i] = -INFINITY;
      }
    }
  }
  chunk_step<kLaneElems>(xb, xq, valid, r, a, best, chunk_id);
}

__device__ __forceinline__ void fail(Ctrl* ctrl, uint32_t* derr) {
  atomicOr(derr, kErrWaitTimeout);
  *reinterpret_cast<volatile int*>(&ctrl->abort) = 1;
}

// Row geometry: the unaligned head and tail (< 16 bytes each) are read
// directly; the 16-byte-aligned body is streamed in tiles.
struct RowGeom {
  int64_t head, body_len, tail, ntiles;
};

template <int DT>
__device__ __forceinline__ RowGeom row_geom(const void* rowb, int64_t V) {
  constexpr int EB = Elem<DT>::kBytes;
  constexpr int E = Elem<DT>::kPerVec;
  constexpr int64_t kStageElems = kStageBytes / EB;
  RowGeom g;
  const uint32_t mis = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(rowb) & 15u);
  g.head = static_cast<int64_t>(((16u - mis) & 15u) / EB);
  if (g.head > V) g.head = V;
  g.body_len = ((V - g.head) / E) * E;
  g.tail = V - g.head - g.body_len;
  g.ntiles = (g.body_len + kStageElems - 1) / kStageElems;
  return g;
}

// Offset (within the body) of element i of lane `lane` in chunk `chunk_id`.
template <int DT>
__device__ __forceinline__ int64_t chunk_elem_offset(int chunk_id, int lane, int i) {
  constexpr int E = Elem<DT>::kPerVec;
  return static_cast<int64_t>(chunk_id) * kChunkElems +
         static_cast<int64_t>((i / E) * 32 + lane) * E + (i % E);
}

// Lowest index holding `m` among the candidate lanes (mask) of one warp's
// published partial; lanes 0..15 of the calling warp each test one element.
template <int DT>
__device__ int rescan_candidates(const void* row, const RowGeom& g, unsigned mask,
                                 const int* locs, float m, int lane) {
  int best = INT_MAX;
  while (mask) {
    const int cl = __ffs(mask) - 1;
    mask &= mask - 1u;
    const int loc = locs[cl];
    int idx = INT_MAX;
    if (lane < kLaneElems && loc >= 0) {
      const int64_t off = chunk_elem_offset<DT>(loc, cl, lane);
      if (off < g.body_len && Elem<DT>::load(row, g.head + off) == m)
        idx = static_cast<int>(g.head + off);
    }
    idx = __reduce_min_sync(0xffffffffu, idx);
    if (idx < best) best = idx;
  }
  return best;
}

template <int DT>
__global__ void __launch_bounds__(kRowThreads, 1)
    kld_rows_kernel(const void* __restrict__ base, const void* __restrict__ quant,
                    const int32_t* __restrict__ tok, int64_t N, int64_t V,
                    kld_row_t* __restrict__ rows, uint32_t* __restrict__ derr) {
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&ctrl->full[s]), 1);
      mbar_init(smem_u32(&ctrl->empty[s]), kConsumerWarps);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(smem_u32(&ctrl->slot_full[s]), kConsumerWarps);
      mbar_init(smem_u32(&ctrl->slot_empty[s]), 1);
    }
    ctrl->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  const char* B = static_cast<const char*>(base);
  const char* Q = static_cast<const char*>(quant);

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = evict_first_policy();
      uint32_t it = 0;
      bool ok = true;
      for (int64_t r = blockIdx.x; r < N && ok; r += gridDim.x) {
        const char* rb = B + r * V * EB;
        const char* rq = Q + r * V * EB;
        const RowGeom g = row_geom<DT>(rb, V);
        for (int64_t t = 0; t < g.ntiles; ++t, ++it) {
          const int s = static_cast<int>(it % kStages);
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(smem_u32(&ctrl->empty[s]), ph ^ 1u, abort)) {
            fail(ctrl, derr);
            ok = false;
            break;
          }
          const int64_t off = g.head + t * kStageElems;
          int64_t len = g.body_len - t * kStageElems;
          if (len > kStageElems) len = kStageElems;
          const uint32_t bytes = static_cast<uint32_t>(len * EB);
          const uint32_t fb = smem_u32(&ctrl->full[s]);
          mbar_arrive_expect_tx(fb, 2u * bytes);
          bulk_load(smem_u32(stage_b + s * kStageBytes), rb + off * EB, bytes, fb, pol);
          bulk_load(smem_u32(stage_q + s * kStageBytes), rq + off * EB, bytes, fb, pol);
        }
      }
      // Never leave with copies in flight: wait (bounded) for the last
      // stages issued. In a normal run they have long completed.
      const uint32_t last = it < kStages ? it : kStages;
      for (uint32_t k = 0; k < last; ++k) {
        const uint32_t j = it - 1u - k;
        const int s = static_cast<int>(j % kStages);
        const uint32_t ph = (j / kStages) & 1u;
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
    return;
  }

  if (warp < kConsumerWarps) {
    // ----------------------------------------------------------- consumers
    constexpr int kChunksPerWarp = kChunksPerTile / kConsumerWarps;
    static_assert(kChunksPerTile % kConsumerWarps == 0, "chunks must split evenly");
    int s = 0;         // stage of the next tile
    uint32_t ph = 0u;  // its phase parity
    int rowk = 0;
    for (int64_t r = blockIdx.x; r < N; r += gridDim.x, ++rowk) {
      const char* rb = B + r * V * EB;
      const RowGeom g = row_geom<DT>(rb, V);
      Ref ref{-INFINITY, -INFINITY, 0.f, 0.f, 0.f};
      Acc acc{0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
      Best best{-INFINITY, -INFINITY, -1, -1};
      const int ntiles = static_cast<int>(g.ntiles);
      for (int t = 0; t < ntiles; ++t) {
        if (!mbar_wait(smem_u32(&ctrl->full[s]), ph, abort)) {
          fail(ctrl, derr);
          return;
        }
        const uint4* tb = reinterpret_cast<const uint4*>(stage_b + s * kStageBytes);
        const uint4* tq = reinterpret_cast<const uint4*>(stage_q + s * kStageBytes);
        const int64_t rem = g.body_len - static_cast<int64_t>(t) * kStageElems;
        if (rem >= kStageElems) {
          // Full tile: this warp's chunks, no masking.
#pragma unroll
          for (int k = 0; k < kChunksPerWarp; ++k) {
            const int c = warp + k * kConsumerWarps;
            process_chunk<DT, false>(tb + c * (kChunkElems / E), tq + c * (kChunkElems / E), lane,
                                     0, ref, acc, best, t * kChunksPerTile + c);
          }
        } else {
          const int len = static_cast<int>(rem);
#pragma unroll 1
          for (int k = 0; k < kChunksPerWarp; ++k) {
            const int c = warp + k * kConsumerWarps;
            const int cstart = c * kChunkElems;
            if (cstart >= len) break;
            process_chunk<DT, true>(tb + cstart / E, tq + cstart / E, lane, (len - cstart) / E,
                                    ref, acc, best, t * kChunksPerTile + c);
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
      const int slot = rowk % kSlots;
      const uint32_t sph = (rowk / kSlots) & 1u;
      const double Sb = warp_sum(acc.Sb), Ap = warp_sum(acc.Ap), C = warp_sum(acc.C);
      const double Ad = warp_sum(acc.Ad), Se = warp_sum(acc.Se), Sh = warp_sum(acc.Sh);
      const float wq = warp_max(best.q);  // the warp's maximum of q
      const unsigned cb_mask = __ballot_sync(0xffffffffu, ref.Mb > -INFINITY && best.b == ref.Mb);
      const unsigned cq_mask = __ballot_sync(0xffffffffu, wq > -INFINITY && best.q == wq);
      if (!mbar_wait(smem_u32(&ctrl->slot_empty[slot]), sph ^ 1u, abort)) {
        fail(ctrl, derr);
        return;
      }
      Slot& sl = ctrl->slot[slot];
      if ((cb_mask >> lane) & 1u) sl.loc_b[warp][lane] = best.lb;
      if ((cq_mask >> lane) & 1u) sl.loc_q[warp][lane] = best.lq;
      if (lane == 0) {
        WarpPart p;
        p.Mb = ref.Mb;
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
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctrl->slot_full[slot]));
    }
    return;
  }

  // ------------------------------------------------------------------ epilogue
  int rowk = 0;
  for (int64_t r = blockIdx.x; r < N; r += gridDim.x, ++rowk) {
    const char* rb = B + r * V * EB;
    const char* rq = Q + r * V * EB;
    const RowGeom g = row_geom<DT>(rb, V);

    // Head/tail elements (one per lane) and the next-token gather, issued
    // before waiting for the consumers' partials.
    const int n_extra = static_cast<int>(g.head + g.tail);
    float xe_b = -INFINITY, xe_q = -INFINITY;
    int idx_e = INT_MAX;
    if (lane < n_extra) {
      const int64_t j = lane < g.head ? lane : g.head + g.body_len + (lane - g.head);
      idx_e = static_cast<int>(j);
      xe_b = Elem<DT>::load(rb, j);
      xe_q = Elem<DT>::load(rq, j);
    }
    int32_t tk = 0;
    bool tok_ok = false;
    float q_tok = 0.f;
    if (tok != nullptr) {
      tk = __ldg(tok + r);
      tok_ok = tk >= 0 && static_cast<int64_t>(tk) < V;
      if (tok_ok && lane == 0) q_tok = Elem<DT>::load(rq, tk);
    }

    // The head/tail as one more partial of the same form.
    Ref eref{-INFINITY, -INFINITY, 0.f, 0.f, 0.f};
    Acc eacc{0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    Best ebest{-INFINITY, -INFINITY, -1, -1};
    if (n_extra > 0) {
      chunk_step<1>(&xe_b, &xe_q, lane < n_extra ? 1u : 0u, eref, eacc, ebest, 0);
    }
    const float eMq = warp_max(xe_q);
    const double eSb = warp_sum(eacc.Sb), eAp = warp_sum(eacc.Ap), eC = warp_sum(eacc.C);
    const double eAd = warp_sum(eacc.Ad), eSe = warp_sum(eacc.Se), eSh = warp_sum(eacc.Sh);

    const int slot = rowk % kSlots;
    const uint32_t sph = (rowk / kSlots) & 1u;
    if (!mbar_wait(smem_u32(&ctrl->slot_full[slot]), sph, abort)) {
      fail(ctrl, derr);
      return;
    }
    const Slot& sl = ctrl->slot[slot];

    // Lane w < 16 takes warp w's partial, lane 16 the head/tail partial.
    WarpPart p;
    if (lane < kConsumerWarps) {
      p = sl.part[lane];
    } else {
      p.Mb = p.Mq = -INFINITY;
      p.Rb = p.Rq = p.K = 0.f;
      p.pad = 0;
      p.Sb = p.Ap = p.C = p.Ad = p.Se = p.Sh = 0.0;
      p.cand_b = p.cand_q = 0u;
      if (lane == kConsumerWarps) {
        p.Mb = eref.Mb;
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
    }
    const float Mb = warp_max(p.Mb);
    const float Mq = warp_max(p.Mq);
    const bool nan_part = isnan(p.Sb) || isnan(p.Sh) || isnan(p.C);
    const bool nonfinite = __any_sync(0xffffffffu, nan_part) || !(Mb < INFINITY) ||
                           !(Mq < INFINITY);
    const bool empty = Mb == -INFINITY || Mq == -INFINITY;

    uint32_t flags = 0;
    if (tok != nullptr && !tok_ok) flags |= KLD_ROW_BAD_TOKEN;
    double kl = __longlong_as_double(0x7ff8000000000000ll);  // NaN
    double nll = kl;
    int ab = -1, aq = -1;
    if (nonfinite) {
      flags |= KLD_ROW_NONFINITE;
    } else if (empty) {
      flags |= KLD_ROW_EMPTY;
    } else {
      // Common frames and centre.
      const float Cb = warp_max(p.Mb > -INFINITY ? p.Rb : -INFINITY);
      // Centre of the part that holds the row maximum of b.
      const unsigned kmask = __ballot_sync(0xffffffffu, p.Mb == Mb);
      const float Kref = __shfl_sync(0xffffffffu, p.K, __ffs(kmask) - 1);
      // Only direct-path sums can be infinite: b_j finite where q_j = -inf.
      const bool inf_kl = __any_sync(0xffffffffu, !isfinite(p.Ad));
      const double dK = static_cast<double>(Kref) - static_cast<double>(p.K);
      const double fb = p.Mb > -INFINITY ? pow2i(p.Rb - Cb) : 0.0;
      // Polynomial-path part of B in the warp's own centre, moved to Kref:
      // e^{l(x+d)} - 1 = e^{l d}(e^{l x} - 1) + (e^{l d} - 1).
      const double Bp = kLambda * p.Ap + p.C;
      const double Sp = p.Sb - p.Se;
      const double em = expm1(kLambda * dK);
      const double BpK = Bp + em * (Bp + Sp);
      // Direct-path quant weights, from their own frame to Cb - Kref*L.
      const double Bh = p.Sh != 0.0
                            ? p.Sh * exp2(static_cast<double>(p.Rq) - static_cast<double>(Cb) +
                                          static_cast<double>(Kref) * kLog2eD)
                            : 0.0;
      const double sb = warp_sum(p.Sb * fb);
      const double sbB = warp_sum(BpK * fb + Bh - p.Se * fb);
      const double sa = warp_sum(inf_kl ? 0.0 : (p.Ap + p.Ad + dK * p.Sb) * fb);
      if (inf_kl) {
        kl = INFINITY;
        flags |= KLD_ROW_INF_KL;
      } else {
        kl = -kLambda * (sa / sb) + log1p(sbB / sb);
      }
      if (tok_ok) {
        const float qt = __shfl_sync(0xffffffffu, q_tok, 0);
        if (qt == -INFINITY) {
          nll = INFINITY;
          flags |= KLD_ROW_INF_NLL;
        } else {
          // B + S is the sum of all quant weights in frame Cb - Kref*L.
          nll = log(sbB + sb) +
                kLn2 * (static_cast<double>(Cb) -
                        (static_cast<double>(Kref) + static_cast<double>(qt)) * kLog2eD);
        }
      }
      // Lowest index of each row maximum.
      int amb = (xe_b == Mb) ? idx_e : INT_MAX;
      int amq = (xe_q == Mq) ? idx_e : INT_MAX;
      amb = __reduce_min_sync(0xffffffffu, amb);
      amq = __reduce_min_sync(0xffffffffu, amq);
      unsigned wb = __ballot_sync(0xffffffffu, lane < kConsumerWarps && p.Mb == Mb);
      unsigned wq = __ballot_sync(0xffffffffu, lane < kConsumerWarps && p.Mq == Mq);
      while (wb) {
        const int w = __ffs(wb) - 1;
        wb &= wb - 1u;
        const unsigned cm = __shfl_sync(0xffffffffu, p.cand_b, w);
        const int i = rescan_candidates<DT>(rb, g, cm, sl.loc_b[w], Mb, lane);
        if (i < amb) amb = i;
      }
      while (wq) {
        const int w = __ffs(wq) - 1;
        wq &= wq - 1u;
        const unsigned cm = __shfl_sync(0xffffffffu, p.cand_q, w);
        const int i = rescan_candidates<DT>(rq, g, cm, sl.loc_q[w], Mq, lane);
        if (i < amq) amq = i;
      }
      ab = amb;
      aq = amq;
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(smem_u32(&ctrl->slot_empty[slot]));
      kld_row_t rec;
      rec.kld = kl;
      rec.nll = nll;
      rec.argmax_base = ab;
      rec.argmax_quant = aq;
      rec.flags = flags;
      rec.reserved = 0u;
      rows[r] = rec;
    }
  }
}

}  // namespace

cudaError_t prepare_rows_kernels() {
  cudaError_t e;
  e = cudaFuncSetAttribute(kld_rows_kernel<KLD_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kRowSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kld_rows_kernel<KLD_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kRowSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kld_rows_kernel<KLD_F16>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, kRowSmemBytes);
}

cudaError_t launch_rows(const void* base, const void* quant, const int32_t* token_ids, int64_t N,
                        int64_t V, kld_dtype_t dtype, kld_row_t* rows, uint32_t* derr, int grid,
                        cudaStream_t stream) {
  const dim3 g(static_cast<unsigned>(grid)), b(kRowThreads);
  switch (dtype) {
    case KLD_F32:
      kld_rows_kernel<KLD_F32><<<g, b, kRowSmemBytes, stream>>>(base, quant, token_ids, N, V, rows,
                                                                 derr);
      break;
    case KLD_BF16:
      kld_rows_kernel<KLD_BF16><<<g, b, kRowSmemBytes, stream>>>(base, quant, token_ids, N, V,
                                                                  rows, derr);
      break;
    case KLD_F16:
      kld_rows_kernel<KLD_F16><<<g, b, kRowSmemBytes, stream>>>(base, quant, token_ids, N, V, rows,
                                                                 derr);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace kld
