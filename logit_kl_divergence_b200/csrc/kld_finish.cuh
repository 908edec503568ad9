// kld_finish.cuh -- the last steps of the statistic, shared by the reduction
// kernel and the row kernel's few-row path: order-preserving keys of the
// per-row KL values, the type-7 interpolation between two order statistics,
// a one-warp sort, and the assembly of kld_result_t from the fixed-order
// sums and the selected order statistics ("Qwen3.6 27B Quantization
// Benchmark", "Raw benchmark data" table: Mean KLD, Same top p (%), Mean
// PPL(Q); the percentiles are order statistics of the same per-row values).
// Device code only; included by .cu files of this library.
#pragma once

#include <stdint.h>

#include "kld_stats.h"

namespace kld {
namespace fin {

constexpr int kTargets = 7;  // ranks floor(p(n-1)) and +1 for p = .5, .9, .99, then n-1
constexpr uint32_t kExcluded = KLD_ROW_NONFINITE | KLD_ROW_EMPTY;

__device__ __forceinline__ uint64_t order_key(double x) {
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x));
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_value(uint64_t k) {
  const uint64_t b = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
  return __longlong_as_double(static_cast<long long>(b));
}

// Type-7 interpolation between the two selected order statistics, with
// explicitly rounded operations (no FMA contraction), so it rounds exactly as
// the plain expression lo + frac * (hi - lo) evaluated step by step.
__device__ __forceinline__ double interpolate(double pos, double lo, double hi) {
  const double k = floor(pos);
  const double frac = __dsub_rn(pos, k);
  if (frac == 0.0 || lo == hi) return lo;
  return __dadd_rn(lo, __dmul_rn(frac, __dsub_rn(hi, lo)));
}

// Ascending bitonic sort of one 64-bit key per lane.
__device__ __forceinline__ unsigned long long warp_sort(unsigned long long key, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, j);
      const bool up = (lane & k) == 0;
      const bool lower = (lane & j) == 0;
      key = (lower == up) ? (key < other ? key : other) : (key > other ? key : other);
    }
  }
  return key;
}

// Rank (among the nv valid values, ascending) of target t.
__device__ __forceinline__ long long target_rank(int t, long long nv) {
  if (t == 6) return nv - 1;
  const double ps[3] = {0.5, 0.9, 0.99};
  const double pos = ps[t >> 1] * static_cast<double>(nv - 1);
  long long k = static_cast<long long>(floor(pos)) + (t & 1);
  return k > nv - 1 ? nv - 1 : k;
}

// Fixed-order sums over the valid rows.
struct Sums {
  double kl, nll, nll_base, dp, dp2;
  long long n_valid, agree, n_nll, n_flag;
  unsigned flags_or;
};

// kld_result_t from the sums and the keys of the seven target ranks
// (tval[t] = key of the value of rank target_rank(t, n_valid)).
__device__ __forceinline__ kld_result_t make_result(int64_t N, const Sums& s,
                                                    const unsigned long long* tval, int has_nll,
                                                    uint32_t device_error) {
  kld_result_t r;
  const double nan = __longlong_as_double(0x7ff8000000000000ll);
  const long long nv = s.n_valid;
  r.n_rows = N;
  r.n_valid = nv;
  r.top1_agree = s.agree;
  r.has_nll = has_nll ? 1 : 0;
  r.reserved0 = 0;
  r.n_nll = s.n_nll;
  r.n_flagged = s.n_flag;
  r.flags_or = s.flags_or;
  r.device_error = device_error;
  if (nv > 0) {
    const double dn = static_cast<double>(nv - 1);
    r.mean_kld = s.kl / static_cast<double>(nv);
    r.median_kld = interpolate(0.5 * dn, key_value(tval[0]), key_value(tval[1]));
    r.p90_kld = interpolate(0.9 * dn, key_value(tval[2]), key_value(tval[3]));
    r.p99_kld = interpolate(0.99 * dn, key_value(tval[4]), key_value(tval[5]));
    r.max_kld = key_value(tval[6]);
    r.top1_agree_pct = 100.0 * static_cast<double>(s.agree) / static_cast<double>(nv);
  } else {
    r.mean_kld = r.median_kld = r.p90_kld = r.p99_kld = r.max_kld = nan;
    r.top1_agree_pct = nan;
  }
  if (has_nll && s.n_nll > 0) {
    const double nn = static_cast<double>(s.n_nll);
    r.mean_nll = s.nll / nn;
    r.ppl = exp(r.mean_nll);
    r.mean_nll_base = s.nll_base / nn;
    r.ppl_base = exp(r.mean_nll_base);
    r.ln_ppl_ratio = r.mean_nll - r.mean_nll_base;
    r.mean_dp = s.dp / nn;
    r.rms_dp = sqrt(s.dp2 / nn);
  } else {
    r.mean_nll = r.ppl = nan;
    r.mean_nll_base = r.ppl_base = r.ln_ppl_ratio = nan;
    r.mean_dp = r.rms_dp = nan;
  }
  return r;
}

// Adds one record to a thread's running sums (the reduction's per-thread
// step). Returns whether the row is valid.
__device__ __forceinline__ bool add_record(Sums& s, const kld_row_t& rc, int has_nll) {
  const bool valid = !(rc.flags & kExcluded);
  s.flags_or |= rc.flags;
  if (rc.flags) ++s.n_flag;
  if (valid) {
    ++s.n_valid;
    s.kl += rc.kld;
    if (rc.argmax_base == rc.argmax_quant) ++s.agree;
    if (has_nll && !(rc.flags & KLD_ROW_BAD_TOKEN)) {
      s.nll += rc.nll;
      s.nll_base += rc.nll_base;
      const double dp = static_cast<double>(rc.dp);
      s.dp += dp;
      s.dp2 += dp * dp;
      ++s.n_nll;
    }
  }
  return valid;
}

// Shuffle-down tree over the 32 lanes of a warp (lane 0 ends with the total).
__device__ __forceinline__ void warp_tree(Sums& s) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s.kl += __shfl_down_sync(0xffffffffu, s.kl, o);
    s.nll += __shfl_down_sync(0xffffffffu, s.nll, o);
    s.nll_base += __shfl_down_sync(0xffffffffu, s.nll_base, o);
    s.dp += __shfl_down_sync(0xffffffffu, s.dp, o);
    s.dp2 += __shfl_down_sync(0xffffffffu, s.dp2, o);
    s.n_valid += __shfl_down_sync(0xffffffffu, s.n_valid, o);
    s.agree += __shfl_down_sync(0xffffffffu, s.agree, o);
    s.n_nll += __shfl_down_sync(0xffffffffu, s.n_nll, o);
    s.n_flag += __shfl_down_sync(0xffffffffu, s.n_flag, o);
    s.flags_or |= __shfl_down_sync(0xffffffffu, s.flags_or, o);
  }
}

__device__ __forceinline__ Sums zero_sums() {
  Sums s;
  s.kl = s.nll = s.nll_base = s.dp = s.dp2 = 0.0;
  s.n_valid = s.agree = s.n_nll = s.n_flag = 0;
  s.flags_or = 0u;
  return s;
}

// The whole statistic of N <= 32 records by one warp, in the same
// arithmetic order as the reduction kernel takes for so few rows (lane i
// holds record i, a shuffle tree within the warp, then the tree over the
// per-warp totals, where every other warp's total is zero), so both give
// identical bits. Records are read through L2 (they were written by other
// SMs); the device error word is read and cleared; the result goes to *out.
__device__ __forceinline__ void reduce_few_rows(const kld_row_t* rows, int N, int has_nll,
                                                uint32_t* derr, kld_result_t* out, int lane) {
  // The error word is taken first: its round trip overlaps the record loads.
  // Every row's record is written, so every consumer and epilogue wait of
  // the pass has ended. The one wait that can still end later is a
  // producer's bounded drain of its own last bulk copies, after its CTA's
  // part is done; those copies were consumed before the record could be
  // written, so the drain finds them complete. Were one still to time out,
  // its bit would be reported by the next run of the same handle, not this.
  const uint32_t de = (lane == 0 && derr) ? atomicExch(derr, 0u) : 0u;
  Sums s = zero_sums();
  unsigned long long key = ~0ull;  // lanes past N sort last
  if (lane < N) {
    const kld_row_t* p = rows + lane;
    kld_row_t rc;
    rc.kld = __ldcg(&p->kld);
    rc.nll = __ldcg(&p->nll);
    rc.nll_base = __ldcg(&p->nll_base);
    rc.argmax_base = __ldcg(&p->argmax_base);
    rc.argmax_quant = __ldcg(&p->argmax_quant);
    rc.flags = __ldcg(&p->flags);
    rc.dp = __ldcg(&p->dp);
    key = add_record(s, rc, has_nll) ? order_key(rc.kld) : 0ull;
  }
  warp_tree(s);
  // second level: lane 0 holds this warp's total, the others zeros
  if (lane != 0) s = zero_sums();
  warp_tree(s);
  Sums t;
  t.kl = __shfl_sync(0xffffffffu, s.kl, 0);
  t.nll = __shfl_sync(0xffffffffu, s.nll, 0);
  t.nll_base = __shfl_sync(0xffffffffu, s.nll_base, 0);
  t.dp = __shfl_sync(0xffffffffu, s.dp, 0);
  t.dp2 = __shfl_sync(0xffffffffu, s.dp2, 0);
  t.n_valid = __shfl_sync(0xffffffffu, s.n_valid, 0);
  t.agree = __shfl_sync(0xffffffffu, s.agree, 0);
  t.n_nll = __shfl_sync(0xffffffffu, s.n_nll, 0);
  t.n_flag = __shfl_sync(0xffffffffu, s.n_flag, 0);
  t.flags_or = __shfl_sync(0xffffffffu, s.flags_or, 0);
  // excluded rows carry key 0 and sort first, offsetting the ranks
  key = warp_sort(key, lane);
  unsigned long long tval[kTargets];
  const long long nv = t.n_valid;
#pragma unroll
  for (int q = 0; q < kTargets; ++q) {
    const int src = nv > 0 ? static_cast<int>(target_rank(q, nv) + (N - nv)) : 0;
    tval[q] = __shfl_sync(0xffffffffu, key, src);
  }
  if (lane == 0) *out = make_result(N, t, tval, has_nll, de);
}

}  // namespace fin
}  // namespace kld
