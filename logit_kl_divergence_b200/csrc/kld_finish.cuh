// kld_finish.cuh -- the last steps of the statistic, shared by the reduction
// kernel and the row kernel's few-row path: order-preserving keys of the
// per-row KL values, the type-7 interpolation between two order statistics,
// a one-warp sort, fixed-order sums, the exact MSB radix selection of the
// order statistics, and the assembly of kld_result_t ("Qwen3.6 27B
// Quantization Benchmark", "Raw benchmark data" table: Mean KLD, Same top p
// (%), Mean PPL(Q); the percentiles are order statistics of the same per-row
// values). Device code only; included by .cu files of this library.
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


// ------------------------------------------------------------- selection

constexpr int kAhead = 4;       // keys each thread loads before using them
constexpr int kDigitBits = 11;  // radix digit of the selection
constexpr int kBins = 1 << kDigitBits;
constexpr int kSmall = 32;      // a group this small is finished by one warp

// Selection state in shared memory: groups of targets whose keys share the
// digits decided so far.
struct SelectShared {
  unsigned long long gprefix[kTargets];
  unsigned long long tnext[kTargets];  // a target's prefix after this level
  unsigned long long trank[kTargets];  // its rank among its group's keys
  unsigned long long tval[kTargets];   // its key, once found
  unsigned int gcount[kTargets];
  unsigned int gfill[kTargets];
  unsigned int tcount[kTargets];  // size of a target's group after this level
  int tgroup[kTargets];           // -1 once found
  int ngroups;
  unsigned int hist[kTargets][kBins];
  unsigned long long gbuf[kTargets][kSmall];
};

// Exact order statistics by an MSB-first radix select with 11-bit digits,
// run by all nt threads of the CTA from `decided` known leading bits on.
// On entry (visible to all threads): ngroups groups with prefix gprefix[g]
// (the decided bits) and key count gcount[g]; every open target t has
// tgroup[t] >= 0 and its rank trank[t] among its group's keys; found targets
// have tgroup[t] = -1. src.at(i), i < n_keys, gives the keys (keys outside
// every group are ignored). Per level: one shared histogram per group, a warp
// per target finds its digit and residual rank, and warp 0 regroups the
// targets by their new prefix; a group of at most kSmall keys is gathered and
// sorted by one warp, which ends its targets; a group still open after all 64
// bits holds equal keys. On return tval[t] holds every target's key.
// Where select_levels reads its keys: an array of keys (shared or global
// memory, read through L2), or the KL values of records (key 0 for excluded
// rows).
struct KeySource {
  const unsigned long long* keys;  // nullable
  const kld_row_t* rows;           // used when keys is null
  bool global;                     // keys in global memory written by this kernel
  __device__ __forceinline__ unsigned long long at(int64_t i) const {
    if (keys != nullptr) return global ? __ldcg(keys + i) : keys[i];
    return (rows[i].flags & kExcluded) ? 0ull : order_key(rows[i].kld);
  }
};

__device__ __forceinline__ void select_levels(SelectShared& sh, KeySource src, int64_t n_keys,
                                              int decided, int nt) {
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int nw = nt >> 5;
  for (;;) {
    bool open = false;
    for (int t = 0; t < kTargets; ++t) open |= sh.tgroup[t] >= 0;
    if (!open) break;
    const int ng = sh.ngroups;
    if (decided >= 64) {
      // every key of a remaining group equals its prefix
      if (tid < kTargets && sh.tgroup[tid] >= 0) {
        sh.tval[tid] = sh.gprefix[sh.tgroup[tid]];
        sh.tgroup[tid] = -1;
      }
      __syncthreads();
      break;
    }
    const int bits = 64 - decided < kDigitBits ? 64 - decided : kDigitBits;
    const int shift = 64 - decided - bits;
    const unsigned long long himask = decided == 0 ? 0ull : (~0ull << (64 - decided));
    for (int i = tid; i < ng * kBins; i += nt)
      if (sh.gcount[i / kBins] > static_cast<unsigned>(kSmall)) (&sh.hist[0][0])[i] = 0u;
    if (tid < ng) sh.gfill[tid] = 0u;
    __syncthreads();

    // One pass over the keys: gather the keys of small groups, count the
    // next digit of the keys of large ones.
    for (int64_t base = 0; base < n_keys; base += static_cast<int64_t>(kAhead) * nt) {
      unsigned long long kv[kAhead];
      bool ok[kAhead];
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        const int64_t i = base + static_cast<int64_t>(u) * nt + tid;
        ok[u] = i < n_keys;
        kv[u] = ok[u] ? src.at(i) : 0ull;
      }
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        int g = -1;
        if (ok[u]) {
          for (int h = 0; h < ng; ++h) {
            if (((kv[u] ^ sh.gprefix[h]) & himask) == 0ull) {
              g = h;
              break;
            }
          }
        }
        const bool small = g >= 0 && sh.gcount[g] <= static_cast<unsigned>(kSmall);
        if (small) {
          const unsigned p = atomicAdd(&sh.gfill[g], 1u);
          if (p < static_cast<unsigned>(kSmall)) sh.gbuf[g][p] = kv[u];
        }
        const int slot = (g >= 0 && !small)
                             ? g * kBins + static_cast<int>((kv[u] >> shift) & (kBins - 1))
                             : -1;
        if (decided == 0) {
          // first digit: few distinct bins, one atomic per bin and warp
          const unsigned peers = __match_any_sync(0xffffffffu, slot);
          if (slot >= 0 && lane == __ffs(peers) - 1)
            atomicAdd(&(&sh.hist[0][0])[slot], static_cast<unsigned>(__popc(peers)));
        } else if (slot >= 0) {
          atomicAdd(&(&sh.hist[0][0])[slot], 1u);  // later digits spread out
        }
      }
    }
    __syncthreads();

    // A warp per open target: finish a small group by sorting its keys, or
    // find the target's digit in its group's histogram. Lane L sums bins
    // [64L, 64L + 64) (rotated start: conflict-free), a warp scan finds the
    // lane whose range holds the rank, and the warp scans those 64 bins.
    for (int t = warp; t < kTargets; t += nw) {
      const int g = sh.tgroup[t];
      if (g < 0) continue;
      const unsigned cnt = sh.gcount[g];
      const unsigned long long r = sh.trank[t];
      if (cnt <= static_cast<unsigned>(kSmall)) {
        const unsigned long long key =
            warp_sort(lane < static_cast<int>(cnt) ? sh.gbuf[g][lane] : ~0ull, lane);
        const unsigned long long v = __shfl_sync(0xffffffffu, key, static_cast<int>(r & 31));
        if (lane == 0) sh.tval[t] = v;
        continue;
      }
      constexpr int kPer = kBins / 32;
      const unsigned* hg = sh.hist[g];
      unsigned long long part = 0;
#pragma unroll 8
      for (int b = 0; b < kPer; ++b) part += hg[lane * kPer + ((b + lane) & (kPer - 1))];
      unsigned long long incl = part;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const unsigned long long excl = incl - part;
      const unsigned hit = __ballot_sync(0xffffffffu, r >= excl && r < incl);
      const int owner = hit ? __ffs(hit) - 1 : 31;  // 31: unreachable for consistent counts
      const unsigned long long before = __shfl_sync(0xffffffffu, excl, owner);
      const unsigned c0 = hg[owner * kPer + lane], c1 = hg[owner * kPer + 32 + lane];
      unsigned long long s0 = c0, s1 = c1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long v0 = __shfl_up_sync(0xffffffffu, s0, o);
        const unsigned long long v1 = __shfl_up_sync(0xffffffffu, s1, o);
        if (lane >= o) {
          s0 += v0;
          s1 += v1;
        }
      }
      s1 += __shfl_sync(0xffffffffu, s0, 31);
      const unsigned long long rr = r - before;  // rank within the owner's 64 bins
      const unsigned m0 = __ballot_sync(0xffffffffu, s0 > rr);
      const unsigned m1 = __ballot_sync(0xffffffffu, s1 > rr);
      const int j = m0 ? __ffs(m0) - 1 : 32 + (m1 ? __ffs(m1) - 1 : 31);
      const unsigned long long incl_j = __shfl_sync(0xffffffffu, j < 32 ? s0 : s1, j & 31);
      const unsigned cnt_j = __shfl_sync(0xffffffffu, j < 32 ? c0 : c1, j & 31);
      if (lane == 0) {
        const int bin = owner * kPer + j;
        sh.tnext[t] = sh.gprefix[g] | (static_cast<unsigned long long>(bin) << shift);
        sh.trank[t] = rr - (incl_j - cnt_j);
        sh.tcount[t] = cnt_j;
      }
    }
    __syncthreads();
    if (warp == 0) {
      // Targets of small groups are done; the others regroup by their new
      // prefix (lane t = target t; groups numbered in lane order).
      const int g0 = lane < kTargets ? sh.tgroup[lane] : -1;
      const bool act = g0 >= 0 && sh.gcount[g0] > static_cast<unsigned>(kSmall);
      const unsigned long long p = act ? sh.tnext[lane] : ~0ull;
      const unsigned cnt = act ? sh.tcount[lane] : 0u;
      const unsigned peers = __match_any_sync(0xffffffffu, p);
      const int leader = __ffs(peers) - 1;
      const unsigned leaders = __ballot_sync(0xffffffffu, act && lane == leader);
      const int gid = __popc(leaders & ((1u << leader) - 1u));
      __syncwarp();
      if (act && lane == leader) {
        sh.gprefix[gid] = p;
        sh.gcount[gid] = cnt;
      }
      if (lane < kTargets) sh.tgroup[lane] = act ? gid : -1;
      if (lane == 0) sh.ngroups = __popc(leaders);
    }
    decided += bits;
    __syncthreads();
  }
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
