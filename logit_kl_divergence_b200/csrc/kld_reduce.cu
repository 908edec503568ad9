// kld_reduce.cu -- fixed-order reduction and exact percentile selection over
// the per-row records of the row pass.
//
// Statistics ("Qwen3.6 27B Quantization Benchmark", "Raw benchmark data"
// table: Mean KLD, Same top p (%), Mean PPL(Q); median / p90 / p99 / max KLD
// are order statistics of the same per-row values):
//   mean KLD   = sum of the valid rows' KL / n_valid,
//   agreement  = valid rows whose two argmaxes are equal, and its percentage,
//   mean NLL   = sum over valid rows with an in-range token / their count,
//   PPL        = exp(mean NLL), and the same for the base model's NLL,
//   ln ratio   = mean NLL - mean base NLL = ln(PPL(Q) / PPL(base)),
//   dp         = exp(-NLL) - exp(-base NLL) = P_quant(tok) - P_base(tok) per
//                row (in the record, from the row pass); its mean and
//                sqrt(mean dp^2) ("Mistral-Small-4-119B-2603
//                GSQ-RCO IQ3_S GGUF", "Quality"; the Qwen3.6 table's RMS dp),
//   percentile = x_(k) + (pos - k) * (x_(k+1) - x_(k)),  pos = p*(n-1),
//                k = floor(pos), over the sorted valid KL values; max = x_(n-1).
//
// One CTA of T threads (T = 1024, or N rounded up to a warp multiple between
// 128 and 1024 when N is smaller, so small inputs pay for few threads):
//   1. thread t sums records t, t+T, ... in order; the T partials are
//      combined by a fixed shuffle tree, so the fp64 sums are deterministic
//      for a given N.
//   2. the up to seven ranks the percentiles need are selected exactly with
//      an MSB-first radix select on order-preserving 64-bit keys of the
//      doubles (8 bits per pass, one shared histogram per distinct prefix,
//      warp-aggregated shared atomics). As soon as the ranks' candidate sets
//      together hold at most kGatherCap keys, those keys are gathered into
//      shared memory and sorted (bitonic), which finishes the selection.
#include <climits>

#include "kld_internal.h"

namespace kld {
namespace {

constexpr int kTargets = 7;
constexpr int kAhead = 4;  // records each thread loads before using them
constexpr int kGatherCap = 4096;
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
__device__ double interpolate(double pos, double lo, double hi) {
  const double k = floor(pos);
  const double frac = __dsub_rn(pos, k);
  if (frac == 0.0 || lo == hi) return lo;
  return __dadd_rn(lo, __dmul_rn(frac, __dsub_rn(hi, lo)));
}

struct ReduceShared {
  double dsum[32][5];
  long long isum[32][4];
  unsigned int flags_or[32];
  // selection state
  unsigned long long prefix[kTargets];
  unsigned long long rank[kTargets];
  unsigned long long gprefix[kTargets];
  unsigned long long gcount[kTargets];
  int tgroup[kTargets];
  int ngroups;
  int done;
  int ncand;
  unsigned int hist[kTargets][256];
  unsigned long long cand[kGatherCap];
};

__global__ void __launch_bounds__(kReduceThreads, 1)
    kld_reduce_kernel(const kld_row_t* __restrict__ rows, int64_t N, int has_nll,
                      uint32_t* __restrict__ derr, kld_result_t* __restrict__ out) {
  __shared__ ReduceShared sh;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int nt = static_cast<int>(blockDim.x);
  // Launched as a programmatic dependent of the row pass: its launch may
  // overlap the row pass, the records are read only after it completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---------------------------------------------------------------- sums
  double s_kl = 0.0, s_nll = 0.0, s_nllb = 0.0, s_dp = 0.0, s_dp2 = 0.0;
  long long n_valid = 0, agree = 0, n_nll = 0, n_flag = 0;
  unsigned int f_or = 0;
  // Records t, t + T, ... in order; kAhead loads in flight per thread.
  for (int64_t i0 = tid; i0 < N; i0 += static_cast<int64_t>(kAhead) * nt) {
    kld_row_t rec[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int64_t i = i0 + static_cast<int64_t>(u) * nt;
      if (i < N) rec[u] = rows[i];
    }
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      if (i0 + static_cast<int64_t>(u) * nt >= N) break;
      const kld_row_t& rc = rec[u];
      f_or |= rc.flags;
      if (rc.flags) ++n_flag;
      if (rc.flags & kExcluded) continue;
      ++n_valid;
      s_kl += rc.kld;
      if (rc.argmax_base == rc.argmax_quant) ++agree;
      if (has_nll && !(rc.flags & KLD_ROW_BAD_TOKEN)) {
        s_nll += rc.nll;
        s_nllb += rc.nll_base;
        const double dp = static_cast<double>(rc.dp);  // computed per row by the row pass
        s_dp += dp;
        s_dp2 += dp * dp;
        ++n_nll;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s_kl += __shfl_down_sync(0xffffffffu, s_kl, o);
    s_nll += __shfl_down_sync(0xffffffffu, s_nll, o);
    s_nllb += __shfl_down_sync(0xffffffffu, s_nllb, o);
    s_dp += __shfl_down_sync(0xffffffffu, s_dp, o);
    s_dp2 += __shfl_down_sync(0xffffffffu, s_dp2, o);
    n_valid += __shfl_down_sync(0xffffffffu, n_valid, o);
    agree += __shfl_down_sync(0xffffffffu, agree, o);
    n_nll += __shfl_down_sync(0xffffffffu, n_nll, o);
    n_flag += __shfl_down_sync(0xffffffffu, n_flag, o);
    f_or |= __shfl_down_sync(0xffffffffu, f_or, o);
  }
  if (lane == 0) {
    sh.dsum[warp][0] = s_kl;
    sh.dsum[warp][1] = s_nll;
    sh.dsum[warp][2] = s_nllb;
    sh.dsum[warp][3] = s_dp;
    sh.dsum[warp][4] = s_dp2;
    sh.isum[warp][0] = n_valid;
    sh.isum[warp][1] = agree;
    sh.isum[warp][2] = n_nll;
    sh.isum[warp][3] = n_flag;
    sh.flags_or[warp] = f_or;
  }
  __syncthreads();
  if (warp == 0) {
    const bool has = lane < (nt >> 5);
    s_kl = has ? sh.dsum[lane][0] : 0.0;
    s_nll = has ? sh.dsum[lane][1] : 0.0;
    s_nllb = has ? sh.dsum[lane][2] : 0.0;
    s_dp = has ? sh.dsum[lane][3] : 0.0;
    s_dp2 = has ? sh.dsum[lane][4] : 0.0;
    n_valid = has ? sh.isum[lane][0] : 0;
    agree = has ? sh.isum[lane][1] : 0;
    n_nll = has ? sh.isum[lane][2] : 0;
    n_flag = has ? sh.isum[lane][3] : 0;
    f_or = has ? sh.flags_or[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s_kl += __shfl_down_sync(0xffffffffu, s_kl, o);
      s_nll += __shfl_down_sync(0xffffffffu, s_nll, o);
      s_nllb += __shfl_down_sync(0xffffffffu, s_nllb, o);
      s_dp += __shfl_down_sync(0xffffffffu, s_dp, o);
      s_dp2 += __shfl_down_sync(0xffffffffu, s_dp2, o);
      n_valid += __shfl_down_sync(0xffffffffu, n_valid, o);
      agree += __shfl_down_sync(0xffffffffu, agree, o);
      n_nll += __shfl_down_sync(0xffffffffu, n_nll, o);
      n_flag += __shfl_down_sync(0xffffffffu, n_flag, o);
      f_or |= __shfl_down_sync(0xffffffffu, f_or, o);
    }
    if (lane == 0) {
      sh.dsum[0][0] = s_kl;
      sh.dsum[0][1] = s_nll;
      sh.dsum[0][2] = s_nllb;
      sh.dsum[0][3] = s_dp;
      sh.dsum[0][4] = s_dp2;
      sh.isum[0][0] = n_valid;
      sh.isum[0][1] = agree;
      sh.isum[0][2] = n_nll;
      sh.isum[0][3] = n_flag;
      sh.flags_or[0] = f_or;
    }
  }
  __syncthreads();
  const long long nv = sh.isum[0][0];

  // ------------------------------------------------------------- selection
  const double ps[3] = {0.5, 0.9, 0.99};
  if (nv > 0) {
    if (tid < kTargets) {
      long long k;
      if (tid < 6) {
        const double pos = ps[tid >> 1] * static_cast<double>(nv - 1);
        k = static_cast<long long>(floor(pos)) + (tid & 1);
        if (k > nv - 1) k = nv - 1;
      } else {
        k = nv - 1;
      }
      sh.prefix[tid] = 0ull;
      sh.rank[tid] = static_cast<unsigned long long>(k);
    }
    if (tid == 0) {
      sh.done = 0;
      sh.ngroups = 1;
      sh.gprefix[0] = 0ull;
      sh.gcount[0] = static_cast<unsigned long long>(nv);
      for (int t = 0; t < kTargets; ++t) sh.tgroup[t] = 0;
    }
    __syncthreads();

    int decided = 0;  // number of high key bits fixed so far
    for (int shift = 56; shift >= 0; shift -= 8) {
      // Few candidates left: gather them and finish by sorting.
      unsigned long long total = 0;
      for (int g = 0; g < sh.ngroups; ++g) total += sh.gcount[g];
      if (total <= static_cast<unsigned long long>(kGatherCap)) break;

      const int ng = sh.ngroups;
      for (int i = tid; i < ng * 256; i += nt) (&sh.hist[0][0])[i] = 0u;
      __syncthreads();
      const uint64_t himask = decided == 0 ? 0ull : (~0ull << (64 - decided));
      // four records per thread in flight, then the warp-aggregated counts
      for (int64_t base_i = 0; base_i < N; base_i += static_cast<int64_t>(kAhead) * nt) {
        double kv[kAhead];
        uint32_t fv[kAhead];
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
          const int64_t i = base_i + static_cast<int64_t>(u) * nt + tid;
          fv[u] = kExcluded;
          if (i < N) {
            fv[u] = rows[i].flags;
            kv[u] = rows[i].kld;
          }
        }
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
          int slot = -1;
          if (!(fv[u] & kExcluded)) {
            const uint64_t key = order_key(kv[u]);
            for (int g = 0; g < ng; ++g) {
              if (((key ^ sh.gprefix[g]) & himask) == 0ull) {
                slot = g * 256 + static_cast<int>((key >> shift) & 0xffu);
                break;
              }
            }
          }
          const unsigned peers = __match_any_sync(0xffffffffu, slot);
          if (slot >= 0 && lane == __ffs(peers) - 1)
            atomicAdd(&(&sh.hist[0][0])[slot], static_cast<unsigned>(__popc(peers)));
        }
      }
      __syncthreads();
      for (int t = warp; t < kTargets; t += nt >> 5) {
        // One warp per target: 8 bins per lane, a warp prefix scan, then the
        // lane holding the rank finds its bin.
        const int g = sh.tgroup[t];
        const unsigned long long r = sh.rank[t];
        unsigned long long part = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) part += sh.hist[g][lane * 8 + b];
        unsigned long long incl = part;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const unsigned long long excl = incl - part;
        const unsigned hit = __ballot_sync(0xffffffffu, r >= excl && r < incl);
        const int owner = hit ? __ffs(hit) - 1 : 31;  // 31: unreachable for consistent counts
        if (lane == owner) {
          unsigned long long before = excl;
          int bin = lane * 8;
          for (int b = 0; b < 8; ++b) {
            bin = lane * 8 + b;
            const unsigned long long c = sh.hist[g][bin];
            if (r < before + c) break;
            before += c;
          }
          sh.prefix[t] = sh.gprefix[g] | (static_cast<unsigned long long>(bin) << shift);
          sh.rank[t] = r - before;
          sh.gcount[t] = sh.hist[g][bin];  // temporarily per target
        }
      }
      __syncthreads();
      if (tid == 0) {
        // Distinct prefixes become the next pass's groups.
        unsigned long long cnt[kTargets];
        for (int t = 0; t < kTargets; ++t) cnt[t] = sh.gcount[t];
        int n = 0;
        for (int t = 0; t < kTargets; ++t) {
          int g = -1;
          for (int j = 0; j < n; ++j)
            if (sh.gprefix[j] == sh.prefix[t]) g = j;
          if (g < 0) {
            g = n++;
            sh.gprefix[g] = sh.prefix[t];
            sh.gcount[g] = cnt[t];
          }
          sh.tgroup[t] = g;
        }
        sh.ngroups = n;
      }
      decided += 8;
      __syncthreads();
    }

    if (decided < 64) {
      // Gather every key whose decided bits match a group, sort, and index.
      if (tid == 0) sh.ncand = 0;
      __syncthreads();
      const uint64_t himask = decided == 0 ? 0ull : (~0ull << (64 - decided));
      const int ng = sh.ngroups;
      for (int64_t base_i = 0; base_i < N; base_i += nt) {
        const int64_t i = base_i + tid;
        bool take = false;
        uint64_t key = 0;
        if (i < N && !(rows[i].flags & kExcluded)) {
          key = order_key(rows[i].kld);
          for (int g = 0; g < ng; ++g)
            if (((key ^ sh.gprefix[g]) & himask) == 0ull) take = true;
        }
        // one shared atomic per warp
        const unsigned m = __ballot_sync(0xffffffffu, take);
        int basepos = 0;
        if (lane == 0 && m) basepos = atomicAdd(&sh.ncand, __popc(m));
        basepos = __shfl_sync(0xffffffffu, basepos, 0);
        if (take) {
          const int pos = basepos + __popc(m & ((1u << lane) - 1u));
          if (pos < kGatherCap) sh.cand[pos] = key;
        }
      }
      __syncthreads();
      int n = sh.ncand;
      if (n > kGatherCap) n = kGatherCap;  // unreachable: counts bound it
      int p2 = 1;
      while (p2 < n) p2 <<= 1;
      for (int i = n + tid; i < p2; i += nt) sh.cand[i] = ~0ull;
      __syncthreads();
      for (int k = 2; k <= p2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
          for (int i = tid; i < p2; i += nt) {
            const int ixj = i ^ j;
            if (ixj > i) {
              const unsigned long long a = sh.cand[i], b = sh.cand[ixj];
              const bool up = (i & k) == 0;
              if ((a > b) == up) {
                sh.cand[i] = b;
                sh.cand[ixj] = a;
              }
            }
          }
          __syncthreads();
        }
      }
      if (tid < kTargets) {
        // Groups are disjoint key ranges: a target's group starts after all
        // candidates of groups with smaller prefixes.
        const int g = sh.tgroup[tid];
        unsigned long long off = 0;
        for (int h = 0; h < ng; ++h)
          if (sh.gprefix[h] < sh.gprefix[g]) off += sh.gcount[h];
        const unsigned long long idx = off + sh.rank[tid];
        sh.prefix[tid] = idx < static_cast<unsigned long long>(n) ? sh.cand[idx] : ~0ull;
      }
      __syncthreads();
    }
  }

  if (tid == 0) {
    kld_result_t r;
    const double nan = __longlong_as_double(0x7ff8000000000000ll);
    r.n_rows = N;
    r.n_valid = nv;
    r.top1_agree = sh.isum[0][1];
    r.has_nll = has_nll ? 1 : 0;
    r.reserved0 = 0;
    r.n_nll = sh.isum[0][2];
    r.n_flagged = sh.isum[0][3];
    r.flags_or = sh.flags_or[0];
    r.device_error = 0u;
    if (derr) {  // report and clear the row pass's error word
      r.device_error = *derr;
      *derr = 0u;
    }
    if (nv > 0) {
      const double dn = static_cast<double>(nv - 1);
      r.mean_kld = sh.dsum[0][0] / static_cast<double>(nv);
      r.median_kld = interpolate(0.5 * dn, key_value(sh.prefix[0]), key_value(sh.prefix[1]));
      r.p90_kld = interpolate(0.9 * dn, key_value(sh.prefix[2]), key_value(sh.prefix[3]));
      r.p99_kld = interpolate(0.99 * dn, key_value(sh.prefix[4]), key_value(sh.prefix[5]));
      r.max_kld = key_value(sh.prefix[6]);
      r.top1_agree_pct = 100.0 * static_cast<double>(sh.isum[0][1]) / static_cast<double>(nv);
    } else {
      r.mean_kld = r.median_kld = r.p90_kld = r.p99_kld = r.max_kld = nan;
      r.top1_agree_pct = nan;
    }
    if (has_nll && sh.isum[0][2] > 0) {
      const double nn = static_cast<double>(sh.isum[0][2]);
      r.mean_nll = sh.dsum[0][1] / nn;
      r.ppl = exp(r.mean_nll);
      r.mean_nll_base = sh.dsum[0][2] / nn;
      r.ppl_base = exp(r.mean_nll_base);
      r.ln_ppl_ratio = r.mean_nll - r.mean_nll_base;
      r.mean_dp = sh.dsum[0][3] / nn;
      r.rms_dp = sqrt(sh.dsum[0][4] / nn);
    } else {
      r.mean_nll = r.ppl = nan;
      r.mean_nll_base = r.ppl_base = r.ln_ppl_ratio = nan;
      r.mean_dp = r.rms_dp = nan;
    }
    *out = r;
  }
}

}  // namespace

cudaError_t launch_reduce(const kld_row_t* rows, int64_t N, int has_nll, uint32_t* derr,
                          kld_result_t* out, cudaStream_t stream) {
  int threads = kReduceThreads;
  if (N < kReduceThreads) {
    threads = static_cast<int>((N + 31) / 32 * 32);
    if (threads < 128) threads = 128;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kld_reduce_kernel, rows, N, has_nll, derr, out);
}

}  // namespace kld
