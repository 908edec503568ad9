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
//      for a given N. The same pass appends the order-preserving 64-bit keys
//      of the valid rows' KL to shared memory (N <= kKeyCap; larger inputs
//      re-read the records for every level instead).
//   2. the up to seven ranks the percentiles need are selected exactly: for
//      at most kCountMax keys by counting each key's rank (ties ordered by
//      index); otherwise by an MSB-first radix select with 11-bit digits: per level, one shared
//      histogram per distinct group of targets (keys that share the digits
//      decided so far), a warp per group scans its 2048 bins and finds the
//      digit and residual rank of each of its targets. A group of at most
//      32 keys is gathered and sorted in one warp instead, which ends its
//      targets; a group still large after all 64 bits holds equal keys.

#include <atomic>
#include <climits>

#include "kld_finish.cuh"
#include "kld_internal.h"

namespace kld {
namespace {

using fin::kExcluded;
using fin::kTargets;
using fin::order_key;
using fin::warp_sort;
using fin::kAhead;
constexpr int kKeyCap = 19968;  // keys kept in shared memory (N up to this)
constexpr int kCountMax = 512;  // up to this many keys: ranks by counting instead of radix levels

struct ReduceShared {
  double dsum[32][5];
  long long isum[32][4];
  unsigned int flags_or[32];
  fin::SelectShared sel;
};
constexpr size_t kReduceSmemMax = sizeof(ReduceShared) + sizeof(unsigned long long) * kKeyCap;
static_assert(kReduceSmemMax <= 227 * 1024, "reduction shared memory");

__global__ void __launch_bounds__(kReduceThreads, 1)
    kld_reduce_kernel(const kld_row_t* __restrict__ rows, int64_t N, int has_nll,
                      uint32_t* __restrict__ derr, kld_result_t* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char reduce_smem[];
  ReduceShared& sh = *reinterpret_cast<ReduceShared*>(reduce_smem);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(reduce_smem + sizeof(ReduceShared));
  const bool in_smem = N <= kKeyCap;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int nt = static_cast<int>(blockDim.x);
  // Launched as a programmatic dependent of the row pass: its launch may
  // overlap the row pass, the records are read only after it completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ------------------------------------------------------- sums and keys
  double s_kl = 0.0, s_nll = 0.0, s_nllb = 0.0, s_dp = 0.0, s_dp2 = 0.0;
  long long n_valid = 0, agree = 0, n_nll = 0, n_flag = 0;
  unsigned int f_or = 0;
  // Records t, t + T, ... in order; kAhead loads in flight per thread.
  for (int64_t base = 0; base < N; base += static_cast<int64_t>(kAhead) * nt) {
    kld_row_t rec[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int64_t i = base + static_cast<int64_t>(u) * nt + tid;
      if (i < N) rec[u] = rows[i];
    }
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const bool in = base + static_cast<int64_t>(u) * nt + tid < N;
      const kld_row_t& rc = rec[u];
      const bool valid = in && !(rc.flags & kExcluded);
      if (in) {
        f_or |= rc.flags;
        if (rc.flags) ++n_flag;
      }
      if (valid) {
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
      // Key of every record in place; excluded rows get key 0, below every
      // key of a non-NaN value, and the ranks are offset by their number.
      if (in_smem && in) keys[base + static_cast<int64_t>(u) * nt + tid] = valid ? order_key(rc.kld) : 0ull;
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
  fin::SelectShared& sel = sh.sel;
  if (tid < kTargets) {
    sel.tval[tid] = 0ull;
    sel.tgroup[tid] = -1;
  }
  __syncthreads();
  if (nv > 0) {
    if (tid < kTargets) {
      sel.trank[tid] = static_cast<unsigned long long>(fin::target_rank(tid, nv));
      sel.tgroup[tid] = 0;
    }
    // Excluded rows have key 0, below every other key: they come first and
    // offset the ranks.
    __syncthreads();
    if (in_smem && N <= 32) {
      // Few rows: one warp sorts all keys.
      if (warp == 0) {
        const unsigned long long key = warp_sort(lane < N ? keys[lane] : ~0ull, lane);
        for (int t = 0; t < kTargets; ++t) {
          const unsigned long long v =
              __shfl_sync(0xffffffffu, key, static_cast<int>(sel.trank[t] + (N - nv)));
          if (lane == 0) {
            sel.tval[t] = v;
            sel.tgroup[t] = -1;
          }
        }
      }
      __syncthreads();
    }
    if (tid < kTargets) sel.trank[tid] += static_cast<unsigned long long>(N - nv);
    if (in_smem && N > 32 && N <= kCountMax) {
      // A few hundred keys: each key's rank by counting the keys before it
      // (equal keys ordered by index, so the ranks are 0..N-1, each once),
      // and the keys at the target ranks read off directly. At this size
      // that is cheaper than the radix levels, whose fixed costs (clearing
      // and scanning 2048-bin histograms, a barrier per step) dominate.
      __syncthreads();
      for (int i = tid; i < N; i += nt) {
        const unsigned long long k = keys[i];
        unsigned rank = 0u;
#pragma unroll 4
        for (int j = 0; j < N; ++j) {
          const unsigned long long y = keys[j];  // same address in every lane: broadcast
          rank += (y < k || (y == k && j < i)) ? 1u : 0u;
        }
#pragma unroll
        for (int t = 0; t < kTargets; ++t)
          if (sel.trank[t] == rank) sel.tval[t] = k;
      }
      __syncthreads();
    } else {
      if (tid == 0) {
        sel.ngroups = 1;
        sel.gprefix[0] = 0ull;
        sel.gcount[0] = static_cast<unsigned int>(N);
      }
      __syncthreads();
      fin::select_levels(sel, in_smem ? fin::KeySource{keys, nullptr, false}
                                      : fin::KeySource{nullptr, rows, false},
                         N, 0, nt);
    }
  }

  if (tid == 0) {
    fin::Sums s;
    s.kl = sh.dsum[0][0];
    s.nll = sh.dsum[0][1];
    s.nll_base = sh.dsum[0][2];
    s.dp = sh.dsum[0][3];
    s.dp2 = sh.dsum[0][4];
    s.n_valid = nv;
    s.agree = sh.isum[0][1];
    s.n_nll = sh.isum[0][2];
    s.n_flag = sh.isum[0][3];
    s.flags_or = sh.flags_or[0];
    uint32_t de = 0u;
    if (derr) {  // report and clear the row pass's error word
      de = *derr;
      *derr = 0u;
    }
    *out = fin::make_result(N, s, sel.tval, has_nll, de);
  }
}

// Per-field arrays from the records, one thread per row.
__global__ void kld_split_records_kernel(const kld_row_t* __restrict__ rows, int64_t N,
                                         double* __restrict__ kld, double* __restrict__ nll,
                                         int32_t* __restrict__ amax_b, int32_t* __restrict__ amax_q) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < N;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const kld_row_t r = rows[i];
    kld[i] = r.kld;
    nll[i] = r.nll;
    amax_b[i] = r.argmax_base;
    amax_q[i] = r.argmax_quant;
  }
}

}  // namespace

cudaError_t launch_split_records(const kld_row_t* rows, int64_t N, double* kld, double* nll,
                                 int32_t* amax_b, int32_t* amax_q, cudaStream_t stream) {
  if (N < 1) return cudaSuccess;
  constexpr int kThreads = 256;
  int64_t blocks = (N + kThreads - 1) / kThreads;
  if (blocks > 4096) blocks = 4096;
  kld_split_records_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      rows, N, kld, nll, amax_b, amax_q);
  return cudaGetLastError();
}

cudaError_t launch_reduce(const kld_row_t* rows, int64_t N, int has_nll, uint32_t* derr,
                          kld_result_t* out, cudaStream_t stream) {
  if (N < 0 || N > static_cast<int64_t>(UINT32_MAX)) return cudaErrorInvalidValue;  // 32-bit counts
  int threads = kReduceThreads;
  if (N < kReduceThreads) {
    threads = static_cast<int>((N + 31) / 32 * 32);
    if (threads < 128) threads = 128;
  }
  // Shared memory beyond the static 48 KB: allowed once per device.
  static std::atomic<unsigned long long> smem_set{0ull};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(smem_set.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kld_reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kReduceSmemMax));
    if (e != cudaSuccess) return e;
    smem_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  const size_t smem = sizeof(ReduceShared) +
                      (N <= kKeyCap ? static_cast<size_t>(N) * sizeof(unsigned long long) : 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kld_reduce_kernel, rows, N, has_nll, derr, out);
}

}  // namespace kld
