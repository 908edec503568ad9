// kld_rows.cu -- launches of the fused row kernel (kld_rows_kernel.cuh):
// the launch plan of the row pass (whole-row rounds, split rows), the
// vocabulary-slice merge, the bounded-wait self-test. The row kernel with
// the top-k scan is instantiated in kld_rows_scan.cu instead.

#include <atomic>

#include "kld_rows_kernel.cuh"

namespace kld {
namespace {

// Vocabulary-sharded rows: one warp per row merges the row's G slice
// partials (lane g holds slice g; G <= 32) exactly as the split-row path
// merges its parts, takes the token logits from the slice that holds the
// token, and writes the record.
constexpr int kMergeWarps = 8;
__global__ void __launch_bounds__(kMergeWarps * 32)
    kld_merge_kernel(const MPart* __restrict__ parts, int G, int64_t N,
                     const int32_t* __restrict__ tok, int64_t v_total,
                     kld_row_t* __restrict__ rows) {
  const int lane = threadIdx.x & 31;
  for (int64_t r = blockIdx.x * static_cast<int64_t>(kMergeWarps) + (threadIdx.x >> 5); r < N;
       r += static_cast<int64_t>(gridDim.x) * kMergeWarps) {
    MPart q = empty_part();
    if (lane < G) {
      const ulonglong2* src = reinterpret_cast<const ulonglong2*>(parts + static_cast<int64_t>(lane) * N + r);
      unsigned long long wds[8];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const ulonglong2 v = __ldg(src + w);
        wds[2 * w] = v.x;
        wds[2 * w + 1] = v.y;
      }
      q = part_from_words(wds);
    }
    const unsigned holder = __ballot_sync(0xffffffffu, (q.flags & kPartHasTok) != 0u);
    const unsigned long long tw = __shfl_sync(0xffffffffu, q.pad2, holder ? __ffs(holder) - 1 : 0);
    q.flags &= ~kPartHasTok;
    const MPart m = warp_merge(q);
    bool tok_ok = false;
    float q_tok = 0.f, b_tok = 0.f;
    if (tok != nullptr) {
      const int32_t tk = __ldg(tok + r);
      tok_ok = tk >= 0 && static_cast<int64_t>(tk) < v_total && holder != 0u;
      q_tok = __uint_as_float(static_cast<unsigned>(tw));
      b_tok = __uint_as_float(static_cast<unsigned>(tw >> 32));
    }
    const kld_row_t rec = finalize_row(m, tok != nullptr, tok_ok, q_tok, b_tok);
    if (lane == 0) rows[r] = rec;
  }
}

// Self-test of the bounded waits: warp 0 waits on an mbarrier that nothing
// ever arrives at; it must give up after limit_ns (or, with use_abort, as
// soon as warp 1 raises the abort flag after ~1 ms) and record the timeout
// in the error word, leaving the context usable.
__global__ void kld_wait_selftest_kernel(uint64_t limit_ns, int use_abort, uint32_t* derr,
                                         unsigned long long* waited_ns) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    const uint64_t t0 = globaltimer();
    const bool ok = mbar_wait_slow(smem_u32(&bar), 0u, &abort_flag, limit_ns);
    if (threadIdx.x == 0) {
      *waited_ns = globaltimer() - t0;
      if (!ok) atomicOr(derr, kErrWaitTimeout);
    }
  } else if (use_abort && threadIdx.x == 32) {
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 1000000ull) {
    }
    *reinterpret_cast<volatile int*>(&abort_flag) = 1;
  }
}

template <int DT>
int max_active_clusters(int cluster_ctas) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cluster_ctas * 32));
  cfg.blockDim = dim3(kRowThreads);
  cfg.dynamicSmemBytes = kRowSmemBytes;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = static_cast<unsigned>(cluster_ctas);
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kld_rows_kernel<DT, false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <int DT>
cudaError_t launch_typed(const RowParams& prm, const RowPlan& pl, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
  cfg.blockDim = dim3(kRowThreads);
  cfg.dynamicSmemBytes = kRowSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = static_cast<unsigned>(pl.cluster_ctas);
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = pl.cluster_ctas > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kld_rows_kernel<DT, false>, prm);
}

}  // namespace

cudaError_t prepare_rows_kernels() {
  const void* kernels[3] = {reinterpret_cast<const void*>(kld_rows_kernel<KLD_F32, false>),
                            reinterpret_cast<const void*>(kld_rows_kernel<KLD_BF16, false>),
                            reinterpret_cast<const void*>(kld_rows_kernel<KLD_F16, false>)};
  for (const void* k : kernels) {
    const cudaError_t e =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kRowSmemBytes);
    if (e != cudaSuccess) return e;
  }
  return prepare_rows_scan_kernels();
}

// Whole-row rounds after which a last partial wave is still split.
constexpr int64_t kTailSplitRounds = 2;

RowPlan plan_rows(int64_t N, int64_t V, int sm_count, const int fit[4], int max_cluster_ctas) {
  RowPlan pl;
  pl.parts_per_row = 1;
  pl.cluster_ctas = 1;
  pl.tail_rows = 0;
  pl.tail_ctas = 0;
  pl.tail_chunks = 0;
  const int64_t nchv = (V + kChunkElems - 1) / kChunkElems;
  pl.nchv = static_cast<int>(nchv);
  const int64_t G = sm_count > 0 ? sm_count : 1;
  if (max_cluster_ctas < 1) {  // whole rows, round robin
    pl.grid = static_cast<int>(N < G ? N : G);
    if (pl.grid < 1) pl.grid = 1;
    pl.whole = static_cast<int>((N + pl.grid - 1) / pl.grid);
    return pl;
  }
  if (max_cluster_ctas >= 2 && N * 2 <= G) {
    int lg = 0;
    while (lg < 3 && (2 << lg) <= max_cluster_ctas) ++lg;
    for (; lg >= 1; --lg) {
      const int C0 = 1 << lg;
      const int f = fit != nullptr && fit[lg] > 0 ? fit[lg] : static_cast<int>(G / C0);
      if (f < N) continue;  // not one cluster per row in one wave
      int C = static_cast<int>(f / N);
      if (C > kPartSlots) C = kPartSlots;  // a row's clusters are merged by one warp
      pl.cluster_ctas = C0;
      pl.parts_per_row = C0 * C;
      pl.grid = static_cast<int>(N) * pl.parts_per_row;
      pl.whole = 0;
      return pl;
    }
  }
  // Whole-row rounds, then a last partial wave of R <= G/2 rows split over
  // the CTAs by balanced chunk ranges: a CTA's range then covers at most
  // two rows, and a range of at least ceil(nchv / 30) chunks keeps every
  // row within 31 CTAs. Below one wave, rows are split into P row-aligned
  // parts (one part per CTA, as many as the SMs hold, at most 32 per row).
  // A larger last wave, or N between G/2 and G, takes whole rows: splitting
  // it would give most CTAs two partial rows to finish, which measured
  // slower than letting the wave's CTAs stream whole rows. So does a last
  // wave after more than kTailSplitRounds whole rounds: the idle time it
  // saves is then a small share of the launch, and the whole-row-only
  // launch runs a leaner consumer loop (measured: 149 and 300 rows of
  // V = 151936 gain 8-12 % and 2.5-6 % from the split; 600 rows or more
  // gain nothing or lose up to 2 %).
  const int64_t W = N / G, R = N % G;
  pl.whole = static_cast<int>(W);
  pl.grid = static_cast<int>(G);
  int64_t Gt = 0;
  if (W == 0) {
    int64_t P = G / N;
    if (P > kPartSlots) P = kPartSlots;
    if (P > nchv) P = nchv;
    if (N * 2 > G || P < 2) {  // whole rows, one per CTA
      pl.grid = static_cast<int>(N);
      pl.whole = 1;
      return pl;
    }
    Gt = N * P;  // ranges of the balanced split fall on row boundaries
  } else if (R > 0) {
    if (R * 2 > G || W > kTailSplitRounds) {  // whole rows, one more round
      pl.whole = static_cast<int>(W + 1);
      return pl;
    }
    const int64_t q = (nchv + 29) / 30;
    Gt = (R * nchv) / q;
    if (Gt > G) Gt = G;
    if (Gt < R) Gt = R;
  }
  if (R > 0) {
    const int64_t Tc = R * nchv;
    pl.tail_rows = static_cast<int>(R);
    pl.tail_ctas = static_cast<int>(Gt);
    pl.tail_chunks = Tc;
    if (W == 0) pl.grid = static_cast<int>(Gt);
    int most = 1;
    for (int64_t rt = 0; rt < R; ++rt) {
      const int64_t first = ((rt * nchv + 1) * Gt - 1) / Tc;
      const int64_t last = (((rt + 1) * nchv) * Gt - 1) / Tc;
      if (last - first + 1 > most) most = static_cast<int>(last - first + 1);
    }
    pl.parts_per_row = most;
  }
  return pl;
}

// Clusters of 2^lg CTAs the current device holds at once, asked once per
// device, element type and size (0 if the query fails).
int active_clusters(kld_dtype_t dtype, int lg) {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cache[kMaxDevices][3][4];  // 0: not asked yet; else count + 1
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  const int t = dtype == KLD_F32 ? 0 : (dtype == KLD_BF16 ? 1 : 2);
  const int c = cache[dev][t][lg].load(std::memory_order_relaxed);
  if (c > 0) return c - 1;
  int n = 0;
  switch (dtype) {
    case KLD_F32: n = max_active_clusters<KLD_F32>(1 << lg); break;
    case KLD_BF16: n = max_active_clusters<KLD_BF16>(1 << lg); break;
    case KLD_F16: n = max_active_clusters<KLD_F16>(1 << lg); break;
  }
  cache[dev][t][lg].store(n + 1, std::memory_order_relaxed);
  return n;
}

cudaError_t launch_merge(const void* parts, int G, int64_t N, const int32_t* token_ids,
                         int64_t V_total, kld_row_t* rows, cudaStream_t stream) {
  if (G < 1 || G > 32 || N < 1) return cudaErrorInvalidValue;
  int64_t blocks = (N + kMergeWarps - 1) / kMergeWarps;
  if (blocks > 65535) blocks = 65535;
  kld_merge_kernel<<<static_cast<unsigned>(blocks), kMergeWarps * 32, 0, stream>>>(
      static_cast<const MPart*>(parts), G, N, token_ids, V_total, rows);
  return cudaGetLastError();
}

cudaError_t launch_rows(const void* base, const void* quant, const int32_t* token_ids, int64_t N,
                        int64_t V, kld_dtype_t dtype, kld_row_t* rows, uint32_t* derr,
                        int sm_count, const SplitScratch* split, RowAux* aux,
                        cudaStream_t stream, void* part_out, int64_t col_offset,
                        kld_result_t* result_out, bool* reduced, const TopkScan* topk) {
  if (reduced) *reduced = false;
  if (topk != nullptr) {
    if (part_out != nullptr) return cudaErrorInvalidValue;
    return launch_rows_scan(base, quant, token_ids, N, V, dtype, rows, derr, sm_count, aux, *topk,
                            stream);
  }
  // Vocabulary-slice partials and launches without split scratch take
  // whole rows only.
  const bool can_split = split != nullptr && part_out == nullptr && split->max_cluster_ctas >= 1;
  RowPlan pl = plan_rows(N, V, sm_count, nullptr, can_split ? 1 : 0);
  if (can_split) {
    int fit[4] = {0, 0, 0, 0};
    if (split->max_cluster_ctas >= 2 && N * 2 <= sm_count)
      for (int lg = 1; lg < 4 && (1 << lg) <= split->max_cluster_ctas; ++lg)
        fit[lg] = active_clusters(dtype, lg);
    pl = plan_rows(N, V, sm_count, fit, split->max_cluster_ctas);
    const int64_t split_rows = pl.cluster_ctas > 1 ? N : pl.tail_rows;
    if (split_rows > split->capacity || pl.grid > split->capacity)
      pl = plan_rows(N, V, sm_count, nullptr, 0);
  }
  RowParams prm = {};
  prm.base = base;
  prm.quant = quant;
  prm.tok = token_ids;
  prm.N = N;
  prm.V = V;
  prm.rows = rows;
  prm.derr = derr;
  prm.sc.P = pl.cluster_ctas > 1 ? pl.parts_per_row : 0;
  prm.sc.W = pl.whole;
  prm.sc.R = pl.tail_rows;
  prm.sc.Gt = pl.tail_ctas;
  prm.sc.nchv = pl.nchv;
  prm.sc.Tc = pl.tail_chunks;
  // row-aligned parts (no whole rounds): nchv * A stays within 32 bits
  prm.sc.A = (pl.cluster_ctas == 1 && pl.whole == 0 && pl.tail_rows > 0 &&
              pl.tail_ctas == pl.tail_rows * pl.parts_per_row &&
              static_cast<int64_t>(pl.nchv) * pl.parts_per_row < (int64_t{1} << 32))
                 ? pl.parts_per_row
                 : 0;
  prm.gparts = split ? static_cast<MPart*>(split->parts) : nullptr;
  prm.tickets = split ? split->tickets : nullptr;
  prm.aux = aux;
  prm.part_out = static_cast<MPart*>(part_out);
  prm.col0 = col_offset;
  // Few split rows (no whole-row round): the row pass reduces its own
  // records (the launch counter is the ticket after the last split row's).
  const bool fuse = result_out != nullptr && can_split && pl.whole == 0 &&
                    N <= kFusedReduceRows && N + 1 <= split->capacity;
  if (fuse) {
    prm.out = result_out;
    prm.counter = split->tickets + N;
  }
  cudaError_t e = cudaErrorInvalidValue;
  switch (dtype) {
    case KLD_F32: e = launch_typed<KLD_F32>(prm, pl, stream); break;
    case KLD_BF16: e = launch_typed<KLD_BF16>(prm, pl, stream); break;
    case KLD_F16: e = launch_typed<KLD_F16>(prm, pl, stream); break;
  }
  if (e == cudaSuccess && reduced) *reduced = fuse;
  return e;
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, int use_abort, uint32_t* derr,
                                 unsigned long long* waited_ns, cudaStream_t stream) {
  kld_wait_selftest_kernel<<<1, 64, 0, stream>>>(limit_ns, use_abort, derr, waited_ns);
  return cudaGetLastError();
}

}  // namespace kld
