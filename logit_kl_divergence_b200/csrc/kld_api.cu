// kld_api.cu -- host side of the C ABI declared in include/kld_stats.h.
//
// Owns the per-handle device workspace (one 40-byte record per row, an
// error word, the split-row scratch), the mapped pinned host result that the
// reduction kernel writes directly, and the staging buffers of the
// host-memory path; validates arguments before anything is enqueued and maps
// CUDA failures to status codes. Every step of the statistic runs in the
// kernels of kld_rows_kernel.cuh (launched from kld_rows.cu and kld_rows_scan.cu),
// kld_reduce.cu, kld_grad.cu and kld_topk.cu.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <string>

#include "kld_internal.h"
#include "kld_probe.h"

namespace {

thread_local std::string g_last_cuda_error;

kld_status_t cuda_fail(cudaError_t e, const char* what) {
  g_last_cuda_error = std::string(what) + ": " + cudaGetErrorString(e);
  if (e == cudaErrorMemoryAllocation) return KLD_ERR_OOM;
  if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver ||
      e == cudaErrorNoKernelImageForDevice)
    return KLD_ERR_NO_DEVICE;
  return KLD_ERR_CUDA;
}

#define KLD_CUDA(call)                                 \
  do {                                                 \
    cudaError_t _e = (call);                           \
    if (_e != cudaSuccess) return cuda_fail(_e, #call); \
  } while (0)

// Makes the handle's device current for the duration of a call.
class DeviceGuard {
 public:
  explicit DeviceGuard(int dev) {
    ok_ = cudaGetDevice(&prev_) == cudaSuccess;
    if (ok_ && prev_ != dev) ok_ = cudaSetDevice(dev) == cudaSuccess;
    switched_ = ok_ && prev_ != dev;
  }
  ~DeviceGuard() {
    if (switched_) cudaSetDevice(prev_);
  }
  bool ok() const { return ok_; }

 private:
  int prev_ = 0;
  bool ok_ = false;
  bool switched_ = false;
};

// Host-path staging: two buffers, each holding a chunk of base rows, quant
// rows and token ids.
constexpr size_t kStageTargetBytes = 128ull << 20;  // per operand per buffer

}  // namespace

struct kld_stats_s {
  int device = 0;
  int sm_count = 0;
  int64_t max_rows = 0;
  kld_row_t* rows = nullptr;
  // kld_stats_rows: per-field arrays filled from the records on request
  double* soa_kld = nullptr;  // one allocation: kld, nll (double), then amax_b, amax_q
  double* soa_nll = nullptr;
  int32_t* soa_amax_b = nullptr;
  int32_t* soa_amax_q = nullptr;
  cudaStream_t last_stream = nullptr;  // stream of the last run that wrote `rows`
  bool rows_written = false;
  void* split_mem = nullptr;  // split-row scratch (kld::SplitScratch)
  kld::RowAux* aux = nullptr;  // per-row normalisers for the gradient and top-k passes
  bool grad_timing_valid = false;
  kld::SplitScratch split = {nullptr, nullptr, 0, kld::kDefaultClusterCtas};
  uint32_t* derr = nullptr;  // the device error word, then the top-k exact-path row count
  unsigned long long* topk_exact = nullptr;
  cudaEvent_t topk_done = nullptr;  // after the last top-k pass
  bool has_topk = false;
  kld_result_t* hres = nullptr;      // pinned, mapped host memory
  kld_result_t* hres_dev = nullptr;  // its device-side pointer
  cudaEvent_t done = nullptr;
  bool has_result = false;
  int64_t last_rows = 0;
  bool timing = false;
  bool timing_valid = false;
  bool rows_pending = false;  // a timed kld_stats_run_rows awaits its reduction
  // row pass start / end, reduction end, second pass end, top-k threshold start
  cudaEvent_t tev[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
  bool threshold_timed = false;  // the last timed second pass had a threshold kernel
  // top-k scan workspace (kld::TopkScan), allocated by the first scanned run_topk
  void* topk_mem = nullptr;
  kld::TopkScan topk_scan = {nullptr, nullptr, nullptr};
  // host path
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t copied[2] = {nullptr, nullptr};
  cudaEvent_t freed[2] = {nullptr, nullptr};
  void* stage[2] = {nullptr, nullptr};
  size_t stage_bytes = 0;  // per buffer
};

namespace {

bool valid_dtype(kld_dtype_t dt) { return dt == KLD_F32 || dt == KLD_BF16 || dt == KLD_F16; }

kld_status_t check_inputs(const void* base, const void* quant, const int32_t* tok, int64_t N,
                          int64_t V, kld_dtype_t dtype, bool device_ptrs) {
  if (!valid_dtype(dtype)) return KLD_ERR_DTYPE;
  if (!base || !quant) return KLD_ERR_INVALID_ARG;
  if (N < 1 || V < 1 || V > INT32_MAX) return KLD_ERR_INVALID_ARG;
  const uintptr_t eb = static_cast<uintptr_t>(kld::elem_bytes(dtype));
  const uintptr_t ab = reinterpret_cast<uintptr_t>(base);
  const uintptr_t aq = reinterpret_cast<uintptr_t>(quant);
  if (ab % eb || aq % eb) return KLD_ERR_INVALID_ARG;
  if (device_ptrs && ((ab - aq) & 15u)) return KLD_ERR_INVALID_ARG;
  if (tok && (reinterpret_cast<uintptr_t>(tok) & 3u)) return KLD_ERR_INVALID_ARG;
  return KLD_OK;
}

cudaError_t launch_rows(kld_stats_s* h, const void* base, const void* quant, const int32_t* tok,
                        int64_t N, int64_t V, kld_dtype_t dtype, kld_row_t* rows, cudaStream_t s,
                        kld::RowAux* aux = nullptr) {
  return kld::launch_rows(base, quant, tok, N, V, dtype, rows, h->derr, h->sm_count, &h->split,
                          aux, s);
}

kld_status_t enqueue_reduce(kld_stats_t h, const kld_row_t* rows, int64_t N, int has_nll,
                            cudaStream_t s) {
  // The reduction writes the result straight into the handle's mapped
  // pinned host buffer: no separate device-to-host copy.
  KLD_CUDA(kld::launch_reduce(rows, N, has_nll, h->derr, h->hres_dev, s));
  if (h->timing && h->timing_valid) KLD_CUDA(cudaEventRecord(h->tev[2], s));
  KLD_CUDA(cudaEventRecord(h->done, s));
  h->has_result = true;
  return KLD_OK;
}

// The row pass, then the reduction (in the row pass itself for few split
// rows), each timed when timing is on. aux: per-row normalisers for a second
// pass (nullable).
kld_status_t run_statistic(kld_stats_t h, const void* base, const void* quant, const int32_t* tok,
                           int64_t N, int64_t V, kld_dtype_t dtype, cudaStream_t s,
                           kld::RowAux* aux, const kld::TopkScan* topk = nullptr) {
  h->timing_valid = h->timing;
  h->rows_pending = false;
  if (h->timing) KLD_CUDA(cudaEventRecord(h->tev[0], s));
  bool reduced = false;
  KLD_CUDA(kld::launch_rows(base, quant, tok, N, V, dtype, h->rows, h->derr, h->sm_count,
                            &h->split, aux, s, nullptr, 0, h->hres_dev, &reduced, topk));
  if (h->timing) KLD_CUDA(cudaEventRecord(h->tev[1], s));
  h->last_rows = N;
  h->last_stream = s;
  h->rows_written = true;
  if (!reduced) return enqueue_reduce(h, h->rows, N, tok != nullptr, s);
  if (h->timing) KLD_CUDA(cudaEventRecord(h->tev[2], s));
  KLD_CUDA(cudaEventRecord(h->done, s));
  h->has_result = true;
  return KLD_OK;
}

}  // namespace

extern "C" {

int kld_abi_version(void) { return KLD_ABI_VERSION; }

const char* kld_status_string(kld_status_t s) {
  switch (s) {
    case KLD_OK: return "ok";
    case KLD_ERR_INVALID_ARG: return "invalid argument";
    case KLD_ERR_DTYPE: return "unknown element type";
    case KLD_ERR_OOM: return "out of memory";
    case KLD_ERR_CUDA: return "CUDA error";
    case KLD_ERR_NONFINITE: return "rows with NaN/+inf or all -inf were excluded";
    case KLD_ERR_BAD_TOKEN: return "token ids outside [0, V) were excluded from PPL";
    case KLD_ERR_TIMEOUT: return "a bounded device wait gave up";
    case KLD_ERR_NO_DEVICE: return "no usable sm_100 device";
    case KLD_ERR_NOT_READY: return "no run to report";
    case KLD_ERR_CAPACITY: return "more rows than the fixed scratch of kld_stats_run_static";
  }
  return "unknown status";
}

const char* kld_last_cuda_error(void) { return g_last_cuda_error.c_str(); }

kld_status_t kld_plan(int64_t N, int64_t V, kld_dtype_t dtype, int sm_count, kld_plan_t* out) {
  if (!out) return KLD_ERR_INVALID_ARG;
  if (!valid_dtype(dtype)) return KLD_ERR_DTYPE;
  if (N < 1 || V < 1 || V > INT32_MAX || sm_count < 1) return KLD_ERR_INVALID_ARG;
  std::memset(out, 0, sizeof(*out));
  const kld::RowPlan pl = kld::plan_rows(N, V, sm_count, nullptr, kld::kDefaultClusterCtas);
  out->variant = pl.cluster_ctas > 1 ? 1 : (pl.tail_rows > 0 ? 2 : 0);
  out->grid = pl.grid;
  out->ctas_per_row = pl.parts_per_row;
  out->cluster_ctas = pl.cluster_ctas;
  out->whole_rounds = pl.whole;
  out->tail_rows = pl.tail_rows;
  out->tail_ctas = pl.tail_ctas;
  out->threads = kld::kRowThreads;
  out->smem_bytes = kld::kRowSmemBytes;
  out->stage_bytes = kld::kStageBytes;
  out->stages = kld::kStages;
  return KLD_OK;
}

kld_status_t kld_stats_create(kld_stats_t* out, int64_t max_rows, int device) {
  if (!out) return KLD_ERR_INVALID_ARG;
  *out = nullptr;
  if (max_rows < 1 || device < 0) return KLD_ERR_INVALID_ARG;
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess || ndev == 0) {
    g_last_cuda_error = e != cudaSuccess ? cudaGetErrorString(e) : "no CUDA device";
    return KLD_ERR_NO_DEVICE;
  }
  if (device >= ndev) return KLD_ERR_INVALID_ARG;
  int major = 0, minor = 0, sms = 0;
  KLD_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device));
  KLD_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device));
  KLD_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device));
  if (major != 10 || minor != 0) {
    g_last_cuda_error = "device is not compute capability 10.0";
    return KLD_ERR_NO_DEVICE;
  }
  DeviceGuard guard(device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  KLD_CUDA(kld::prepare_rows_kernels());

  kld_stats_s* h = new kld_stats_s();
  h->device = device;
  h->sm_count = sms;
  h->max_rows = max_rows;
  kld_status_t st = KLD_OK;
  do {
    cudaError_t err;
    if ((err = cudaMalloc(&h->rows, sizeof(kld_row_t) * static_cast<size_t>(max_rows))) !=
        cudaSuccess) { st = cuda_fail(err, "cudaMalloc(rows)"); break; }
    if ((err = cudaMalloc(&h->aux, sizeof(kld::RowAux) * static_cast<size_t>(max_rows))) !=
        cudaSuccess) { st = cuda_fail(err, "cudaMalloc(row normalisers)"); break; }
    if ((err = cudaMalloc(&h->soa_kld, 24 * static_cast<size_t>(max_rows))) != cudaSuccess) {
      st = cuda_fail(err, "cudaMalloc(per-field rows)"); break; }
    h->soa_nll = h->soa_kld + max_rows;
    h->soa_amax_b = reinterpret_cast<int32_t*>(h->soa_nll + max_rows);
    h->soa_amax_q = h->soa_amax_b + max_rows;
    if ((err = cudaMalloc(&h->derr, 16)) != cudaSuccess) {
      st = cuda_fail(err, "cudaMalloc(error word)"); break; }
    if ((err = cudaMemset(h->derr, 0, 16)) != cudaSuccess) {
      st = cuda_fail(err, "cudaMemset"); break; }
    h->topk_exact = reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(h->derr) + 8);
    if ((err = cudaEventCreateWithFlags(&h->topk_done, cudaEventDisableTiming)) != cudaSuccess) {
      st = cuda_fail(err, "cudaEventCreate"); break; }
    {
      // Split-row scratch (see kld::SplitScratch): partial slots and a
      // ticket for each of up to SMs split rows, plus the few-row launch
      // counter, all zeroed once here (each launch leaves them zero).
      auto up = [](size_t b) { return (b + 255) & ~static_cast<size_t>(255); };
      const size_t pbytes = up(static_cast<size_t>(sms) * kld::kPartSlotsPerRow * kld::kSplitPartBytes);
      const size_t tbytes = up(static_cast<size_t>(sms + 1) * sizeof(unsigned));
      if ((err = cudaMalloc(&h->split_mem, pbytes + tbytes)) != cudaSuccess) {
        st = cuda_fail(err, "cudaMalloc(split scratch)"); break; }
      if ((err = cudaMemset(h->split_mem, 0, pbytes + tbytes)) != cudaSuccess) {
        st = cuda_fail(err, "cudaMemset"); break; }
      h->split.parts = h->split_mem;
      h->split.tickets = reinterpret_cast<unsigned*>(static_cast<char*>(h->split_mem) + pbytes);
      h->split.capacity = sms;
    }
    if ((err = cudaHostAlloc(reinterpret_cast<void**>(&h->hres), sizeof(kld_result_t),
                             cudaHostAllocMapped | cudaHostAllocPortable)) != cudaSuccess) {
      st = cuda_fail(err, "cudaHostAlloc"); break; }
    std::memset(h->hres, 0, sizeof(kld_result_t));
    if ((err = cudaHostGetDevicePointer(reinterpret_cast<void**>(&h->hres_dev), h->hres, 0)) !=
        cudaSuccess) { st = cuda_fail(err, "cudaHostGetDevicePointer"); break; }
    if ((err = cudaEventCreateWithFlags(&h->done, cudaEventDisableTiming)) != cudaSuccess) {
      st = cuda_fail(err, "cudaEventCreate"); break; }
    for (int i = 0; i < 5 && st == KLD_OK; ++i)
      if ((err = cudaEventCreate(&h->tev[i])) != cudaSuccess) st = cuda_fail(err, "cudaEventCreate");
  } while (0);
  if (st != KLD_OK) {
    kld_stats_destroy(h);
    return st;
  }
  *out = h;
  return KLD_OK;
}

void kld_stats_destroy(kld_stats_t h) {
  if (!h) return;
  DeviceGuard guard(h->device);
  if (h->copy_stream) cudaStreamSynchronize(h->copy_stream);
  if (h->done && h->has_result) cudaEventSynchronize(h->done);
  for (int i = 0; i < 2; ++i) {
    if (h->freed[i]) cudaEventSynchronize(h->freed[i]);
    if (h->stage[i]) cudaFree(h->stage[i]);
    if (h->copied[i]) cudaEventDestroy(h->copied[i]);
    if (h->freed[i]) cudaEventDestroy(h->freed[i]);
  }
  if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
  for (int i = 0; i < 5; ++i)
    if (h->tev[i]) cudaEventDestroy(h->tev[i]);
  if (h->done) cudaEventDestroy(h->done);
  if (h->topk_done) {
    if (h->has_topk) cudaEventSynchronize(h->topk_done);
    cudaEventDestroy(h->topk_done);
  }
  if (h->hres) cudaFreeHost(h->hres);
  if (h->derr) cudaFree(h->derr);
  if (h->rows) cudaFree(h->rows);
  if (h->soa_kld) cudaFree(h->soa_kld);
  if (h->split_mem) cudaFree(h->split_mem);
  if (h->aux) cudaFree(h->aux);
  if (h->topk_mem) cudaFree(h->topk_mem);
  delete h;
}

kld_status_t kld_stats_run_rows(kld_stats_t h, const void* base, const void* quant,
                                const int32_t* token_ids, int64_t N, int64_t V,
                                kld_dtype_t dtype, kld_row_t* rows_out, void* stream) {
  if (!h) return KLD_ERR_INVALID_ARG;
  kld_status_t st = check_inputs(base, quant, token_ids, N, V, dtype, true);
  if (st != KLD_OK) return st;
  if (!rows_out && N > h->max_rows) return KLD_ERR_INVALID_ARG;
  if (rows_out && (reinterpret_cast<uintptr_t>(rows_out) & 7u)) return KLD_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Timed like kld_stats_run: the reduction that follows records the end.
  h->timing_valid = h->timing;
  h->rows_pending = h->timing;
  h->grad_timing_valid = false;
  h->threshold_timed = false;
  if (h->timing) KLD_CUDA(cudaEventRecord(h->tev[0], s));
  KLD_CUDA(launch_rows(h, base, quant, token_ids, N, V, dtype, rows_out ? rows_out : h->rows, s));
  if (h->timing) KLD_CUDA(cudaEventRecord(h->tev[1], s));
  if (!rows_out) {
    h->last_rows = N;
    h->last_stream = s;
    h->rows_written = true;
  }
  return KLD_OK;
}

kld_status_t kld_stats_reduce(kld_stats_t h, const kld_row_t* rows_dev, int64_t N, int has_nll,
                              void* stream) {
  if (!h) return KLD_ERR_INVALID_ARG;
  if (N < 1) return KLD_ERR_INVALID_ARG;
  if (!rows_dev && N > h->max_rows) return KLD_ERR_INVALID_ARG;
  if (rows_dev && (reinterpret_cast<uintptr_t>(rows_dev) & 7u)) return KLD_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  // Timed only as the reduction that follows a timed kld_stats_run_rows
  // (whose start and end events are recorded): then the end of this
  // reduction completes the measurement.
  h->timing_valid = h->timing_valid && h->rows_pending;
  h->rows_pending = false;
  h->grad_timing_valid = false;
  h->threshold_timed = false;
  return enqueue_reduce(h, rows_dev ? rows_dev : h->rows, N, has_nll ? 1 : 0,
                        static_cast<cudaStream_t>(stream));
}

kld_status_t kld_stats_run(kld_stats_t h, const void* base, const void* quant,
                           const int32_t* token_ids, int64_t N, int64_t V, kld_dtype_t dtype,
                           void* stream) {
  if (!h) return KLD_ERR_INVALID_ARG;
  kld_status_t st = check_inputs(base, quant, token_ids, N, V, dtype, true);
  if (st != KLD_OK) return st;
  if (N > h->max_rows) return KLD_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  h->grad_timing_valid = false;
  h->threshold_timed = false;
  return run_statistic(h, base, quant, token_ids, N, V, dtype, static_cast<cudaStream_t>(stream),
                       nullptr);
}

kld_status_t kld_stats_run_grad(kld_stats_t h, const void* base, const void* quant,
                                const int32_t* token_ids, int64_t N, int64_t V,
                                kld_dtype_t dtype, void* grad, kld_dtype_t grad_dtype,
                                double scale, void* stream) {
  if (!h) return KLD_ERR_INVALID_ARG;
  kld_status_t st = check_inputs(base, quant, token_ids, N, V, dtype, true);
  if (st != KLD_OK) return st;
  if (!valid_dtype(grad_dtype)) return KLD_ERR_DTYPE;
  if (!grad || (reinterpret_cast<uintptr_t>(grad) % kld::elem_bytes(grad_dtype))) return KLD_ERR_INVALID_ARG;
  if (N > h->max_rows || !(scale == scale)) return KLD_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->grad_timing_valid = h->timing;
  h->threshold_timed = false;
  st = run_statistic(h, base, quant, token_ids, N, V, dtype, s, h->aux);
  if (st != KLD_OK) return st;
  KLD_CUDA(kld::launch_grad(base, quant, h->aux, N, V, dtype, grad, grad_dtype,
                            static_cast<float>(scale), h->sm_count, s));
  if (h->timing) KLD_CUDA(cudaEventRecord(h->tev[3], s));
  return KLD_OK;
}

kld_status_t kld_stats_run_partials(kld_stats_t h, const void* base, const void* quant,
                                    const int32_t* token_ids, int64_t N, int64_t V,
                                    int64_t col_offset, int64_t V_total, kld_dtype_t dtype,
                                    void* parts_out, void* stream) {
  if (!h) return KLD_ERR_INVALID_ARG;
  kld_status_t st = check_inputs(base, quant, token_ids, N, V, dtype, true);
  if (st != KLD_OK) return st;
  if (!parts_out || (reinterpret_cast<uintptr_t>(parts_out) & 15u)) return KLD_ERR_INVALID_ARG;
  if (col_offset < 0 || V_total > INT32_MAX || col_offset + V > V_total) return KLD_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->timing_valid = false;
  h->rows_pending = false;
  h->grad_timing_valid = false;
  h->threshold_timed = false;
  KLD_CUDA(kld::launch_rows(base, quant, token_ids, N, V, dtype, h->rows, h->derr, h->sm_count,
                            &h->split, nullptr, s, parts_out, col_offset));
  return KLD_OK;
}

kld_status_t kld_stats_merge_partials(kld_stats_t h, const void* parts, int G, int64_t N,
                                      const int32_t* token_ids, int64_t V_total, void* stream) {
  if (!h || !parts || G < 1 || G > 32 || N < 1 || N > h->max_rows) return KLD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(parts) & 15u) || V_total < 1 || V_total > INT32_MAX)
    return KLD_ERR_INVALID_ARG;
  if (token_ids && (reinterpret_cast<uintptr_t>(token_ids) & 3u)) return KLD_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->timing_valid = false;
  h->rows_pending = false;
  h->grad_timing_valid = false;
  h->threshold_timed = false;
  KLD_CUDA(kld::launch_merge(parts, G, N, token_ids, V_total, h->rows, s));
  h->last_rows = N;
  h->last_stream = s;
  h->rows_written = true;
  return enqueue_reduce(h, h->rows, N, token_ids != nullptr, s);
}

kld_status_t kld_stats_run_topk(kld_stats_t h, const void* base, const void* quant,
                                const int32_t* token_ids, int64_t N, int64_t V,
                                kld_dtype_t dtype, int k, int32_t* idx_out, float* logp_out,
                                float* rest_out, double* kl_out, void* stream) {
  if (!h) return KLD_ERR_INVALID_ARG;
  kld_status_t st = check_inputs(base, quant, token_ids, N, V, dtype, true);
  if (st != KLD_OK) return st;
  if (N > h->max_rows || k < 1 || k > kld::kMaxTopk || !kl_out) return KLD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(kl_out) & 7u) || (reinterpret_cast<uintptr_t>(idx_out) & 3u) ||
      (reinterpret_cast<uintptr_t>(logp_out) & 3u) || (reinterpret_cast<uintptr_t>(rest_out) & 3u))
    return KLD_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Rows longer than the top-k pass's candidate capacity: a threshold per
  // row first, so that the row pass can list the lanes holding candidates.
  const bool scan = V > kld::kTopkCap;
  if (scan && !h->topk_mem) {
    // Synchronises the device once (the first scanned call of the handle).
    auto up = [](size_t b) { return (b + 255) & ~static_cast<size_t>(255); };
    const size_t rows = static_cast<size_t>(h->max_rows);
    const size_t tf_b = up(rows * sizeof(float));
    const size_t rg_b = up(rows * kld::kConsumerWarps * kld::kRegionVecs * sizeof(uint4));
    const size_t ct_b = up(rows * kld::kConsumerWarps * sizeof(int));
    const cudaError_t err = cudaMalloc(&h->topk_mem, tf_b + rg_b + ct_b);
    if (err != cudaSuccess) {
      h->topk_mem = nullptr;
      return cuda_fail(err, "cudaMalloc(top-k scan)");
    }
    char* m = static_cast<char*>(h->topk_mem);
    h->topk_scan.tf = reinterpret_cast<float*>(m);
    h->topk_scan.regions = reinterpret_cast<uint4*>(m + tf_b);
    h->topk_scan.counts = reinterpret_cast<int*>(m + tf_b + rg_b);
  }
  h->grad_timing_valid = h->timing;
  h->threshold_timed = h->timing && scan;
  if (scan) {
    if (h->timing) KLD_CUDA(cudaEventRecord(h->tev[4], s));
    KLD_CUDA(kld::launch_topk_threshold(base, N, V, dtype, k, h->topk_scan.tf,
                                        h->sm_count, s));
  }
  st = run_statistic(h, base, quant, token_ids, N, V, dtype, s, h->aux,
                     scan ? &h->topk_scan : nullptr);
  if (st != KLD_OK) return st;
  KLD_CUDA(cudaMemsetAsync(h->topk_exact, 0, sizeof(unsigned long long), s));
  KLD_CUDA(kld::launch_topk(base, quant, h->aux, N, V, dtype, k, idx_out, logp_out, rest_out,
                            kl_out, h->sm_count, s, scan ? &h->topk_scan : nullptr, h->topk_exact));
  if (h->timing) KLD_CUDA(cudaEventRecord(h->tev[3], s));
  KLD_CUDA(cudaEventRecord(h->topk_done, s));
  h->has_topk = true;
  return KLD_OK;
}

kld_status_t kld_selftest_bounded_wait(int device, uint64_t limit_ns, int use_abort,
                                       uint64_t* waited_ns) {
  if (device < 0 || limit_ns < 1000 || limit_ns > 10000000000ull) return KLD_ERR_INVALID_ARG;
  DeviceGuard guard(device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  void* mem = nullptr;
  KLD_CUDA(cudaMalloc(&mem, 16));
  uint32_t* derr = static_cast<uint32_t*>(mem);
  unsigned long long* waited = reinterpret_cast<unsigned long long*>(static_cast<char*>(mem) + 8);
  kld_status_t st = KLD_OK;
  uint32_t err_word = 0;
  unsigned long long w = 0;
  cudaError_t e = cudaMemset(mem, 0, 16);
  if (e == cudaSuccess) e = kld::launch_wait_selftest(limit_ns, use_abort, derr, waited, nullptr);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&err_word, derr, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(&w, waited, 8, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) st = cuda_fail(e, "bounded-wait self-test");
  cudaFree(mem);
  if (st != KLD_OK) return st;
  if (waited_ns) *waited_ns = w;
  return err_word ? KLD_ERR_TIMEOUT : KLD_OK;
}

kld_status_t kld_stats_read_probe(kld_stats_t h, const void* a, const void* b, int64_t bytes,
                                  void* stream) {
  if (!h || !a || !b || bytes <= 0 || (bytes & 15)) return KLD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 15u)
    return KLD_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  KLD_CUDA(kld::launch_read_probe(a, b, bytes, h->derr, h->sm_count,
                                  static_cast<cudaStream_t>(stream)));
  return KLD_OK;
}

kld_status_t kld_stats_second_pass_timing(kld_stats_t h, float* pass_ms) {
  if (!h || !pass_ms) return KLD_ERR_INVALID_ARG;
  if (!h->grad_timing_valid || !h->has_result) return KLD_ERR_NOT_READY;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  KLD_CUDA(cudaEventSynchronize(h->tev[3]));
  KLD_CUDA(cudaEventElapsedTime(pass_ms, h->tev[2], h->tev[3]));
  if (h->threshold_timed) {
    float t = 0.f;
    KLD_CUDA(cudaEventElapsedTime(&t, h->tev[4], h->tev[0]));
    *pass_ms += t;
  }
  return KLD_OK;
}

kld_status_t kld_stats_topk_exact_rows(kld_stats_t h, int64_t* rows) {
  if (!h || !rows) return KLD_ERR_INVALID_ARG;
  if (!h->has_topk) return KLD_ERR_NOT_READY;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  KLD_CUDA(cudaEventSynchronize(h->topk_done));
  unsigned long long n = 0;
  KLD_CUDA(cudaMemcpy(&n, h->topk_exact, sizeof(n), cudaMemcpyDeviceToHost));
  *rows = static_cast<int64_t>(n);
  return KLD_OK;
}

kld_status_t kld_stats_result(kld_stats_t h, kld_result_t* out) {
  if (!h || !out) return KLD_ERR_INVALID_ARG;
  if (!h->has_result) return KLD_ERR_NOT_READY;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  KLD_CUDA(cudaEventSynchronize(h->done));
  *out = *h->hres;
  if (out->device_error) return KLD_ERR_TIMEOUT;
  if (out->flags_or & (KLD_ROW_NONFINITE | KLD_ROW_EMPTY)) return KLD_ERR_NONFINITE;
  if (out->flags_or & KLD_ROW_BAD_TOKEN) return KLD_ERR_BAD_TOKEN;
  return KLD_OK;
}

kld_status_t kld_stats_records(kld_stats_t h, const kld_row_t** rows_dev, int64_t* n_rows) {
  if (!h || !rows_dev || !n_rows) return KLD_ERR_INVALID_ARG;
  *rows_dev = h->rows;
  *n_rows = h->last_rows;
  return KLD_OK;
}

kld_status_t kld_stats_rows(kld_stats_t h, const double** kld, const double** nll,
                            const int32_t** amax_b, const int32_t** amax_q) {
  if (!h) return KLD_ERR_INVALID_ARG;
  if (!h->rows_written) return KLD_ERR_NOT_READY;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  KLD_CUDA(kld::launch_split_records(h->rows, h->last_rows, h->soa_kld, h->soa_nll,
                                     h->soa_amax_b, h->soa_amax_q, h->last_stream));
  if (kld) *kld = h->soa_kld;
  if (nll) *nll = h->soa_nll;
  if (amax_b) *amax_b = h->soa_amax_b;
  if (amax_q) *amax_q = h->soa_amax_q;
  return KLD_OK;
}

kld_status_t kld_stats_set_split(kld_stats_t h, int cluster_ctas) {
  if (!h) return KLD_ERR_INVALID_ARG;
  switch (cluster_ctas) {
    case -1: h->split.max_cluster_ctas = 0; return KLD_OK;
    case 0: h->split.max_cluster_ctas = kld::kDefaultClusterCtas; return KLD_OK;
    case 1: case 2: case 4: case 8: h->split.max_cluster_ctas = cluster_ctas; return KLD_OK;
    default: return KLD_ERR_INVALID_ARG;
  }
}

kld_status_t kld_stats_set_timing(kld_stats_t h, int enable) {
  if (!h) return KLD_ERR_INVALID_ARG;
  h->timing = enable != 0;
  h->timing_valid = false;
  h->rows_pending = false;
  h->grad_timing_valid = false;
  h->threshold_timed = false;
  return KLD_OK;
}

kld_status_t kld_stats_timing(kld_stats_t h, float* row_pass_ms, float* reduce_ms) {
  if (!h || !row_pass_ms || !reduce_ms) return KLD_ERR_INVALID_ARG;
  if (!h->timing_valid || !h->has_result) return KLD_ERR_NOT_READY;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  KLD_CUDA(cudaEventSynchronize(h->done));
  KLD_CUDA(cudaEventElapsedTime(row_pass_ms, h->tev[0], h->tev[1]));
  KLD_CUDA(cudaEventElapsedTime(reduce_ms, h->tev[1], h->tev[2]));
  return KLD_OK;
}

}  // extern "C"

namespace {

// Host-memory row pass: rows [0, N) copied to the device in chunks on the
// handle's copy stream (two staging buffers, so the copy of one chunk
// overlaps the row pass of the previous one), records to rows_out[0, N).
kld_status_t host_rows(kld_stats_t h, const void* base_host, const void* quant_host,
                       const int32_t* token_ids_host, int64_t N, int64_t V, kld_dtype_t dtype,
                       kld_row_t* rows_out, cudaStream_t s) {
  const size_t row_bytes = static_cast<size_t>(V) * static_cast<size_t>(kld::elem_bytes(dtype));
  int64_t chunk = static_cast<int64_t>(kStageTargetBytes / row_bytes);
  if (chunk < 1) chunk = 1;
  if (chunk > N) chunk = N;
  // Each buffer: [chunk rows of base][chunk rows of quant][chunk token ids],
  // every part starting on a 256-byte boundary.
  const size_t part = ((static_cast<size_t>(chunk) * row_bytes) + 255) & ~static_cast<size_t>(255);
  const size_t need = 2 * part + ((static_cast<size_t>(chunk) * 4 + 255) & ~static_cast<size_t>(255));
  if (!h->copy_stream) {
    KLD_CUDA(cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking));
    for (int i = 0; i < 2; ++i) {
      KLD_CUDA(cudaEventCreateWithFlags(&h->copied[i], cudaEventDisableTiming));
      KLD_CUDA(cudaEventCreateWithFlags(&h->freed[i], cudaEventDisableTiming));
    }
  }
  if (need > h->stage_bytes) {
    for (int i = 0; i < 2; ++i) {
      KLD_CUDA(cudaEventSynchronize(h->freed[i]));
      if (h->stage[i]) cudaFree(h->stage[i]);
      h->stage[i] = nullptr;
    }
    h->stage_bytes = 0;
    for (int i = 0; i < 2; ++i) KLD_CUDA(cudaMalloc(&h->stage[i], need));
    h->stage_bytes = need;
  }
  // Earlier work of `stream` may still read the staging buffers.
  for (int i = 0; i < 2; ++i) KLD_CUDA(cudaEventRecord(h->freed[i], s));

  h->timing_valid = false;
  h->rows_pending = false;
  h->grad_timing_valid = false;
  h->threshold_timed = false;
  const char* hb = static_cast<const char*>(base_host);
  const char* hq = static_cast<const char*>(quant_host);
  const int64_t nchunks = (N + chunk - 1) / chunk;
  for (int64_t c = 0; c < nchunks; ++c) {
    const int b = static_cast<int>(c & 1);
    const int64_t r0 = c * chunk;
    const int64_t n = (N - r0) < chunk ? (N - r0) : chunk;
    char* sb = static_cast<char*>(h->stage[b]);
    char* sq = sb + part;
    int32_t* stok = reinterpret_cast<int32_t*>(sb + 2 * part);
    KLD_CUDA(cudaStreamWaitEvent(h->copy_stream, h->freed[b], 0));
    KLD_CUDA(cudaMemcpyAsync(sb, hb + static_cast<size_t>(r0) * row_bytes,
                             static_cast<size_t>(n) * row_bytes, cudaMemcpyHostToDevice,
                             h->copy_stream));
    KLD_CUDA(cudaMemcpyAsync(sq, hq + static_cast<size_t>(r0) * row_bytes,
                             static_cast<size_t>(n) * row_bytes, cudaMemcpyHostToDevice,
                             h->copy_stream));
    if (token_ids_host)
      KLD_CUDA(cudaMemcpyAsync(stok, token_ids_host + r0, static_cast<size_t>(n) * 4,
                               cudaMemcpyHostToDevice, h->copy_stream));
    KLD_CUDA(cudaEventRecord(h->copied[b], h->copy_stream));
    KLD_CUDA(cudaStreamWaitEvent(s, h->copied[b], 0));
    KLD_CUDA(launch_rows(h, sb, sq, token_ids_host ? stok : nullptr, n, V, dtype, rows_out + r0,
                         s));
    KLD_CUDA(cudaEventRecord(h->freed[b], s));
  }
  if (rows_out == h->rows) {
    h->last_rows = N;
    h->last_stream = s;
    h->rows_written = true;
  }
  return KLD_OK;
}

}  // namespace

extern "C" {

kld_status_t kld_stats_run_host(kld_stats_t h, const void* base_host, const void* quant_host,
                                const int32_t* token_ids_host, int64_t N, int64_t V,
                                kld_dtype_t dtype, void* stream) {
  if (!h) return KLD_ERR_INVALID_ARG;
  kld_status_t st = check_inputs(base_host, quant_host, token_ids_host, N, V, dtype, false);
  if (st != KLD_OK) return st;
  if (N > h->max_rows) return KLD_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = host_rows(h, base_host, quant_host, token_ids_host, N, V, dtype, h->rows, s);
  if (st != KLD_OK) return st;
  return enqueue_reduce(h, h->rows, N, token_ids_host != nullptr, s);
}

kld_status_t kld_stats_run_rows_host(kld_stats_t h, const void* base_host, const void* quant_host,
                                     const int32_t* token_ids_host, int64_t N, int64_t V,
                                     kld_dtype_t dtype, kld_row_t* rows_out, void* stream) {
  if (!h) return KLD_ERR_INVALID_ARG;
  kld_status_t st = check_inputs(base_host, quant_host, token_ids_host, N, V, dtype, false);
  if (st != KLD_OK) return st;
  if (!rows_out && N > h->max_rows) return KLD_ERR_INVALID_ARG;
  if (rows_out && (reinterpret_cast<uintptr_t>(rows_out) & 7u)) return KLD_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok()) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
  return host_rows(h, base_host, quant_host, token_ids_host, N, V, dtype,
                   rows_out ? rows_out : h->rows, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
