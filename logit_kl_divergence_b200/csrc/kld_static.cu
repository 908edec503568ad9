// kld_static.cu -- allocation-free variant of kld_stats_run.
//
// Some callers cannot allocate device memory at the point where they need the
// statistic: an inference server that reserves nearly all HBM for its own
// pool (KV cache, activations) at start-up and forbids other allocations, or
// a latency-critical loop that cannot afford the implicit device
// synchronisation cudaMalloc/cudaFree may perform. kld_stats_run_static serves
// them: the per-row records and the error word live in one fixed-size
// file-scope device array below, so the call enqueues the same row pass and
// reduction as kld_stats_run without allocating anything. The caller supplies
// the inputs and a device buffer for the result.
//
// The array is part of this library's device image: every GPU that loads the
// library holds it (KLD_STATIC_MAX_ROWS records, 2.5 MiB plus 256 bytes) until
// the process exits. Host code never dereferences it: the array's name on the
// host is only a stand-in, so the first call on each device (with that device
// current) looks up its device address with cudaGetSymbolAddress and keeps it.
// That first call also sets the row kernel's shared-memory attribute, so it
// should come before any stream capture. Every call shares the one array, and
// each call overwrites what the previous one left there: calls whose work
// overlaps on the GPU (other streams, other threads) race and must be ordered
// by the caller.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "kld_internal.h"

namespace {

constexpr int64_t kMaxRows = KLD_STATIC_MAX_ROWS;
constexpr size_t kRowsBytes = static_cast<size_t>(kMaxRows) * sizeof(kld_row_t);
constexpr size_t kScratchBytes = kRowsBytes + 256;  // records, then the error word

static __device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

struct DeviceSetup {
  void* scratch = nullptr;  // device address of g_static_scratch on that device
  int sm_count = 0;
};

std::mutex g_setup_mu;
DeviceSetup g_setup[kMaxDevices];

kld_status_t fail_cuda(cudaError_t e) {
  if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver ||
      e == cudaErrorNoKernelImageForDevice)
    return KLD_ERR_NO_DEVICE;
  return KLD_ERR_CUDA;
}

// Once per device, with that device current: the scratch address and the
// kernel attributes.
kld_status_t setup_current_device(DeviceSetup* out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e);
  if (dev < 0 || dev >= kMaxDevices) return KLD_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  DeviceSetup& s = g_setup[dev];
  if (!s.scratch) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return fail_cuda(e);
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return fail_cuda(e);
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return fail_cuda(e);
    if (major != 10 || minor != 0) return KLD_ERR_NO_DEVICE;
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_static_scratch)) != cudaSuccess)
      return fail_cuda(e);
    if ((e = kld::prepare_rows_kernels()) != cudaSuccess)
      return fail_cuda(e);
    s.sm_count = sms;
    s.scratch = p;
  }
  *out = s;
  return KLD_OK;
}

}  // namespace

extern "C" kld_status_t kld_stats_run_static(const void* base, const void* quant,
                                             const int32_t* token_ids, int64_t N, int64_t V,
                                             kld_dtype_t dtype, kld_result_t* result_dev,
                                             void* stream) {
  if (dtype != KLD_F32 && dtype != KLD_BF16 && dtype != KLD_F16) return KLD_ERR_DTYPE;
  if (!base || !quant || !result_dev) return KLD_ERR_INVALID_ARG;
  if (N < 1 || V < 1 || V > INT32_MAX) return KLD_ERR_INVALID_ARG;
  if (N > kMaxRows) return KLD_ERR_CAPACITY;  // more rows than the fixed scratch holds
  const uintptr_t eb = static_cast<uintptr_t>(kld::elem_bytes(dtype));
  const uintptr_t ab = reinterpret_cast<uintptr_t>(base);
  const uintptr_t aq = reinterpret_cast<uintptr_t>(quant);
  if (ab % eb || aq % eb || ((ab - aq) & 15u)) return KLD_ERR_INVALID_ARG;
  if (token_ids && (reinterpret_cast<uintptr_t>(token_ids) & 3u)) return KLD_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(result_dev) & 7u) return KLD_ERR_INVALID_ARG;

  DeviceSetup dev;
  kld_status_t st = setup_current_device(&dev);
  if (st != KLD_OK) return st;

  unsigned char* scratch = static_cast<unsigned char*>(dev.scratch);
  kld_row_t* rows = reinterpret_cast<kld_row_t*>(scratch);
  uint32_t* derr = reinterpret_cast<uint32_t*>(scratch + kRowsBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // The array keeps the previous call's contents: the error word must start
  // at zero (the records are rewritten for every row before they are read).
  cudaError_t e = cudaMemsetAsync(derr, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return fail_cuda(e);
  // Whole-row mode only: split rows would need scratch beyond the fixed array.
  e = kld::launch_rows(base, quant, token_ids, N, V, dtype, rows, derr, dev.sm_count, nullptr,
                       nullptr, s);
  if (e != cudaSuccess) return fail_cuda(e);
  e = kld::launch_reduce(rows, N, token_ids != nullptr, derr, result_dev, s);
  if (e != cudaSuccess) return fail_cuda(e);
  return KLD_OK;
}
