// kld_probe.cu -- read-bandwidth probe for the row pass's roofline.
//
// One CTA per SM streams 32 KB tiles of two buffers (alternating; tile t of
// the pair goes to CTA t mod grid) from HBM into a ring of kProbeStages
// shared-memory stages with bulk copies, as the row pass's producer does, and
// does nothing else with them. The rate it reaches is what an
// HBM-to-shared-memory stream of the row pass's shape can reach on the
// device: the read-only roofline of the row pass, beside the copy bandwidth
// (a read+write stream) the benchmark is also compared with. One thread per
// CTA issues and waits; every wait is bounded, and a wait that gives up sets
// the error word and stops issuing (the CTA still waits, bounded, for the
// copies it has in flight).
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "kld_internal.h"
#include "kld_probe.h"

namespace kld {
namespace {

constexpr int kProbeTileBytes = 32 * 1024;
constexpr int kProbeStages = 6;
constexpr size_t kProbeSmemBytes = kProbeStages * static_cast<size_t>(kProbeTileBytes) + 256;
constexpr uint64_t kProbeWaitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool phase_done(uint32_t bar, uint32_t parity) {
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
// Bounded wait for the phase of `parity`.
__device__ bool wait_phase(uint32_t bar, uint32_t parity) {
  if (phase_done(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  while (!phase_done(bar, parity))
    if (now_ns() - t0 > kProbeWaitNs) return false;
  return true;
}

__global__ void __launch_bounds__(32, 1)
    kld_read_probe_kernel(const char* __restrict__ a, const char* __restrict__ b, int64_t bytes,
                          uint32_t* __restrict__ derr) {
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned long long* full =
      reinterpret_cast<unsigned long long*>(smem + kProbeStages * kProbeTileBytes);
  if (threadIdx.x != 0) return;
  for (int s = 0; s < kProbeStages; ++s)
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(&full[s])));
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  const int64_t tiles = (bytes + kProbeTileBytes - 1) / kProbeTileBytes;  // per buffer
  int64_t issued = 0;
  for (int64_t t = blockIdx.x; t < 2 * tiles; t += gridDim.x) {
    const int s = static_cast<int>(issued % kProbeStages);
    const uint32_t bar = saddr(&full[s]);
    if (issued >= kProbeStages &&
        !wait_phase(bar, static_cast<uint32_t>((issued / kProbeStages - 1) & 1))) {
      atomicOr(derr, kErrWaitTimeout);
      break;
    }
    const int64_t tile = t >> 1;
    const char* src = ((t & 1) ? b : a) + tile * kProbeTileBytes;
    const int64_t rem = bytes - tile * kProbeTileBytes;
    const uint32_t len = static_cast<uint32_t>(rem < kProbeTileBytes ? rem : kProbeTileBytes);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(len)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(saddr(smem + s * kProbeTileBytes)),
        "l"(src), "r"(len), "r"(bar), "l"(pol)
        : "memory");
    ++issued;
  }
  // Never leave with copies in flight.
  const int64_t first = issued > kProbeStages ? issued - kProbeStages : 0;
  for (int64_t i = first; i < issued; ++i) {
    const int s = static_cast<int>(i % kProbeStages);
    if (!wait_phase(saddr(&full[s]), static_cast<uint32_t>((i / kProbeStages) & 1))) {
      atomicOr(derr, kErrWaitTimeout);
      break;
    }
  }
}

}  // namespace

// a and b 16-byte aligned, bytes a positive multiple of 16 (checked by the
// caller); one CTA of one warp per SM.
cudaError_t launch_read_probe(const void* a, const void* b, int64_t bytes, uint32_t* derr,
                              int sm_count, cudaStream_t stream) {
  static std::atomic<unsigned long long> smem_set{0ull};  // attribute set once per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(smem_set.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kld_read_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kProbeSmemBytes));
    if (e != cudaSuccess) return e;
    smem_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  kld_read_probe_kernel<<<sm_count, 32, kProbeSmemBytes, stream>>>(
      static_cast<const char*>(a), static_cast<const char*>(b), bytes, derr);
  return cudaGetLastError();
}

}  // namespace kld
