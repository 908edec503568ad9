// kld_rows_scan.cu -- the row kernel with the top-k scan
// (kld_rows_kernel<DT, true>, see TopkScan), whole rows only.
//
// A translation unit of its own: instantiated beside the plain row kernel,
// it changed how the compiler inlined the helpers the two share, and the
// plain kernel then spilled registers in its hot loop and ran at less than
// half its speed.

#include "kld_rows_kernel.cuh"

namespace kld {
namespace {

template <int DT>
cudaError_t launch_scan_typed(const RowParams& prm, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kRowThreads);
  cfg.dynamicSmemBytes = kRowSmemBytes + kScanSmemBytes;
  cfg.stream = stream;
  return cudaLaunchKernelEx(&cfg, kld_rows_kernel<DT, true>, prm);
}

}  // namespace

cudaError_t prepare_rows_scan_kernels() {
  const void* kernels[3] = {reinterpret_cast<const void*>(kld_rows_kernel<KLD_F32, true>),
                            reinterpret_cast<const void*>(kld_rows_kernel<KLD_BF16, true>),
                            reinterpret_cast<const void*>(kld_rows_kernel<KLD_F16, true>)};
  for (const void* k : kernels) {
    const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               kRowSmemBytes + kScanSmemBytes);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_rows_scan(const void* base, const void* quant, const int32_t* token_ids,
                             int64_t N, int64_t V, kld_dtype_t dtype, kld_row_t* rows,
                             uint32_t* derr, int sm_count, RowAux* aux, const TopkScan& topk,
                             cudaStream_t stream) {
  if (topk.tf == nullptr || topk.regions == nullptr || topk.counts == nullptr || aux == nullptr)
    return cudaErrorInvalidValue;
  const RowPlan pl = plan_rows(N, V, sm_count, nullptr, 0);  // whole rows, round robin
  RowParams prm = {};
  prm.base = base;
  prm.quant = quant;
  prm.tok = token_ids;
  prm.N = N;
  prm.V = V;
  prm.rows = rows;
  prm.derr = derr;
  prm.sc.W = pl.whole;
  prm.sc.nchv = pl.nchv;
  prm.aux = aux;
  prm.scan = topk;
  switch (dtype) {
    case KLD_F32: return launch_scan_typed<KLD_F32>(prm, pl.grid, stream);
    case KLD_BF16: return launch_scan_typed<KLD_BF16>(prm, pl.grid, stream);
    case KLD_F16: return launch_scan_typed<KLD_F16>(prm, pl.grid, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kld
