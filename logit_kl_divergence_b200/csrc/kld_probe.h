// kld_probe.h -- launcher of the read-bandwidth probe (kld_probe.cu), kept
// apart from kld_internal.h: the probe shares nothing with the statistic's
// kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kld {

// Streams `bytes` of each of a and b (16-byte aligned, bytes a positive
// multiple of 16) from HBM into shared memory with bulk copies, one CTA per
// SM; a wait that gives up sets *derr (see kld_stats_read_probe).
cudaError_t launch_read_probe(const void* a, const void* b, int64_t bytes, uint32_t* derr,
                              int sm_count, cudaStream_t stream);

}  // namespace kld
