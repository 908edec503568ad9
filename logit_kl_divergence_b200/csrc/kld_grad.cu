// kld_grad.cu -- gradient of KL(P_base || P_quant) with respect to the quant
// logits, the objective of end-to-end tuning ("Mistral-Small-4-119B-2603
// GSQ-RCO IQ3_S GGUF", "How it was made", step 7: the continuous values are
// tuned to minimise KL(BF16 || quantized) of the next-token distributions):
//
//   grad[i][j] = scale * (softmax(q_i)_j - softmax(b_i)_j),
//
// zero on rows that the statistics exclude (NaN / +inf, all -inf). The row
// pass has already produced each row's normalisers (kld_rows_kernel.cuh,
// row_aux): softmax(b)_j = 2^(b_j*L - Fb) * mb with an integer frame Fb
// and mb in (0.5, 1], the same for q. This second pass streams b and q once
// more and writes the gradient: a pure HBM-bound elementwise kernel (reads
// 2*s, writes s_out bytes per element), 16-byte vector loads and stores,
// grid sized to the SM count.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kld_internal.h"

namespace kld {
namespace {

constexpr float kL = 1.4426950408889634f;  // log2(e) rounded to fp32, as in the row pass
constexpr int kGradThreads = 256;
constexpr int kUnit = 8;  // elements per thread step (one or two 16-byte vectors)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int DT>
struct In;
template <>
struct In<KLD_F32> {
  __device__ static void load8(const void* p, float* o) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
  __device__ static float load1(const void* p) { return *static_cast<const float*>(p); }
  static constexpr int kBytes = 4;
};
template <>
struct In<KLD_BF16> {
  __device__ static void load8(const void* p, float* o) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      o[2 * k] = __uint_as_float(w[k] << 16);
      o[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
  __device__ static float load1(const void* p) {
    return __uint_as_float(static_cast<uint32_t>(*static_cast<const unsigned short*>(p)) << 16);
  }
  static constexpr int kBytes = 2;
};
template <>
struct In<KLD_F16> {
  __device__ static void load8(const void* p, float* o) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
      o[2 * k] = f.x;
      o[2 * k + 1] = f.y;
    }
  }
  __device__ static float load1(const void* p) {
    return __half2float(*static_cast<const __half*>(p));
  }
  static constexpr int kBytes = 2;
};

template <int OT>
struct Out;
template <>
struct Out<KLD_F32> {
  __device__ static void store8(void* p, const float* g) {
    reinterpret_cast<float4*>(p)[0] = make_float4(g[0], g[1], g[2], g[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(g[4], g[5], g[6], g[7]);
  }
  __device__ static void store1(void* p, float g) { *static_cast<float*>(p) = g; }
  static constexpr int kBytes = 4;
};
template <>
struct Out<KLD_BF16> {
  __device__ static void store8(void* p, const float* g) {
    uint4 v;
    uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(g[2 * k], g[2 * k + 1]);
      w[k] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = v;
  }
  __device__ static void store1(void* p, float g) {
    *static_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(g);
  }
  static constexpr int kBytes = 2;
};
template <>
struct Out<KLD_F16> {
  __device__ static void store8(void* p, const float* g) {
    uint4 v;
    uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __half2 h = __floats2half2_rn(g[2 * k], g[2 * k + 1]);
      w[k] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = v;
  }
  __device__ static void store1(void* p, float g) { *static_cast<__half*>(p) = __float2half_rn(g); }
  static constexpr int kBytes = 2;
};

// One gradient value from the row's normalisers (nb.x = Fb is NaN on
// excluded rows: the caller writes zeros there).
// Products are rounded separately (no contraction into r - p), so equal
// rows give exactly zero.
__device__ __forceinline__ float grad_of(float b, float q, const float4& nb, float scale) {
  const float p = __fmul_rn(ex2(fmaf(b, kL, -nb.x)), nb.y);  // softmax(b)_j; 0 where b = -inf
  const float r = __fmul_rn(ex2(fmaf(q, kL, -nb.z)), nb.w);  // softmax(q)_j
  return __fmul_rn(scale, __fsub_rn(r, p));
}

// Vector path (V % 8 == 0 and 16-byte aligned rows): each thread takes units
// of 8 elements, u = tid + k * threads over the flattened [N, V/8] units,
// grid-stride; the row of a unit is u / (V/8).
template <int DT, int OT>
__global__ void __launch_bounds__(kGradThreads)
    kld_grad_vec_kernel(const void* __restrict__ base, const void* __restrict__ quant,
                        const RowAux* __restrict__ aux, int64_t N, int64_t V,
                        void* __restrict__ grad, float scale) {
  const int64_t upr = V / kUnit;  // units per row
  const int64_t total = N * upr;
  const char* B = static_cast<const char*>(base);
  const char* Q = static_cast<const char*>(quant);
  char* G = static_cast<char*>(grad);
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = u / upr;
    const int64_t e = u * kUnit;  // flattened element index (= r * V + column)
    const float4 nb = __ldg(reinterpret_cast<const float4*>(aux + r));
    float g[kUnit];
    if (isnan(nb.x)) {
#pragma unroll
      for (int k = 0; k < kUnit; ++k) g[k] = 0.f;
    } else {
      float b[kUnit], q[kUnit];
      In<DT>::load8(B + e * In<DT>::kBytes, b);
      In<DT>::load8(Q + e * In<DT>::kBytes, q);
#pragma unroll
      for (int k = 0; k < kUnit; ++k) g[k] = grad_of(b[k], q[k], nb, scale);
    }
    Out<OT>::store8(G + e * Out<OT>::kBytes, g);
  }
}

// Scalar path for any V and alignment: one element per thread step.
template <int DT, int OT>
__global__ void __launch_bounds__(kGradThreads)
    kld_grad_scalar_kernel(const void* __restrict__ base, const void* __restrict__ quant,
                           const RowAux* __restrict__ aux, int64_t N, int64_t V,
                           void* __restrict__ grad, float scale) {
  const int64_t total = N * V;
  const char* B = static_cast<const char*>(base);
  const char* Q = static_cast<const char*>(quant);
  char* G = static_cast<char*>(grad);
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 nb = __ldg(reinterpret_cast<const float4*>(aux + e / V));
    float g = 0.f;
    if (!isnan(nb.x))
      g = grad_of(In<DT>::load1(B + e * In<DT>::kBytes), In<DT>::load1(Q + e * In<DT>::kBytes),
                  nb, scale);
    Out<OT>::store1(G + e * Out<OT>::kBytes, g);
  }
}

template <int DT, int OT>
cudaError_t launch_typed(const void* base, const void* quant, const RowAux* aux, int64_t N,
                         int64_t V, void* grad, float scale, int sm_count, cudaStream_t s) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(base) | reinterpret_cast<uintptr_t>(quant) |
                      reinterpret_cast<uintptr_t>(grad);
  const bool vec = (V % kUnit) == 0 && (a & 15u) == 0;
  // Enough resident threads to keep HBM busy: 8 CTAs of 256 per SM.
  const int grid = sm_count * 8;
  if (vec) {
    kld_grad_vec_kernel<DT, OT><<<grid, kGradThreads, 0, s>>>(base, quant, aux, N, V, grad,
                                                              scale);
  } else {
    kld_grad_scalar_kernel<DT, OT><<<grid, kGradThreads, 0, s>>>(base, quant, aux, N, V, grad,
                                                                 scale);
  }
  return cudaGetLastError();
}

template <int DT>
cudaError_t launch_out(const void* base, const void* quant, const RowAux* aux, int64_t N,
                       int64_t V, void* grad, kld_dtype_t ot, float scale, int sm_count,
                       cudaStream_t s) {
  switch (ot) {
    case KLD_F32: return launch_typed<DT, KLD_F32>(base, quant, aux, N, V, grad, scale, sm_count, s);
    case KLD_BF16: return launch_typed<DT, KLD_BF16>(base, quant, aux, N, V, grad, scale, sm_count, s);
    case KLD_F16: return launch_typed<DT, KLD_F16>(base, quant, aux, N, V, grad, scale, sm_count, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_grad(const void* base, const void* quant, const RowAux* aux, int64_t N,
                        int64_t V, kld_dtype_t dtype, void* grad, kld_dtype_t grad_dtype,
                        float scale, int sm_count, cudaStream_t stream) {
  switch (dtype) {
    case KLD_F32:
      return launch_out<KLD_F32>(base, quant, aux, N, V, grad, grad_dtype, scale, sm_count, stream);
    case KLD_BF16:
      return launch_out<KLD_BF16>(base, quant, aux, N, V, grad, grad_dtype, scale, sm_count, stream);
    case KLD_F16:
      return launch_out<KLD_F16>(base, quant, aux, N, V, grad, grad_dtype, scale, sm_count, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kld
