// kld_rows.cu -- fused single-pass row kernel for sm_100a.
//
// For every row i it reads base b[i, :] and quant q[i, :] from HBM exactly
// once and produces KL(P_base || P_quant) over the full vocabulary, the
// lowest-index argmax of both rows and, with token ids, the quantized row's
// NLL of the given token ("Qwen3.6 27B Quantization Benchmark", sections
// "Measurement method" and "Understand KLD and Same Top P"; direction and
// full vocabulary from "Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S GGUF", "How it
// was made", step 5).
//
// Streaming form of the statistic. With L = log2(e) rounded to fp32 and a
// reference c per row operand (the running maximum),
//   u_j = (b_j - c_b) * L,  v_j = (q_j - c_q) * L
//   S_b = sum 2^u_j,  S_q = sum 2^v_j,  T = sum 2^u_j * (u_j - v_j)
//   KL  = ln2 * T / S_b + ln(S_q / S_b)
// The references cancel exactly in KL; they only keep every term max-
// relative, so a constant shift of a whole row (e.g. quant = base + 1000)
// does not cancel catastrophically, the maximum contributes exactly 2^0 = 1,
// and an exact shift gives bit-identical u and v (KL exactly 0). Raising c_b
// by D rescales S_b and T by 2^-(D*L) and subtracts D*L*S_b from T; raising
// c_q by D adds D*L*S_b to T and rescales S_q by 2^-(D*L). (Since L is fp32,
// exponentials are of (1 + 1.4e-8) * x; KL and NLL change by that factor.)
//
// Structure (one CTA per row at a time, persistent over rows):
//   - warp 8 (producer): one lane streams the row's 16-byte-aligned body in
//     32 KB tiles per operand into a 3-stage shared-memory ring with
//     cp.async.bulk (no multicast), completing on mbarriers; it runs ahead
//     across row boundaries.
//   - warps 0..7 (consumers): each takes 1024-element chunks of a tile (32
//     elements per lane, conflict-free 16-byte shared loads). Per chunk: lane
//     max, warp max (redux.sync), a warp-uniform reference raise when the
//     max grew, then 2 exp2 + a few FMA per element pair in fp32, folded
//     into per-lane fp64 accumulators once per chunk.
//   - argmax: each lane remembers the first chunk in which its own maximum
//     appeared (strict >, increasing index order); at the end of the row
//     only lanes whose maximum equals the row maximum re-read that chunk's
//     32 elements to find the lowest matching index.
//   - the unaligned head/tail (< 16 bytes each) is read directly by warp 0.
//   - all intra-CTA waits are mbarrier waits bounded by wall time; a wait
//     that gives up sets an error bit the reduction reports.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <climits>

#include "kld_internal.h"

namespace kld {
namespace {

constexpr float kLog2e = 1.4426950408889634f;  // log2(e) rounded to fp32
constexpr double kLog2eD = static_cast<double>(kLog2e);  // the same value
constexpr double kLn2 = 0.6931471805599453;    // ln(2)
constexpr float kNegBig = -1.0e30f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// ------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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
// Wait for the phase of `parity` to complete; gives up after kWaitLimitNs or
// as soon as another thread of the CTA has raised *abort.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                       volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort) return false;
      if (globaltimer() - t0 > kWaitLimitNs) return false;
    }
  }
}
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src,
                                          uint32_t bytes, uint32_t bar,
                                          uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float warp_max(float x) {
  float y;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

// ------------------------------------------------------------ element types

template <int DT>
struct Elem;

template <>
struct Elem<KLD_F32> {
  static constexpr int kBytes = 4;
  static constexpr int kPerVec = 4;
  __device__ static float load(const void* row, int64_t j) {
    return __ldg(static_cast<const float*>(row) + j);
  }
  __device__ static void unpack(const uint4& v, float* o) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
};

template <>
struct Elem<KLD_BF16> {
  static constexpr int kBytes = 2;
  static constexpr int kPerVec = 8;
  __device__ static float load(const void* row, int64_t j) {
    const unsigned short h = __ldg(static_cast<const unsigned short*>(row) + j);
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
  }
  // bf16 is the top half of an fp32: widening is a shift / mask.
  __device__ static void unpack(const uint4& v, float* o) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      o[2 * k] = __uint_as_float(w[k] << 16);
      o[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
};

template <>
struct Elem<KLD_F16> {
  static constexpr int kBytes = 2;
  static constexpr int kPerVec = 8;
  __device__ static float load(const void* row, int64_t j) {
    const unsigned short h = __ldg(static_cast<const unsigned short*>(row) + j);
    return __half2float(__ushort_as_half(h));
  }
  __device__ static void unpack(const uint4& v, float* o) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
      o[2 * k] = f.x;
      o[2 * k + 1] = f.y;
    }
  }
};

// ------------------------------------------------------------- per-row state

// Warp-uniform reference of one row operand pair.
struct WarpRef {
  float Mb, Mq;  // running maxima seen by this warp (-inf before any)
  float cb, cq;  // references: the running maxima once finite, 0 before
};

// Per-lane accumulators and argmax memory.
struct LaneAcc {
  double Sb, Sq, T;
  float best_b, best_q;  // lane maximum over its chunks so far
  int loc_b, loc_q;      // chunk in which it first appeared
};

// Per-warp partial handed to the row combine.
struct WarpPart {
  float Mb, Mq, cb, cq;
  double Sb, Sq, T;
};

struct Ctrl {
  unsigned long long full[kStages];
  unsigned long long empty[kStages];
  unsigned long long part_bar;
  unsigned long long cand_bar;
  WarpPart part[2][kConsumerWarps];
  int amax[2][2];
  int abort;
};
static_assert(sizeof(Ctrl) <= kRowCtrlBytes, "control block too large");

__device__ __forceinline__ void raise_base(float wmax, WarpRef& r, LaneAcc& a) {
  if (r.Mb != -INFINITY) {  // accumulators are exactly 0 before any finite max
    const double d = (static_cast<double>(wmax) - static_cast<double>(r.cb)) * kLog2eD;
    const double sc = exp2(-d);
    a.T = (a.T - d * a.Sb) * sc;
    a.Sb *= sc;
  }
  r.cb = wmax;
  r.Mb = wmax;
}

__device__ __forceinline__ void raise_quant(float wmax, WarpRef& r, LaneAcc& a) {
  const double d = (static_cast<double>(wmax) - static_cast<double>(r.cq)) * kLog2eD;
  a.T += d * a.Sb;
  if (r.Mq != -INFINITY) a.Sq *= exp2(-d);
  r.cq = wmax;
  r.Mq = wmax;
}

// Accumulate 32 element pairs per lane (already widened to fp32) whose warp
// maxima are wmb / wmq and lane maxima mb / mq.
__device__ __forceinline__ void accumulate32(const float* xb, const float* xq,
                                             float mb, float mq, WarpRef& ref,
                                             LaneAcc& acc, int chunk_id) {
  const float wmb = warp_max(mb);
  const float wmq = warp_max(mq);
  if (wmb > ref.Mb) raise_base(wmb, ref, acc);
  if (wmq > ref.Mq) raise_quant(wmq, ref, acc);
  const float cb = ref.cb, cq = ref.cq;
  float sb0 = 0.f, sb1 = 0.f, sq0 = 0.f, sq1 = 0.f, t0 = 0.f, t1 = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float u0 = __fmul_rn(__fsub_rn(xb[i], cb), kLog2e);
    const float v0 = __fmul_rn(__fsub_rn(xq[i], cq), kLog2e);
    const float u1 = __fmul_rn(__fsub_rn(xb[i + 1], cb), kLog2e);
    const float v1 = __fmul_rn(__fsub_rn(xq[i + 1], cq), kLog2e);
    const float e0 = ex2(u0), f0 = ex2(v0);
    const float e1 = ex2(u1), f1 = ex2(v1);
    sb0 += e0;
    sq0 += f0;
    sb1 += e1;
    sq1 += f1;
    // d < -1e30 only where 2^u underflows to 0; the clamp turns the
    // (-inf) - (-inf) of masked entries into a harmless finite value.
    t0 = fmaf(e0, fmaxf(u0 - v0, kNegBig), t0);
    t1 = fmaf(e1, fmaxf(u1 - v1, kNegBig), t1);
  }
  acc.Sb += static_cast<double>(sb0 + sb1);
  acc.Sq += static_cast<double>(sq0 + sq1);
  acc.T += static_cast<double>(t0 + t1);
  if (mb > acc.best_b) {
    acc.best_b = mb;
    acc.loc_b = chunk_id;
  }
  if (mq > acc.best_q) {
    acc.best_q = mq;
    acc.loc_q = chunk_id;
  }
}

// One 1024-element chunk of the current tile. `valid_vecs` < 32*VPC marks a
// ragged last chunk whose vectors beyond it are treated as -inf.
template <int DT, bool kMasked>
__device__ __forceinline__ void process_chunk(const uint4* cb, const uint4* cq,
                                              int lane, int valid_vecs,
                                              WarpRef& ref, LaneAcc& acc,
                                              int chunk_id) {
  constexpr int E = Elem<DT>::kPerVec;
  constexpr int VPC = 32 / E;
  float xb[32], xq[32];
#pragma unroll
  for (int k = 0; k < VPC; ++k) {
    const int vi = k * 32 + lane;
    const uint4 vb = cb[vi];
    const uint4 vq = cq[vi];
    Elem<DT>::unpack(vb, &xb[k * E]);
    Elem<DT>::unpack(vq, &xq[k * E]);
    if (kMasked && vi >= valid_vecs) {
#pragma unroll
      for (int i = 0; i < E; ++i) {
        xb[k * E + i] = -INFINITY;
        xq[k * E + i] = -INFINITY;
      }
    }
  }
  float mb = max3(xb[0], xb[1], xb[2]);
  float mq = max3(xq[0], xq[1], xq[2]);
#pragma unroll
  for (int i = 3; i < 31; i += 2) {
    mb = max3(mb, xb[i], xb[i + 1]);
    mq = max3(mq, xq[i], xq[i + 1]);
  }
  mb = fmaxf(mb, xb[31]);
  mq = fmaxf(mq, xq[31]);
  accumulate32(xb, xq, mb, mq, ref, acc, chunk_id);
}

// Lowest index in a lane's chunk whose value equals m (INT_MAX if none).
template <int DT>
__device__ int rescan_chunk(const void* row, int64_t body_start, int64_t body_len,
                            int chunk_id, int lane, float m) {
  constexpr int E = Elem<DT>::kPerVec;
  constexpr int VPC = 32 / E;
  const int64_t c0 = static_cast<int64_t>(chunk_id) * kChunkElems;
  for (int k = 0; k < VPC; ++k) {
    for (int i = 0; i < E; ++i) {
      const int64_t off = c0 + static_cast<int64_t>(k * 32 + lane) * E + i;
      if (off >= body_len) return INT_MAX;
      if (Elem<DT>::load(row, body_start + off) == m)
        return static_cast<int>(body_start + off);
    }
  }
  return INT_MAX;
}

__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ void fail(Ctrl* ctrl, uint32_t* derr) {
  atomicOr(derr, kErrWaitTimeout);
  *reinterpret_cast<volatile int*>(&ctrl->abort) = 1;
}

// Row geometry: the unaligned head and tail (< 16 bytes each) are read
// directly; the 16-byte-aligned body is streamed in tiles.
struct RowGeom {
  int64_t head, body_len, tail, ntiles;
};

template <int DT>
__device__ __forceinline__ RowGeom row_geom(const void* rowb, int64_t V) {
  constexpr int EB = Elem<DT>::kBytes;
  constexpr int E = Elem<DT>::kPerVec;
  constexpr int64_t kStageElems = kStageBytes / EB;
  RowGeom g;
  const uint32_t mis = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(rowb) & 15u);
  g.head = static_cast<int64_t>(((16u - mis) & 15u) / EB);
  if (g.head > V) g.head = V;
  g.body_len = ((V - g.head) / E) * E;
  g.tail = V - g.head - g.body_len;
  g.ntiles = (g.body_len + kStageElems - 1) / kStageElems;
  return g;
}

template <int DT>
__global__ void __launch_bounds__(kRowThreads, 1)
    kld_rows_kernel(const void* __restrict__ base, const void* __restrict__ quant,
                    const int32_t* __restrict__ tok, int64_t N, int64_t V,
                    kld_row_t* __restrict__ rows, uint32_t* __restrict__ derr) {
  constexpr int EB = Elem<DT>::kBytes;
  constexpr int E = Elem<DT>::kPerVec;
  constexpr int kStageElems = kStageBytes / EB;
  constexpr int kChunksPerTile = kStageElems / kChunkElems;

  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stage_b = smem;
  unsigned char* stage_q = smem + kStages * kStageBytes;
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + 2 * kStages * kStageBytes);
  volatile int* abort = &ctrl->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&ctrl->full[s]), 1);
      mbar_init(smem_u32(&ctrl->empty[s]), kConsumerWarps);
    }
    mbar_init(smem_u32(&ctrl->part_bar), kConsumerWarps);
    mbar_init(smem_u32(&ctrl->cand_bar), kConsumerWarps);
    ctrl->amax[0][0] = ctrl->amax[0][1] = INT_MAX;
    ctrl->amax[1][0] = ctrl->amax[1][1] = INT_MAX;
    ctrl->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  const char* B = static_cast<const char*>(base);
  const char* Q = static_cast<const char*>(quant);

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = evict_first_policy();
      uint32_t it = 0;
      bool ok = true;
      for (int64_t r = blockIdx.x; r < N && ok; r += gridDim.x) {
        const char* rb = B + r * V * EB;
        const char* rq = Q + r * V * EB;
        const RowGeom g = row_geom<DT>(rb, V);
        for (int64_t t = 0; t < g.ntiles; ++t, ++it) {
          const int s = static_cast<int>(it % kStages);
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(smem_u32(&ctrl->empty[s]), ph ^ 1u, abort)) {
            fail(ctrl, derr);
            ok = false;
            break;
          }
          const int64_t off = g.head + t * kStageElems;
          int64_t len = g.body_len - t * kStageElems;
          if (len > kStageElems) len = kStageElems;
          const uint32_t bytes = static_cast<uint32_t>(len * EB);
          const uint32_t fb = smem_u32(&ctrl->full[s]);
          mbar_arrive_expect_tx(fb, 2u * bytes);
          bulk_load(smem_u32(stage_b + s * kStageBytes), rb + off * EB, bytes, fb, pol);
          bulk_load(smem_u32(stage_q + s * kStageBytes), rq + off * EB, bytes, fb, pol);
        }
      }
      // Never leave with copies in flight: wait (bounded) for the last
      // stages issued. In a normal run they have long completed.
      const uint32_t last = it < kStages ? it : kStages;
      for (uint32_t k = 0; k < last; ++k) {
        const uint32_t j = it - 1u - k;
        const int s = static_cast<int>(j % kStages);
        const uint32_t ph = (j / kStages) & 1u;
        const uint32_t fb = smem_u32(&ctrl->full[s]);
        if (!mbar_try_wait(fb, ph)) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(fb, ph)) {
            if (globaltimer() - t0 > kWaitLimitNs) {
              atomicOr(derr, kErrWaitTimeout);
              break;
            }
          }
        }
      }
    }
    return;
  }

  // ---------------------------------------------------------------- consumers
  uint32_t it = 0;
  int rowk = 0;
  for (int64_t r = blockIdx.x; r < N; r += gridDim.x, ++rowk) {
    const char* rb = B + r * V * EB;
    const char* rq = Q + r * V * EB;
    const RowGeom g = row_geom<DT>(rb, V);
    const int pb = rowk & 1;

    WarpRef ref{-INFINITY, -INFINITY, 0.f, 0.f};
    LaneAcc acc{0.0, 0.0, 0.0, -INFINITY, -INFINITY, -1, -1};

    // Head/tail elements (warp 0), loaded now and used at the row end.
    float xe_b = -INFINITY, xe_q = -INFINITY;
    int idx_e = INT_MAX;
    const int n_extra = static_cast<int>(g.head + g.tail);
    if (warp == 0 && lane < n_extra) {
      const int64_t j = lane < g.head ? lane : g.head + g.body_len + (lane - g.head);
      idx_e = static_cast<int>(j);
      xe_b = Elem<DT>::load(rb, j);
      xe_q = Elem<DT>::load(rq, j);
    }
    // Next-token gather (thread 0), also issued early.
    int32_t tk = 0;
    bool tok_ok = false;
    float q_tok = 0.f;
    if (threadIdx.x == 0 && tok != nullptr) {
      tk = __ldg(tok + r);
      tok_ok = tk >= 0 && static_cast<int64_t>(tk) < V;
      if (tok_ok) q_tok = Elem<DT>::load(rq, tk);
    }

    bool ok = true;
    for (int64_t t = 0; t < g.ntiles; ++t, ++it) {
      const int s = static_cast<int>(it % kStages);
      const uint32_t ph = (it / kStages) & 1u;
      if (!mbar_wait(smem_u32(&ctrl->full[s]), ph, abort)) {
        fail(ctrl, derr);
        ok = false;
        break;
      }
      int64_t len = g.body_len - t * kStageElems;
      if (len > kStageElems) len = kStageElems;
      const uint4* tb = reinterpret_cast<const uint4*>(stage_b + s * kStageBytes);
      const uint4* tq = reinterpret_cast<const uint4*>(stage_q + s * kStageBytes);
      for (int c = warp; c < kChunksPerTile; c += kConsumerWarps) {
        const int cstart = c * kChunkElems;
        if (cstart >= len) break;
        const int gid = static_cast<int>(t) * kChunksPerTile + c;
        const uint4* cb = tb + cstart / E;
        const uint4* cq = tq + cstart / E;
        if (cstart + kChunkElems <= len) {
          process_chunk<DT, false>(cb, cq, lane, 0, ref, acc, gid);
        } else {
          process_chunk<DT, true>(cb, cq, lane, static_cast<int>((len - cstart) / E),
                                  ref, acc, gid);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctrl->empty[s]));
    }
    if (!ok) return;

    // Head/tail as one more (sparse) step of warp 0: one element per lane.
    if (warp == 0 && n_extra > 0) {
      const float wmb = warp_max(xe_b);
      const float wmq = warp_max(xe_q);
      if (wmb > ref.Mb) raise_base(wmb, ref, acc);
      if (wmq > ref.Mq) raise_quant(wmq, ref, acc);
      const float u = __fmul_rn(__fsub_rn(xe_b, ref.cb), kLog2e);
      const float v = __fmul_rn(__fsub_rn(xe_q, ref.cq), kLog2e);
      const float e = ex2(u);
      acc.Sb += static_cast<double>(e);
      acc.Sq += static_cast<double>(ex2(v));
      acc.T += static_cast<double>(e * fmaxf(u - v, kNegBig));
    }

    // Warp partial -> shared memory.
    const double Sb = warp_sum(acc.Sb);
    const double Sq = warp_sum(acc.Sq);
    const double T = warp_sum(acc.T);
    if (lane == 0) ctrl->part[pb][warp] = WarpPart{ref.Mb, ref.Mq, ref.cb, ref.cq, Sb, Sq, T};
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&ctrl->part_bar));
    if (!mbar_wait(smem_u32(&ctrl->part_bar), rowk & 1, abort)) {
      fail(ctrl, derr);
      return;
    }

    // Row maxima, then the lowest index holding each.
    float Mb = -INFINITY, Mq = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      Mb = fmaxf(Mb, ctrl->part[pb][w].Mb);
      Mq = fmaxf(Mq, ctrl->part[pb][w].Mq);
    }
    const bool finite_max = Mb > -INFINITY && Mb < INFINITY && Mq > -INFINITY && Mq < INFINITY;
    if (finite_max) {
      int cb_idx = INT_MAX, cq_idx = INT_MAX;
      if (acc.best_b == Mb) cb_idx = rescan_chunk<DT>(rb, g.head, g.body_len, acc.loc_b, lane, Mb);
      if (acc.best_q == Mq) cq_idx = rescan_chunk<DT>(rq, g.head, g.body_len, acc.loc_q, lane, Mq);
      if (warp == 0 && xe_b == Mb && idx_e < cb_idx) cb_idx = idx_e;
      if (warp == 0 && xe_q == Mq && idx_e < cq_idx) cq_idx = idx_e;
      cb_idx = __reduce_min_sync(0xffffffffu, cb_idx);
      cq_idx = __reduce_min_sync(0xffffffffu, cq_idx);
      if (lane == 0) {
        if (cb_idx != INT_MAX) atomicMin(&ctrl->amax[pb][0], cb_idx);
        if (cq_idx != INT_MAX) atomicMin(&ctrl->amax[pb][1], cq_idx);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&ctrl->cand_bar));

    if (threadIdx.x == 0) {
      if (!mbar_wait(smem_u32(&ctrl->cand_bar), rowk & 1, abort)) {
        fail(ctrl, derr);
        return;
      }
      uint32_t flags = 0;
      if (tok != nullptr && !tok_ok) flags |= KLD_ROW_BAD_TOKEN;
      bool nonfinite = !(Mb < INFINITY) || !(Mq < INFINITY);
      for (int w = 0; w < kConsumerWarps; ++w) {
        const WarpPart& p = ctrl->part[pb][w];
        if (isnan(p.Sb) || isnan(p.Sq)) nonfinite = true;
      }
      double kl = __longlong_as_double(0x7ff8000000000000ll);  // NaN
      double nll = kl;
      int ab = -1, aq = -1;
      if (nonfinite) {
        flags |= KLD_ROW_NONFINITE;
      } else if (Mb == -INFINITY || Mq == -INFINITY) {
        flags |= KLD_ROW_EMPTY;
      } else {
        // Common references: the largest per-warp reference of warps that
        // saw a finite maximum.
        float Cb = -INFINITY, Cq = -INFINITY;
        for (int w = 0; w < kConsumerWarps; ++w) {
          const WarpPart& p = ctrl->part[pb][w];
          if (p.Mb > -INFINITY) Cb = fmaxf(Cb, p.cb);
          if (p.Mq > -INFINITY) Cq = fmaxf(Cq, p.cq);
        }
        double sb = 0.0, sq = 0.0, tt = 0.0;
        bool inf_kl = false;
        for (int w = 0; w < kConsumerWarps; ++w) {
          const WarpPart& p = ctrl->part[pb][w];
          const double dq = (static_cast<double>(Cq) - static_cast<double>(p.cq)) * kLog2eD;
          if (p.Mb > -INFINITY) {
            const double db = (static_cast<double>(Cb) - static_cast<double>(p.cb)) * kLog2eD;
            const double sc = exp2(-db);
            sb += p.Sb * sc;
            if (!isfinite(p.T)) {
              inf_kl = true;
            } else {
              tt += sc * (p.T - (db - dq) * p.Sb);
            }
          }
          if (p.Mq > -INFINITY) sq += p.Sq * exp2(-dq);
        }
        if (inf_kl) {
          kl = INFINITY;
          flags |= KLD_ROW_INF_KL;
        } else {
          kl = kLn2 * (tt / sb) + log(sq / sb);
        }
        if (tok_ok) {
          if (q_tok == -INFINITY) {
            nll = INFINITY;
            flags |= KLD_ROW_INF_NLL;
          } else {
            nll = log(sq) +
                  kLn2 * ((static_cast<double>(Cq) - static_cast<double>(q_tok)) * kLog2eD);
          }
        }
        ab = ctrl->amax[pb][0];
        aq = ctrl->amax[pb][1];
      }
      kld_row_t rec;
      rec.kld = kl;
      rec.nll = nll;
      rec.argmax_base = ab;
      rec.argmax_quant = aq;
      rec.flags = flags;
      rec.reserved = 0u;
      rows[r] = rec;
      ctrl->amax[pb][0] = INT_MAX;
      ctrl->amax[pb][1] = INT_MAX;
    }
  }
}

}  // namespace

cudaError_t prepare_rows_kernels() {
  cudaError_t e;
  e = cudaFuncSetAttribute(kld_rows_kernel<KLD_F32>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, kRowSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kld_rows_kernel<KLD_BF16>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, kRowSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kld_rows_kernel<KLD_F16>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, kRowSmemBytes);
}

cudaError_t launch_rows(const void* base, const void* quant, const int32_t* token_ids,
                        int64_t N, int64_t V, kld_dtype_t dtype, kld_row_t* rows,
                        uint32_t* derr, int grid, cudaStream_t stream) {
  const dim3 g(static_cast<unsigned>(grid)), b(kRowThreads);
  switch (dtype) {
    case KLD_F32:
      kld_rows_kernel<KLD_F32><<<g, b, kRowSmemBytes, stream>>>(base, quant, token_ids, N, V,
                                                                 rows, derr);
      break;
    case KLD_BF16:
      kld_rows_kernel<KLD_BF16><<<g, b, kRowSmemBytes, stream>>>(base, quant, token_ids, N, V,
                                                                  rows, derr);
      break;
    case KLD_F16:
      kld_rows_kernel<KLD_F16><<<g, b, kRowSmemBytes, stream>>>(base, quant, token_ids, N, V,
                                                                 rows, derr);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace kld
