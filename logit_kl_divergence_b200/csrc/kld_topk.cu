// kld_topk.cu -- top-k compression of the base row and the KL of the quant
// row against it ("Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S GGUF", "How it
// was made", step 7: tuning "against the top-128 distributions (and the rest
// of the mass)").
//
// Per row, T = the k largest base logits (ties to the lowest index), listed
// in that order with log P_base, plus log of the rest mass, and
//   KL_topk = sum_{j in T} p_j log(p_j / r_j) + p_rest log(p_rest / r_rest).
// Runs after the row pass, which leaves each row's normalisers (RowAux:
// lse_b, log1p(B/S), the centre K and fp32 frames) so that, for j in T,
//   log p_j = lambda*b_j - lse_b,  log(p_j / r_j) = log1p(B/S) - lambda*x_j,
// x_j = q_j - b_j + K formed as the row pass forms it (kShiftForm), the
// rest in fp64.
//
// One CTA per row (persistent over rows, three per SM). Fast path: 4096
// samples of the base row (512 evenly spaced runs of 8 adjacent elements,
// one memory sector each) give a threshold key t0 (the m-th
// largest sample, m ~ 1.5 k * 4096 / V + 8, to 21 bits by two 11-bit
// histogram levels), and every element with key >= t0 goes to a shared
// candidate list, every other one to the rest masses. For rows of more than
// kCap elements the thresholds come first (kld_topk_threshold_kernel), and
// the row pass, in its top-k scan form, copies out the 16-element lanes
// that hold such an element and sums the rest masses of all others
// (TopkScan): this pass then reads only the copies (copied_pass), and each
// logit is read from memory once in all. Without a scan, one fused pass
// over both rows here (gather_pass) does the same. If fewer than k or
// more than kCap elements pass the threshold (ties or extreme rows), an exact
// path takes the row instead: an MSB radix select over order-preserving
// 32-bit keys (11/11/10-bit levels, stopping as soon as the candidates fit
// in shared memory; for a tie group at the threshold larger than that, the
// lowest indices in it by a radix select over the index), the candidates,
// and a last pass for the rest masses (the row is read 2-4 times). T is the
// first k candidates by (key desc, index asc): ranked by counting when there
// are at most kRankMax of them (the fast path's usual few hundred; with many
// more than k, a histogram of the candidates' keys first leaves only those
// in or above the bin of the k-th largest to be ranked), else by a bitonic
// sort in shared memory; candidates beyond T join the rest.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <climits>

#include "kld_internal.h"

namespace kld {
namespace {

constexpr int kTopkThreads = 256;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkCtasPerSm = 3;  // 85 registers a thread: the copies' loads stay in flight
constexpr int kHistBins = 2048;
constexpr int kCap = kTopkCap;  // candidates sorted in shared memory
constexpr int kSample = 4096;  // samples of a row for the threshold
constexpr int kRankMax = 1536;  // at most this many candidates: rank by counting
constexpr int kSetBase = 2048;  // where the boundary set of the ranking is kept in cand[]
static_assert(kSetBase >= kRankMax && kSetBase + kRankMax <= kCap, "boundary set layout");
constexpr float kL = 1.4426950408889634f;  // log2(e) rounded to fp32, as the row pass
constexpr double kLn2 = 0.6931471805599453;
constexpr int kGatherUnroll = 2;  // 16-byte vectors per operand per thread per step
static_assert(kSample % kTopkThreads == 0, "sample loads per thread");

template <int DT>
__device__ __forceinline__ float load_el(const char* row, int64_t j);
template <>
__device__ __forceinline__ float load_el<KLD_F32>(const char* row, int64_t j) {
  return __ldg(reinterpret_cast<const float*>(row) + j);
}
template <>
__device__ __forceinline__ float load_el<KLD_BF16>(const char* row, int64_t j) {
  return __uint_as_float(static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(row) + j)) << 16);
}
template <>
__device__ __forceinline__ float load_el<KLD_F16>(const char* row, int64_t j) {
  return __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short*>(row) + j)));
}

// Order-preserving key of a float (larger float, larger key).
__device__ __forceinline__ uint32_t okey(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u >> 31) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct TopkShared {
  unsigned hist[kHistBins];
  unsigned long long cand[kCap + kMaxTopk];  // candidates, then T sorted by rank
  double red[kTopkWarps][4];
  unsigned wmax[kTopkWarps];
  int ncand;
  int nset;
  unsigned sel[3];  // bin, count above it, count in it
  int fcnt[kConsumerWarps];  // scanned rows: lanes copied by each consumer warp of the row pass
};

// Block-wide: the bin holding the `need`-th element counting from the top
// (descending = true) or the bottom of hist[0..bins). Returns (bin, count
// before it in that direction, count in it) through sh.sel. Warp 0 scans the
// lanes' contiguous segments of bins/32 bins, then the owner segment again
// with a few bins per lane, so no lane walks more than a couple of bins.
__device__ __forceinline__ unsigned warp_incl_scan(unsigned v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}
template <class Sh>
__device__ void find_bin(Sh& sh, int bins, unsigned need, bool descending) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    auto bin_at = [&](int pos) { return descending ? bins - 1 - pos : pos; };  // pos: scan order
    const int per = bins / 32;  // bins per lane, contiguous in scan order
    unsigned part = 0;
    for (int i = 0; i < per; ++i) part += sh.hist[bin_at(lane * per + i)];
    const unsigned incl = warp_incl_scan(part, lane);
    const unsigned excl = incl - part;
    const unsigned hit = __ballot_sync(0xffffffffu, excl < need && incl >= need);
    const int owner = hit ? __ffs(hit) - 1 : 31;
    const unsigned cum0 = __shfl_sync(0xffffffffu, excl, owner);
    // the owner's segment, a few bins per lane
    const int sub = (per + 31) / 32;
    const int p0 = owner * per + min(lane * sub, per), p1 = owner * per + min((lane + 1) * sub, per);
    unsigned part2 = 0;
    for (int q = p0; q < p1; ++q) part2 += sh.hist[bin_at(q)];
    const unsigned incl2 = warp_incl_scan(part2, lane) + cum0;
    const unsigned excl2 = incl2 - part2;
    const unsigned hit2 = __ballot_sync(0xffffffffu, p1 > p0 && excl2 < need && incl2 >= need);
    const int own2 = hit2 ? __ffs(hit2) - 1 : 31;
    if (lane == own2) {
      unsigned cum = excl2;
      int bin = bin_at(p0 < p1 ? p0 : p1 - 1);
      for (int q = p0; q < p1; ++q) {
        bin = bin_at(q);
        if (cum + sh.hist[bin] >= need) break;
        cum += sh.hist[bin];
      }
      sh.sel[0] = static_cast<unsigned>(bin);
      sh.sel[1] = cum;
      sh.sel[2] = sh.hist[bin];
    }
  }
  __syncthreads();
}

// Block sums of four values at once (one barrier pair); the totals come
// back in the same variables, summed in a fixed order (lanes by the shuffle
// tree, then warps in index order), so a row's result does not depend on
// timing.
__device__ void block_sum4(TopkShared& sh, double& v0, double& v1, double& v2, double& v3) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  double v[4] = {v0, v1, v2, v3};
#pragma unroll
  for (int s = 0; s < 4; ++s) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[s] += __shfl_down_sync(0xffffffffu, v[s], o);
  }
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < 4; ++s) sh.red[warp][s] = v[s];
  }
  __syncthreads();
  double t[4] = {0.0, 0.0, 0.0, 0.0};
  for (int w = 0; w < kTopkWarps; ++w) {
#pragma unroll
    for (int s = 0; s < 4; ++s) t[s] += sh.red[w][s];
  }
  __syncthreads();
  v0 = t[0];
  v1 = t[1];
  v2 = t[2];
  v3 = t[3];
}

// Inverse of okey.
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k >> 31) ? (k & 0x7fffffffu) : ~k);
}

// Fast-path threshold: a key t0 with, by the samples, comfortably more than
// kt but fewer than kCap elements of the row at or above it (block-wide).
template <int DT, class Sh>
__device__ uint32_t sample_threshold(Sh& sh, const char* rb, int64_t V, int kt) {
  const int tid = threadIdx.x;
  uint32_t* skey = reinterpret_cast<uint32_t*>(sh.cand);  // kSample keys
  double mm = 1.5 * static_cast<double>(kt) * kSample / static_cast<double>(V) + 8.0;
  const unsigned m = mm > kSample ? static_cast<unsigned>(kSample) : static_cast<unsigned>(mm);
  // kSample / 8 evenly spaced runs of 8 adjacent elements (one sector each);
  // every thread issues all of its loads before using any, so the sampling
  // costs one memory latency instead of one per load
  constexpr int kPer = kSample / kTopkThreads;
  float sv[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = tid + u * kTopkThreads;
    const int64_t start = (static_cast<int64_t>(i >> 3) * (V - 8) / (kSample / 8)) & ~static_cast<int64_t>(7);
    sv[u] = load_el<DT>(rb, start + (i & 7));
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) skey[tid + u * kTopkThreads] = okey(sv[u]);
  for (int i = tid; i < kHistBins; i += kTopkThreads) sh.hist[i] = 0u;
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kPer; ++u) atomicAdd(&sh.hist[okey(sv[u]) >> 21], 1u);
  __syncthreads();
  find_bin(sh, kHistBins, m, true);
  const uint32_t bin = sh.sel[0], above = sh.sel[1], inbin = sh.sel[2];
  uint32_t t0 = bin << 21;
  if (inbin > 1) {
    // the next 11 bits of the samples in the bin (a bin of the first digit
    // spans a quarter of a binade: too coarse near the top of a row)
    __syncthreads();
    for (int i = tid; i < kHistBins; i += kTopkThreads) sh.hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < kSample; i += kTopkThreads)
      if ((skey[i] >> 21) == bin) atomicAdd(&sh.hist[(skey[i] >> 10) & (kHistBins - 1)], 1u);
    __syncthreads();
    find_bin(sh, kHistBins, m - above, true);
    t0 |= sh.sel[0] << 10;
  }
  __syncthreads();  // the sample keys share memory with the candidates
  return t0;
}


// Rest-mass terms of one element (fp32, as the row pass rounds them).
__device__ __forceinline__ float rest_b(float bj, const RowAux& a) {
  return __fmul_rn(ex2(fmaf(bj, kL, -a.Fb)), a.mb);
}
__device__ __forceinline__ float rest_q(float qj, const RowAux& a) {
  return __fmul_rn(ex2(fmaf(qj, kL, -a.Fq)), a.mq);
}

// Fused pass: elements with key >= t0 become candidates (the count goes on
// past kCap, which sends the row to the exact path); all others add to the
// rest masses (fp32 over one vector, fp64 across vectors).
template <int DT>
__device__ void gather_pass(TopkShared& sh, const char* rb, const char* rq, int64_t V,
                            uint32_t t0, const RowAux& a, double& prest, double& rrest) {
  const int tid = threadIdx.x;
  auto take = [&](float bj, int64_t j, float& sp, float& sr, float qj) {
    const uint32_t key = okey(bj);
    if (key >= t0) {
      const int pos = atomicAdd(&sh.ncand, 1);
      if (pos < kCap)
        sh.cand[pos] = (static_cast<unsigned long long>(key) << 32) | (0xffffffffu - static_cast<uint32_t>(j));
    } else {
      sp += rest_b(bj, a);
      sr += rest_q(qj, a);
    }
  };
  constexpr int EB = DT == KLD_F32 ? 4 : 2;
  constexpr int E = 16 / EB;  // elements per 16-byte vector
  const bool vec = ((reinterpret_cast<uintptr_t>(rb) | reinterpret_cast<uintptr_t>(rq)) & 15u) == 0 &&
                   (V % E) == 0;
  if (vec) {
    const uint4* vb = reinterpret_cast<const uint4*>(rb);
    const uint4* vq = reinterpret_cast<const uint4*>(rq);
    const int64_t nv = V / E;
    for (int64_t v0 = tid; v0 < nv; v0 += kGatherUnroll * kTopkThreads) {
      uint4 xb[kGatherUnroll], xq[kGatherUnroll];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int64_t v = v0 + u * kTopkThreads;
        if (v < nv) {
          xb[u] = __ldg(vb + v);
          xq[u] = __ldg(vq + v);
        }
      }
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int64_t v = v0 + u * kTopkThreads;
        if (v >= nv) continue;
        float fb[E], fq[E];
        const uint32_t wb[4] = {xb[u].x, xb[u].y, xb[u].z, xb[u].w};
        const uint32_t wq[4] = {xq[u].x, xq[u].y, xq[u].z, xq[u].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          if (DT == KLD_F32) {
            fb[w] = __uint_as_float(wb[w]);
            fq[w] = __uint_as_float(wq[w]);
          } else if (DT == KLD_BF16) {
            fb[2 * w] = __uint_as_float(wb[w] << 16);
            fb[2 * w + 1] = __uint_as_float(wb[w] & 0xffff0000u);
            fq[2 * w] = __uint_as_float(wq[w] << 16);
            fq[2 * w + 1] = __uint_as_float(wq[w] & 0xffff0000u);
          } else {
            fb[2 * w] = __half2float(__ushort_as_half(static_cast<unsigned short>(wb[w] & 0xffffu)));
            fb[2 * w + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(wb[w] >> 16)));
            fq[2 * w] = __half2float(__ushort_as_half(static_cast<unsigned short>(wq[w] & 0xffffu)));
            fq[2 * w + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(wq[w] >> 16)));
          }
        }
        float sp = 0.f, sr = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) take(fb[e], v * E + e, sp, sr, fq[e]);
        prest += static_cast<double>(sp);
        rrest += static_cast<double>(sr);
      }
    }
  } else {
    for (int64_t j = tid; j < V; j += kTopkThreads) {
      float sp = 0.f, sr = 0.f;
      take(load_el<DT>(rb, j), j, sp, sr, load_el<DT>(rq, j));
      prest += static_cast<double>(sp);
      rrest += static_cast<double>(sr);
    }
  }
}

// Rows the row pass scanned (TopkScan): the same split into candidates and
// rest as gather_pass, over the lane records the row pass copied and the
// row's head and tail; the rest masses of all other elements come with the
// row (RowAux.rest_b, rest_q). Every thread takes whole lane records; a
// warp's records are contiguous, so the loads coalesce. False (for the
// whole block, before anything is taken) if a consumer warp copied more
// lanes than its region holds: the row then reads both rows once
// (gather_pass) with the same threshold.
template <int DT>
__device__ bool copied_pass(TopkShared& sh, const char* rb, const char* rq, int64_t V,
                            uint32_t t0, const RowAux& a, const uint4* regions, const int* cnt,
                            double& prest, double& rrest) {
  const int tid = threadIdx.x;
  constexpr int EB = DT == KLD_F32 ? 4 : 2;
  constexpr int E = 16 / EB;        // elements per 16-byte vector
  constexpr int VPC = 16 / E;       // vectors per lane and row
  if (tid < kConsumerWarps) sh.fcnt[tid] = cnt[tid];
  __syncthreads();
  bool over = false;
#pragma unroll
  for (int w = 0; w < kConsumerWarps; ++w) over |= sh.fcnt[w] > kCopyCap;
  if (over) return false;
  auto take = [&](float bj, int64_t j, float qj, float& sp, float& sr) {
    const uint32_t key = okey(bj);
    if (key >= t0) {
      const int pos = atomicAdd(&sh.ncand, 1);
      if (pos < kCap)
        sh.cand[pos] = (static_cast<unsigned long long>(key) << 32) | (0xffffffffu - static_cast<uint32_t>(j));
    } else {
      sp += rest_b(bj, a);
      sr += rest_q(qj, a);
    }
  };
  const RowSpan g = row_span(rb, V, EB);
  // head and tail (< 16 bytes each)
  const int n_extra = static_cast<int>(g.head + g.tail);
  if (tid < n_extra) {
    const int64_t j = tid < g.head ? tid : g.head + g.body + (tid - g.head);
    float sp = 0.f, sr = 0.f;
    take(load_el<DT>(rb, j), j, load_el<DT>(rq, j), sp, sr);
    prest += static_cast<double>(sp);
    rrest += static_cast<double>(sr);
  }
  for (int i = tid; i < kConsumerWarps * kCopyCap; i += kTopkThreads) {
    const int w = i / kCopyCap, e = i % kCopyCap;
    if (e >= sh.fcnt[w]) continue;
    const uint4* reg = regions + w * kRegionVecs;
    const uint32_t id = reinterpret_cast<const uint32_t*>(reg + kCopyCap * kCopyVecs)[e];
    const uint4* rec = reg + e * kCopyVecs;
    uint4 xb[VPC], xq[VPC];
#pragma unroll
    for (int k = 0; k < VPC; ++k) {
      xb[k] = rec[k];
      xq[k] = rec[VPC + k];
    }
    const int64_t chunk = id >> 5;
    const int ln = static_cast<int>(id & 31u);
    float sp = 0.f, sr = 0.f;
#pragma unroll
    for (int k = 0; k < VPC; ++k) {
      const int64_t off = chunk * kChunkElems + static_cast<int64_t>(k * 32 + ln) * E;
      if (off >= g.body) break;
      float fb[E], fq[E];
      const uint32_t wb[4] = {xb[k].x, xb[k].y, xb[k].z, xb[k].w};
      const uint32_t wq[4] = {xq[k].x, xq[k].y, xq[k].z, xq[k].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (DT == KLD_F32) {
          fb[u] = __uint_as_float(wb[u]);
          fq[u] = __uint_as_float(wq[u]);
        } else if (DT == KLD_BF16) {
          fb[2 * u] = __uint_as_float(wb[u] << 16);
          fb[2 * u + 1] = __uint_as_float(wb[u] & 0xffff0000u);
          fq[2 * u] = __uint_as_float(wq[u] << 16);
          fq[2 * u + 1] = __uint_as_float(wq[u] & 0xffff0000u);
        } else {
          fb[2 * u] = __half2float(__ushort_as_half(static_cast<unsigned short>(wb[u] & 0xffffu)));
          fb[2 * u + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(wb[u] >> 16)));
          fq[2 * u] = __half2float(__ushort_as_half(static_cast<unsigned short>(wq[u] & 0xffffu)));
          fq[2 * u + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(wq[u] >> 16)));
        }
      }
#pragma unroll
      for (int u = 0; u < E; ++u) take(fb[u], g.head + off + u, fq[u], sp, sr);
    }
    prest += static_cast<double>(sp);
    rrest += static_cast<double>(sr);
  }
  return true;
}

// The first kt of the n (unique) candidates in descending order, by counting
// for each candidate how many are larger: for the few hundred candidates of
// the fast path this beats a bitonic network and its barriers. When there
// are many more candidates than kt, a histogram of their keys above t0 first
// finds the bin that holds the kt-th largest: every candidate below that bin
// is outside T, and only the ones in it or above (about kt) are ranked
// against each other. T goes to sh.cand[kCap .. kCap + kt) (the sorted list
// the outputs read), candidates beyond T add to the rest masses.
template <int DT>
__device__ void rank_select(TopkShared& sh, int n, int kt, uint32_t t0, const char* rq,
                            const RowAux& a, double& prest, double& rrest) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned long long* out = sh.cand + kCap;
  auto to_rest = [&](unsigned long long x) {
    const uint32_t j = 0xffffffffu - static_cast<uint32_t>(x);
    prest += static_cast<double>(rest_b(key_float(static_cast<uint32_t>(x >> 32)), a));
    rrest += static_cast<double>(rest_q(load_el<DT>(rq, j), a));
  };
  const unsigned long long* set = sh.cand;
  int ns = n;
  if (n > 2 * kt + 64) {
    // digit = (key - t0) >> s over 2048 bins, s from the largest key
    unsigned mx = 0u;
    for (int e = tid; e < n; e += kTopkThreads)
      mx = max(mx, static_cast<uint32_t>(sh.cand[e] >> 32) - t0);
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) sh.wmax[warp] = mx;
    for (int i = tid; i < kHistBins; i += kTopkThreads) sh.hist[i] = 0u;
    if (tid == 0) sh.nset = 0;
    __syncthreads();
    mx = 0u;
#pragma unroll
    for (int w = 0; w < kTopkWarps; ++w) mx = max(mx, sh.wmax[w]);
    const int bits = 32 - __clz(mx);  // mx < 2^bits
    const int s = bits > 11 ? bits - 11 : 0;
    for (int e = tid; e < n; e += kTopkThreads)
      atomicAdd(&sh.hist[(static_cast<uint32_t>(sh.cand[e] >> 32) - t0) >> s], 1u);
    __syncthreads();
    find_bin(sh, kHistBins, static_cast<unsigned>(kt), true);
    const uint32_t B = sh.sel[0];
    unsigned long long* setw = sh.cand + kSetBase;
    // two candidates per thread and step, so that the quant logits of those
    // that join the rest are fetched together (one memory latency)
    for (int e0 = tid; e0 < n; e0 += 2 * kTopkThreads) {
      const int e1 = e0 + kTopkThreads;
      const unsigned long long x0 = sh.cand[e0], x1 = e1 < n ? sh.cand[e1] : 0ull;
      const bool in0 = ((static_cast<uint32_t>(x0 >> 32) - t0) >> s) >= B;
      const bool in1 = e1 < n && ((static_cast<uint32_t>(x1 >> 32) - t0) >> s) >= B;
      const bool out1 = e1 < n && !in1;
      const float q0 = in0 ? 0.f : load_el<DT>(rq, 0xffffffffu - static_cast<uint32_t>(x0));
      const float q1 = out1 ? load_el<DT>(rq, 0xffffffffu - static_cast<uint32_t>(x1)) : 0.f;
      if (in0) {
        setw[atomicAdd(&sh.nset, 1)] = x0;
      } else {
        prest += static_cast<double>(rest_b(key_float(static_cast<uint32_t>(x0 >> 32)), a));
        rrest += static_cast<double>(rest_q(q0, a));
      }
      if (in1) {
        setw[atomicAdd(&sh.nset, 1)] = x1;
      } else if (out1) {
        prest += static_cast<double>(rest_b(key_float(static_cast<uint32_t>(x1 >> 32)), a));
        rrest += static_cast<double>(rest_q(q1, a));
      }
    }
    __syncthreads();
    set = setw;
    ns = sh.nset;
  }
  for (int e0 = tid; e0 < ns; e0 += 2 * kTopkThreads) {
    const int e1 = e0 + kTopkThreads;
    const unsigned long long x0 = set[e0];
    const unsigned long long x1 = e1 < ns ? set[e1] : ~0ull;
    int r0 = 0, r1 = 0;
    for (int i = 0; i < ns; ++i) {
      const unsigned long long y = set[i];  // same address in every lane: broadcast
      r0 += y > x0;
      r1 += y > x1;
    }
    const unsigned long long xs[2] = {x0, x1};
    const int rs[2] = {r0, r1};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (u == 1 && e1 >= ns) break;
      if (rs[u] < kt)
        out[rs[u]] = xs[u];
      else
        to_rest(xs[u]);
    }
  }
  __syncthreads();
}

// Bitonic sort of sh.cand[0..n) descending; zeros pad to a power of 2.
__device__ void sort_cand(TopkShared& sh, int n) {
  const int tid = threadIdx.x;
  int p2 = 1;
  while (p2 < n) p2 <<= 1;
  for (int i = n + tid; i < p2; i += kTopkThreads) sh.cand[i] = 0ull;
  __syncthreads();
  for (int kk = 2; kk <= p2; kk <<= 1) {
    for (int jj = kk >> 1; jj > 0; jj >>= 1) {
      for (int i = tid; i < p2; i += kTopkThreads) {
        const int ixj = i ^ jj;
        if (ixj > i) {
          const unsigned long long x = sh.cand[i], y = sh.cand[ixj];
          const bool desc = (i & kk) == 0;
          if (desc ? (x < y) : (x > y)) {
            sh.cand[i] = y;
            sh.cand[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// T (the first kt sorted candidates): indices, log P_base and this thread's
// share of sum_T p_j log(p_j / r_j); inf_t = 1 if the quant row gives an
// element of T no mass.
template <int DT>
__device__ void t_terms(const unsigned long long* sorted, const char* rb, const char* rq,
                        const RowAux& a, int64_t r, int k, int kt, double lambda,
                        int32_t* idx_out, float* logp_out, double& kl_t, double& inf_t) {
  for (int i = threadIdx.x; i < k; i += kTopkThreads) {
    if (i < kt) {
      const uint32_t j = 0xffffffffu - static_cast<uint32_t>(sorted[i]);
      const float bj = load_el<DT>(rb, j), qj = load_el<DT>(rq, j);
      const double lp = lambda * static_cast<double>(bj) - a.lse_b;
      if (idx_out) idx_out[r * k + i] = static_cast<int32_t>(j);
      if (logp_out) logp_out[r * k + i] = static_cast<float>(lp);
      if (bj != -INFINITY) {
        if (qj == -INFINITY) {
          inf_t = 1.0;
        } else {
          // x formed as the row pass forms it, so that it agrees with the
          // log1p(B/S) that pass summed: rounded as (q - b) + K for small
          // centres (an exact x would leave the sums' mean rounding error
          // in the result), exact for fp32 rows offset by a large constant
          // (where the row pass's order keeps x exact)
          double x;
          if (DT == KLD_F32 && fabsf(a.K) >= kShiftForm)
            x = (static_cast<double>(qj) - static_cast<double>(bj)) + static_cast<double>(a.K);
          else
            x = static_cast<double>(__fadd_rn(__fsub_rn(qj, bj), a.K));
          const double lratio = a.lr - lambda * x;  // log p_j - log r_j
          kl_t += exp(lp) * lratio;
        }
      }
    } else {
      if (idx_out) idx_out[r * k + i] = -1;
      if (logp_out) logp_out[r * k + i] = -INFINITY;
    }
  }
}

// Block sums and the row's outputs.
__device__ void finish_row(TopkShared& sh, int64_t r, double kl_t, double inf_t, double prest,
                           double rrest, float* rest_out, double* kl_out) {
  block_sum4(sh, kl_t, inf_t, prest, rrest);
  if (threadIdx.x == 0) {
    double kl = kl_t;
    bool inf = inf_t > 0.0;
    if (prest > 0.0) {
      if (rrest > 0.0)
        kl += prest * (log(prest) - log(rrest));
      else
        inf = true;
    }
    if (rest_out) rest_out[r] = prest > 0.0 ? static_cast<float>(log(prest)) : -INFINITY;
    kl_out[r] = inf ? INFINITY : kl;
  }
}

template <int DT>
__global__ void __launch_bounds__(kTopkThreads, kTopkCtasPerSm)
    kld_topk_kernel(const void* __restrict__ base, const void* __restrict__ quant,
                    const RowAux* __restrict__ aux, int64_t N, int64_t V, int k,
                    int32_t* __restrict__ idx_out, float* __restrict__ logp_out,
                    float* __restrict__ rest_out, double* __restrict__ kl_out,
                    const float* __restrict__ scan_tf, const uint4* __restrict__ scan_regions,
                    const int* __restrict__ scan_counts, unsigned long long* __restrict__ exact_rows) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  constexpr int EB = DT == KLD_F32 ? 4 : 2;
  const double lambda = static_cast<double>(kL) * kLn2;
  const float nanf = __int_as_float(0x7fc00000);
  const int tid = threadIdx.x;
  const int kt = static_cast<int>(V < k ? V : k);

  for (int64_t r = blockIdx.x; r < N; r += gridDim.x) {
    const char* rb = static_cast<const char*>(base) + r * V * EB;
    const char* rq = static_cast<const char*>(quant) + r * V * EB;
    const RowAux a = aux[r];
    if (isnan(a.Fb)) {  // excluded row
      for (int i = tid; i < k; i += kTopkThreads) {
        if (idx_out) idx_out[r * k + i] = -1;
        if (logp_out) logp_out[r * k + i] = nanf;
      }
      if (tid == 0) {
        if (rest_out) rest_out[r] = nanf;
        kl_out[r] = __longlong_as_double(0x7ff8000000000000ll);
      }
      continue;
    }

    // ---- fast path: a threshold, then every element at or above it is a
    // candidate and every other one adds to the rest masses. Rows the row
    // pass scanned read the lanes it copied (all their candidates) and the
    // head and tail; the others sample their threshold here and read both
    // rows once.
    {
      const bool scanned = scan_tf != nullptr;
      const uint32_t t0 = scanned ? okey(scan_tf[r])
                                  : (V > kCap ? sample_threshold<DT>(sh, rb, V, kt) : 0u);
      if (tid == 0) sh.ncand = 0;
      __syncthreads();
      double prest = 0.0, rrest = 0.0;
      if (scanned) {
        if (copied_pass<DT>(sh, rb, rq, V, t0, a, scan_regions + r * kConsumerWarps * kRegionVecs,
                            scan_counts + r * kConsumerWarps, prest, rrest)) {
          if (tid == 0) {  // the unflagged lanes' shares, added once
            prest += a.rest_b;
            rrest += a.rest_q;
          }
        } else {  // a region overflowed: both rows once, with the same threshold
          gather_pass<DT>(sh, rb, rq, V, t0, a, prest, rrest);
        }
      } else {
        gather_pass<DT>(sh, rb, rq, V, t0, a, prest, rrest);
      }
      __syncthreads();
      const int n = sh.ncand;
      if (n >= kt && n <= kCap) {
        double kl_t = 0.0, inf_t = 0.0;
        if (n <= kRankMax) {
          rank_select<DT>(sh, n, kt, t0, rq, a, prest, rrest);
          t_terms<DT>(sh.cand + kCap, rb, rq, a, r, k, kt, lambda, idx_out, logp_out, kl_t, inf_t);
        } else {
          sort_cand(sh, n);
          t_terms<DT>(sh.cand, rb, rq, a, r, k, kt, lambda, idx_out, logp_out, kl_t, inf_t);
          // candidates beyond T join the rest
          for (int i = kt + tid; i < n; i += kTopkThreads) {
            const uint32_t j = 0xffffffffu - static_cast<uint32_t>(sh.cand[i]);
            prest += static_cast<double>(rest_b(key_float(static_cast<uint32_t>(sh.cand[i] >> 32)), a));
            rrest += static_cast<double>(rest_q(load_el<DT>(rq, j), a));
          }
        }
        __syncthreads();  // everyone is done with cand before the next row reuses it
        finish_row(sh, r, kl_t, inf_t, prest, rrest, rest_out, kl_out);
        continue;
      }
    }

    // ---- exact path. Threshold key: MSB radix select for the kt-th largest key
    if (tid == 0 && exact_rows != nullptr) atomicAdd(exact_rows, 1ull);
    uint32_t prefix = 0u, mask = 0u;
    unsigned need = static_cast<unsigned>(kt);
    unsigned ncount = static_cast<unsigned>(V);  // elements matching the prefix
    const int shifts[3] = {21, 10, 0}, widths[3] = {11, 11, 10};
    int levels = 0;
    for (; levels < 3; ++levels) {
      if ((static_cast<unsigned>(kt) - need) + ncount <= static_cast<unsigned>(kCap)) break;
      const int sh_ = shifts[levels], bins = 1 << widths[levels];
      for (int i = tid; i < kHistBins; i += kTopkThreads) sh.hist[i] = 0u;
      __syncthreads();
      // warp-aggregated shared atomics: the bins of a row are few and crowded
      for (int64_t j0 = 0; j0 < V; j0 += kTopkThreads) {
        const int64_t j = j0 + tid;
        int bin = -1;
        if (j < V) {
          const uint32_t key = okey(load_el<DT>(rb, j));
          if ((key & mask) == prefix) bin = static_cast<int>((key >> sh_) & (bins - 1));
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin >= 0 && (tid & 31) == __ffs(peers) - 1) atomicAdd(&sh.hist[bin], __popc(peers));
      }
      __syncthreads();
      find_bin(sh, bins, need, true);
      const unsigned bin = sh.sel[0], above = sh.sel[1], inbin = sh.sel[2];
      __syncthreads();
      need -= above;
      prefix |= bin << sh_;
      mask |= static_cast<uint32_t>(bins - 1) << sh_;
      ncount = inbin;
    }

    // ---- collect the candidates
    if (tid == 0) sh.ncand = 0;
    __syncthreads();
    if ((static_cast<unsigned>(kt) - need) + ncount <= static_cast<unsigned>(kCap)) {
      // every element above the prefix, and every element in it
      for (int64_t j = tid; j < V; j += kTopkThreads) {
        const uint32_t key = okey(load_el<DT>(rb, j));
        if ((key & mask) >= prefix) {
          const int pos = atomicAdd(&sh.ncand, 1);
          sh.cand[pos] = (static_cast<unsigned long long>(key) << 32) | (0xffffffffu - static_cast<uint32_t>(j));
        }
      }
    } else {
      // all 32 key bits fixed and a tie group too large to sort: the `need`
      // lowest indices among keys equal to the threshold (radix select on the
      // index from the bottom), then every key above it
      const uint32_t tau = prefix;
      uint32_t jp = 0u, jm = 0u;
      unsigned jneed = need;
      const int jshifts[3] = {20, 10, 0}, jwidths[3] = {11, 10, 10};
      for (int lv = 0; lv < 3; ++lv) {
        const int sh_ = jshifts[lv], bins = 1 << jwidths[lv];
        for (int i = tid; i < kHistBins; i += kTopkThreads) sh.hist[i] = 0u;
        __syncthreads();
        for (int64_t j0 = 0; j0 < V; j0 += kTopkThreads) {
          const int64_t j = j0 + tid;
          int bin = -1;
          if (j < V) {
            const uint32_t uj = static_cast<uint32_t>(j);
            if ((uj & jm) == jp && okey(load_el<DT>(rb, j)) == tau)
              bin = static_cast<int>((uj >> sh_) & (bins - 1));
          }
          const unsigned peers = __match_any_sync(0xffffffffu, bin);
          if (bin >= 0 && (tid & 31) == __ffs(peers) - 1) atomicAdd(&sh.hist[bin], __popc(peers));
        }
        __syncthreads();
        find_bin(sh, bins, jneed, false);
        const unsigned bin = sh.sel[0], below = sh.sel[1];
        __syncthreads();
        jneed -= below;
        jp |= bin << sh_;
        jm |= static_cast<uint32_t>(bins - 1) << sh_;
      }
      const uint32_t jlast = jp;  // the need-th lowest index with key == tau
      for (int64_t j = tid; j < V; j += kTopkThreads) {
        const uint32_t key = okey(load_el<DT>(rb, j));
        if (key > tau || (key == tau && static_cast<uint32_t>(j) <= jlast)) {
          const int pos = atomicAdd(&sh.ncand, 1);
          sh.cand[pos] = (static_cast<unsigned long long>(key) << 32) | (0xffffffffu - static_cast<uint32_t>(j));
        }
      }
    }
    __syncthreads();

    sort_cand(sh, sh.ncand);
    double kl_t = 0.0, inf_t = 0.0;
    t_terms<DT>(sh.cand, rb, rq, a, r, k, kt, lambda, idx_out, logp_out, kl_t, inf_t);
    // membership of T: key above the last selected, or equal with an index
    // no larger than its
    const unsigned long long last = sh.cand[kt - 1];
    const uint32_t tau_f = static_cast<uint32_t>(last >> 32);
    const uint32_t j_f = 0xffffffffu - static_cast<uint32_t>(last);
    double prest = 0.0, rrest = 0.0;
    for (int64_t j = tid; j < V; j += kTopkThreads) {
      const float bj = load_el<DT>(rb, j);
      const uint32_t key = okey(bj);
      if (key > tau_f || (key == tau_f && static_cast<uint32_t>(j) <= j_f)) continue;
      prest += static_cast<double>(rest_b(bj, a));
      rrest += static_cast<double>(rest_q(load_el<DT>(rq, j), a));
    }
    __syncthreads();  // everyone is done with cand before the next row reuses it
    finish_row(sh, r, kl_t, inf_t, prest, rrest, rest_out, kl_out);
  }
}

// Thresholds of the top-k scan: the fast path's sampled threshold of each
// row, as the float whose order key it is. Only the histogram and the
// sample keys in shared memory, so that more rows are in flight per SM
// (each row is a chain of dependent steps).
struct ThresholdShared {
  unsigned hist[kHistBins];
  unsigned long long cand[kSample / 2];  // the kSample sample keys
  unsigned sel[3];
};
constexpr int kThresholdCtasPerSm = 4;
template <int DT>
__global__ void __launch_bounds__(kTopkThreads, kThresholdCtasPerSm)
    kld_topk_threshold_kernel(const void* __restrict__ base, int64_t N, int64_t V, int kt,
                              float* __restrict__ tf) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ThresholdShared& sh = *reinterpret_cast<ThresholdShared*>(smem_raw);
  constexpr int EB = DT == KLD_F32 ? 4 : 2;
  for (int64_t r = blockIdx.x; r < N; r += gridDim.x) {
    const uint32_t t0 = sample_threshold<DT>(sh, static_cast<const char*>(base) + r * V * EB, V, kt);
    if (threadIdx.x == 0) tf[r] = key_float(t0);
  }
}

int64_t topk_grid(int sm_count, int64_t N) {
  const int64_t grid = static_cast<int64_t>(sm_count) * kTopkCtasPerSm;
  return grid > N ? N : grid;
}

template <int DT>
cudaError_t launch_typed(const void* base, const void* quant, const RowAux* aux, int64_t N,
                         int64_t V, int k, int32_t* idx, float* logp, float* rest, double* kl,
                         int sm_count, cudaStream_t s, const TopkScan* scan,
                         unsigned long long* exact_rows) {
  const size_t smem = sizeof(TopkShared);
  cudaError_t e = cudaFuncSetAttribute(kld_topk_kernel<DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kld_topk_kernel<DT><<<static_cast<unsigned>(topk_grid(sm_count, N)), kTopkThreads, smem, s>>>(
      base, quant, aux, N, V, k, idx, logp, rest, kl, scan ? scan->tf : nullptr,
      scan ? scan->regions : nullptr, scan ? scan->counts : nullptr, exact_rows);
  return cudaGetLastError();
}

template <int DT>
cudaError_t launch_threshold_typed(const void* base, int64_t N, int64_t V, int kt, float* tf,
                                   int sm_count, cudaStream_t s) {
  const size_t smem = sizeof(ThresholdShared);
  cudaError_t e = cudaFuncSetAttribute(kld_topk_threshold_kernel<DT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int64_t grid = static_cast<int64_t>(sm_count) * kThresholdCtasPerSm;
  if (grid > N) grid = N;
  kld_topk_threshold_kernel<DT><<<static_cast<unsigned>(grid), kTopkThreads, smem, s>>>(
      base, N, V, kt, tf);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk(const void* base, const void* quant, const RowAux* aux, int64_t N,
                        int64_t V, kld_dtype_t dtype, int k, int32_t* idx, float* logp,
                        float* rest, double* kl, int sm_count, cudaStream_t stream,
                        const TopkScan* scan, unsigned long long* exact_rows) {
  if (k < 1 || k > kMaxTopk) return cudaErrorInvalidValue;
  if (scan != nullptr && (V <= kCap || !scan->tf || !scan->regions || !scan->counts))
    return cudaErrorInvalidValue;
  switch (dtype) {
    case KLD_F32:
      return launch_typed<KLD_F32>(base, quant, aux, N, V, k, idx, logp, rest, kl, sm_count, stream, scan, exact_rows);
    case KLD_BF16:
      return launch_typed<KLD_BF16>(base, quant, aux, N, V, k, idx, logp, rest, kl, sm_count, stream, scan, exact_rows);
    case KLD_F16:
      return launch_typed<KLD_F16>(base, quant, aux, N, V, k, idx, logp, rest, kl, sm_count, stream, scan, exact_rows);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_topk_threshold(const void* base, int64_t N, int64_t V, kld_dtype_t dtype,
                                  int k, float* tf, int sm_count, cudaStream_t stream) {
  if (k < 1 || k > kMaxTopk || V <= kCap || N < 1 || !tf) return cudaErrorInvalidValue;
  const int kt = static_cast<int>(V < k ? V : k);
  switch (dtype) {
    case KLD_F32: return launch_threshold_typed<KLD_F32>(base, N, V, kt, tf, sm_count, stream);
    case KLD_BF16: return launch_threshold_typed<KLD_BF16>(base, N, V, kt, tf, sm_count, stream);
    case KLD_F16: return launch_threshold_typed<KLD_F16>(base, N, V, kt, tf, sm_count, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kld
