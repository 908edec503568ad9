// kld_internal.h -- declarations shared by the library's translation units
// (row pass, reduction, host API). Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kld_stats.h"

namespace kld {

// Device error word bits (kld_result_t.device_error).
constexpr uint32_t kErrWaitTimeout = 1u << 0;  // a bounded mbarrier wait gave up

// Row-pass geometry: a producer warp streams both rows through a ring of
// shared-memory stages with bulk copies; kConsumerWarps warps consume them in
// chunks of kLaneElems elements per lane; one epilogue warp combines each
// row's partials (published through a ring of kSlots slots).
constexpr int kConsumerWarps = 16;
constexpr int kRowThreads = (kConsumerWarps + 2) * 32;
constexpr int kStageBytes = 32 * 1024;  // per operand per stage
constexpr int kStages = 3;
constexpr int kLaneElems = 16;
constexpr int kChunkElems = kLaneElems * 32;  // elements per warp-chunk
constexpr int kSlots = 4;

// Split-row mode: up to kMaxClusterCtas CTAs per thread-block cluster share
// one row; their partials meet in the cluster leader's shared memory.
constexpr int kMaxClusterCtas = 8;

// Per-handle global scratch of split rows (parts of one row on several
// CTAs): kPartSlotsPerRow 64-byte partials and one arrival ticket per split
// row; a launch splits at most `capacity` rows (>= the SM count), and the
// ticket after the last split row's counts a few-row launch's finished rows
// (its in-pass reduction). Tickets start at zero and whoever finishes with
// one puts it back.
constexpr int kSplitPartBytes = 64;
constexpr int kPartSlotsPerRow = 32;
struct SplitScratch {
  void* parts;
  unsigned* tickets;
  int capacity;
  int max_cluster_ctas;  // largest cluster the plan may use (1: plain CTAs; 0: never split)
};
// Cluster size split rows use unless the caller asks otherwise.
constexpr int kDefaultClusterCtas = 1;

// Dynamic shared memory of the row kernel: stages for both operands, then the
// control block (mbarriers and the partial slots).
constexpr int kRowCtrlBytes = 24 * 1024;
constexpr int kRowSmemBytes = kStages * 2 * kStageBytes + kRowCtrlBytes;

// Reduction kernel geometry.
constexpr int kReduceThreads = 1024;

inline int elem_bytes(kld_dtype_t dt) { return dt == KLD_F32 ? 4 : 2; }

// The row pass forms the log-ratio x = q - b + K of fp32 inputs in the order
// that keeps it exact for rows offset by a large constant: when |K| >= this,
// (q + K) - b or q - (b - K); below it, (q - b) + K (the order 16-bit
// inputs always take, where q - b is exact). Passes that reuse the row
// pass's sums form x the same way.
constexpr float kShiftForm = 8.0f;

// Per-row normalisers the row pass leaves for the gradient and top-k passes
// (64 bytes; the first 16 are read as a float4 by the gradient pass).
struct RowAux {
  float Fb, mb, Fq, mq;  // softmax(b)_j = 2^(b_j L - Fb) mb, softmax(q)_j likewise;
                         // Fb NaN on rows excluded from the statistics
  double lse_b;          // ln sum_j exp(lambda b_j)
  double lr;             // log1p(B/S) = lse_q - lse_b + lambda K
  float K;               // centre of the log-ratio x = q - b + K
  uint32_t flags;        // the row's KLD_ROW_* flags
  uint64_t pad;
  // Top-k scan launches only (TopkScan), else 0: softmax(b) and softmax(q)
  // summed over the elements of the lanes the scan left unflagged.
  double rest_b, rest_q;
};
static_assert(sizeof(RowAux) == 64, "RowAux layout");

// Where a row's elements lie for the row pass: `head` elements before the
// row's first 16-byte boundary, a 16-byte-aligned body of `body` elements
// streamed in chunks of kChunkElems, then `tail` elements (the head and
// tail are read apart, < 16 bytes each). Inside the body, element i < 16 of
// lane l in chunk c is at c * kChunkElems + ((i / E) * 32 + l) * E + i % E,
// E = 16 / (element bytes): each lane reads 16-byte vectors, a warp 512
// contiguous bytes per vector step.
struct RowSpan {
  int64_t head, body, tail;
};
__host__ __device__ __forceinline__ RowSpan row_span(const void* row, int64_t V, int eb) {
  RowSpan g;
  const uint32_t mis = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(row) & 15u);
  g.head = static_cast<int64_t>(((16u - mis) & 15u) / static_cast<uint32_t>(eb));
  if (g.head > V) g.head = V;
  const int64_t e = 16 / eb;
  g.body = ((V - g.head) / e) * e;
  g.tail = V - g.head - g.body;
  return g;
}

// Top-k scan of the row pass (launch_rows with `topk` set; whole rows
// only), for a threshold tf[r] on the base logits of row r. In every chunk a
// consumer warp streams, each lane whose 16 elements hold a base logit >=
// tf[r] copies them, both rows' 16-byte vectors as they sit in shared
// memory, to its warp's region of kCopyCap lane records, and notes the
// chunk and lane in ids; every lane of a chunk that takes the direct path
// of the log-ratio sums does the same. The other lanes add their elements'
// softmax weights to rest sums, which go to RowAux.rest_b / rest_q (as
// shares of softmax(b) and softmax(q)). counts[r][w]: the lanes warp w
// copied (it runs on past kCopyCap; the top-k pass then takes that row by
// its exact path). So the top-k pass reads the copies and the row's head
// and tail, never the rows again.
constexpr int kCopyCap = 96;
constexpr int kCopyVecs = 8;  // 16-byte vectors of a lane record: both rows' 16 elements (fp32)
// One warp's region of one row: kCopyCap records, then their kCopyCap ids
// (chunk index in the body * 32 + lane), in 16-byte vectors.
constexpr int kRegionVecs = kCopyCap * kCopyVecs + kCopyCap / 4;
static_assert(kCopyCap % 4 == 0, "ids pack four to a vector");
struct TopkScan {
  float* tf;        // [N], written by launch_topk_threshold
  uint4* regions;   // [N][kConsumerWarps][kRegionVecs]: records (b vectors, then q vectors), ids
  int* counts;      // [N][kConsumerWarps]
};

// Launchers (defined in the .cu files). They enqueue on `stream` and return
// the launch error.
// Row pass. With split == nullptr every CTA handles whole rows; otherwise
// the plan of plan_rows (whole-row rounds, then the last partial wave's rows
// split over all CTAs; few rows over clusters when asked) using the split
// scratch.
// aux (nullable): per-row normalisers for the gradient and top-k passes.
// part_out (nullable): vocabulary-slice mode, the row is columns
// [col_offset, col_offset + V) of a wider vocabulary and each row's merged
// 64-byte partial goes to part_out[r] instead of a record (see
// launch_merge); whole rows only.
// result_out (nullable): a launch whose rows are all split (fewer rows than
// SMs) and at most kFusedReduceRows of them also reduces its records into
// *result_out (the launch's last finaliser does it; no reduction kernel
// needed) and sets *reduced.
constexpr int kFusedReduceRows = 32;
cudaError_t launch_rows(const void* base, const void* quant,
                        const int32_t* token_ids, int64_t N, int64_t V,
                        kld_dtype_t dtype, kld_row_t* rows, uint32_t* derr,
                        int sm_count, const SplitScratch* split, RowAux* aux,
                        cudaStream_t stream, void* part_out = nullptr,
                        int64_t col_offset = 0, kld_result_t* result_out = nullptr,
                        bool* reduced = nullptr, const TopkScan* topk = nullptr);

// The row pass with the top-k scan (TopkScan; whole rows, aux required):
// what launch_rows does when given `topk`. prepare_rows_scan_kernels: its
// per-device attribute setup (called by prepare_rows_kernels).
cudaError_t launch_rows_scan(const void* base, const void* quant, const int32_t* token_ids,
                             int64_t N, int64_t V, kld_dtype_t dtype, kld_row_t* rows,
                             uint32_t* derr, int sm_count, RowAux* aux, const TopkScan& topk,
                             cudaStream_t stream);
cudaError_t prepare_rows_scan_kernels();

// Records from the G vocabulary-slice partials of each row (parts: [G][N]
// 64-byte partials, rank/slice order), tokens checked against V_total.
constexpr int kPartialBytes = 64;
cudaError_t launch_merge(const void* parts, int G, int64_t N, const int32_t* token_ids,
                         int64_t V_total, kld_row_t* rows, cudaStream_t stream);

// Launch shape of the row pass.
//   cluster_ctas > 1: few rows split over thread-block clusters: grid =
//     N * parts_per_row CTAs, parts_per_row / cluster_ctas clusters per row.
//   otherwise: `whole` rounds of whole rows (CTA b takes rows b + j * grid),
//     then the tail_rows remaining rows split over tail_ctas CTAs by balanced
//     ranges of their tail_chunks chunks (nchv per row); parts_per_row is
//     the most CTAs any tail row is split over (1 without a tail).
struct RowPlan {
  int grid, parts_per_row, cluster_ctas;
  int whole, tail_rows, tail_ctas, nchv;
  int64_t tail_chunks;
};
// fit[i]: clusters of 2^i CTAs the device holds at once (i = 0..3; <= 0:
// unknown, estimated as sm_count >> i). max_cluster_ctas: 0 = whole rows
// only (grid = min(N, SMs), rows round robin); 1 = whole rounds plus a split
// tail; 2, 4, 8: as 1, but N <= sm_count / 2 rows are split over clusters of
// the largest power of two <= max_cluster_ctas that leaves one cluster per
// row in one wave, each row taking as many clusters (<= 32) as still fit.
RowPlan plan_rows(int64_t N, int64_t V, int sm_count, const int fit[4], int max_cluster_ctas);
cudaError_t prepare_rows_kernels();  // per-device attribute setup

// Gradient pass: grad[i][j] = scale * (softmax(q_i)_j - softmax(b_i)_j)
// from the per-row normalisers of the row pass (zero on excluded rows);
// grad in grad_dtype, [N, V] row-major.
cudaError_t launch_grad(const void* base, const void* quant, const RowAux* aux, int64_t N,
                        int64_t V, kld_dtype_t dtype, void* grad, kld_dtype_t grad_dtype,
                        float scale, int sm_count, cudaStream_t stream);

// Top-k compression of the base rows and KL of the quant rows against it
// (k <= kMaxTopk), from the row pass's RowAux; idx, logp, rest nullable.
// scan (nullable): the row pass ran the top-k scan with these thresholds
// (from launch_topk_threshold), so only the flagged lanes are read back.
// exact_rows (nullable): counts the rows that took the exact path.
// Rows of at most kTopkCap elements take no threshold (every element is a
// candidate) and no scan.
constexpr int kMaxTopk = 1024;
constexpr int kTopkCap = 4096;
cudaError_t launch_topk(const void* base, const void* quant, const RowAux* aux, int64_t N,
                        int64_t V, kld_dtype_t dtype, int k, int32_t* idx, float* logp,
                        float* rest, double* kl, int sm_count, cudaStream_t stream,
                        const TopkScan* scan = nullptr,
                        unsigned long long* exact_rows = nullptr);
// Per-row base thresholds for the top-k scan: tf[r] from 4096 samples of
// row r, with comfortably more than k but (by the samples) at most
// kTopkCap elements at or above it.
cudaError_t launch_topk_threshold(const void* base, int64_t N, int64_t V, kld_dtype_t dtype,
                                  int k, float* tf, int sm_count, cudaStream_t stream);

// Bounded-wait self-test (see kld_selftest_bounded_wait).
cudaError_t launch_wait_selftest(uint64_t limit_ns, int use_abort, uint32_t* derr,
                                 unsigned long long* waited_ns, cudaStream_t stream);

cudaError_t launch_reduce(const kld_row_t* rows, int64_t N, int has_nll,
                          uint32_t* derr, kld_result_t* out,
                          cudaStream_t stream);

// Per-field copies of N records (kld_stats_rows): kld[i], nll[i], amax_b[i],
// amax_q[i] from rows[i].
cudaError_t launch_split_records(const kld_row_t* rows, int64_t N, double* kld, double* nll,
                                 int32_t* amax_b, int32_t* amax_q, cudaStream_t stream);

}  // namespace kld
