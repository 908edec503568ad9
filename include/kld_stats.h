/*
 * kld_stats.h -- C ABI of the B200 (sm_100a) logit KL-divergence statistics
 * library (libkld_stats.so).
 *
 * The statistic is the one `llama-perplexity --kl-divergence` prints when a
 * quantized model is scored against its BF16 base ("Qwen3.6 27B Quantization
 * Benchmark", sections "Measurement method" and "Understand KLD and Same Top
 * P", and the "Raw benchmark data" table). For each of N token positions the
 * library takes a base logit row b and a quantized logit row q over a
 * vocabulary of V entries and computes, in one pass over HBM:
 *
 *   KL_i   = sum_j P_j (log P_j - log R_j),  P = softmax(b), R = softmax(q),
 *            natural log, over the full vocabulary, base first
 *            ("Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S GGUF", "How it was
 *            made", step 5: KL(BF16 || quantized) over the full vocabulary);
 *   amax_i = argmax_j b_j and argmax_j q_j, lowest index on ties
 *            ("Same Top P": how often both models pick the same token);
 *   NLL_i  = -log R_{tok_i} when next-token ids are given (the table's
 *            "Mean PPL(Q)" column is exp(mean NLL));
 *
 * and reduces them over the rows to mean / median / p90 / p99 / max KLD,
 * the top-1 agreement count and percentage, mean NLL and PPL. Percentiles
 * interpolate linearly between order statistics at pos = p*(n-1).
 *
 * Conventions shared by every call:
 *   - Logit tensors are row-major [N, V], contiguous, in device memory
 *     (except kld_stats_run_host), element type kld_dtype_t. Row i of base
 *     and row i of quant are paired. Both pointers must be aligned to their
 *     element size and have the same address modulo 16 (true for any two
 *     tensors from cudaMalloc or the PyTorch allocator).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Work is enqueued asynchronously; inputs must stay valid and
 *     unchanged until kld_stats_result() returns.
 *   - Memory passed in is owned by the caller; memory a handle allocates is
 *     owned by the handle and released by kld_stats_destroy().
 *   - Errors are reported by return codes only: nothing on the device traps
 *     or aborts. Arguments are checked before anything is enqueued; errors
 *     that arise on the device (a bounded wait giving up, rows that must be
 *     excluded) surface in kld_stats_result().
 *   - A handle is bound to one device and is not thread-safe; use one handle
 *     per concurrent stream.
 *
 * Row policy (the pages are silent; both this library and its test oracle
 * follow it):
 *   - a row holding NaN or +inf in b or q: flag NONFINITE, KL/NLL = NaN,
 *     argmaxes -1, excluded from every statistic;
 *   - a row whose b or q entries are all -inf: flag EMPTY, treated the same;
 *   - entries with b_j = -inf have P_j = 0 and add nothing (padding masks);
 *     b_j finite with q_j = -inf gives KL = +inf (flag INF_KL, row kept);
 *   - token id outside [0, V): flag BAD_TOKEN, row left out of NLL/PPL;
 *     q[tok] = -inf gives NLL = +inf (flag INF_NLL, row kept).
 */
#ifndef KLD_STATS_H
#define KLD_STATS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KLD_ABI_VERSION 4

typedef enum {
  KLD_OK = 0,
  KLD_ERR_INVALID_ARG = 1, /* null/unaligned pointer, N or V out of range  */
  KLD_ERR_DTYPE = 2,       /* unknown element type                         */
  KLD_ERR_OOM = 3,         /* a device or pinned allocation failed          */
  KLD_ERR_CUDA = 4,        /* a CUDA call failed; see kld_last_cuda_error() */
  KLD_ERR_NONFINITE = 5,   /* some rows were NONFINITE or EMPTY (excluded);
                              the statistics of the other rows are valid     */
  KLD_ERR_BAD_TOKEN = 6,   /* some token ids were outside [0, V); PPL uses
                              the other rows                                 */
  KLD_ERR_TIMEOUT = 7,     /* a bounded device-side wait gave up            */
  KLD_ERR_NO_DEVICE = 8,   /* no usable sm_100 device                       */
  KLD_ERR_NOT_READY = 9,   /* kld_stats_result() before any run             */
  KLD_ERR_CAPACITY = 10    /* more rows than kld_stats_run_static can hold  */
} kld_status_t;

typedef enum { KLD_F32 = 0, KLD_BF16 = 1, KLD_F16 = 2 } kld_dtype_t;

/* Per-row flag bits (kld_row_t.flags). */
#define KLD_ROW_NONFINITE (1u << 0)
#define KLD_ROW_EMPTY     (1u << 1)
#define KLD_ROW_INF_KL    (1u << 2)
#define KLD_ROW_BAD_TOKEN (1u << 3)
#define KLD_ROW_INF_NLL   (1u << 4)
#define KLD_ROW_INF_NLL_BASE (1u << 5)  /* b[tok] = -inf: nll_base = +inf */

/* One 40-byte record per row, written by the row pass. */
typedef struct {
  double kld;            /* KL(P_base || P_quant) in nats (NaN if excluded) */
  double nll;            /* -log P_quant(tok) (NaN if no/bad token)        */
  double nll_base;       /* -log P_base(tok), same conditions               */
  int32_t argmax_base;   /* lowest index of the row maximum, -1 if excluded */
  int32_t argmax_quant;
  uint32_t flags;        /* KLD_ROW_* bits                                  */
  float dp;              /* P_quant(tok) - P_base(tok) (NaN if no/bad token) */
} kld_row_t;

/* Summary statistics (caller-owned plain struct). */
typedef struct {
  int64_t n_rows;        /* rows reduced                                      */
  int64_t n_valid;       /* rows that are neither NONFINITE nor EMPTY         */
  double mean_kld;       /* statistics over the valid rows (NaN if none)      */
  double median_kld;
  double p90_kld;
  double p99_kld;
  double max_kld;
  int64_t top1_agree;    /* valid rows whose two argmaxes are equal           */
  double top1_agree_pct; /* 100 * top1_agree / n_valid                        */
  int32_t has_nll;       /* token ids were given                              */
  int32_t reserved0;
  int64_t n_nll;         /* valid rows with an in-range token id              */
  double mean_nll;
  double ppl;            /* exp(mean_nll)                                     */
  int64_t n_flagged;     /* rows with any flag                                */
  uint32_t flags_or;     /* OR of all row flags                               */
  uint32_t device_error; /* nonzero if a bounded device wait gave up          */
  /* Over the same rows as mean_nll (NaN without token ids). The perplexity
   * ratio and the probability the quantized model gives the token against
   * the base ("Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S GGUF", "Quality";
   * "Qwen3.6 27B Quantization Benchmark", table column RMS dp (%)). */
  double mean_nll_base;  /* mean of -log P_base(tok)                         */
  double ppl_base;       /* exp(mean_nll_base)                                */
  double ln_ppl_ratio;   /* mean_nll - mean_nll_base = ln(PPL(Q)/PPL(base))   */
  double mean_dp;        /* mean of dp = P_quant(tok) - P_base(tok)           */
  double rms_dp;         /* sqrt(mean of dp^2)                                */
} kld_result_t;

typedef struct kld_stats_s* kld_stats_t;

/* ABI version this library was built with (KLD_ABI_VERSION). */
int kld_abi_version(void);

/* Static description of a status code. Never NULL. */
const char* kld_status_string(kld_status_t status);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char* kld_last_cuda_error(void);

/*
 * Create a handle on `device` for runs of up to `max_rows` rows.
 * Allocates a device workspace of max_rows records (40 bytes each), the
 * per-field arrays of kld_stats_rows (24 bytes per row), the per-row
 * normalisers of the gradient and top-k passes (64 bytes per row) plus a few
 * KB, and a pinned host copy of the result. The first kld_stats_run_topk on
 * rows of more than 4096 elements adds the top-k scan's workspace (about
 * 200 KB per row of max_rows). Returns KLD_ERR_NO_DEVICE if the
 * device is not a compute-capability 10.0 (B200-class) GPU.
 */
kld_status_t kld_stats_create(kld_stats_t* out, int64_t max_rows, int device);

/* Release everything the handle owns. Waits for its pending work. NULL ok. */
void kld_stats_destroy(kld_stats_t h);

/*
 * The whole statistic for rows [0, N): the fused row pass, then the
 * fixed-order reduction and the exact percentile selection, which writes the
 * result straight into the handle's pinned host buffer (read it with
 * kld_stats_result). A launch whose rows are all split over several CTAs
 * (at most 32 rows, fewer than half the SMs) reduces its own records at the
 * end of the row pass and needs no second kernel.
 * token_ids (device, int32[N]) may be NULL: no NLL/PPL.
 * 1 <= N <= max_rows, 1 <= V <= 2^31-1. Asynchronous.
 */
kld_status_t kld_stats_run(kld_stats_t h, const void* base, const void* quant,
                           const int32_t* token_ids, int64_t N, int64_t V,
                           kld_dtype_t dtype, void* stream);

/*
 * Wait for the last run/reduce of this handle and copy its statistics to
 * *out. Returns KLD_OK, or KLD_ERR_NONFINITE / KLD_ERR_BAD_TOKEN (statistics
 * of the remaining rows still filled in), KLD_ERR_TIMEOUT, KLD_ERR_CUDA.
 */
kld_status_t kld_stats_result(kld_stats_t h, kld_result_t* out);

/*
 * Per-row results of the last run that wrote the handle's workspace
 * (kld_stats_run, kld_stats_run_rows with rows_out NULL, kld_stats_run_host,
 * kld_stats_run_grad, kld_stats_run_topk, kld_stats_merge_partials) as four
 * contiguous DEVICE arrays of N values each, row i at index i:
 *   *kld    KL(P_base || P_quant) in nats, NaN on excluded rows;
 *   *nll    -log P_quant(tok), NaN without tokens or with a bad token;
 *   *amax_b lowest index of the base row's maximum, -1 on excluded rows;
 *   *amax_q the same for the quant row.
 * Any of the four output pointers may be NULL (that array is not returned).
 * The arrays are owned by the handle. The call enqueues a small kernel, on
 * the stream of that run, that copies the fields out of the run's records
 * (kld_stats_records); the arrays are valid in that stream's order after it
 * and until the next run or kld_stats_destroy. KLD_ERR_NOT_READY before any
 * such run.
 */
kld_status_t kld_stats_rows(kld_stats_t h, const double** kld, const double** nll,
                            const int32_t** amax_b, const int32_t** amax_q);

/*
 * The same rows as 40-byte records (kld_row_t, with the flags, the base
 * model's NLL and dp as well): device pointer to the workspace's N records
 * and their count, stream-ordered after the run that wrote them. Valid until
 * the next run or destroy. No kernel is enqueued.
 */
kld_status_t kld_stats_records(kld_stats_t h, const kld_row_t** rows_dev,
                               int64_t* n_rows);

/*
 * The row pass alone: per-row records for rows [0, N) written to rows_out
 * (device, N records, caller-owned; NULL = the handle's workspace). This is
 * the unit a row-sharded multi-GPU run executes on each GPU before the
 * records are gathered and reduced. Asynchronous.
 */
kld_status_t kld_stats_run_rows(kld_stats_t h, const void* base,
                                const void* quant, const int32_t* token_ids,
                                int64_t N, int64_t V, kld_dtype_t dtype,
                                kld_row_t* rows_out, void* stream);

/*
 * Reduction and percentile selection over N records in device memory
 * (rows_dev; NULL = the handle's workspace), e.g. the records of all GPUs
 * after a gather. has_nll: whether token ids were given to the row pass.
 * N may exceed max_rows. Result through kld_stats_result(). Asynchronous.
 */
kld_status_t kld_stats_reduce(kld_stats_t h, const kld_row_t* rows_dev,
                              int64_t N, int has_nll, void* stream);

/*
 * kld_stats_run for logits in HOST memory (e.g. logits saved by a base-model
 * run): rows are copied to the device in chunks on an internal copy stream,
 * overlapped with the row pass of the previous chunk, then reduced as in
 * kld_stats_run. Pinned host memory gives full PCIe bandwidth; pageable
 * memory works but is slower. token_ids is a host pointer or NULL. The first
 * call allocates two device staging buffers (kept until destroy).
 */
kld_status_t kld_stats_run_host(kld_stats_t h, const void* base_host,
                                const void* quant_host,
                                const int32_t* token_ids_host, int64_t N,
                                int64_t V, kld_dtype_t dtype, void* stream);

/*
 * The row pass alone for logits in HOST memory: the chunked, overlapped
 * copies of kld_stats_run_host, then per-row records for rows [0, N) in
 * rows_out (device, N records, caller-owned; NULL = the handle's
 * workspace), without the reduction. This is what one rank of a
 * row-sharded run executes when its shard of logits lives in host memory,
 * before the records are gathered and reduced (kld_stats_reduce).
 * Asynchronous on `stream`; errors as kld_stats_run_host.
 */
kld_status_t kld_stats_run_rows_host(kld_stats_t h, const void* base_host,
                                     const void* quant_host,
                                     const int32_t* token_ids_host, int64_t N,
                                     int64_t V, kld_dtype_t dtype,
                                     kld_row_t* rows_out, void* stream);

/*
 * How the row pass splits rows (see kld_plan):
 *   -1: never split: whole rows round robin at any N (the last partial wave
 *       may leave SMs idle);
 *    0: the library default (currently 1);
 *    1: whole rows, with the rows of a last partial wave (all rows when
 *       N < SMs) split over plain CTAs by balanced chunk ranges, merged
 *       through global memory;
 *    2, 4, 8: as 1, but few rows (N <= SMs / 2) are split over thread-block
 *       clusters of up to that many CTAs, merged first through distributed
 *       shared memory, then across the row's clusters through global memory.
 * Results agree within rounding whatever the shape. Measured on B200 with
 * V = 262144 fp32 rows, plain CTAs were as fast as or up to ~10% faster than
 * clusters, hence the default. Other values: KLD_ERR_INVALID_ARG.
 */
kld_status_t kld_stats_set_split(kld_stats_t h, int cluster_ctas);

/*
 * The statistic plus its gradient with respect to the quant logits, the
 * objective of end-to-end tuning ("Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S
 * GGUF", "How it was made", step 7: minimise KL(BF16 || quantized)):
 *   grad[i][j] = scale * (softmax(q_i)_j - softmax(b_i)_j)
 * (e.g. scale = 1/N for the gradient of the mean over N rows), zero on rows
 * the statistics exclude (NONFINITE / EMPTY). Inputs as for kld_stats_run;
 * grad: caller-owned DEVICE memory for N*V values of grad_dtype (KLD_F32,
 * KLD_BF16 or KLD_F16; row-major [N, V], aligned to its element size; 16-byte
 * aligned with V % 8 == 0 takes the vectorised path). Enqueues the row pass
 * (which also keeps per-row normalisers in the handle), the reduction (the
 * same result as kld_stats_run) and a second streaming pass that reads b and q
 * again and writes grad. Asynchronous on `stream`; kld_stats_result() waits
 * for the statistics, the stream for grad. Errors as kld_stats_run, plus
 * KLD_ERR_DTYPE for an unknown grad_dtype and KLD_ERR_INVALID_ARG for a NULL
 * or misaligned grad or a NaN scale.
 */
kld_status_t kld_stats_run_grad(kld_stats_t h, const void* base, const void* quant,
                                const int32_t* token_ids, int64_t N, int64_t V,
                                kld_dtype_t dtype, void* grad, kld_dtype_t grad_dtype,
                                double scale, void* stream);

/*
 * Vocabulary-sharded rows (a tensor-parallel lm_head leaves each GPU with a
 * column slice of the logits). kld_stats_run_partials takes this GPU's slice:
 * [N, V] row-major logits holding columns [col_offset, col_offset + V) of a
 * vocabulary of V_total entries (same pointer rules as kld_stats_run), and
 * writes one 64-byte partial per row to parts_out (caller-owned DEVICE
 * memory of N * KLD_PARTIAL_BYTES bytes, 16-byte aligned): the slice's
 * maxima with their lowest global indices, its softmax sums in an exact
 * frame, flags, and the token's two logits when token_ids[r] falls in the
 * slice. Gather every slice's partials (any transport; [G][N] in slice
 * order, G <= 32, the slices covering [0, V_total) without overlap) and
 * call kld_stats_merge_partials: it merges each row's G partials into the
 * handle's records (token ids checked against V_total) and enqueues the
 * reduction; kld_stats_result() then returns the statistics of the full
 * rows. Both are asynchronous on `stream`. Errors: KLD_ERR_INVALID_ARG for
 * bad sizes, offsets or alignment, else as kld_stats_run.
 */
#define KLD_PARTIAL_BYTES 64
kld_status_t kld_stats_run_partials(kld_stats_t h, const void* base, const void* quant,
                                    const int32_t* token_ids, int64_t N, int64_t V,
                                    int64_t col_offset, int64_t V_total, kld_dtype_t dtype,
                                    void* parts_out, void* stream);
kld_status_t kld_stats_merge_partials(kld_stats_t h, const void* parts, int G, int64_t N,
                                      const int32_t* token_ids, int64_t V_total, void* stream);

/*
 * The statistic plus a top-k compression of each base row and the KL of the
 * quant row against it ("Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S GGUF",
 * "How it was made", step 7: tuning "against the top-128 distributions (and
 * the rest of the mass)"). Per row r, T = the k largest base logits (ties to
 * the lowest index; 1 <= k <= 1024):
 *   idx_out[r*k + i]  index of the i-th entry of T (int32; -1 past V)
 *   logp_out[r*k + i] its log P_base (float; -inf past V)
 *   rest_out[r]       log of P_base outside T (float; -inf if none)
 *   kl_out[r]         sum_{T} p log(p/r) + p_rest log(p_rest/r_rest) (double)
 * with p = softmax(base), r = softmax(quant). Rows the statistics exclude get
 * idx -1 and NaN. idx_out, logp_out and rest_out may be NULL; all are
 * caller-owned DEVICE memory, naturally aligned. For V > 4096 it enqueues
 * a threshold kernel (a base threshold per row from 4096 samples, with
 * comfortably more than k elements at or above it), the row pass in its
 * top-k scan form (it also copies out the 16-element lanes that hold an
 * element at or above the threshold, about 5 % of the row, and sums the
 * rest masses of all other lanes), the reduction (read with
 * kld_stats_result) and the top-k pass, which selects T in the copies: each
 * logit is read from memory once. For V <=
 * 4096 the top-k pass reads both rows once after the row pass instead.
 * Rows whose threshold holds fewer than k or too many elements (large tie
 * groups, masked rows) fall back to an exact radix selection that reads
 * the base row 2-4 times. The first call with V > 4096 allocates the scan's
 * workspace (cudaMalloc, synchronising the device): make one such call
 * before capturing this call into a CUDA graph.
 */
#define KLD_MAX_TOPK 1024
kld_status_t kld_stats_run_topk(kld_stats_t h, const void* base, const void* quant,
                                const int32_t* token_ids, int64_t N, int64_t V,
                                kld_dtype_t dtype, int k, int32_t* idx_out, float* logp_out,
                                float* rest_out, double* kl_out, void* stream);

/*
 * Allocation-free kld_stats_run (no counterpart on the source pages: it is a
 * deployment convenience of this library).
 *
 * For callers that cannot allocate device memory when they need the
 * statistic -- e.g. a server that reserves almost all HBM for its own pool at
 * start-up, or a loop that cannot afford the device synchronisation
 * cudaMalloc/cudaFree may cause. It takes no handle and allocates nothing:
 * per-row records and the error word live in one fixed array compiled into
 * the library (KLD_STATIC_MAX_ROWS records, about 2.5 MiB), which every GPU
 * that loads the library keeps until the process exits.
 *
 * Runs on the calling thread's current device and enqueues the row pass and
 * the reduction on `stream`; inputs as for kld_stats_run (device pointers).
 * result_dev: caller-owned DEVICE memory for one kld_result_t (8-byte
 * aligned), written asynchronously; its flags_or / device_error fields carry
 * what kld_stats_result() would report as status. 1 <= N <=
 * KLD_STATIC_MAX_ROWS, else KLD_ERR_CAPACITY (nothing enqueued).
 *
 * The first call on a device (with it current) looks up the array's device
 * address and sets kernel attributes; make that first call before any stream
 * capture. All calls share the one array and each overwrites the previous
 * call's records, so calls whose GPU work overlaps (other streams or threads)
 * race: order them.
 */
#define KLD_STATIC_MAX_ROWS 65536
kld_status_t kld_stats_run_static(const void* base, const void* quant,
                                  const int32_t* token_ids, int64_t N,
                                  int64_t V, kld_dtype_t dtype,
                                  kld_result_t* result_dev, void* stream);

/* ======================================================================
 * Diagnostics. None of these computes anything the pages define: they
 * expose timing, launch shape and self-checks of this library, for
 * benchmarks and tests. A caller of the statistic needs none of them.
 * ====================================================================== */

/*
 * Self-test of failure detection (no counterpart on the source pages; a
 * diagnostic of this library). Every device wait of the kernels is bounded:
 * this runs one small kernel on `device` whose warp waits on an mbarrier
 * that nothing ever completes, with a limit of limit_ns nanoseconds (1e3 ..
 * 1e10) -- or, with use_abort, until a second warp raises the kernel's abort
 * flag after ~1 ms -- and reports what the kernels report: KLD_ERR_TIMEOUT
 * when the wait gave up (the expected outcome), with the time waited in
 * *waited_ns. The context stays usable afterwards. Synchronous.
 */
kld_status_t kld_selftest_bounded_wait(int device, uint64_t limit_ns, int use_abort,
                                       uint64_t* waited_ns);

/*
 * Duration in milliseconds of the second pass of the last
 * kld_stats_run_grad (the gradient pass) or kld_stats_run_topk (the top-k
 * pass that follows the reduction, plus the threshold kernel before the row
 * pass when there is one); timing enabled by kld_stats_set_timing; waits for
 * that run. KLD_ERR_NOT_READY when the last run had no such pass or was not
 * timed.
 */
kld_status_t kld_stats_second_pass_timing(kld_stats_t h, float* pass_ms);

/*
 * Rows of the last kld_stats_run_topk that took the exact path (a radix
 * selection that reads the base row 2-4 times) instead of the threshold's
 * fast path: large tie groups at the threshold, masked rows, or a scanned
 * row whose flagged chunks overflowed the scan's lists (rows of more than
 * 512 * 16 * 64 elements only). Waits for that run. KLD_ERR_NOT_READY if
 * the handle has run no top-k yet.
 */
kld_status_t kld_stats_topk_exact_rows(kld_stats_t h, int64_t* rows);

/*
 * Read-bandwidth probe, a measuring aid with no counterpart in the
 * statistic: streams `bytes` of each of the device buffers a and b from HBM
 * into shared memory with the row pass's bulk copies (32 KB tiles, one CTA
 * per SM, nothing computed), so that the time the caller measures around it
 * (CUDA events on `stream`) gives the read-only bandwidth the row pass can
 * reach on this device. a and b: 16-byte aligned; bytes: a positive
 * multiple of 16; otherwise KLD_ERR_INVALID_ARG and nothing is enqueued.
 * Asynchronous on `stream`. A bounded wait that gives up sets the handle's
 * device error word, which the next kld_stats_result reports
 * (KLD_ERR_TIMEOUT).
 */
kld_status_t kld_stats_read_probe(kld_stats_t h, const void* a, const void* b, int64_t bytes,
                                  void* stream);

/*
 * Kernel timing of the next runs: when enabled, kld_stats_run (and
 * kld_stats_run_grad, kld_stats_run_topk) records CUDA events around its row
 * pass and its reduction; kld_stats_timing() returns the last run's
 * durations in milliseconds (waits for that run). A kld_stats_run_rows
 * followed by kld_stats_reduce on the same stream is timed the same way:
 * row_pass_ms covers the row pass, reduce_ms everything enqueued between
 * the end of the row pass and the end of the reduction (in a row-sharded
 * run, the record gather too). For a run whose row pass reduced its own
 * records (few split rows, see kld_stats_run) the row-pass time includes
 * the reduction and reduce_ms is about zero.
 */
kld_status_t kld_stats_set_timing(kld_stats_t h, int enable);
kld_status_t kld_stats_timing(kld_stats_t h, float* row_pass_ms,
                              float* reduce_ms);

/*
 * Launch plan of the row pass for (N, V, dtype) on a device with sm_count
 * SMs, for the default split setting (kld_stats_set_split). One persistent
 * CTA per SM takes whole rows round robin (rows r, r + grid, ...) for
 * whole_rounds rounds; the tail_rows rows that would leave most SMs idle in
 * a last partial wave (all N rows when N < sm_count) are instead split over
 * tail_ctas CTAs, each taking a balanced, contiguous range of the tail's
 * 512-element chunks (at most two rows' worth); a row's parts meet through a
 * small global scratch and a per-row arrival counter. variant: 0 = whole
 * rows only, 1 = few rows split over thread-block clusters (only when asked
 * for with kld_stats_set_split), 2 = whole rounds plus a split tail.
 * ctas_per_row: the most CTAs any row is split over. Also: threads per CTA,
 * dynamic shared memory bytes, stage bytes per operand, stages. Pure host
 * logic; enqueues nothing.
 */
typedef struct {
  int32_t variant;
  int32_t grid;
  int32_t ctas_per_row;
  int32_t threads;
  int32_t smem_bytes;
  int32_t stage_bytes;
  int32_t stages;
  int32_t cluster_ctas;
  int32_t whole_rounds;
  int32_t tail_rows;
  int32_t tail_ctas;
  int32_t reserved;
} kld_plan_t;

kld_status_t kld_plan(int64_t N, int64_t V, kld_dtype_t dtype, int sm_count,
                      kld_plan_t* out);

#ifdef __cplusplus
}
#endif
#endif /* KLD_STATS_H */
