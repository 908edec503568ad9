/*
 * kld_oracle.h -- plain fp64 CPU oracle for the logit KL-divergence statistic.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library includes, links or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do. It shares no header, constant or helper with the CUDA path.
 *
 * What it computes (per row i of two [N, V] logit tensors, base b and quant q):
 *   - log-softmax of both rows over the full vocabulary,
 *   - KL(P_base || P_quant) in nats,
 *   - argmax of each row, lowest index on ties ("Same Top P"),
 *   - optionally NLL_i = -log P_quant(tok_i) and NLLB_i = -log P_base(tok_i),
 * and over all rows: mean / median / p90 / p99 / max KLD, top-1 agreement
 * count and percentage, mean NLL and PPL = exp(mean NLL), the same for the
 * base row (PPL(base)), ln(PPL(Q)/PPL(base)) = mean NLL - mean NLLB, and the
 * token-probability shift dp_i = P_quant(tok_i) - P_base(tok_i): its mean
 * and its root mean square ("RMS dp").
 *
 * Sources:
 *   "Qwen3.6 27B Quantization Benchmark" (huy.rocks), sections "Measurement
 *     method", "Understand KLD and Same Top P" and the "Raw benchmark data"
 *     table (columns Mean PPL(Q), Mean KLD, Same top p).
 *   "Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S GGUF" model card, "Quality" and
 *     "How it was made" steps 5 and 7: the direction is KL(BF16 || quantized)
 *     over the full vocabulary. Its "Quality" section also reads the
 *     perplexity ratio and how many points of probability the quantized
 *     model gives the correct token less than BF16 on average (mean dp);
 *     the Qwen3.6 page's table has the "RMS dp (%)" column.
 *   Percentiles (median/p90/p99) are not printed on any page; they follow the
 *   linear-interpolation ("type 7") order-statistic rule stated below.
 */
#ifndef KLD_ORACLE_H
#define KLD_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of the logit tensors. */
enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_F16 = 2 };

/* Per-row flag bits (same meaning and values as the product library states). */
enum {
  ORACLE_ROW_NONFINITE = 1u << 0, /* a NaN or +inf in either row: row excluded */
  ORACLE_ROW_EMPTY     = 1u << 1, /* every entry of a row is -inf: row excluded */
  ORACLE_ROW_INF_KL    = 1u << 2, /* b_j finite where q_j = -inf: KL = +inf   */
  ORACLE_ROW_BAD_TOKEN = 1u << 3, /* token id outside [0, V): no NLL for row  */
  ORACLE_ROW_INF_NLL   = 1u << 4, /* q[tok] = -inf: NLL = +inf                 */
  ORACLE_ROW_INF_NLLB  = 1u << 5  /* b[tok] = -inf: NLLB = +inf                */
};

typedef struct {
  int64_t n_rows;     /* rows given                                         */
  int64_t n_valid;    /* rows without NONFINITE / EMPTY                     */
  double mean_kld;    /* left-to-right sum over valid rows / n_valid        */
  double median_kld;  /* type-7 percentiles of the valid KL values          */
  double p90_kld;
  double p99_kld;
  double max_kld;
  int64_t top1_agree; /* valid rows with argmax_base == argmax_quant        */
  double top1_agree_pct;
  int32_t has_nll;
  int32_t _pad;
  int64_t n_nll;      /* valid rows with an in-range token id               */
  double mean_nll;
  double ppl;
  int64_t n_flagged;  /* rows with any flag set                             */
  uint32_t flags_or;  /* OR of all row flags                                */
  uint32_t _pad2;
  /* over the same rows as mean_nll (NaN without token ids): */
  double mean_nll_base; /* mean of NLLB                                     */
  double ppl_base;      /* exp(mean_nll_base)                               */
  double ln_ppl_ratio;  /* mean_nll - mean_nll_base = ln(PPL(Q)/PPL(base))  */
  double mean_dp;       /* mean of dp = exp(-NLL) - exp(-NLLB)              */
  double rms_dp;        /* sqrt(mean of dp^2)                               */
} oracle_result_t;

/* Per-row statistics of rows [0, N). `tok` may be NULL (no NLL). Rows are
 * independent; nthreads > 1 spreads whole rows over std::threads, which
 * leaves every per-row value bit-identical. Returns 0, or -1 on bad args. */
int oracle_rows(const void* base, const void* quant, const int32_t* tok,
                int64_t N, int64_t V, int dtype, double* kld, double* nll,
                double* nll_base, int32_t* amax_b, int32_t* amax_q,
                uint32_t* flags, int nthreads);

/* Reduction of per-row values to the summary statistics. */
int oracle_reduce(const double* kld, const double* nll, const double* nll_base,
                  const int32_t* amax_b, const int32_t* amax_q,
                  const uint32_t* flags, int64_t N, int has_nll,
                  oracle_result_t* out);

/* Gradient of KL(P_base || P_quant) with respect to the quant logits, per
 * row i and entry j: grad[i][j] = scale * (P_quant_j - P_base_j), i.e.
 * softmax(q_i) - softmax(b_i) (the objective minimised in
 * "Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S GGUF", "How it was made", step 7).
 * Rows that are NONFINITE or EMPTY (excluded from the statistics) get zeros.
 * Returns 0, or -1 on bad args. */
int oracle_grad(const void* base, const void* quant, int64_t N, int64_t V,
                int dtype, double scale, double* grad);

/* Top-k compression of the base row and the KL against it ("Mistral-Small-
 * 4-119B-2603 GSQ-RCO IQ3_S GGUF", "How it was made", step 7: tuning
 * "against the top-128 distributions (and the rest of the mass)"). Per row:
 * T = the k entries with the largest base logits (ties: lowest index
 * first), listed in that order in idx[r*k ..] with log P_base in
 * logp[r*k ..] (entries past V: index -1, logp -inf); rest[r] =
 * log(sum of P_base outside T) (-inf when T holds everything), and
 *   kl_topk[r] = sum_{j in T} p_j log(p_j / r_j) + p_rest log(p_rest / r_rest),
 * with p = softmax(b), r = softmax(q), p_rest = sum_{j not in T} p_j,
 * r_rest likewise (a term with p = 0 is 0; p > 0 with r = 0 is +inf).
 * Excluded rows (NONFINITE / EMPTY): idx -1, logp and rest NaN, kl NaN.
 * Returns 0, or -1 on bad args. */
int oracle_topk(const void* base, const void* quant, int64_t N, int64_t V,
                int dtype, int k, int32_t* idx, double* logp, double* rest,
                double* kl_topk);

/* Type-7 percentile of an ascending array x[0..n): pos = p*(n-1). */
double oracle_percentile_sorted(const double* x, int64_t n, double p);

#ifdef __cplusplus
}
#endif
#endif /* KLD_ORACLE_H */
