/*
 * kld_oracle.cpp -- plain, slow fp64 CPU oracle (two passes per row).
 *
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).
 * No code here is shared with, or called by, the CUDA library.
 *
 * Every step follows the textbook definitions, in the order the quantities
 * are defined, with no fusion or streaming:
 *   "Qwen3.6 27B Quantization Benchmark", section "Understand KLD and Same
 *   Top P": KLD measures how far the quantized model's next-token
 *   distribution drifts from the base model's over the whole vocabulary;
 *   Same Top P is how often both models pick the same top token.
 *   Same page, "Raw benchmark data" table: Mean KLD, Same top p (%) and Mean
 *   PPL(Q), the perplexity of the quantized model on the evaluated text.
 *   "Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S GGUF", "How it was made", step 5:
 *   the divergence is KL(BF16 || quantized) over the full vocabulary.
 *
 * Readings where the pages are silent (each one is also listed with the
 * design notes of the repository):
 *   - natural logarithm (nats);
 *   - argmax ties go to the lowest index;
 *   - a row holding a NaN or +inf is flagged NONFINITE and excluded;
 *   - a row whose entries are all -inf is flagged EMPTY and excluded;
 *   - a vocabulary entry with b_j = -inf has P_base = 0 and adds nothing;
 *     b_j finite with q_j = -inf makes the KL +inf (flag INF_KL, kept);
 *   - percentiles use linear interpolation between order statistics,
 *     pos = p*(n-1) (the "type 7" rule); max is the largest order statistic;
 *   - means run over the valid rows; PPL = exp(mean NLL);
 *   - the base model's NLL of the same token (NLLB) gives PPL(base) and the
 *     perplexity ratio ("Mistral-Small-4-119B-2603 GSQ-RCO IQ3_S GGUF",
 *     "Quality"); dp = P_quant(tok) - P_base(tok), averaged and as a root
 *     mean square over the rows with a token (the Qwen3.6 table's "RMS dp
 *     (%)" column, the same card's points of probability); b[tok] = -inf
 *     makes NLLB +inf (flag INF_NLLB) and P_base(tok) = 0.
 */
#include "kld_oracle.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

/* bf16 is the top half of an IEEE binary32: widening is exact. */
double widen_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

/* IEEE binary16 -> double, decoded field by field (exact). */
double widen_f16(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0x1f) {
    v = m ? std::numeric_limits<double>::quiet_NaN()
          : std::numeric_limits<double>::infinity();
  } else if (e == 0) {
    v = std::ldexp((double)m, -24); /* subnormal: m * 2^-24 */
  } else {
    v = std::ldexp((double)(m + 1024), e - 25); /* (1 + m/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

/* Row r of a [N, V] tensor, widened exactly to double. */
void load_row(const void* t, int dtype, int64_t r, int64_t V, double* out) {
  if (dtype == ORACLE_F32) {
    const float* p = (const float*)t + r * V;
    for (int64_t j = 0; j < V; ++j) out[j] = (double)p[j];
  } else if (dtype == ORACLE_BF16) {
    const uint16_t* p = (const uint16_t*)t + r * V;
    for (int64_t j = 0; j < V; ++j) out[j] = widen_bf16(p[j]);
  } else {
    const uint16_t* p = (const uint16_t*)t + r * V;
    for (int64_t j = 0; j < V; ++j) out[j] = widen_f16(p[j]);
  }
}

const double kNaN = std::numeric_limits<double>::quiet_NaN();
const double kInf = std::numeric_limits<double>::infinity();

/* Statistics of one row pair, by the definitions, two passes per row. */
void one_row(const double* b, const double* q, int64_t V, int has_tok,
             int32_t tok, double* kld, double* nll, double* nllb, int32_t* ab,
             int32_t* aq, uint32_t* flags) {
  uint32_t f = 0;
  *kld = kNaN;
  *nll = kNaN;
  *nllb = kNaN;
  *ab = -1;
  *aq = -1;

  /* Inputs that are NaN or +inf make the distribution undefined. */
  for (int64_t j = 0; j < V; ++j) {
    if (std::isnan(b[j]) || std::isnan(q[j]) || b[j] == kInf || q[j] == kInf) {
      f |= ORACLE_ROW_NONFINITE;
      break;
    }
  }
  if (f) {
    if (has_tok && (tok < 0 || (int64_t)tok >= V)) f |= ORACLE_ROW_BAD_TOKEN;
    *flags = f;
    return;
  }

  /* Step 1: row maxima. */
  double m_b = -kInf, m_q = -kInf;
  for (int64_t j = 0; j < V; ++j) {
    if (b[j] > m_b) m_b = b[j];
    if (q[j] > m_q) m_q = q[j];
  }
  if (m_b == -kInf || m_q == -kInf) {
    f |= ORACLE_ROW_EMPTY;
    if (has_tok && (tok < 0 || (int64_t)tok >= V)) f |= ORACLE_ROW_BAD_TOKEN;
    *flags = f;
    return;
  }

  /* Step 2: argmax = the smallest index holding the maximum. */
  int32_t amax_b = -1, amax_q = -1;
  for (int64_t j = 0; j < V; ++j) {
    if (amax_b < 0 && b[j] == m_b) amax_b = (int32_t)j;
    if (amax_q < 0 && q[j] == m_q) amax_q = (int32_t)j;
  }

  /* Step 3: log-sum-exp of each row, plain left-to-right sums. */
  double s_b = 0.0, s_q = 0.0;
  for (int64_t j = 0; j < V; ++j) s_b += std::exp(b[j] - m_b);
  for (int64_t j = 0; j < V; ++j) s_q += std::exp(q[j] - m_q);
  const double lse_b = m_b + std::log(s_b);
  const double lse_q = m_q + std::log(s_q);

  /* Steps 4-5: KL = sum_j p_j * (log p_j - log r_j) over entries with
   * p_j > 0, i.e. b_j > -inf. log p_j = b_j - lse_b, log r_j = q_j - lse_q. */
  double kl = 0.0;
  bool inf_kl = false;
  for (int64_t j = 0; j < V; ++j) {
    if (b[j] == -kInf) continue;
    if (q[j] == -kInf) {
      inf_kl = true;
      continue;
    }
    const double logp = b[j] - lse_b;
    const double logr = q[j] - lse_q;
    kl += std::exp(logp) * (logp - logr);
  }
  if (inf_kl) {
    kl = kInf;
    f |= ORACLE_ROW_INF_KL;
  }

  /* Step 6: NLL of the given next token under the quantized row, and under
   * the base row. */
  if (has_tok) {
    if (tok < 0 || (int64_t)tok >= V) {
      f |= ORACLE_ROW_BAD_TOKEN;
    } else {
      if (q[tok] == -kInf) {
        *nll = kInf;
        f |= ORACLE_ROW_INF_NLL;
      } else {
        *nll = lse_q - q[tok];
      }
      if (b[tok] == -kInf) {
        *nllb = kInf;
        f |= ORACLE_ROW_INF_NLLB;
      } else {
        *nllb = lse_b - b[tok];
      }
    }
  }

  *kld = kl;
  *ab = amax_b;
  *aq = amax_q;
  *flags = f;
}

void rows_range(const void* base, const void* quant, const int32_t* tok,
                int64_t r0, int64_t r1, int64_t V, int dtype, double* kld,
                double* nll, double* nllb, int32_t* ab, int32_t* aq,
                uint32_t* flags) {
  std::vector<double> b((size_t)V), q((size_t)V);
  for (int64_t r = r0; r < r1; ++r) {
    load_row(base, dtype, r, V, b.data());
    load_row(quant, dtype, r, V, q.data());
    one_row(b.data(), q.data(), V, tok != nullptr, tok ? tok[r] : 0, &kld[r],
            &nll[r], &nllb[r], &ab[r], &aq[r], &flags[r]);
  }
}

}  // namespace

extern "C" int oracle_rows(const void* base, const void* quant,
                           const int32_t* tok, int64_t N, int64_t V, int dtype,
                           double* kld, double* nll, double* nll_base,
                           int32_t* amax_b, int32_t* amax_q, uint32_t* flags,
                           int nthreads) {
  if (!base || !quant || !kld || !nll || !nll_base || !amax_b || !amax_q ||
      !flags)
    return -1;
  if (N < 0 || V < 1 || V > 0x7fffffffLL) return -1;
  if (dtype != ORACLE_F32 && dtype != ORACLE_BF16 && dtype != ORACLE_F16)
    return -1;
  if (nthreads <= 1 || N < 2) {
    rows_range(base, quant, tok, 0, N, V, dtype, kld, nll, nll_base, amax_b,
               amax_q, flags);
    return 0;
  }
  /* Whole rows per thread: every row is computed by the same code in the same
   * order as the single-threaded run. */
  int64_t T = std::min<int64_t>(nthreads, N);
  std::vector<std::thread> pool;
  for (int64_t t = 0; t < T; ++t) {
    int64_t r0 = N * t / T, r1 = N * (t + 1) / T;
    pool.emplace_back(rows_range, base, quant, tok, r0, r1, V, dtype, kld, nll,
                      nll_base, amax_b, amax_q, flags);
  }
  for (auto& th : pool) th.join();
  return 0;
}

extern "C" int oracle_grad(const void* base, const void* quant, int64_t N,
                           int64_t V, int dtype, double scale, double* grad) {
  if (!base || !quant || !grad || N < 0 || V < 1 || V > 0x7fffffffLL) return -1;
  if (dtype != ORACLE_F32 && dtype != ORACLE_BF16 && dtype != ORACLE_F16)
    return -1;
  std::vector<double> b((size_t)V), q((size_t)V);
  for (int64_t r = 0; r < N; ++r) {
    load_row(base, dtype, r, V, b.data());
    load_row(quant, dtype, r, V, q.data());
    double* g = grad + r * V;
    /* Excluded rows (NaN/+inf anywhere, or a row of -inf) add nothing to
     * the mean over valid rows, so their gradient is zero. */
    bool excluded = false;
    double m_b = -kInf, m_q = -kInf;
    for (int64_t j = 0; j < V; ++j) {
      if (std::isnan(b[j]) || std::isnan(q[j]) || b[j] == kInf || q[j] == kInf)
        excluded = true;
      if (b[j] > m_b) m_b = b[j];
      if (q[j] > m_q) m_q = q[j];
    }
    if (excluded || m_b == -kInf || m_q == -kInf) {
      for (int64_t j = 0; j < V; ++j) g[j] = 0.0;
      continue;
    }
    /* log-sum-exp of both rows, plain left-to-right sums */
    double zb = 0.0, zq = 0.0;
    for (int64_t j = 0; j < V; ++j) zb += std::exp(b[j] - m_b);
    for (int64_t j = 0; j < V; ++j) zq += std::exp(q[j] - m_q);
    const double lse_b = m_b + std::log(zb);
    const double lse_q = m_q + std::log(zq);
    for (int64_t j = 0; j < V; ++j)
      g[j] = scale * (std::exp(q[j] - lse_q) - std::exp(b[j] - lse_b));
  }
  return 0;
}

extern "C" int oracle_topk(const void* base, const void* quant, int64_t N,
                           int64_t V, int dtype, int k, int32_t* idx,
                           double* logp, double* rest, double* kl_topk) {
  if (!base || !quant || !idx || !logp || !rest || !kl_topk) return -1;
  if (N < 0 || V < 1 || V > 0x7fffffffLL || k < 1) return -1;
  if (dtype != ORACLE_F32 && dtype != ORACLE_BF16 && dtype != ORACLE_F16)
    return -1;
  std::vector<double> b((size_t)V), q((size_t)V);
  std::vector<int64_t> order((size_t)V);
  std::vector<char> in_top((size_t)V);
  for (int64_t r = 0; r < N; ++r) {
    load_row(base, dtype, r, V, b.data());
    load_row(quant, dtype, r, V, q.data());
    int32_t* id = idx + r * k;
    double* lp = logp + r * k;
    /* Excluded rows, as for the statistics. */
    bool excluded = false;
    double m_b = -kInf, m_q = -kInf;
    for (int64_t j = 0; j < V; ++j) {
      if (std::isnan(b[j]) || std::isnan(q[j]) || b[j] == kInf || q[j] == kInf)
        excluded = true;
      if (b[j] > m_b) m_b = b[j];
      if (q[j] > m_q) m_q = q[j];
    }
    if (excluded || m_b == -kInf || m_q == -kInf) {
      for (int i = 0; i < k; ++i) {
        id[i] = -1;
        lp[i] = kNaN;
      }
      rest[r] = kNaN;
      kl_topk[r] = kNaN;
      continue;
    }
    /* The k largest base logits, ties to the lowest index: a stable sort of
     * the indices by descending logit. */
    for (int64_t j = 0; j < V; ++j) order[(size_t)j] = j;
    std::stable_sort(order.begin(), order.end(),
                     [&](int64_t x, int64_t y) { return b[x] > b[y]; });
    const int64_t kt = std::min<int64_t>(k, V);
    std::fill(in_top.begin(), in_top.end(), 0);
    for (int64_t i = 0; i < kt; ++i) in_top[(size_t)order[(size_t)i]] = 1;
    /* Both distributions over the full row. */
    double zb = 0.0, zq = 0.0;
    for (int64_t j = 0; j < V; ++j) zb += std::exp(b[j] - m_b);
    for (int64_t j = 0; j < V; ++j) zq += std::exp(q[j] - m_q);
    const double lse_b = m_b + std::log(zb);
    const double lse_q = m_q + std::log(zq);
    double kl = 0.0, p_rest = 0.0, r_rest = 0.0;
    bool inf_kl = false;
    for (int64_t i = 0; i < k; ++i) {
      if (i >= kt) {
        id[i] = -1;
        lp[i] = -kInf;
        continue;
      }
      const int64_t j = order[(size_t)i];
      id[i] = (int32_t)j;
      lp[i] = b[j] - lse_b;
      if (b[j] == -kInf) continue; /* p_j = 0 adds nothing */
      if (q[j] == -kInf) {
        inf_kl = true;
        continue;
      }
      const double logp_j = b[j] - lse_b, logr_j = q[j] - lse_q;
      kl += std::exp(logp_j) * (logp_j - logr_j);
    }
    for (int64_t j = 0; j < V; ++j) {
      if (in_top[(size_t)j]) continue;
      p_rest += std::exp(b[j] - lse_b);
      r_rest += std::exp(q[j] - lse_q);
    }
    if (p_rest > 0.0) {
      if (r_rest > 0.0)
        kl += p_rest * (std::log(p_rest) - std::log(r_rest));
      else
        inf_kl = true;
    }
    rest[r] = p_rest > 0.0 ? std::log(p_rest) : -kInf;
    kl_topk[r] = inf_kl ? kInf : kl;
  }
  return 0;
}

extern "C" double oracle_percentile_sorted(const double* x, int64_t n,
                                           double p) {
  if (n <= 0) return kNaN;
  const double pos = p * (double)(n - 1);
  int64_t k = (int64_t)std::floor(pos);
  if (k < 0) k = 0;
  if (k >= n - 1) return x[n - 1];
  const double frac = pos - (double)k;
  const double lo = x[k], hi = x[k + 1];
  if (frac == 0.0 || lo == hi) return lo;
  return lo + frac * (hi - lo);
}

extern "C" int oracle_reduce(const double* kld, const double* nll,
                             const double* nll_base, const int32_t* amax_b,
                             const int32_t* amax_q, const uint32_t* flags,
                             int64_t N, int has_nll, oracle_result_t* out) {
  if (!kld || !amax_b || !amax_q || !flags || !out || N < 0) return -1;
  if (has_nll && (!nll || !nll_base)) return -1;
  std::memset(out, 0, sizeof(*out));
  out->n_rows = N;
  out->has_nll = has_nll ? 1 : 0;

  std::vector<double> valid;
  valid.reserve((size_t)N);
  double sum_kl = 0.0, sum_nll = 0.0, sum_nllb = 0.0, sum_dp = 0.0, sum_dp2 = 0.0;
  int64_t agree = 0, n_nll = 0, n_flagged = 0;
  uint32_t f_or = 0;
  for (int64_t i = 0; i < N; ++i) {
    const uint32_t f = flags[i];
    f_or |= f;
    if (f) ++n_flagged;
    if (f & (ORACLE_ROW_NONFINITE | ORACLE_ROW_EMPTY)) continue;
    valid.push_back(kld[i]);
    sum_kl += kld[i];
    if (amax_b[i] == amax_q[i]) ++agree;
    if (has_nll && !(f & ORACLE_ROW_BAD_TOKEN)) {
      sum_nll += nll[i];
      sum_nllb += nll_base[i];
      /* P(tok) = exp(-NLL) for each model; exp(-inf) = 0. */
      const double dp = std::exp(-nll[i]) - std::exp(-nll_base[i]);
      sum_dp += dp;
      sum_dp2 += dp * dp;
      ++n_nll;
    }
  }
  const int64_t n = (int64_t)valid.size();
  out->n_valid = n;
  out->n_flagged = n_flagged;
  out->flags_or = f_or;
  out->top1_agree = agree;
  if (n > 0) {
    std::sort(valid.begin(), valid.end());
    out->mean_kld = sum_kl / (double)n;
    out->median_kld = oracle_percentile_sorted(valid.data(), n, 0.5);
    out->p90_kld = oracle_percentile_sorted(valid.data(), n, 0.9);
    out->p99_kld = oracle_percentile_sorted(valid.data(), n, 0.99);
    out->max_kld = valid[(size_t)n - 1];
    out->top1_agree_pct = 100.0 * (double)agree / (double)n;
  } else {
    out->mean_kld = out->median_kld = out->p90_kld = out->p99_kld =
        out->max_kld = out->top1_agree_pct = kNaN;
  }
  out->n_nll = n_nll;
  if (has_nll && n_nll > 0) {
    out->mean_nll = sum_nll / (double)n_nll;
    out->ppl = std::exp(out->mean_nll);
    out->mean_nll_base = sum_nllb / (double)n_nll;
    out->ppl_base = std::exp(out->mean_nll_base);
    out->ln_ppl_ratio = out->mean_nll - out->mean_nll_base;
    out->mean_dp = sum_dp / (double)n_nll;
    out->rms_dp = std::sqrt(sum_dp2 / (double)n_nll);
  } else {
    out->mean_nll = out->ppl = kNaN;
    out->mean_nll_base = out->ppl_base = out->ln_ppl_ratio = kNaN;
    out->mean_dp = out->rms_dp = kNaN;
  }
  return 0;
}
