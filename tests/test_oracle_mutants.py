"""The oracle's pins must catch plausible mistakes.

Each case compiles a copy of the oracle with one planted mistake (on the CPU,
into a temporary directory) and runs the pin suite against it through
``KLD_ORACLE_LIB``; the suite has to fail for every mutant.
"""
import os
import subprocess
import sys
import tempfile

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "kld_oracle.cpp")

MUTANTS = {
    "kl_direction_swapped": ("kl += std::exp(logp) * (logp - logr);",
                             "kl += std::exp(logr) * (logr - logp);"),
    "kl_sign_flipped": ("kl += std::exp(logp) * (logp - logr);",
                        "kl += std::exp(logp) * (logr - logp);"),
    "log_softmax_drops_normaliser": ("const double logp = b[j] - lse_b;",
                                     "const double logp = b[j] - m_b;"),
    "quant_normaliser_from_base": ("const double logr = q[j] - lse_q;",
                                   "const double logr = q[j] - lse_b;"),
    "last_vocab_entry_dropped": ("for (int64_t j = 0; j < V; ++j) s_b += std::exp(b[j] - m_b);",
                                 "for (int64_t j = 0; j + 1 < V; ++j) s_b += std::exp(b[j] - m_b);"),
    "argmax_ties_to_highest": ("if (amax_b < 0 && b[j] == m_b) amax_b = (int32_t)j;",
                               "if (b[j] == m_b) amax_b = (int32_t)j;"),
    "percentile_position_off": ("const double pos = p * (double)(n - 1);",
                                "const double pos = p * (double)n;"),
    "nll_sign_flipped": ("*nll = lse_q - q[tok];", "*nll = q[tok] - lse_q;"),
    "nll_under_base_row": ("*nll = lse_q - q[tok];", "*nll = lse_b - b[tok];"),
    "excluded_rows_enter_mean": ("if (f & (ORACLE_ROW_NONFINITE | ORACLE_ROW_EMPTY)) continue;",
                                 "if (f & ORACLE_ROW_NONFINITE) continue;"),
    "masked_quant_entry_ignored": ("      inf_kl = true;\n      continue;", "      continue;"),
    "bf16_widening_wrong": ("uint32_t u = (uint32_t)h << 16;", "uint32_t u = (uint32_t)h << 15;"),
    "agreement_counts_all_rows": ("if (amax_b[i] == amax_q[i]) ++agree;", "++agree;"),
    "base_nll_under_quant_row": ("*nllb = lse_b - b[tok];", "*nllb = lse_q - q[tok];"),
    "base_nll_without_normaliser": ("*nllb = lse_b - b[tok];", "*nllb = m_b - b[tok];"),
    "dp_sign_flipped": ("const double dp = std::exp(-nll[i]) - std::exp(-nll_base[i]);",
                        "const double dp = std::exp(-nll_base[i]) - std::exp(-nll[i]);"),
    "rms_dp_without_root": ("out->rms_dp = std::sqrt(sum_dp2 / (double)n_nll);",
                            "out->rms_dp = sum_dp2 / (double)n_nll;"),
    "grad_sign_flipped": ("g[j] = scale * (std::exp(q[j] - lse_q) - std::exp(b[j] - lse_b));",
                          "g[j] = scale * (std::exp(b[j] - lse_b) - std::exp(q[j] - lse_q));"),
    "grad_quant_normaliser_from_base": ("g[j] = scale * (std::exp(q[j] - lse_q) - std::exp(b[j] - lse_b));",
                                        "g[j] = scale * (std::exp(q[j] - lse_b) - std::exp(b[j] - lse_b));"),
    "topk_selected_by_quant": ("[&](int64_t x, int64_t y) { return b[x] > b[y]; });",
                               "[&](int64_t x, int64_t y) { return q[x] > q[y]; });"),
    "topk_rest_term_dropped": ("kl += p_rest * (std::log(p_rest) - std::log(r_rest));",
                               "kl += 0.0 * (std::log(p_rest) - std::log(r_rest));"),
    "topk_rest_from_quant_side": ("      p_rest += std::exp(b[j] - lse_b);",
                                  "      p_rest += std::exp(q[j] - lse_q);"),
    "ppl_ratio_inverted": ("out->ln_ppl_ratio = out->mean_nll - out->mean_nll_base;",
                           "out->ln_ppl_ratio = out->mean_nll_base - out->mean_nll;"),
    "kl_in_bits": ("kl += std::exp(logp) * (logp - logr);",
                   "kl += std::exp(logp) * (logp - logr) / std::log(2.0);"),
    "lse_without_the_maximum": ("const double lse_b = m_b + std::log(s_b);",
                                "const double lse_b = std::log(s_b);"),
    "mean_kld_over_all_rows": ("out->mean_kld = sum_kl / (double)n;",
                               "out->mean_kld = sum_kl / (double)N;"),
    "agreement_pct_over_all_rows": ("out->top1_agree_pct = 100.0 * (double)agree / (double)n;",
                                    "out->top1_agree_pct = 100.0 * (double)agree / (double)N;"),
    "ppl_in_base_two": ("out->ppl = std::exp(out->mean_nll);",
                        "out->ppl = std::exp2(out->mean_nll);"),
    "percentile_takes_the_upper_neighbour": ("return lo + frac * (hi - lo);", "return hi;"),
    "topk_ties_to_highest_index": ("for (int64_t j = 0; j < V; ++j) order[(size_t)j] = j;",
                                   "for (int64_t j = 0; j < V; ++j) order[(size_t)j] = V - 1 - j;"),
    "plus_inf_treated_as_finite": (
        "if (std::isnan(b[j]) || std::isnan(q[j]) || b[j] == kInf || q[j] == kInf) {",
        "if (std::isnan(b[j]) || std::isnan(q[j])) {"),
    "empty_quant_row_not_excluded": ("if (m_b == -kInf || m_q == -kInf) {", "if (m_b == -kInf) {"),
    "masked_token_not_flagged": ("        f |= ORACLE_ROW_INF_NLL;\n", ""),
    "grad_scale_dropped": ("g[j] = scale * (std::exp(q[j] - lse_q) - std::exp(b[j] - lse_b));",
                           "g[j] = (std::exp(q[j] - lse_q) - std::exp(b[j] - lse_b));"),
}


@pytest.fixture(scope="module")
def mutant_dir():
    with tempfile.TemporaryDirectory() as d:
        yield d


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, mutant_dir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not unique/present: {name}"
    msrc = os.path.join(mutant_dir, f"{name}.cpp")
    with open(msrc, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(mutant_dir, f"{name}.so")
    subprocess.run(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                    "-I", os.path.join(ROOT, "oracle"), "-o", lib, msrc], check=True)
    env = dict(os.environ, KLD_ORACLE_LIB=lib)
    proc = subprocess.run(
        [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
         os.path.join(ROOT, "tests", "test_oracle_pins.py")],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert proc.returncode != 0, f"pins did not catch mutant {name}:\n{proc.stdout[-2000:]}"


def test_unmutated_oracle_passes_the_same_way():
    oracle.build()
    proc = subprocess.run(
        [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
         os.path.join(ROOT, "tests", "test_oracle_pins.py")],
        cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert proc.returncode == 0, proc.stdout[-2000:]
