"""Pins of the fp64 CPU oracle against facts that do not come from the oracle.

Each check uses something independent of the oracle's code path: a closed
form, an invariant of KL divergence, a brute-force evaluation of the textbook
formula sum p*log(p/r) in Python (no max subtraction, no log-softmax), the
worked example printed in "Qwen3.6 27B Quantization Benchmark" (section
"Understand KLD and Same Top P"), or a library routine (numpy argmax,
numpy.percentile, math.fsum, numpy's float16 widening).
"""
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(12345)
NEG_INF = np.float32(-np.inf)


def _run(b, q, tok=None, dtype=oracle.F32, nthreads=1):
    return oracle.run(b, q, tok, dtype, nthreads)


def _brute_kl(b_row, q_row):
    """sum_j p_j log(p_j / r_j) with p, r from exp(x) / sum exp(x) directly."""
    eb = [math.exp(float(x)) for x in b_row]
    eq = [math.exp(float(x)) for x in q_row]
    sb, sq = math.fsum(eb), math.fsum(eq)
    terms = []
    for x, y in zip(eb, eq):
        p, r = x / sb, y / sq
        if p > 0:
            terms.append(p * math.log(p / r))
    return math.fsum(terms)


# ---------------------------------------------------------------- KL basics

@pytest.mark.parametrize("V", [1, 2, 7, 33, 1000, 32000])
def test_kl_of_identical_rows_is_exactly_zero(V):
    b = RNG.normal(0, 2.5, size=(6, V)).astype(np.float32)
    r, res = _run(b, b.copy())
    assert np.all(r["kld"] == 0.0)
    assert np.array_equal(r["amax_b"], r["amax_q"])
    assert res["top1_agree"] == 6 and res["top1_agree_pct"] == 100.0
    assert res["mean_kld"] == 0.0 and res["max_kld"] == 0.0


def test_kl_is_nonnegative():
    b = RNG.normal(0, 2.5, size=(200, 257)).astype(np.float32)
    q = (b + RNG.normal(0, 0.5, size=b.shape)).astype(np.float32)
    r, _ = _run(b, q)
    assert np.all(r["kld"] >= 0.0)
    assert np.all(r["kld"] > 0.0)  # noise makes every row differ


@pytest.mark.parametrize("shift_b,shift_q", [(4.0, 0.0), (0.0, -8.0), (2.0, 512.0)])
def test_kl_invariant_to_adding_a_constant(shift_b, shift_q):
    # values on a 2^-10 grid with |x| < 2^12: adding these constants is exact
    b = (np.round(RNG.normal(0, 2.5, size=(8, 513)) * 1024) / 1024).astype(np.float32)
    q = (np.round((b + RNG.normal(0, 0.3, size=b.shape)) * 1024) / 1024).astype(np.float32)
    b2 = (b + np.float32(shift_b)).astype(np.float32)
    q2 = (q + np.float32(shift_q)).astype(np.float32)
    assert np.array_equal(b2.astype(np.float64) - shift_b, b.astype(np.float64))
    r1, _ = _run(b, q)
    r2, _ = _run(b2, q2)
    np.testing.assert_allclose(r2["kld"], r1["kld"], rtol=1e-11, atol=1e-13)
    assert np.array_equal(r1["amax_b"], r2["amax_b"])
    assert np.array_equal(r1["amax_q"], r2["amax_q"])


def test_kl_invariant_to_common_vocab_permutation():
    b = RNG.normal(0, 2.5, size=(10, 999)).astype(np.float32)
    q = (b + RNG.normal(0, 0.4, size=b.shape)).astype(np.float32)
    perm = RNG.permutation(999)
    r1, _ = _run(b, q)
    r2, _ = _run(np.ascontiguousarray(b[:, perm]), np.ascontiguousarray(q[:, perm]))
    np.testing.assert_allclose(r2["kld"], r1["kld"], rtol=1e-11, atol=1e-14)
    # argmax moves with the permutation (random data: no ties)
    assert np.array_equal(perm[r2["amax_b"]], r1["amax_b"])
    assert np.array_equal(perm[r2["amax_q"]], r1["amax_q"])


def test_kl_direction_is_base_first():
    # P = base, R = quant; swapping the operands changes the value
    b = np.array([[0.0, -1.0, -3.0]], np.float32)
    q = np.array([[-2.0, 0.5, 0.0]], np.float32)
    r_bq, _ = _run(b, q)
    r_qb, _ = _run(q, b)
    assert abs(r_bq["kld"][0] - _brute_kl(b[0], q[0])) < 1e-14
    assert abs(r_qb["kld"][0] - _brute_kl(q[0], b[0])) < 1e-14
    assert abs(r_bq["kld"][0] - r_qb["kld"][0]) > 1e-3


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("V", [1, 2, 5, 32000, 151936])
def test_one_hot_base_against_uniform_quant_is_log_V(V):
    hot = V // 3
    b = np.full((1, V), NEG_INF, np.float32)
    b[0, hot] = 1.25
    q = np.zeros((1, V), np.float32)
    r, _ = _run(b, q)
    assert abs(r["kld"][0] - math.log(V)) <= 1e-12 * max(1.0, math.log(V))
    assert r["amax_b"][0] == hot
    assert r["amax_q"][0] == 0  # all equal: lowest index wins
    assert r["flags"][0] == 0


def test_uniform_base_against_one_hot_quant_is_infinite():
    V = 16
    b = np.zeros((1, V), np.float32)
    q = np.full((1, V), NEG_INF, np.float32)
    q[0, 3] = 0.0
    r, res = _run(b, q)
    assert r["kld"][0] == math.inf
    assert r["flags"][0] == oracle.ROW_INF_KL
    assert res["n_valid"] == 1 and res["mean_kld"] == math.inf


@pytest.mark.parametrize("b0,b1,q0,q1", [
    (0.0, 0.0, 0.0, 1.0), (0.3, -1.7, 2.0, 0.5), (-4.0, 4.0, 1.0, -1.0),
    (10.0, 9.5, 10.0, 10.5), (100.0, 101.0, -50.0, -49.0),
])
def test_two_token_rows_match_bernoulli_closed_form(b0, b1, q0, q1):
    b = np.array([[b0, b1]], np.float32)
    q = np.array([[q0, q1]], np.float32)
    x0, x1, y0, y1 = (float(v) for v in (b[0, 0], b[0, 1], q[0, 0], q[0, 1]))
    p = 1.0 / (1.0 + math.exp(x0 - x1))  # sigmoid(b1 - b0) = P_base(token 1)
    s = 1.0 / (1.0 + math.exp(y0 - y1))
    want = p * math.log(p / s) + (1 - p) * math.log((1 - p) / (1 - s))
    r, _ = _run(b, q)
    assert abs(r["kld"][0] - want) <= 1e-12 * max(1.0, abs(want))


def test_small_vocab_brute_force():
    for V in range(1, 9):
        b = RNG.normal(0, 2.0, size=(40, V)).astype(np.float32)
        q = (b + RNG.normal(0, 1.0, size=b.shape)).astype(np.float32)
        r, _ = _run(b, q)
        for i in range(40):
            want = _brute_kl(b[i], q[i])
            assert abs(r["kld"][i] - want) <= 1e-13 + 1e-11 * want, (V, i)
            assert r["amax_b"][i] == int(np.argmax(b[i]))
            assert r["amax_q"][i] == int(np.argmax(q[i]))


def test_second_order_expansion_for_small_perturbations():
    # KL(softmax(b) || softmax(b + e)) = Var_p(e) / 2 + O(|e|^3)
    V = 20000
    b = RNG.normal(0, 2.0, size=(4, V)).astype(np.float32)
    q = (b + RNG.normal(0, 2e-3, size=b.shape)).astype(np.float32)
    r, _ = _run(b, q)
    for i in range(4):
        x = b[i].astype(np.float64)
        e = q[i].astype(np.float64) - x  # exact perturbation of the stored values
        p = np.exp(x - x.max())
        p /= p.sum()
        mean_e = np.dot(p, e)
        half_var = 0.5 * np.dot(p, (e - mean_e) ** 2)
        assert abs(r["kld"][i] - half_var) <= 2e-2 * half_var


# ---------------------------------------------------------------- worked example

def _homework_case(golden_dir, key):
    with open(os.path.join(golden_dir, "worked_example_homework.json")) as f:
        case = json.load(f)[key]
    return case


def test_page_worked_example_renormalised(golden_dir):
    case = _homework_case(golden_dir, "renormalised")
    pb = [Decimal(x) / Decimal(100) for x in case["base_percent"]]
    pq = [Decimal(x) / Decimal(100) for x in case["quant_percent"]]
    getcontext().prec = 50
    zb, zq = sum(pb), sum(pq)
    want = sum((x / zb) * ((x / zb) / (y / zq)).ln() for x, y in zip(pb, pq))
    b = np.array([[math.log(float(x)) for x in pb]], np.float32)
    q = np.array([[math.log(float(y)) for y in pq]], np.float32)
    # the logits are fp32-rounded logs, so compare with the stored values too
    r, res = _run(b, q)
    assert abs(r["kld"][0] - _brute_kl(b[0], q[0])) < 1e-14
    assert abs(r["kld"][0] - float(want)) < 1e-6  # fp32 rounding of the logs
    # by hand: p = (.9375, .052083, .010417), r = (.5, .3, .2);
    # .9375 ln 1.875 + .052083 ln .17361 + .010417 ln .052083
    # = .589321 - .091195 - .030780 = .467346
    assert abs(float(want) - 0.467346) < 2e-6
    assert r["amax_b"][0] == case["top_index"] == r["amax_q"][0]
    assert res["top1_agree_pct"] == 100.0


def test_page_worked_example_with_residual_mass(golden_dir):
    case = _homework_case(golden_dir, "residual")
    b = np.array([[math.log(x / 100) if x > 0 else -np.inf
                   for x in case["base_percent"]]], np.float32)
    q = np.array([[math.log(x / 100) if x > 0 else -np.inf
                   for x in case["quant_percent"]]], np.float32)
    r, _ = _run(b, q)
    assert r["kld"][0] == math.inf
    assert r["flags"][0] & oracle.ROW_INF_KL
    assert r["amax_b"][0] == r["amax_q"][0] == case["top_index"]


# ---------------------------------------------------------------- NLL / PPL

@pytest.mark.parametrize("V", [3, 1000, 151936])
def test_uniform_quant_gives_nll_log_V_and_ppl_V(V):
    b = RNG.normal(0, 1, size=(5, V)).astype(np.float32)
    q = np.full((5, V), -3.5, np.float32)
    tok = RNG.integers(0, V, size=5).astype(np.int32)
    r, res = _run(b, q, tok)
    np.testing.assert_allclose(r["nll"], math.log(V), rtol=1e-13)
    assert abs(res["ppl"] - V) <= 1e-10 * V


def test_one_hot_quant_nll():
    V = 64
    b = RNG.normal(0, 1, size=(2, V)).astype(np.float32)
    q = np.full((2, V), NEG_INF, np.float32)
    q[:, 9] = 2.0
    tok = np.array([9, 10], np.int32)
    r, res = _run(b, q, tok)
    assert r["nll"][0] == 0.0
    assert r["nll"][1] == math.inf and r["flags"][1] & oracle.ROW_INF_NLL
    assert res["ppl"] == math.inf


def test_nll_matches_brute_force_log_prob():
    V = 7
    b = RNG.normal(0, 1, size=(30, V)).astype(np.float32)
    q = RNG.normal(0, 2, size=(30, V)).astype(np.float32)
    tok = RNG.integers(0, V, size=30).astype(np.int32)
    r, res = _run(b, q, tok)
    want = []
    for i in range(30):
        e = [math.exp(float(x)) for x in q[i]]
        want.append(-math.log(e[tok[i]] / math.fsum(e)))
    np.testing.assert_allclose(r["nll"], want, rtol=1e-13)
    assert abs(res["mean_nll"] - math.fsum(want) / 30) < 1e-13
    assert abs(res["ppl"] - math.exp(math.fsum(want) / 30)) < 1e-12 * res["ppl"]


def test_bad_token_ids_are_flagged_and_excluded_from_ppl():
    V = 10
    b = RNG.normal(0, 1, size=(4, V)).astype(np.float32)
    q = RNG.normal(0, 1, size=(4, V)).astype(np.float32)
    tok = np.array([0, -1, V, 3], np.int32)
    r, res = _run(b, q, tok)
    assert list(r["flags"] & oracle.ROW_BAD_TOKEN) == [0, oracle.ROW_BAD_TOKEN,
                                                       oracle.ROW_BAD_TOKEN, 0]
    assert res["n_nll"] == 2 and res["n_valid"] == 4
    assert abs(res["mean_nll"] - (r["nll"][0] + r["nll"][3]) / 2) < 1e-15


# ------------------------------------------- base NLL, PPL(base), ratio, dp

def test_base_nll_matches_brute_force_and_dp_statistics():
    V, n = 9, 40
    b = RNG.normal(0, 1.5, size=(n, V)).astype(np.float32)
    q = RNG.normal(0, 2, size=(n, V)).astype(np.float32)
    tok = RNG.integers(0, V, size=n).astype(np.int32)
    r, res = _run(b, q, tok)
    pb, pq = [], []
    for i in range(n):
        eb = [math.exp(float(x)) for x in b[i]]
        eq = [math.exp(float(x)) for x in q[i]]
        pb.append(eb[tok[i]] / math.fsum(eb))
        pq.append(eq[tok[i]] / math.fsum(eq))
    np.testing.assert_allclose(r["nll_base"], [-math.log(x) for x in pb], rtol=1e-13)
    dp = [x - y for x, y in zip(pq, pb)]  # P_quant(tok) - P_base(tok)
    assert abs(res["mean_dp"] - math.fsum(dp) / n) < 1e-14
    assert abs(res["rms_dp"] - math.sqrt(math.fsum(d * d for d in dp) / n)) < 1e-14
    want_b = math.fsum(-math.log(x) for x in pb) / n
    assert abs(res["mean_nll_base"] - want_b) < 1e-13
    assert abs(res["ppl_base"] - math.exp(want_b)) < 1e-12 * res["ppl_base"]
    assert abs(res["ln_ppl_ratio"] - (res["mean_nll"] - want_b)) < 1e-13
    assert abs(math.exp(res["ln_ppl_ratio"]) - res["ppl"] / res["ppl_base"]) < 1e-12


def test_uniform_base_against_one_hot_quant_at_the_token():
    # P_base(tok) = 1/V, P_quant(tok) = 1: dp = 1 - 1/V on every row, so the
    # mean and the root mean square both equal it (a dropped square root or a
    # flipped sign shows); NLLB = log V, NLL = 0, ln(PPL(Q)/PPL(base)) = -log V.
    V = 50
    b = np.zeros((6, V), np.float32)
    q = np.full((6, V), NEG_INF, np.float32)
    tok = np.arange(6, dtype=np.int32) * 7
    q[np.arange(6), tok] = 3.0
    r, res = _run(b, q, tok)
    np.testing.assert_allclose(r["nll_base"], math.log(V), rtol=1e-14)
    assert np.all(r["nll"] == 0.0)
    assert abs(res["mean_dp"] - (1 - 1 / V)) < 1e-15
    assert abs(res["rms_dp"] - (1 - 1 / V)) < 1e-15
    assert abs(res["ln_ppl_ratio"] + math.log(V)) < 1e-14
    assert abs(res["ppl_base"] - V) < 1e-11


def test_identical_rows_have_zero_dp_and_unit_ppl_ratio():
    b = RNG.normal(0, 2, size=(25, 3000)).astype(np.float32)
    tok = RNG.integers(0, 3000, size=25).astype(np.int32)
    r, res = _run(b, b.copy(), tok)
    assert np.array_equal(r["nll"], r["nll_base"])
    assert res["mean_dp"] == 0.0 and res["rms_dp"] == 0.0 and res["ln_ppl_ratio"] == 0.0
    assert res["ppl"] == res["ppl_base"]


def test_base_nll_invariant_to_adding_a_constant_and_masked_token():
    V = 300
    # logits on a 2^-10 grid, so that adding 64 is exact in fp32
    b = (np.round(RNG.normal(0, 1, size=(3, V)) * 1024) / 1024).astype(np.float32)
    q = RNG.normal(0, 1, size=(3, V)).astype(np.float32)
    tok = np.array([5, 17, 200], np.int32)
    r0, _ = _run(b, q, tok)
    assert np.array_equal((b + np.float32(64.0)).astype(np.float64) - 64.0, b.astype(np.float64))
    r1, _ = _run(b + np.float32(64.0), q, tok)
    np.testing.assert_allclose(r1["nll_base"], r0["nll_base"], rtol=1e-13)
    b2 = b.copy()
    b2[2, 200] = NEG_INF   # the base gives the token no probability
    r2, res2 = _run(b2, q, tok)
    assert r2["nll_base"][2] == math.inf and r2["flags"][2] & oracle.ROW_INF_NLLB
    assert res2["ppl_base"] == math.inf
    # P_base(tok) = 0 there, so that row's dp is P_quant(tok), still finite
    pq = math.exp(-r2["nll"][2])
    dp = [math.exp(-r2["nll"][i]) - math.exp(-r2["nll_base"][i]) for i in range(3)]
    assert abs(dp[2] - pq) < 1e-16 and abs(res2["mean_dp"] - math.fsum(dp) / 3) < 1e-15


def test_without_tokens_base_statistics_are_nan():
    b = RNG.normal(0, 1, size=(4, 50)).astype(np.float32)
    r, res = _run(b, b + np.float32(0.1))
    assert np.all(np.isnan(r["nll_base"]))
    for k in ("mean_nll_base", "ppl_base", "ln_ppl_ratio", "mean_dp", "rms_dp"):
        assert math.isnan(res[k]), k


# ---------------------------------------------------------------- argmax / ties

def test_argmax_ties_go_to_lowest_index():
    V = 50
    b = RNG.normal(0, 1, size=(20, V)).astype(np.float32)
    q = b.copy()
    for i in range(20):
        idx = np.sort(RNG.choice(V, size=2 + i % 7, replace=False))
        b[i, idx] = 9.0
        q[i, idx[::-1][: max(2, len(idx) - 1)]] = 9.5
    r, _ = _run(b, q)
    for i in range(20):
        assert r["amax_b"][i] == int(np.argmax(b[i]))  # numpy: first occurrence
        assert r["amax_q"][i] == int(np.argmax(q[i]))


def test_same_top_p_counts_index_agreement():
    b = np.array([[0, 5, 5], [1, 0, 0], [0, 0, 2]], np.float32)
    q = np.array([[0, 5, 5], [0, 1, 0], [0, 0, 3]], np.float32)
    r, res = _run(b, q)
    assert list(r["amax_b"]) == [1, 0, 2] and list(r["amax_q"]) == [1, 1, 2]
    assert res["top1_agree"] == 2
    assert abs(res["top1_agree_pct"] - 200.0 / 3) < 1e-12


# ---------------------------------------------------------------- reductions

def test_percentiles_hand_values():
    x = np.array([1.0, 2.0, 3.0, 4.0, 5.0])
    assert oracle.percentile_sorted(x, 0.5) == 3.0
    assert abs(oracle.percentile_sorted(x, 0.9) - 4.6) < 1e-15
    assert abs(oracle.percentile_sorted(x, 0.99) - 4.96) < 1e-15
    assert oracle.percentile_sorted(np.array([1.0, 2.0]), 0.5) == 1.5
    assert oracle.percentile_sorted(np.array([7.0]), 0.99) == 7.0


@pytest.mark.parametrize("n", [1, 2, 3, 10, 101, 4096, 32768])
def test_percentiles_match_numpy_linear(n):
    x = np.sort(RNG.gamma(0.5, 0.1, size=n))
    for p in (0.5, 0.9, 0.99):
        want = np.percentile(x, 100 * p, method="linear")
        got = oracle.percentile_sorted(x, p)
        assert abs(got - want) <= 1e-15 * max(1.0, abs(want)) + 1e-300


def test_reduction_against_library_sums():
    b = RNG.normal(0, 2.5, size=(301, 211)).astype(np.float32)
    q = (b + RNG.normal(0, 0.3, size=b.shape)).astype(np.float32)
    tok = RNG.integers(0, 211, size=301).astype(np.int32)
    r, res = _run(b, q, tok)
    assert abs(res["mean_kld"] - math.fsum(r["kld"]) / 301) <= 1e-13 * res["mean_kld"]
    want_nll = math.fsum(r["nll"]) / 301
    assert abs(res["mean_nll"] - want_nll) <= 1e-13 * want_nll
    srt = np.sort(r["kld"])
    assert res["median_kld"] == np.percentile(srt, 50, method="linear")
    assert abs(res["p99_kld"] - np.percentile(srt, 99, method="linear")) <= 1e-15
    assert res["max_kld"] == srt[-1]
    assert res["top1_agree"] == int(np.sum(r["amax_b"] == r["amax_q"]))


# ---------------------------------------------------------------- flags

def test_nonfinite_and_empty_rows_are_flagged_and_excluded():
    V = 12
    b = RNG.normal(0, 1, size=(6, V)).astype(np.float32)
    q = (b + 0.1).astype(np.float32)
    b[1, 3] = np.nan
    q[2, 5] = np.inf
    b[3, :] = -np.inf
    q[4, :] = -np.inf
    r, res = _run(b, q)
    fl = list(r["flags"])
    assert fl[0] == 0 and fl[5] == 0
    assert fl[1] == oracle.ROW_NONFINITE and fl[2] == oracle.ROW_NONFINITE
    assert fl[3] == oracle.ROW_EMPTY and fl[4] == oracle.ROW_EMPTY
    for i in (1, 2, 3, 4):
        assert math.isnan(r["kld"][i]) and r["amax_b"][i] == -1 and r["amax_q"][i] == -1
    assert res["n_valid"] == 2 and res["n_flagged"] == 4
    assert abs(res["mean_kld"] - (r["kld"][0] + r["kld"][5]) / 2) < 1e-15


def test_statistics_are_over_the_valid_rows_only():
    # excluded rows (NaN, all -inf) count in n_rows but in none of the
    # means, percentages or order statistics: each is the same statistic of
    # the valid rows alone
    V = 64
    b = RNG.normal(0, 2, size=(10, V)).astype(np.float32)
    q = (b + RNG.normal(0, 0.7, size=b.shape)).astype(np.float32)
    b[2, 7] = np.nan
    q[6, :] = -np.inf
    r, res = _run(b, q)
    keep = [i for i in range(10) if i not in (2, 6)]
    valid = np.array([r["kld"][i] for i in keep])
    assert res["n_rows"] == 10 and res["n_valid"] == 8
    assert abs(res["mean_kld"] - math.fsum(valid) / 8) <= 1e-14 * res["mean_kld"]
    agree = sum(int(r["amax_b"][i] == r["amax_q"][i]) for i in keep)
    assert res["top1_agree"] == agree
    assert abs(res["top1_agree_pct"] - 100.0 * agree / 8) <= 1e-12
    assert res["median_kld"] == np.percentile(np.sort(valid), 50, method="linear")
    assert res["max_kld"] == valid.max()
    # the valid rows alone give the same statistics
    _, alone = _run(b[keep], q[keep])
    for k in ("mean_kld", "median_kld", "p90_kld", "p99_kld", "max_kld", "top1_agree_pct"):
        assert abs(res[k] - alone[k]) <= 1e-14 * abs(alone[k]) + 1e-300, k


def test_masked_vocab_entries_contribute_nothing():
    # -inf in both rows on the same entries == dropping those entries
    V = 300
    b = RNG.normal(0, 2, size=(5, V)).astype(np.float32)
    q = (b + RNG.normal(0, 0.3, size=b.shape)).astype(np.float32)
    bm, qm = b.copy(), q.copy()
    bm[:, -37:] = -np.inf
    qm[:, -37:] = -np.inf
    r1, _ = _run(bm, qm)
    r2, _ = _run(np.ascontiguousarray(b[:, :-37]), np.ascontiguousarray(q[:, :-37]))
    np.testing.assert_allclose(r1["kld"], r2["kld"], rtol=1e-14, atol=0)
    assert np.all(r1["flags"] == 0)


# ---------------------------------------------------------------- dtypes, threads

def test_bf16_input_equals_widened_fp32_input():
    b32 = RNG.normal(0, 2.5, size=(9, 515)).astype(np.float32)
    q32 = (b32 + RNG.normal(0, 0.2, size=b32.shape)).astype(np.float32)
    # round to bf16 by keeping the top 16 bits with round-to-nearest-even
    def to_bf16_bits(x):
        u = x.view(np.uint32).astype(np.uint64)
        u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
        return u.astype(np.uint16)
    bb, qb = to_bf16_bits(b32), to_bf16_bits(q32)
    bw = (bb.astype(np.uint32) << 16).view(np.float32)
    qw = (qb.astype(np.uint32) << 16).view(np.float32)
    r16, s16 = _run(bb, qb, dtype=oracle.BF16)
    r32, s32 = _run(bw, qw, dtype=oracle.F32)
    for k in ("kld", "amax_b", "amax_q", "flags"):
        assert np.array_equal(r16[k], r32[k])


def test_f16_input_equals_numpy_widening():
    x = RNG.normal(0, 3, size=(7, 333)).astype(np.float16)
    x[0, :20] = np.array([6e-8, -6e-8, 1e-5, 65504, -65504] * 4, np.float16)
    y = (x.astype(np.float32) + RNG.normal(0, 0.5, size=x.shape)).astype(np.float16)
    r16, _ = _run(x.view(np.uint16), y.view(np.uint16), dtype=oracle.F16)
    r32, _ = _run(x.astype(np.float32), y.astype(np.float32), dtype=oracle.F32)
    for k in ("kld", "amax_b", "amax_q", "flags"):
        assert np.array_equal(r16[k], r32[k])


def test_threaded_rows_are_bit_identical():
    b = RNG.normal(0, 2.5, size=(37, 1001)).astype(np.float32)
    q = (b + RNG.normal(0, 0.3, size=b.shape)).astype(np.float32)
    tok = RNG.integers(0, 1001, size=37).astype(np.int32)
    r1, s1 = _run(b, q, tok, nthreads=1)
    r4, s4 = _run(b, q, tok, nthreads=4)
    for k in r1:
        assert np.array_equal(r1[k], r4[k])
    assert s1 == s4


# ---------------------------------------------------------------- KL gradient

def _brute_kl64(b_row, q_row):
    """KL in fp64 straight from sum p log(p/r), no max subtraction."""
    eb = [math.exp(x) for x in b_row]
    eq = [math.exp(x) for x in q_row]
    sb, sq = math.fsum(eb), math.fsum(eq)
    return math.fsum((x / sb) * math.log((x / sb) / (y / sq)) for x, y in zip(eb, eq) if x > 0)


def test_grad_matches_central_differences_of_the_kl():
    V = 6
    b = RNG.normal(0, 1, size=(4, V)).astype(np.float32)
    q = RNG.normal(0, 1, size=(4, V)).astype(np.float32)
    g = oracle.grad(b, q)
    h = 1e-5
    for i in range(4):
        bi = [float(x) for x in b[i]]
        for j in range(V):
            up = [float(x) for x in q[i]]
            dn = list(up)
            up[j] += h
            dn[j] -= h
            fd = (_brute_kl64(bi, up) - _brute_kl64(bi, dn)) / (2 * h)
            assert abs(g[i, j] - fd) < 1e-8, (i, j, g[i, j], fd)


def test_grad_rows_sum_to_zero_and_scale_linearly():
    b = RNG.normal(0, 2, size=(5, 2000)).astype(np.float32)
    q = (b + RNG.normal(0, 0.3, size=(5, 2000))).astype(np.float32)
    g1 = oracle.grad(b, q)
    assert np.all(np.abs(g1.sum(axis=1)) < 1e-14)
    g3 = oracle.grad(b, q, scale=-0.25)
    np.testing.assert_allclose(g3, -0.25 * g1, rtol=1e-15, atol=0)


def test_grad_closed_forms():
    V = 40
    # identical rows: exactly zero
    b = RNG.normal(0, 1, size=(2, V)).astype(np.float32)
    assert np.all(oracle.grad(b, b.copy()) == 0.0)
    # one-hot base (entry 7) against a uniform quant: 1/V - [j == 7]
    b1 = np.full((1, V), NEG_INF, np.float32)
    b1[0, 7] = 0.0
    q1 = np.zeros((1, V), np.float32)
    want = np.full(V, 1.0 / V)
    want[7] -= 1.0
    np.testing.assert_allclose(oracle.grad(b1, q1)[0], want, rtol=0, atol=1e-16)


def test_grad_of_excluded_rows_is_zero_and_masks_are_zero():
    V = 10
    b = RNG.normal(0, 1, size=(3, V)).astype(np.float32)
    q = RNG.normal(0, 1, size=(3, V)).astype(np.float32)
    b[0, 3] = np.nan
    q[1, :] = NEG_INF
    b[2, 4] = NEG_INF      # P_base = 0 there
    q[2, 5] = NEG_INF      # P_quant = 0 there
    g = oracle.grad(b, q)
    assert np.all(g[0] == 0.0) and np.all(g[1] == 0.0)
    e = np.exp(q[2].astype(np.float64) - q[2].max())
    r = e / e.sum()
    assert g[2, 5] < 0 and abs(g[2, 4] - r[4]) < 1e-16


# ---------------------------------------------------- top-k compression + KL

def _softmax_np(x):
    x = x.astype(np.float64)
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=1, keepdims=True)


def test_topk_with_k_at_least_V_is_the_full_kl():
    b = RNG.normal(0, 2, size=(6, 50)).astype(np.float32)
    q = (b + RNG.normal(0, 0.5, size=(6, 50))).astype(np.float32)
    t = oracle.topk(b, q, k=64)
    r, _ = _run(b, q)
    np.testing.assert_allclose(t["kl_topk"], r["kld"], rtol=1e-11, atol=1e-15)
    assert np.all(np.isneginf(t["rest"]))
    assert np.all(t["idx"][:, 50:] == -1) and np.all(np.isneginf(t["logp"][:, 50:]))
    np.testing.assert_array_equal(t["idx"][:, :50], np.argsort(-b, axis=1, kind="stable"))


def test_topk_one_is_the_binary_kl_of_the_top_entry():
    b = RNG.normal(0, 1.5, size=(10, 300)).astype(np.float32)
    q = (b + RNG.normal(0, 0.4, size=(10, 300))).astype(np.float32)
    t = oracle.topk(b, q, k=1)
    p, r = _softmax_np(b), _softmax_np(q)
    for i in range(10):
        j = int(np.argmax(b[i]))
        assert t["idx"][i, 0] == j
        p1, r1 = p[i, j], r[i, j]
        want = p1 * math.log(p1 / r1) + (1 - p1) * math.log((1 - p1) / (1 - r1))
        assert abs(t["kl_topk"][i] - want) < 1e-12
        assert abs(t["rest"][i] - math.log1p(-p1)) < 1e-12


def test_topk_kl_grows_with_k_up_to_the_full_kl():
    # merging categories never increases KL (data processing), and the top-k
    # partitions refine each other as k grows
    b = RNG.normal(0, 2.5, size=(8, 2000)).astype(np.float32)
    q = (b + RNG.normal(0, 0.3, size=(8, 2000))).astype(np.float32)
    full, _ = _run(b, q)
    prev = np.zeros(8)
    for k in (1, 2, 8, 32, 128, 512, 2000):
        cur = oracle.topk(b, q, k=k)["kl_topk"]
        assert np.all(cur >= prev - 1e-15) and np.all(cur <= full["kld"] + 1e-12)
        prev = cur
    np.testing.assert_allclose(prev, full["kld"], rtol=1e-11)


def test_topk_indices_logp_and_rest_by_numpy_and_ties():
    b = RNG.normal(0, 1, size=(5, 1000)).astype(np.float32)
    b[0, [900, 3, 500]] = 9.0          # a three-way tie at the top
    q = (b + RNG.normal(0, 0.2, size=(5, 1000))).astype(np.float32)
    t = oracle.topk(b, q, k=128)
    order = np.argsort(-b, axis=1, kind="stable")[:, :128]
    np.testing.assert_array_equal(t["idx"], order)
    assert list(t["idx"][0, :3]) == [3, 500, 900]
    p = _softmax_np(b)
    np.testing.assert_allclose(t["logp"], np.log(np.take_along_axis(p, order, axis=1)), rtol=1e-12)
    mask = np.ones_like(p, bool)
    np.put_along_axis(mask, order, False, axis=1)
    np.testing.assert_allclose(t["rest"], np.log(np.where(mask, p, 0).sum(axis=1)), rtol=1e-12)


def test_topk_identical_rows_masks_and_excluded_rows():
    b = RNG.normal(0, 1, size=(4, 200)).astype(np.float32)
    t = oracle.topk(b, b.copy(), k=16)
    assert np.all(t["kl_topk"] == 0.0)
    b2 = b.copy()
    q2 = b.copy() + np.float32(0.25)
    b2[0, 10:] = NEG_INF                 # only 10 finite base entries: k = 16 reaches p = 0
    b2[1, 5] = np.nan                    # excluded row
    q2[2, int(np.argmax(b2[2]))] = NEG_INF  # the quant gives the top entry nothing
    t2 = oracle.topk(b2, q2, k=16)
    assert np.isneginf(t2["rest"][0]) and np.all(np.isneginf(t2["logp"][0, 10:]))
    assert np.all(t2["idx"][1] == -1) and math.isnan(t2["kl_topk"][1]) and math.isnan(t2["rest"][1])
    assert t2["kl_topk"][2] == math.inf
    assert abs(t2["kl_topk"][3]) < 1e-15   # a constant shift changes no probability
