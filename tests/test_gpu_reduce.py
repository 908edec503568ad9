"""The reduction + exact percentile kernel on synthetic per-row records.

Record arrays are built directly (no row pass) so the radix select meets
distributions the row pass rarely produces: heavy duplicates, all-equal
values, tiny negative KL from rounding, +inf, excluded rows, and sizes from a
single row to well past the gather threshold (several radix passes)."""
import math

import numpy as np
import pytest
import torch

import oracle
from logit_kl_divergence_b200 import KLDStats

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

REC = np.dtype([("kld", "<f8"), ("nll", "<f8"), ("nll_base", "<f8"), ("amax_b", "<i4"),
                ("amax_q", "<i4"), ("flags", "<u4"), ("dp", "<f4")])
assert REC.itemsize == 40


def make_records(kld, rng, flags=None, nll=True):
    n = len(kld)
    r = np.zeros(n, REC)
    r["kld"] = kld
    r["nll"] = rng.gamma(2.0, 1.0, n) if nll else np.nan
    r["nll_base"] = rng.gamma(2.0, 1.0, n) if nll else np.nan
    r["dp"] = np.exp(-r["nll"]) - np.exp(-r["nll_base"])  # as the row pass writes it
    r["amax_b"] = rng.integers(0, 5, n)
    r["amax_q"] = rng.integers(0, 5, n)
    if flags is not None:
        r["flags"] = flags
        excl = (flags & (oracle.ROW_NONFINITE | oracle.ROW_EMPTY)) != 0
        r["kld"][excl] = np.nan
        r["amax_b"][excl] = -1
        r["amax_q"][excl] = -1
    return r


def run_reduce(rec, has_nll=True):
    t = torch.from_numpy(rec.view(np.uint8).copy()).to(DEV)
    st = KLDStats(max_rows=1, device=DEV)
    st.reduce(t, len(rec), has_nll)
    res = st.result()
    st.close()
    return res


def check(rec, has_nll=True):
    g = run_reduce(rec, has_nll)
    d = {"kld": rec["kld"], "nll": rec["nll"], "nll_base": rec["nll_base"], "amax_b": rec["amax_b"],
         "amax_q": rec["amax_q"], "flags": rec["flags"]}
    o = oracle.reduce(d, has_nll)
    for k in ("median_kld", "p90_kld", "p99_kld", "max_kld"):
        assert g[k] == o[k] or (math.isnan(g[k]) and math.isnan(o[k])), (k, g[k], o[k])
    for k in ("n_rows", "n_valid", "top1_agree", "n_nll", "n_flagged", "flags_or"):
        assert int(g[k]) == int(o[k]), k
    for k in ("mean_kld", "mean_nll", "ppl", "top1_agree_pct", "mean_nll_base", "ppl_base"):
        a, b = g[k], o[k]
        if math.isnan(b) or math.isinf(b):
            assert (math.isnan(a) and math.isnan(b)) or a == b, (k, a, b)
        else:
            assert abs(a - b) <= 1e-12 * abs(b) + 1e-300, (k, a, b)
    # a difference of nearly equal sums: absolute bar at fp64 rounding level
    a, b = g["ln_ppl_ratio"], o["ln_ppl_ratio"]
    assert (math.isnan(a) and math.isnan(b)) or a == b or abs(a - b) <= 1e-12, ("ln_ppl_ratio", a, b)
    # dp comes from the records' fp32 field: each value within 2^-24 relative,
    # so the mean within 1e-7 of the mean |dp| and the RMS within 1e-7 relative
    valid = (rec["flags"] & (oracle.ROW_NONFINITE | oracle.ROW_EMPTY | oracle.ROW_BAD_TOKEN)) == 0
    mabs = float(np.mean(np.abs(rec["dp"][valid].astype(np.float64)))) if valid.any() else 0.0
    for k, tol in (("mean_dp", 1e-7 * mabs + 1e-15), ("rms_dp", 1e-7 * abs(o["rms_dp"]) + 1e-15)):
        a, b = g[k], o[k]
        assert (math.isnan(a) and math.isnan(b)) or abs(a - b) <= tol, (k, a, b)
    return g


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 100, 4095, 4096, 4097, 8192, 32768, 100003, 1 << 20])
def test_continuous_values(n):
    rng = np.random.default_rng(n)
    check(make_records(rng.gamma(0.6, 0.08, n), rng))


@pytest.mark.parametrize("n", [10, 5000, 70000])
def test_heavy_duplicates(n):
    rng = np.random.default_rng(7)
    vals = rng.choice(np.array([0.0, 1e-3, 0.05, 0.05000000000000001, 2.0]), size=n)
    check(make_records(vals, rng))


@pytest.mark.parametrize("n", [33, 64, 200, 511, 512, 513])
def test_counted_ranks_around_their_size_limit(n):
    # 33..512 keys take the counting path (equal keys ordered by index),
    # 513 the radix levels: a tie group, signed zeros, infinities and
    # excluded rows on both sides of the limit
    rng = np.random.default_rng(n + 1)
    v = rng.gamma(0.6, 0.08, n)
    v[rng.integers(0, n, n // 4)] = 0.05
    v[rng.integers(0, n, 3)] = -0.0
    v[rng.integers(0, n, 3)] = 0.0
    v[rng.integers(0, n, 2)] = np.inf
    flags = np.zeros(n, np.uint32)
    flags[rng.integers(0, n, n // 10)] |= oracle.ROW_EMPTY
    check(make_records(v, rng, flags))


@pytest.mark.parametrize("n", [1, 300, 4097, 50000])
def test_all_equal(n):
    rng = np.random.default_rng(3)
    check(make_records(np.full(n, 0.0123), rng))


def test_tiny_negatives_zeros_and_infinities():
    rng = np.random.default_rng(11)
    n = 60000
    v = rng.gamma(0.6, 0.08, n)
    v[rng.integers(0, n, 500)] = -1e-13
    v[rng.integers(0, n, 500)] = -0.0
    v[rng.integers(0, n, 500)] = 0.0
    v[rng.integers(0, n, 50)] = np.inf
    check(make_records(v, rng))


@pytest.mark.parametrize("n", [8192, 30000])
def test_outliers_at_both_ends_of_a_narrow_cluster(n):
    # the selection starts from the range of the keys present: a range made
    # huge by outliers (the largest finite double, +inf, the smallest
    # subnormal, tiny negatives) around a cluster narrower than one first digit
    rng = np.random.default_rng(n)
    v = 0.02 + 1e-9 * rng.random(n)
    v[rng.integers(0, n, 3)] = 1.7976931348623157e308
    v[rng.integers(0, n, 2)] = np.inf
    v[rng.integers(0, n, 3)] = 5e-324
    v[rng.integers(0, n, 3)] = -1e-300
    check(make_records(v, rng))


def test_excluded_rows_and_bad_tokens():
    rng = np.random.default_rng(5)
    n = 20000
    flags = np.zeros(n, np.uint32)
    flags[rng.integers(0, n, 300)] |= oracle.ROW_NONFINITE
    flags[rng.integers(0, n, 300)] |= oracle.ROW_EMPTY
    flags[rng.integers(0, n, 300)] |= oracle.ROW_BAD_TOKEN
    check(make_records(rng.gamma(0.6, 0.08, n), rng, flags))


def test_all_rows_excluded():
    rng = np.random.default_rng(2)
    flags = np.full(10, oracle.ROW_EMPTY, np.uint32)
    g = check(make_records(np.zeros(10), rng, flags))
    assert g["n_valid"] == 0 and math.isnan(g["mean_kld"]) and math.isnan(g["median_kld"])


def test_without_nll():
    rng = np.random.default_rng(9)
    g = check(make_records(rng.gamma(0.6, 0.08, 999), rng, nll=False), has_nll=False)
    assert math.isnan(g["ppl"]) and g["has_nll"] == 0
