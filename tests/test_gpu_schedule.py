"""The row pass's schedule against the fp64 oracle.

Whole rows go round robin over one CTA per SM; a last partial wave of at
most SMs/2 rows is split over the CTAs by balanced chunk ranges, fewer rows
than SMs/2 in all into row-aligned parts, and the parts are merged per row;
the reduction follows (fixed-order sums, the
seven order statistics by an exact radix select). The cases sweep row counts
around multiples of the SM count,
cover the mid-range counts of scoring 512-token chunks one chunk per row at
the full vocabulary, and stress the selection with identical, repeated and
excluded rows. Every percentile must be the exact order statistic of the
GPU's own per-row values.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from logit_kl_divergence_b200 import KLDStats, rows_view, synth

from gpu_helpers import (ODT, assert_rows_match, assert_select_exact, assert_stats_match, gpu_run,
                         oracle_rows_chunked)

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _sms():
    return torch.cuda.get_device_properties(DEV).multi_processor_count


def _parity(w, split=None):
    t = None if w.token_ids is None else w.token_ids.to(DEV)
    g_rows, gres = gpu_run(w.base.to(DEV), w.quant.to(DEV), t, split=split)
    o_rows, ores = oracle.run(w.base, w.quant, w.token_ids, ODT[w.dtype], 8)
    assert_rows_match(g_rows, o_rows)
    assert_stats_match(gres, ores)
    assert_select_exact(g_rows, gres, w.token_ids is not None)
    return g_rows, gres


@pytest.mark.parametrize("n_rel", [-1, 0, 1, 2, 74, 148 + 1, 2 * 148 + 3])
@pytest.mark.parametrize("dtype,v", [(synth.F32, 3001), (synth.BF16, 4099)])
def test_rows_around_multiples_of_the_sm_count(n_rel, dtype, v):
    n = _sms() + n_rel
    _parity(synth.make_recipe("ctx", n=n, v=v, dtype=dtype, seed=1000 + n))


@pytest.mark.parametrize("n", [1, 5, 75, 100, 300, 601])
def test_tiny_vocabularies_leave_parts_empty(n):
    # a row of one or two chunks: many CTAs' ranges cover a single chunk
    for v in (1, 513, 1000):
        _parity(synth.make_recipe("edge", n=n, v=v, dtype=synth.F32, seed=v + n))


@pytest.mark.parametrize("n", [75, 100, 149, 300, 600])
def test_mid_range_rows_full_vocabulary(n):
    # 512-token chunks scored one per row at the full vocabulary
    w = synth.make_recipe("ctx", n=n, v=151936, dtype=synth.F32, seed=n, device=DEV)
    g_rows, gres = gpu_run(w.base, w.quant, w.token_ids)
    o_rows = oracle_rows_chunked(w)
    assert_rows_match(g_rows, o_rows)
    ores = oracle.reduce(o_rows, True)
    for k in ("n_valid", "top1_agree", "n_nll"):
        assert int(gres[k]) == int(ores[k]), k
    assert_select_exact(g_rows, gres, True)


def test_split_tail_equals_whole_rows():
    # the same rows through the split tail and through whole-row launches
    w = synth.make_recipe("ctx", n=2 * _sms() + 7, v=20011, dtype=synth.BF16, seed=9)
    a, ares = _parity(w)
    b, bres = _parity(w, split=-1)
    np.testing.assert_array_equal(a["amax_b"], b["amax_b"])
    np.testing.assert_array_equal(a["flags"], b["flags"])
    ok = np.abs(a["kld"] - b["kld"]) <= 1e-6 + 1e-4 * np.abs(b["kld"])
    assert ok.all()


@pytest.mark.parametrize("n", [40, 700, 3000, 24000])
def test_identical_rows_all_give_zero(n):
    # every KL is exactly 0: all keys equal through every radix level; at
    # 24000 rows more keys than shared memory holds, so the selection reads
    # them from the records for every level
    w = synth.make_recipe("ctx", n=n, v=2049, dtype=synth.F32, seed=n)
    w.quant.copy_(w.base)
    g_rows, gres = _parity(w)
    assert np.all(g_rows["kld"] == 0.0)
    assert gres["median_kld"] == 0.0 and gres["max_kld"] == 0.0


def test_repeated_rows_make_heavy_duplicates():
    # four distinct row pairs, each repeated: every order statistic sits in a
    # run of hundreds of equal keys
    base = synth.make_recipe("ctx", n=4, v=3001, dtype=synth.F32, seed=5)
    idx = torch.arange(1500) % 4
    w = synth.make_recipe("ctx", n=1500, v=3001, dtype=synth.F32, seed=6)
    w.base.copy_(base.base[idx])
    w.quant.copy_(base.quant[idx])
    w.token_ids.copy_(base.token_ids[idx])
    g_rows, _ = _parity(w)
    assert len(np.unique(g_rows["kld"])) == 4


def test_excluded_rows_offset_the_ranks():
    w = synth.make_recipe("ctx", n=500, v=3001, dtype=synth.F32, seed=7)
    w.base[::3, 11] = math.nan        # a third of the rows excluded
    w.quant[1::7, :] = -math.inf      # all -inf quant rows: EMPTY
    w.token_ids[2::5] = 3001 + 4      # tokens outside the vocabulary
    _parity(w)


def test_all_rows_excluded():
    w = synth.make_recipe("ctx", n=300, v=1000, dtype=synth.F32, seed=8)
    w.base[:, 3] = math.nan
    g_rows, gres = gpu_run(w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV))
    assert gres["n_valid"] == 0 and math.isnan(gres["median_kld"]) and math.isnan(gres["mean_kld"])
    _, ores = oracle.run(w.base, w.quant, w.token_ids, oracle.F32)
    assert_stats_match(gres, ores)


def test_repeated_launches_leave_the_split_scratch_ready():
    # the split rows' tickets and the few-row launch counter must be back at
    # zero after every launch: different row counts, dtypes and token
    # presence on one handle
    st = KLDStats(max_rows=2 * 148 + 40, device=DEV)
    try:
        for n, v, dt, tok, seed in [(300, 5003, synth.F32, True, 1), (149, 4099, synth.BF16, False, 2),
                                    (7, 70001, synth.F32, True, 3), (148, 3001, synth.F16, True, 4),
                                    (336, 2049, synth.F32, True, 5), (1, 1000, synth.F32, False, 6)]:
            w = synth.make_recipe("ctx", n=n, v=v, dtype=dt, seed=seed)
            t = w.token_ids if tok else None
            st.run(w.base.to(DEV), w.quant.to(DEV), None if t is None else t.to(DEV))
            gres = st.result()
            g = {k: x.cpu().numpy() for k, x in rows_view(st.records()).items()}
            g["flags"] = g["flags"].astype(np.uint32)
            o_rows, ores = oracle.run(w.base, w.quant, t, ODT[dt])
            assert_rows_match(g, o_rows)
            assert_stats_match(dict(gres), ores)
            assert_select_exact(g, gres, t is not None)
    finally:
        st.close()


def test_run_and_rows_then_reduce_agree():
    # the whole statistic and its two halves called one after the other
    # give the same records and the same statistics
    n = 3 * _sms() + 11
    w = synth.make_recipe("ctx", n=n, v=3001, dtype=synth.F32, seed=10)
    b, q, t = w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV)
    st = KLDStats(max_rows=n, device=DEV)
    try:
        st.run(b, q, t)
        fused = st.result()
        st.run_rows(b, q, t)
        st.reduce(None, n, True)
        ref = st.result()
    finally:
        st.close()
    for k in ("median_kld", "p90_kld", "p99_kld", "max_kld", "n_valid", "top1_agree", "n_nll",
              "n_flagged", "flags_or"):
        assert fused[k] == ref[k], k
    for k in ("mean_kld", "mean_nll", "ppl", "mean_nll_base", "mean_dp", "rms_dp"):
        assert math.isclose(fused[k], ref[k], rel_tol=1e-13, abs_tol=1e-15), k
