"""GPU (sm_100a) results against the fp64 CPU oracle, through the C ABI."""
import math

import numpy as np
import pytest
import torch

import oracle
from logit_kl_divergence_b200 import KLDStats, synth

from gpu_helpers import (ODT, assert_rows_match, assert_select_exact, assert_stats_match,
                         gpu_run)

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _parity(w, use_rows_api=False):
    b, q, t = w.base.to(DEV), w.quant.to(DEV), None if w.token_ids is None else w.token_ids.to(DEV)
    g_rows, gres = gpu_run(b, q, t, use_rows_api)
    o_rows, ores = oracle.run(w.base, w.quant, w.token_ids, ODT[w.dtype])
    assert_rows_match(g_rows, o_rows)
    assert_stats_match(gres, ores)
    assert_select_exact(g_rows, gres, w.token_ids is not None)
    return g_rows, gres


def test_small_workload_full_parity():
    _parity(synth.make("small_64x32000_f32"))


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16, synth.F16])
@pytest.mark.parametrize("V", [1, 2, 3, 5, 7, 8, 9, 31, 33, 1023, 1024, 1025, 4097, 8191,
                               8192, 8193, 16385, 32001, 65537])
def test_ragged_vocabularies(V, dtype):
    _parity(synth.make_recipe("ctx", n=7, v=V, dtype=dtype, seed=V))


@pytest.mark.parametrize("dtype,offset", [(synth.F32, 1), (synth.F32, 3), (synth.BF16, 1),
                                          (synth.BF16, 5), (synth.F16, 7)])
def test_misaligned_row_starts(dtype, offset):
    w = synth.make_recipe("ctx", n=9, v=5003, dtype=dtype, seed=3)
    n, v = w.base.shape
    bb = torch.empty(n * v + 16, dtype=w.base.dtype, device=DEV)
    qb = torch.empty(n * v + 16, dtype=w.base.dtype, device=DEV)
    b = bb[offset:offset + n * v].view(n, v)
    q = qb[offset:offset + n * v].view(n, v)
    b.copy_(w.base)
    q.copy_(w.quant)
    g_rows, gres = gpu_run(b, q, w.token_ids.to(DEV))
    o_rows, ores = oracle.run(w.base, w.quant, w.token_ids, ODT[dtype])
    assert_rows_match(g_rows, o_rows)
    assert_stats_match(gres, ores)


def test_rows_api_and_reduce_match_run():
    w = synth.make_recipe("ctx", n=100, v=3000, dtype=synth.BF16, seed=5)
    a_rows, ares = _parity(w, use_rows_api=False)
    b_rows, bres = _parity(w, use_rows_api=True)
    for k in a_rows:
        assert np.array_equal(a_rows[k], b_rows[k], equal_nan=(a_rows[k].dtype.kind == "f"))


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
def test_edge_recipe_at_its_vocabulary(dtype):
    # near-one-hot rows, exact ties, -inf padding masks, constant +1000 shifts
    _parity(synth.make("edge_16384x131072_f32", n=192, dtype=dtype))


def test_identical_rows_give_exactly_zero():
    w = synth.make_recipe("ctx", n=33, v=20000, seed=9)
    b = w.base.to(DEV)
    g_rows, gres = gpu_run(b, b.clone(), w.token_ids.to(DEV))
    assert np.all(g_rows["kld"] == 0.0)
    assert gres["mean_kld"] == 0.0 and gres["max_kld"] == 0.0 and gres["top1_agree_pct"] == 100.0


def test_constant_shift_rows_are_near_zero():
    w = synth.make_recipe("ctx", n=16, v=151936, seed=2)
    b = w.base
    q = (b + 1000.0).to(torch.float32)
    g_rows, _ = gpu_run(b.to(DEV), q.to(DEV))
    o_rows, _ = oracle.run(b, q, None, oracle.F32)
    assert np.all(np.abs(g_rows["kld"]) <= 1e-6)
    assert_rows_match(g_rows, o_rows)


@pytest.mark.parametrize("split", [None, -1])
@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
def test_dominant_element_at_every_gap_above_the_rest(dtype, split):
    # One element far enough above the rest to hold most of the mass, placed
    # late in its row (after the running maximum has settled), at gaps from
    # a fraction of a nat to well past the frame's move threshold; small
    # quant noise so that the KL is tiny and any centring error would show.
    gaps = [0.25, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0, 6.0, 8.0, 10.0, 12.0, 16.0, 24.0]
    v = 32768
    g = torch.Generator().manual_seed(21)
    rows_b, rows_q = [], []
    for gap in gaps:
        for sigma in (0.003, 0.03):
            b = torch.randn(v, generator=g)
            b[-700] = b.max() + gap
            rows_b.append(b)
            rows_q.append(b + sigma * torch.randn(v, generator=g))
    b = torch.stack(rows_b)
    q = torch.stack(rows_q)
    if dtype == synth.BF16:
        b, q = b.to(torch.bfloat16), q.to(torch.bfloat16)
    tok = torch.randint(0, v, (b.shape[0],), generator=g, dtype=torch.int32)
    g_rows, gres = gpu_run(b.contiguous().to(DEV), q.contiguous().to(DEV), tok.to(DEV),
                           split=split)
    o_rows, ores = oracle.run(b.contiguous(), q.contiguous(), tok, ODT[dtype])
    assert_rows_match(g_rows, o_rows)
    assert_stats_match(gres, ores)


def test_planted_ties_lowest_index_wins():
    n, v = 64, 9000
    g = torch.Generator().manual_seed(4)
    b = torch.randn((n, v), generator=g) * 2
    q = b + 0.1 * torch.randn((n, v), generator=g)
    for i in range(n):
        k = 2 + i % 7
        idx = torch.randperm(v, generator=g)[:k]
        if i % 3 != 1:
            b[i, idx] = b[i].max() + 1.0
        if i % 3 != 0:
            q[i, idx] = q[i].max() + 1.0
    # ties straddling warp chunks, tiles and the unaligned head/tail
    b[0, [0, 1, 4095, 8191, 8999]] = 50.0
    q[1, [8999, 3]] = 60.0
    b, q = b.float().contiguous(), q.float().contiguous()
    g_rows, _ = gpu_run(b.to(DEV), q.to(DEV))
    o_rows, _ = oracle.run(b, q, None, oracle.F32)
    assert_rows_match(g_rows, o_rows)
    assert g_rows["amax_b"][0] == 0 and g_rows["amax_q"][1] == 3


def test_special_rows_policy():
    n, v = 12, 777
    gen = torch.Generator().manual_seed(1)
    b = torch.randn((n, v), generator=gen)
    q = b + 0.2 * torch.randn((n, v), generator=gen)
    b[1, 5] = math.nan
    q[2, 700] = math.inf
    b[3, :] = -math.inf
    q[4, :] = -math.inf
    q[5, 17] = -math.inf          # b finite where q = -inf: KL = +inf
    b[6, 3] = -300.0              # exp underflows in fp32, q = -inf there: still +inf
    q[6, 3] = -math.inf
    b[7, 100:] = -math.inf        # padding mask in both
    q[7, 100:] = -math.inf
    b[8, 0] = -math.inf           # base mask only
    q[9, 400] = -math.inf         # target token masked in quant: NLL = +inf
    tok = torch.randint(0, v, (n,), generator=gen, dtype=torch.int32)
    tok[9] = 400
    tok[10] = -1                  # out of range
    tok[11] = v
    b, q = b.contiguous(), q.contiguous()
    g_rows, gres = gpu_run(b.to(DEV), q.to(DEV), tok.to(DEV))
    o_rows, ores = oracle.run(b, q, tok, oracle.F32)
    assert_rows_match(g_rows, o_rows)
    assert_stats_match(gres, ores)
    assert gres["status"] == 5  # KLD_ERR_NONFINITE: rows excluded, stats of the rest valid


def test_without_token_ids():
    w = synth.make_recipe("small", n=20, v=1000)
    g_rows, gres = gpu_run(w.base.to(DEV), w.quant.to(DEV), None)
    o_rows, ores = oracle.run(w.base, w.quant, None, oracle.F32)
    assert_rows_match(g_rows, o_rows)
    assert_stats_match(gres, ores)
    assert gres["has_nll"] == 0 and math.isnan(gres["ppl"])


def test_run_host_matches_device_run():
    w = synth.make_recipe("ctx", n=300, v=8193, dtype=synth.BF16, seed=8)
    b, q, t = w.base.pin_memory(), w.quant.pin_memory(), w.token_ids.pin_memory()
    st = KLDStats(max_rows=300, device=DEV)
    st.run_host(b, q, t)
    hres = st.result()
    st.run(b.to(DEV), q.to(DEV), t.to(DEV))
    dres = st.result()
    st.close()
    for k in dres:
        a, c = hres[k], dres[k]
        assert a == c or (isinstance(a, float) and math.isnan(a) and math.isnan(c)), k


def test_timing_api_reports_kernel_times():
    w = synth.make_recipe("ctx", n=64, v=32000, seed=1)
    st = KLDStats(max_rows=64, device=DEV)
    st.set_timing(True)
    st.run(w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV))
    st.result()
    rp, rd = st.timing()
    st.close()
    assert rp > 0 and rd > 0


def test_handle_reuse_across_sizes_and_dtypes():
    st = KLDStats(max_rows=50, device=DEV)
    for n, v, dt in [(50, 1000, synth.F32), (3, 70000, synth.BF16), (17, 5, synth.F16)]:
        w = synth.make_recipe("ctx", n=n, v=v, dtype=dt, seed=n)
        st.run(w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV))
        gres = st.result()
        _, ores = oracle.run(w.base, w.quant, w.token_ids, ODT[dt])
        assert_stats_match({**gres}, ores)
    st.close()


def test_per_field_row_arrays_match_records_and_oracle():
    # kld_stats_rows: four device arrays (KL, NLL, both argmaxes) taken from
    # the records of the last run, including excluded rows (NaN / -1) and a
    # run that reused the handle with fewer rows.
    import ctypes

    from logit_kl_divergence_b200 import _lib, rows_view

    st = KLDStats(max_rows=300, device=DEV)
    for n, seed in ((300, 8), (37, 9)):
        w = synth.make_recipe("edge", n=n, v=4099, dtype=synth.F32, seed=seed)
        st.run(w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV))
        st.result()
        soa = {k: v.cpu().numpy() for k, v in st.rows().items()}
        rec = {k: v.cpu().numpy() for k, v in rows_view(st.records()).items()}
        # the same call through the C ABI with some outputs not requested
        lib = _lib.load()
        p = ctypes.c_void_p()
        assert lib.kld_stats_rows(st._h, None, None, ctypes.byref(p), None) == _lib.KLD_OK
        assert p.value
        for k in ("kld", "nll"):
            assert soa[k].shape == (n,)
            np.testing.assert_array_equal(soa[k], rec[k])  # NaN positions included
        np.testing.assert_array_equal(soa["amax_b"], rec["amax_b"])
        np.testing.assert_array_equal(soa["amax_q"], rec["amax_q"])
        o_rows, _ = oracle.run(w.base, w.quant, w.token_ids, ODT[synth.F32])
        np.testing.assert_array_equal(soa["amax_b"], o_rows["amax_b"])
        np.testing.assert_array_equal(soa["amax_q"], o_rows["amax_q"])
        ok = np.isnan(o_rows["kld"]) & np.isnan(soa["kld"])
        ok |= np.abs(soa["kld"] - o_rows["kld"]) <= 1e-6 + 1e-4 * np.abs(o_rows["kld"])
        ok |= np.isinf(o_rows["kld"]) & (soa["kld"] == o_rows["kld"])
        assert ok.all()
    st.close()


def test_per_field_rows_before_any_run_is_not_ready():
    import ctypes

    from logit_kl_divergence_b200 import _lib

    st = KLDStats(max_rows=4, device=DEV)
    try:
        d = ctypes.c_void_p()
        lib = _lib.load()
        assert lib.kld_stats_rows(st._h, ctypes.byref(d), None, None, None) == _lib.KLD_ERR_NOT_READY
    finally:
        st.close()
