"""Split-row launches (few rows: each row's chunks spread over several CTAs
whose partial sums merge through global memory, or over thread-block
clusters whose partials merge in shared memory first) against the fp64 CPU
oracle.

Rows fewer than the SMs are all split. By default a row is split over plain
CTAs by balanced chunk ranges (kld_stats_set_split(1)); the cluster shapes
(2, 4, 8 CTAs, combined through distributed shared memory) and whole-row
launches (-1) are selected explicitly here. The cases put maxima, ties, NaN, masks and the target token
in parts other than the first, leave parts with no chunk at small
vocabularies, and reuse one handle so that the per-row arrival counters must
come back to zero after every launch.
"""
import ctypes
import math
import struct

import numpy as np
import pytest
import torch

import oracle
from logit_kl_divergence_b200 import KLDStats, _lib, dtype_code, synth

from gpu_helpers import ODT, assert_rows_match, assert_select_exact, assert_stats_match, gpu_run

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
V_FULL = 151936


def _sm_count():
    return torch.cuda.get_device_properties(DEV).multi_processor_count


SHAPES = [1, 2, 4, 8]  # split over plain CTAs, then clusters of up to 2, 4, 8 CTAs


def _parity(base, quant, tok, odt, split=None):
    g_rows, gres = gpu_run(base.to(DEV), quant.to(DEV), None if tok is None else tok.to(DEV),
                           split=split)
    o_rows, ores = oracle.run(base, quant, tok, odt)
    assert_rows_match(g_rows, o_rows)
    assert_stats_match(gres, ores)
    assert_select_exact(g_rows, gres, tok is not None)
    return g_rows, gres


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("n", [1, 2, 3, 4, 7, 9, 16, 20, 37, 38, 64, 74])
def test_split_rows_full_vocabulary(n, dtype):
    st = KLDStats(max_rows=n, device=DEV)
    p = st.plan(n, V_FULL, _lib.KLD_F32 if dtype == synth.F32 else _lib.KLD_BF16)
    st.close()
    if 2 * n <= _sm_count():
        assert p["variant"] == 2 and p["whole_rounds"] == 0 and p["ctas_per_row"] >= 2
    w = synth.make_recipe("ctx", n=n, v=V_FULL, dtype=dtype, seed=100 + n)
    _parity(w.base, w.quant, w.token_ids, ODT[dtype])


@pytest.mark.parametrize("split", SHAPES + [-1])
@pytest.mark.parametrize("n", [1, 3, 9, 20, 38, 74])
def test_every_launch_shape_full_vocabulary(n, split):
    w = synth.make_recipe("ctx", n=n, v=V_FULL, dtype=synth.F32, seed=200 + n)
    _parity(w.base, w.quant, w.token_ids, oracle.F32, split=split)


@pytest.mark.parametrize("split", [1, 8])
@pytest.mark.parametrize("v", [1, 7, 512, 513, 1024, 4097, 16385, 100003])
def test_split_rows_small_vocabularies_leave_parts_empty(v, split):
    w = synth.make_recipe("ctx", n=2, v=v, dtype=synth.F16, seed=v)
    _parity(w.base, w.quant, w.token_ids, oracle.F16, split=split)


@pytest.mark.parametrize("split", SHAPES)
def test_split_rows_ties_across_parts_lowest_index_wins(split):
    n, v = 3, V_FULL
    g = torch.Generator().manual_seed(11)
    b = torch.randn((n, v), generator=g)
    q = b + 0.1 * torch.randn((n, v), generator=g)
    b[0, [150000, 70001, 70000, 151935]] = 30.0      # lowest tie in a middle part
    q[0, [151935, 99999]] = 40.0
    b[1, [151935, 1]] = 30.0                          # head element vs last element
    q[1, [0, 151935]] = 40.0
    b[2, [151000, 150999]] = 30.0                     # both in the last part
    q[2, [2047, 2048, 4095]] = 40.0
    g_rows, _ = _parity(b.contiguous(), q.contiguous(), None, oracle.F32, split=split)
    assert list(g_rows["amax_b"]) == [70000, 1, 150999]
    assert list(g_rows["amax_q"]) == [99999, 0, 2047]


@pytest.mark.parametrize("split", SHAPES)
def test_split_rows_special_values_in_later_parts(split):
    n, v = 6, V_FULL
    g = torch.Generator().manual_seed(12)
    b = torch.randn((n, v), generator=g)
    q = b + 0.3 * torch.randn((n, v), generator=g)
    b[0, :100000] = -math.inf                         # parts with quant weight only
    q[0, :100000] += 2.0
    b[1] -= 1000.0                                    # deep frames, same masks
    q[1] -= 1000.0
    b[1, :100000] = -math.inf
    b[2, 150000] = math.nan                           # NaN in the last part
    q[3, 140000] = -math.inf                          # KL = +inf from a late part
    b[4, :] = -math.inf                               # one finite base entry, late
    b[4, 151000] = 3.0
    q[5, 120000:] = -math.inf                         # quant mask over the last parts
    b[5, 120000:] = -math.inf
    tok = torch.tensor([5, 50000, 7, 140000, 151000, 130000], dtype=torch.int32)
    g_rows, gres = _parity(b.contiguous(), q.contiguous(), tok, oracle.F32, split=split)
    assert g_rows["amax_b"][4] == 151000
    assert math.isinf(g_rows["kld"][3]) and math.isinf(g_rows["nll"][3])
    assert math.isinf(g_rows["nll"][5])


def test_split_rows_repeat_launches_on_one_handle():
    st = KLDStats(max_rows=8, device=DEV)
    try:
        for n, v, dt, seed, split in [(1, V_FULL, synth.F32, 1, 0), (5, 70001, synth.BF16, 2, 8),
                                      (1, V_FULL, synth.F32, 3, 4), (8, 4097, synth.F16, 4, 1),
                                      (2, V_FULL, synth.BF16, 5, 2), (3, V_FULL, synth.F32, 6, -1),
                                      (1, V_FULL, synth.F32, 7, 0)]:
            st.set_split(split)
            w = synth.make_recipe("ctx", n=n, v=v, dtype=dt, seed=seed)
            st.run(w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV))
            gres = st.result()
            _, ores = oracle.run(w.base, w.quant, w.token_ids, ODT[dt])
            assert_stats_match(dict(gres), ores)
    finally:
        st.close()


def _same_bits(a, b):
    if isinstance(a, float) or isinstance(b, float):
        if math.isnan(a) and math.isnan(b):
            return True
        return struct.pack("<d", a) == struct.pack("<d", b)
    return a == b


@pytest.mark.parametrize("split", [1, 2, 8])
@pytest.mark.parametrize("n", [1, 2, 5, 16, 31, 32, 33])
def test_few_split_rows_reduce_in_the_row_pass_like_the_reduction_kernel(n, split):
    # A split launch of at most 32 rows reduces its own records (the warp
    # that finalises the last row does it): its result must equal the
    # reduction kernel's on the same records bit for bit, with excluded
    # rows, a bad token and no tokens at all, over repeated launches on one
    # handle (the launch counter must come back to zero). 33 rows take the
    # reduction kernel both ways.
    v = 70001
    w = synth.make_recipe("ctx", n=n, v=v, dtype=synth.F32, seed=100 + n)
    b, q, t = w.base.clone(), w.quant.clone(), w.token_ids.clone()
    if n >= 5:
        b[1, 17] = math.nan   # excluded row
        t[3] = v + 5          # token outside the vocabulary
    bd, qd, td = b.to(DEV), q.to(DEV), t.to(DEV)
    st = KLDStats(max_rows=n, device=DEV)
    try:
        st.set_split(split)
        for tok in (td, None, td):
            st.run(bd, qd, tok)
            fused = st.result()
            st.run_rows(bd, qd, tok)
            st.reduce(None, n, tok is not None)
            ref = st.result()
            assert fused.keys() == ref.keys()
            for k in fused:
                assert _same_bits(fused[k], ref[k]), (k, fused[k], ref[k])
            _, ores = oracle.run(b, q, None if tok is None else t, oracle.F32)
            assert_stats_match(fused, ores)
    finally:
        st.close()


def test_split_rows_agree_with_whole_row_launch():
    # kld_stats_run_static keeps whole rows at any N: the same rows through
    # both launch shapes must agree with the oracle.
    w = synth.make_recipe("ctx", n=6, v=V_FULL, dtype=synth.BF16, seed=13)
    b, q, t = w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV)
    lib = _lib.load()
    out = torch.zeros(ctypes.sizeof(_lib.Result), dtype=torch.uint8, device=DEV)
    stream = torch.cuda.current_stream(DEV)
    st = lib.kld_stats_run_static(ctypes.c_void_p(b.data_ptr()), ctypes.c_void_p(q.data_ptr()),
                                  ctypes.c_void_p(t.data_ptr()), 6, V_FULL, dtype_code(b),
                                  ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
    assert st == _lib.KLD_OK
    stream.synchronize()
    res = _lib.Result.from_buffer_copy(bytes(out.cpu().numpy()))
    whole = {name: getattr(res, name) for name, _ in _lib.Result._fields_ if not name.startswith("reserved")}
    _, split = gpu_run(b, q, t)
    _, ores = oracle.run(w.base, w.quant, w.token_ids, oracle.BF16)
    for r in (whole, split):
        assert int(r["top1_agree"]) == int(ores["top1_agree"])
        for k in ("mean_kld", "median_kld", "max_kld", "mean_nll"):
            assert math.isclose(r[k], ores[k], rel_tol=1e-5, abs_tol=1e-9), (k, r[k], ores[k])


def test_set_split_rejects_unknown_shapes():
    st = KLDStats(max_rows=4, device=DEV)
    try:
        for bad in (-2, 3, 5, 16):
            with pytest.raises(_lib.KLDError):
                st.set_split(bad)
        for ok in (-1, 0, 1, 2, 4, 8):
            st.set_split(ok)
    finally:
        st.close()


def test_few_split_rows_time_no_separate_reduction():
    # the row pass of a few-row split launch includes the reduction: the
    # reduction's events sit back to back; whole-row launches still run the
    # reduction kernel after the row pass
    w = synth.make_recipe("ctx", n=4, v=V_FULL, dtype=synth.F32, seed=41)
    b, q, t = w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV)
    st = KLDStats(max_rows=4, device=DEV)
    try:
        st.set_timing(True)
        st.run(b, q, t)
        fused = st.result()
        row_ms, red_ms = st.timing()
        assert row_ms > 0.0 and 0.0 <= red_ms < 0.01, (row_ms, red_ms)
        st.set_split(-1)
        st.run(b, q, t)
        whole = st.result()
        row2_ms, red2_ms = st.timing()
        assert row2_ms > 0.0 and red2_ms > 0.0
        assert fused["top1_agree"] == whole["top1_agree"]
        assert math.isclose(fused["mean_kld"], whole["mean_kld"], rel_tol=1e-5, abs_tol=1e-9)
    finally:
        st.close()
