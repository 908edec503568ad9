"""Top-k compression of the base rows and KL of the quant rows against it
(kld_stats_run_topk) against the fp64 oracle: indices bit-exact (the k
largest base logits, ties to the lowest index, in order); log P_base and
the log rest mass within 2e-6 + 1e-6 * |ref| (fp32 outputs of fp64 values
computed from the row pass's normalisers, whose lambda = 1 + 1.4e-8 moves a
log-probability by ~1e-7); KL_topk within the per-row KL bar
1e-6 + 1e-4 * |ref|; the statistics of the same run as kld_stats_run."""
import math

import numpy as np
import pytest
import torch

import oracle
from logit_kl_divergence_b200 import KLDStats, synth

from gpu_helpers import ODT, assert_stats_match

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _close(g, o, atol, rtol, what):
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    same = (np.isnan(g) & np.isnan(o)) | (np.isinf(g) & np.isinf(o) & (np.sign(g) == np.sign(o)))
    with np.errstate(invalid="ignore"):
        ok = same | (np.abs(g - o) <= atol + rtol * np.abs(o))
    assert ok.all(), (what, np.argwhere(~ok)[:5], g[~ok][:5], o[~ok][:5])


def _check(b, q, tok, dt, k, split=None):
    st = KLDStats(max_rows=b.shape[0], device=DEV)
    if split is not None:
        st.set_split(split)
    out = st.run_topk(b.to(DEV), q.to(DEV), None if tok is None else tok.to(DEV), k=k)
    res = st.result()
    st.close()
    g = {key: t.cpu().numpy() for key, t in out.items()}
    o = oracle.topk(b, q, k, ODT[dt])
    np.testing.assert_array_equal(g["idx"], o["idx"])
    _close(g["logp"], o["logp"], 2e-6, 1e-6, "logp")
    _close(g["rest"], o["rest"], 2e-6, 1e-6, "rest")
    _close(g["kl_topk"], o["kl_topk"], 1e-6, 1e-4, "kl_topk")
    _, ores = oracle.run(b, q, tok, ODT[dt])
    assert_stats_match(res, ores)
    return g, o


@pytest.mark.parametrize("dt", [synth.F32, synth.BF16, synth.F16])
@pytest.mark.parametrize("n,v,k", [(100, 151936, 128), (40, 32000, 1), (40, 32000, 1024),
                                   (7, 4099, 128), (3, 5, 128), (9, 4096, 4096 // 4),
                                   (5, 1000, 128), (4, 1536, 1), (6, 2000, 700)])
def test_topk_matches_oracle(n, v, k, dt):
    w = synth.make_recipe("ctx", n=n, v=v, dtype=dt, seed=n + v + k)
    _check(w.base, w.quant, w.token_ids, dt, k)


def test_topk_edge_rows():
    # near-one-hot rows (T holds almost all the mass), exact ties at the top,
    # the last 1024 entries -inf, constant shifts
    w = synth.make_recipe("edge", n=200, v=131072, dtype=synth.F32, seed=8)
    g, _ = _check(w.base, w.quant, w.token_ids, synth.F32, 128)
    # KL >= 0 up to the per-row absolute bar (the +1000 rows sit at ~1e-10)
    assert np.all(g["kl_topk"][np.isfinite(g["kl_topk"])] >= -1e-6)


def test_topk_huge_tie_group_and_masks():
    n, v = 6, 60000
    gen = torch.Generator().manual_seed(2)
    b = torch.randn((n, v), generator=gen)
    q = b + 0.1 * torch.randn((n, v), generator=gen)
    b[0] = 1.0                        # one value everywhere: the lowest k indices
    b[1, 1000:] = 3.0                 # 59000-way tie above the rest
    b[2, :] = -math.inf
    b[2, 100:150] = 0.5               # 50 finite entries: T reaches p = 0
    q[3, int(torch.argmax(b[3]))] = -math.inf   # quant gives the top entry nothing
    b[4, 7] = math.nan                # excluded row
    g, o = _check(b.contiguous(), q.contiguous(), None, synth.F32, 128)
    assert list(g["idx"][0, :5]) == [0, 1, 2, 3, 4]
    assert list(g["idx"][1, :3]) == [1000, 1001, 1002]
    assert g["kl_topk"][3] == math.inf and np.all(g["idx"][4] == -1)


@pytest.mark.parametrize("dt", [synth.F32, synth.BF16])
def test_topk_tie_group_inside_the_boundary_bin(dt):
    # a few hundred equal logits at the top of a wide row: the candidates
    # hold the whole tie group and more, the bin holding the k-th largest is
    # the tie group itself, and T is its lowest k indices
    n, v = 8, 151936
    w = synth.make_recipe("ctx", n=n, v=v, dtype=synth.F32, seed=31)
    b, q = w.base.clone(), w.quant.clone()
    gen = torch.Generator().manual_seed(4)
    for i in range(n):
        cnt = [130, 300, 600, 129][i % 4]
        idx = torch.randperm(v, generator=gen)[:cnt]
        b[i, idx] = float(b[i].max()) + 1.0
    if dt == synth.BF16:
        b, q = b.to(torch.bfloat16), q.to(torch.bfloat16)
    g, _ = _check(b.contiguous(), q.contiguous(), w.token_ids, dt, 128)
    for i in range(n):
        top = np.sort(np.flatnonzero(b[i].float().numpy() == float(b[i].float().max())))[:128]
        np.testing.assert_array_equal(g["idx"][i, :128], top)


@pytest.mark.parametrize("split", [1, -1])
def test_topk_after_split_row_launches(split):
    w = synth.make_recipe("ctx", n=5, v=151936, dtype=synth.BF16, seed=77)
    _check(w.base, w.quant, w.token_ids, synth.BF16, 128, split=split)


def test_topk_never_exceeds_the_full_kl():
    w = synth.make_recipe("ctx", n=64, v=32000, dtype=synth.F32, seed=5)
    st = KLDStats(max_rows=64, device=DEV)
    out = st.run_topk(w.base.to(DEV), w.quant.to(DEV), None, k=128)
    st.result()
    full = st.rows()["kld"].cpu().numpy()  # the per-field arrays of kld_stats_rows
    st.close()
    assert np.all(out["kl_topk"].cpu().numpy() <= full + 1e-6 + 1e-4 * full)


def test_topk_pass_is_timed():
    # with timing on, the top-k pass is bracketed by its own events
    w = synth.make_recipe("ctx", n=64, v=32000, dtype=synth.F32, seed=12)
    st = KLDStats(max_rows=64, device=DEV)
    try:
        st.set_timing(True)
        st.run_topk(w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV), k=128)
        st.result()
        row_ms, red_ms = st.timing()
        topk_ms = st.second_pass_timing()
        assert 0.0 < row_ms < 100.0 and 0.0 < red_ms < 100.0 and 0.0 < topk_ms < 100.0
    finally:
        st.close()


def _sampled(v):
    # positions the threshold's samples read: 512 evenly spaced runs of 8
    cover = np.zeros(v, bool)
    for i in range(512):
        s = (i * (v - 8) // 512) & ~7
        cover[s:s + 8] = True
    return cover


@pytest.mark.parametrize("dt", [synth.F32, synth.BF16])
def test_topk_scan_takes_the_fast_path(dt):
    # rows longer than the candidate capacity: thresholds first, the row
    # pass copies the lanes holding candidates, the top-k pass reads only
    # those; no row of the benchmark's recipe needs the exact path
    w = synth.make_recipe("ctx", n=48, v=151936, dtype=dt, seed=41)
    st = KLDStats(max_rows=48, device=DEV)
    try:
        out = st.run_topk(w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV), k=128)
        st.result()
        assert st.topk_exact_rows() == 0
        g = {key: t.cpu().numpy() for key, t in out.items()}
    finally:
        st.close()
    o = oracle.topk(w.base, w.quant, 128, ODT[dt])
    np.testing.assert_array_equal(g["idx"], o["idx"])
    _close(g["rest"], o["rest"], 2e-6, 1e-6, "rest")
    _close(g["kl_topk"], o["kl_topk"], 1e-6, 1e-4, "kl_topk")


@pytest.mark.parametrize("dt", [synth.F32, synth.BF16])
def test_topk_scan_overflow_direct_chunks_and_misaligned_rows(dt):
    # row 0: 3000 high logits where the samples do not look, so far more
    # than the copy regions hold pass the threshold (the row is read again
    # with the same threshold); row 1: the quant row far from the base row
    # everywhere (every chunk takes the direct path and is copied whole);
    # row 2: three chunks with quant spikes (a few direct-path chunks);
    # rows 3-5 ordinary; V odd, so rows start at every misalignment
    n, v = 6, 151937
    w = synth.make_recipe("ctx", n=n, v=v, dtype=synth.F32, seed=43)
    b, q = w.base.clone(), w.quant.clone()
    gen = torch.Generator().manual_seed(5)
    free = np.flatnonzero(~_sampled(v))
    pos = torch.from_numpy(free[torch.randperm(len(free), generator=gen)[:3000].numpy()])
    b[0, pos] = float(b[0].max()) + 2.0
    q[1] = b[1] + 5.0 * torch.randn(v, generator=gen)
    for c in (3, 100, 250):
        q[2, c * 512 + 17] = float(q[2].max()) + 30.0
    if dt == synth.BF16:
        b, q = b.to(torch.bfloat16), q.to(torch.bfloat16)
    st = KLDStats(max_rows=n, device=DEV)
    try:
        out = st.run_topk(b.contiguous().to(DEV), q.contiguous().to(DEV), w.token_ids.to(DEV), k=128)
        st.result()
        assert st.topk_exact_rows() == 0
        g = {key: t.cpu().numpy() for key, t in out.items()}
    finally:
        st.close()
    o = oracle.topk(b.contiguous(), q.contiguous(), 128, ODT[dt])
    np.testing.assert_array_equal(g["idx"], o["idx"])
    _close(g["logp"], o["logp"], 2e-6, 1e-6, "logp")
    _close(g["rest"], o["rest"], 2e-6, 1e-6, "rest")
    _close(g["kl_topk"], o["kl_topk"], 1e-6, 1e-4, "kl_topk")


def test_topk_exact_rows_before_any_topk():
    st = KLDStats(max_rows=4, device=DEV)
    try:
        with pytest.raises(Exception):
            st.topk_exact_rows()
    finally:
        st.close()
