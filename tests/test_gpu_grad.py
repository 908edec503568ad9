"""Gradient of KL(P_base || P_quant) with respect to the quant logits
(kld_stats_run_grad) against the fp64 oracle: every element within
|scale| * (4e-6 * (p + r) + 1e-12) for fp32 output, where p and r are the
two softmax values of the element. Each is an fp32 exponential of the row
pass's normalisers: rounding of its argument (<= |arg| * 2^-25 * ln 2, about
6e-7 for |arg| <= 24), ex2.approx (<= 2^-22), the normaliser (2^-24) and the
lambda = 1 + 1.4e-8 of the row pass (<= ~3e-7) add up to ~1.3e-6 per value,
so 4e-6 on the sum is a ~3x margin. The quant normaliser comes from the fp32
log-ratios x = (q - b) + K of the row pass, each rounded by up to
2^-24 * |q - b|: for rows whose quant is offset from the base by a large
constant (the +1000 rows of the edge recipe) that adds
2^-23 * max |q - b| relative to r (6e-5 at an offset of 1000, 2e-7 for
ordinary rows); plus half a rounding step for
16-bit outputs (f16's fixed absolute step below its smallest normal too); zero rows where the statistics exclude the row; the
statistics of the same run equal those of kld_stats_run."""
import math

import numpy as np
import pytest
import torch

import oracle
from logit_kl_divergence_b200 import KLDStats, synth

from gpu_helpers import ODT, assert_stats_match

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _softmax64(x):
    x = x.astype(np.float64)
    m = np.max(x, axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(x - m)
    return e / e.sum(axis=1, keepdims=True)


def _check(b, q, tok, dt, out_dtype, scale=1.0, split=None):
    st = KLDStats(max_rows=b.shape[0], device=DEV)
    if split is not None:
        st.set_split(split)
    g = st.run_grad(b.to(DEV), q.to(DEV), None if tok is None else tok.to(DEV), scale=scale,
                    grad_dtype=out_dtype)
    res = st.result()
    st.close()
    ref = oracle.grad(b, q, ODT[dt], scale)
    got = g.float().cpu().numpy().astype(np.float64)
    bb = b.float().numpy() if dt != synth.F32 else b.numpy()
    qq = q.float().numpy() if dt != synth.F32 else q.numpy()
    with np.errstate(invalid="ignore", over="ignore"):
        p, r = _softmax64(bb), _softmax64(qq)
    with np.errstate(invalid="ignore"):
        d = np.abs(qq.astype(np.float64) - bb.astype(np.float64))
    off = np.nanmax(np.where(np.isfinite(d), d, np.nan), axis=1, initial=0.0)[:, None]
    tol = abs(scale) * (4e-6 * (np.nan_to_num(p) + np.nan_to_num(r))
                        + 2.0 ** -23 * off * np.nan_to_num(r) + 1e-12)
    if out_dtype == torch.bfloat16:
        tol = tol + np.abs(ref) * 2.0 ** -8
    elif out_dtype == torch.float16:
        # half a step of f16 rounding: 2^-11 relative, 2^-25 absolute below
        # the smallest normal (the subnormal spacing is 2^-24)
        tol = tol + np.abs(ref) * 2.0 ** -11 + 2.0 ** -25
    bad = np.abs(got - ref) > tol
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], ref[bad][:5])
    _, ores = oracle.run(b, q, tok, ODT[dt])
    assert_stats_match(res, ores)
    return got


@pytest.mark.parametrize("dt,out", [(synth.F32, torch.float32), (synth.BF16, torch.float32),
                                    (synth.BF16, torch.bfloat16), (synth.F16, torch.float16)])
@pytest.mark.parametrize("n,v", [(64, 32000), (150, 151936), (7, 4099), (3, 5)])
def test_grad_matches_oracle(n, v, dt, out):
    w = synth.make_recipe("ctx", n=n, v=v, dtype=dt, seed=n + v)
    _check(w.base, w.quant, w.token_ids, dt, out, scale=1.0 / n)


def test_grad_rows_sum_to_zero_and_excluded_rows_are_zero():
    w = synth.make_recipe("edge", n=200, v=8192, dtype=synth.F32, seed=3)
    b, q = w.base.clone(), w.quant.clone()
    b[5, 17] = math.nan
    q[9, :] = -math.inf
    got = _check(b, q, w.token_ids, synth.F32, torch.float32, scale=2.0)
    assert np.all(got[5] == 0.0) and np.all(got[9] == 0.0)
    assert np.max(np.abs(got.sum(axis=1))) < 1e-4


@pytest.mark.parametrize("split", [1, 8, -1])
def test_grad_after_split_row_launches(split):
    w = synth.make_recipe("ctx", n=5, v=151936, dtype=synth.BF16, seed=41)
    _check(w.base, w.quant, w.token_ids, synth.BF16, torch.float32, scale=0.5, split=split)


def test_grad_unaligned_output_takes_the_scalar_path():
    w = synth.make_recipe("ctx", n=9, v=5003, dtype=synth.F32, seed=5)
    st = KLDStats(max_rows=9, device=DEV)
    buf = torch.empty(9 * 5003 + 1, dtype=torch.float32, device=DEV)
    out = buf[1:].view(9, 5003)
    st.run_grad(w.base.to(DEV), w.quant.to(DEV), None, out=out)
    st.result()
    st.close()
    ref = oracle.grad(w.base, w.quant)
    assert np.max(np.abs(out.cpu().numpy() - ref)) < 2e-6


def test_identical_rows_give_exactly_zero_gradient():
    w = synth.make_recipe("ctx", n=20, v=20000, seed=9)
    b = w.base.to(DEV)
    st = KLDStats(max_rows=20, device=DEV)
    g = st.run_grad(b, b.clone(), None)
    st.result()
    st.close()
    assert torch.all(g == 0)
