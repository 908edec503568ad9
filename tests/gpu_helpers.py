"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare with the fp64 oracle at the stated tolerances.

Tolerances: argmax indices, flags and agreement counts bit-exact; per-row KL
and NLL (quant and base) |gpu - ref| <= 1e-6 + 1e-4 * |ref|; mean KLD,
percentiles, mean NLL and PPL (quant and base), the PPL ratio and the mean
and RMS of dp within 1e-5 relative, with an absolute floor where the
reference is ~0 (1e-9 nats for KL statistics, 1e-7 nats for mean NLL, i.e.
1e-7 relative for PPL): fp32 inputs do not resolve a log-probability better
than that. The dp statistics take a floor of 5e-8: a row's dp carries the
absolute rounding of its two NLLs (fp32 exponentials in the row pass, ~1e-8
where the NLL is ~0, as in single-token vocabularies), far inside the dp bar
the per-row NLL bars allow (~1e-6). ln(PPL ratio) within 1e-5 absolute is the
ratio within 1e-5 relative.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import oracle
from logit_kl_divergence_b200 import KLDStats, rows_view, synth

ODT = {synth.F32: oracle.F32, synth.BF16: oracle.BF16, synth.F16: oracle.F16}
EXCLUDED = oracle.ROW_NONFINITE | oracle.ROW_EMPTY
ROW_ATOL, ROW_RTOL = 1e-6, 1e-4
STAT_RTOL = 1e-5
STAT_ATOL = {"mean_kld": 1e-9, "median_kld": 1e-9, "p90_kld": 1e-9, "p99_kld": 1e-9,
             "max_kld": 1e-9, "mean_nll": 1e-7, "mean_nll_base": 1e-7, "top1_agree_pct": 0.0,
             "mean_dp": 5e-8, "rms_dp": 5e-8}
CORES = max(1, os.cpu_count() or 1)


def gpu_run(base, quant, tok=None, use_rows_api=False, split=None):
    """The whole statistic on the GPU; returns (per-row numpy dict, result).
    ``split``: the handle's few-row launch shape (kld_stats_set_split)."""
    st = KLDStats(max_rows=base.shape[0], device=base.device)
    if split is not None:
        st.set_split(split)
    try:
        if use_rows_api:
            out = torch.empty((base.shape[0], 40), dtype=torch.uint8, device=base.device)
            st.run_rows(base, quant, tok, out=out)
            st.reduce(out, base.shape[0], tok is not None)
            res = st.result()
            rec = rows_view(out)
        else:
            st.run(base, quant, tok)
            res = st.result()
            rec = rows_view(st.records())
        rows = {k: v.cpu().numpy() for k, v in rec.items()}
        rows["flags"] = rows["flags"].astype(np.uint32)
        return rows, res
    finally:
        st.close()


def _close_rows(g, o, what, idx):
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    both_nan = np.isnan(g) & np.isnan(o)
    both_inf = np.isinf(g) & np.isinf(o) & (np.sign(g) == np.sign(o))
    ok = both_nan | both_inf | (np.abs(g - o) <= ROW_ATOL + ROW_RTOL * np.abs(o))
    if not ok.all():
        bad = np.nonzero(~ok)[0][:8]
        raise AssertionError(f"{what} mismatch at rows {idx[bad]}: gpu={g[bad]} ref={o[bad]}")


def _close_dp(g, o, tol, idx):
    ok = (np.isnan(g) & np.isnan(o)) | (np.abs(g - o) <= tol + 6e-8 * np.abs(o))
    if not ok.all():
        bad = np.nonzero(~ok)[0][:8]
        raise AssertionError(f"dp mismatch at rows {idx[bad]}: gpu={g[bad]} ref={o[bad]}")


def assert_rows_match(g: dict, o: dict, idx=None):
    n = len(o["kld"])
    idx = np.arange(n) if idx is None else np.asarray(idx)
    assert np.array_equal(g["flags"], o["flags"]), (
        f"flags differ at rows {idx[np.nonzero(g['flags'] != o['flags'])[0][:8]]}")
    assert np.array_equal(g["amax_b"], o["amax_b"]), (
        f"argmax_base differs at rows {idx[np.nonzero(g['amax_b'] != o['amax_b'])[0][:8]]}")
    assert np.array_equal(g["amax_q"], o["amax_q"]), (
        f"argmax_quant differs at rows {idx[np.nonzero(g['amax_q'] != o['amax_q'])[0][:8]]}")
    _close_rows(g["kld"], o["kld"], "kld", idx)
    _close_rows(g["nll"], o["nll"], "nll", idx)
    _close_rows(g["nll_base"], o["nll_base"], "nll_base", idx)
    # dp = P_quant(tok) - P_base(tok), fp32 in the record: each NLL within its
    # bar (ROW_ATOL + ROW_RTOL * NLL) moves its probability by that much
    # relative, plus fp32 rounding
    with np.errstate(invalid="ignore", over="ignore"):
        nq, nb = np.asarray(o["nll"], np.float64), np.asarray(o["nll_base"], np.float64)
        pq, pb = np.exp(-nq), np.exp(-nb)
        tol = (pq * (ROW_ATOL + ROW_RTOL * np.nan_to_num(nq, posinf=0.0))
               + pb * (ROW_ATOL + ROW_RTOL * np.nan_to_num(nb, posinf=0.0)) + 1e-12)
    _close_dp(np.asarray(g["dp"], np.float64), pq - pb, tol, idx)


def stat_close(a, b, key):
    if (isinstance(a, float) and math.isnan(a)) or (isinstance(b, float) and math.isnan(b)):
        return math.isnan(a) and math.isnan(b)
    if math.isinf(a) or math.isinf(b):
        return a == b
    if key in ("ppl", "ppl_base"):
        return abs(a - b) <= (STAT_RTOL + 1e-7) * abs(b)
    if key == "ln_ppl_ratio":
        # the ratio PPL(Q)/PPL(base) within STAT_RTOL relative
        return abs(a - b) <= STAT_RTOL
    return abs(a - b) <= STAT_ATOL[key] + STAT_RTOL * abs(b)


def assert_stats_match(gres: dict, ores: dict):
    for k in ("n_rows", "n_valid", "top1_agree", "n_nll", "n_flagged", "flags_or", "has_nll"):
        assert int(gres[k]) == int(ores[k]), (k, gres[k], ores[k])
    for k in ("mean_kld", "median_kld", "p90_kld", "p99_kld", "max_kld", "top1_agree_pct",
              "mean_nll", "ppl", "mean_nll_base", "ppl_base", "ln_ppl_ratio", "mean_dp", "rms_dp"):
        assert stat_close(gres[k], ores[k], k), (k, gres[k], ores[k])
    assert gres["device_error"] == 0


def assert_select_exact(g_rows: dict, gres: dict, has_nll: bool):
    """The GPU's percentiles are the exact order statistics of its own per-row
    array (the oracle's std::sort + interpolation applied to the same values)."""
    ref = oracle.reduce(g_rows, has_nll)
    for k in ("median_kld", "p90_kld", "p99_kld", "max_kld"):
        a, b = gres[k], ref[k]
        assert (a == b) or (math.isnan(a) and math.isnan(b)), (k, a, b)
    for k in ("n_valid", "top1_agree", "n_nll", "n_flagged", "flags_or"):
        assert int(gres[k]) == int(ref[k]), k


def oracle_rows_chunked(w, nthreads=CORES, chunk_rows=1024):
    """Oracle per-row values of a device workload, computed on host chunks."""
    n = w.base.shape[0]
    out = {k: [] for k in ("kld", "nll", "nll_base", "amax_b", "amax_q", "flags")}
    for r0 in range(0, n, chunk_rows):
        r1 = min(n, r0 + chunk_rows)
        b = w.base[r0:r1].cpu()
        q = w.quant[r0:r1].cpu()
        t = w.token_ids[r0:r1].cpu() if w.token_ids is not None else None
        r = oracle.rows(b, q, t, ODT[w.dtype], nthreads)
        for k in out:
            out[k].append(r[k])
    return {k: np.concatenate(v) for k, v in out.items()}
