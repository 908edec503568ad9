"""Parity at the full workload sizes, in the launch configuration the
benchmark times. Inputs are generated on the GPU by the seeded generator; the
oracle recomputes every row on the host cores, chunk by chunk."""
import math

import numpy as np
import pytest
import torch

import oracle
from logit_kl_divergence_b200 import synth

from gpu_helpers import (assert_rows_match, assert_select_exact, assert_stats_match, gpu_run,
                         oracle_rows_chunked)

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _full(name, **kw):
    w = synth.make(name, device=DEV, **kw)
    g_rows, gres = gpu_run(w.base, w.quant, w.token_ids)
    assert_select_exact(g_rows, gres, True)
    o_rows = oracle_rows_chunked(w)
    assert_rows_match(g_rows, o_rows)
    ores = oracle.reduce(o_rows, True)
    assert_stats_match(gres, ores)
    del w
    torch.cuda.empty_cache()
    return gres


def test_context_8192_v151936_f32():
    r = _full("ctx8192_v151936_f32")
    assert 0.001 < r["mean_kld"] < 0.2 and r["status"] == 0


def test_context_8192_v151936_bf16():
    r = _full("ctx8192_v151936_bf16")
    assert 0.001 < r["mean_kld"] < 0.2


def test_four_contexts_v151936_bf16():
    r = _full("ctx4x8192_v151936_bf16")
    assert r["n_rows"] == 32768


@pytest.mark.parametrize("n", [1, 4, 16, 32])
def test_split_row_sizes_v262144(n):
    _full(f"splitrow{n}_v262144_f32")


def test_edge_16384x131072():
    r = _full("edge_16384x131072_f32")
    assert r["status"] == 0 and r["n_valid"] == 16384
