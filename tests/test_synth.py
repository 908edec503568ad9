"""The seeded workload generator draws what its recipes state."""
import math

import numpy as np
import torch

from logit_kl_divergence_b200 import synth


def test_seeded_and_deterministic():
    a = synth.make("small_64x32000_f32", n=8, v=1000)
    b = synth.make("small_64x32000_f32", n=8, v=1000)
    assert torch.equal(a.base, b.base) and torch.equal(a.quant, b.quant)
    assert torch.equal(a.token_ids, b.token_ids)
    c = synth.make("small_64x32000_f32", n=8, v=1000, seed=7)
    assert not torch.equal(a.base, c.base)


def test_named_shapes_and_dtypes():
    w = synth.make("ctx8192_v151936_bf16", n=4, v=2048)
    assert w.base.dtype == torch.bfloat16 and w.base.shape == (4, 2048)
    assert w.token_ids.dtype == torch.int32
    assert synth.WORKLOADS["ctx8192_v151936_f32"][1:4] == (8192, 151936, synth.F32)
    assert synth.WORKLOADS["ctx4x8192_v151936_bf16"][1:4] == (32768, 151936, synth.BF16)
    assert synth.WORKLOADS["edge_16384x131072_f32"][1:4] == (16384, 131072, synth.F32)


def test_small_recipe_has_one_peak_per_row():
    # with the background switched off only the +8 peak remains
    b, _, _ = synth._small(16, 500, synth.F32, 0, torch.device("cpu"), std=0.0)
    assert np.all((b.numpy() == 8.0).sum(axis=1) == 1)
    assert np.all((b.numpy() == 0.0).sum(axis=1) == 499)
    w = synth.make("small_64x32000_f32")
    noise = (w.quant - w.base).numpy()
    assert abs(noise.std() - 0.25) < 0.01


def test_ctx_recipe_noise_levels_and_tokens():
    w = synth.make("ctx8192_v151936_f32", n=64, v=4096)
    sig = (w.quant - w.base).std(dim=1).numpy()
    for s in sig:
        assert min(abs(s - t) for t in (0.05, 0.15, 0.4)) < 0.02
    assert int(w.token_ids.min()) >= 0 and int(w.token_ids.max()) < 4096


def test_edge_recipe_groups():
    n, v = 64, 4096
    w = synth.make("edge_16384x131072_f32", n=n, v=v)
    b, q = w.base.numpy(), w.quant.numpy()
    masked = np.all(np.isneginf(b[:, -1024:]), axis=1) & np.all(np.isneginf(q[:, -1024:]), axis=1)
    shifted = np.all(np.abs((q - b) - 1000.0) < 0.01, axis=1)
    assert masked.sum() == n // 4 and shifted.sum() == n // 4
    ties_b = (b == b.max(axis=1, keepdims=True)).sum(axis=1)
    ties_q = (q == q.max(axis=1, keepdims=True)).sum(axis=1)
    tie_rows = (ties_b >= 2) | (ties_q >= 2)
    assert tie_rows.sum() == n // 4
    assert np.all(np.maximum(ties_b, ties_q)[tie_rows] <= 8)
    hot = (np.sort(b, axis=1)[:, -1] - np.sort(b, axis=1)[:, -2]) > 20
    assert hot.sum() == n // 4
    # sampled tokens never land on masked entries
    assert np.all(np.isfinite(b[np.arange(n), w.token_ids.numpy()]))
