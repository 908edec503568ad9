"""kld_stats_run_static, the entry point for callers that cannot allocate
device memory when they need the statistic (e.g. a server whose allocator
owns nearly all HBM), must give the same statistics as the handle-based
kld_stats_run. Called through the C ABI, twice in a row with different
inputs, so the second call also checks that the shared fixed scratch array
carries nothing over from the first. Collected last on purpose.
"""
import ctypes
import math

import pytest
import torch

from logit_kl_divergence_b200 import KLDStats, _lib, dtype_code, synth

from gpu_helpers import stat_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _static_run(base, quant, tok):
    lib = _lib.load()
    out = torch.zeros(ctypes.sizeof(_lib.Result), dtype=torch.uint8, device=DEV)
    stream = torch.cuda.current_stream(DEV)
    st = lib.kld_stats_run_static(
        ctypes.c_void_p(base.data_ptr()), ctypes.c_void_p(quant.data_ptr()),
        None if tok is None else ctypes.c_void_p(tok.data_ptr()),
        base.shape[0], base.shape[1], dtype_code(base), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(stream.cuda_stream))
    assert st == _lib.KLD_OK, lib.kld_status_string(st)
    stream.synchronize()
    res = _lib.Result.from_buffer_copy(bytes(out.cpu().numpy()))
    return {name: getattr(res, name) for name, _ in _lib.Result._fields_ if not name.startswith("reserved")}


def _handle_run(base, quant, tok):
    st = KLDStats(max_rows=base.shape[0], device=DEV)
    st.run(base, quant, tok)
    res = st.result()
    st.close()
    return res


@pytest.mark.parametrize("first,second", [
    (("ctx", 300, 32001, synth.BF16, 21), ("edge", 1000, 4099, synth.F32, 22)),
])
def test_static_entry_matches_handle_entry_twice(first, second):
    for recipe, n, v, dt, seed in (first, second):
        w = synth.make_recipe(recipe, n=n, v=v, dtype=dt, seed=seed, device=DEV)
        a = _static_run(w.base, w.quant, w.token_ids)
        b = _handle_run(w.base, w.quant, w.token_ids)
        for k in ("n_rows", "n_valid", "top1_agree", "n_nll", "n_flagged", "flags_or",
                  "has_nll", "device_error"):
            assert int(a[k]) == int(b[k]), k
        for k in ("mean_kld", "median_kld", "p90_kld", "p99_kld", "max_kld", "top1_agree_pct",
                  "mean_nll", "ppl"):
            assert stat_close(a[k], b[k], k), (k, a[k], b[k])
        assert not math.isnan(a["mean_kld"])


def test_static_entry_rejects_more_rows_than_its_scratch():
    lib = _lib.load()
    p = torch.zeros(16, dtype=torch.float32, device=DEV)
    out = torch.zeros(ctypes.sizeof(_lib.Result), dtype=torch.uint8, device=DEV)
    st = lib.kld_stats_run_static(ctypes.c_void_p(p.data_ptr()), ctypes.c_void_p(p.data_ptr()),
                                  None, _lib.KLD_STATIC_MAX_ROWS + 1, 1, _lib.KLD_F32,
                                  ctypes.c_void_p(out.data_ptr()), None)
    assert st == _lib.KLD_ERR_CAPACITY
