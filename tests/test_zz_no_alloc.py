"""kld_stats_run_static, the entry point for callers that cannot allocate
device memory when they need the statistic (e.g. a server whose allocator
owns nearly all HBM), must give the same statistics as the handle-based
kld_stats_run and as the fp64 oracle. Every call goes through the C ABI.

Each case runs two calls in a row with different inputs, so the second call
also checks that the shared fixed scratch array carries nothing over from
the first. One case fills the fixed array exactly (KLD_STATIC_MAX_ROWS rows),
where the reduction reads its keys back from the records in global memory.
A separate case checks the contract itself: after a warm-up call, a call
leaves the device's free memory and the PyTorch allocator unchanged.
Collected last on purpose.
"""
import ctypes
import math

import pytest
import torch

import oracle
from logit_kl_divergence_b200 import KLDStats, _lib, dtype_code, synth

from gpu_helpers import ODT, assert_stats_match, stat_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

INT_FIELDS = ("n_rows", "n_valid", "top1_agree", "n_nll", "n_flagged", "flags_or", "has_nll",
              "device_error")
FLOAT_FIELDS = ("mean_kld", "median_kld", "p90_kld", "p99_kld", "max_kld", "top1_agree_pct",
                "mean_nll", "ppl", "mean_nll_base", "ppl_base", "ln_ppl_ratio", "mean_dp", "rms_dp")


def _static_call(base, quant, tok, out):
    lib = _lib.load()
    stream = torch.cuda.current_stream(DEV)
    st = lib.kld_stats_run_static(
        ctypes.c_void_p(base.data_ptr()), ctypes.c_void_p(quant.data_ptr()),
        None if tok is None else ctypes.c_void_p(tok.data_ptr()),
        base.shape[0], base.shape[1], dtype_code(base), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(stream.cuda_stream))
    assert st == _lib.KLD_OK, lib.kld_status_string(st)


def _static_run(base, quant, tok):
    out = torch.zeros(ctypes.sizeof(_lib.Result), dtype=torch.uint8, device=DEV)
    _static_call(base, quant, tok, out)
    torch.cuda.current_stream(DEV).synchronize()
    res = _lib.Result.from_buffer_copy(bytes(out.cpu().numpy()))
    return {name: getattr(res, name) for name, _ in _lib.Result._fields_ if not name.startswith("reserved")}


def _handle_run(base, quant, tok):
    st = KLDStats(max_rows=base.shape[0], device=DEV)
    st.run(base, quant, tok)
    res = st.result()
    st.close()
    return res


def _check_against_handle_and_oracle(w):
    a = _static_run(w.base, w.quant, w.token_ids)
    b = _handle_run(w.base, w.quant, w.token_ids)
    for k in INT_FIELDS:
        assert int(a[k]) == int(b[k]), k
    for k in FLOAT_FIELDS:
        assert stat_close(a[k], b[k], k), (k, a[k], b[k])
    tok = None if w.token_ids is None else w.token_ids.cpu()
    _, ref = oracle.run(w.base.cpu(), w.quant.cpu(), tok, ODT[w.dtype])
    assert_stats_match(a, ref)  # every field, at the parity tolerances
    assert not math.isnan(a["mean_kld"])


@pytest.mark.parametrize("first,second", [
    (("ctx", 300, 32001, synth.BF16, 21), ("edge", 1000, 4099, synth.F32, 22)),
    # the full fixed array, then a small call reusing it
    (("ctx", _lib.KLD_STATIC_MAX_ROWS, 257, synth.F32, 23), ("small", 5, 1000, synth.F32, 24)),
])
def test_static_entry_matches_handle_entry_and_oracle_twice(first, second):
    for recipe, n, v, dt, seed in (first, second):
        w = synth.make_recipe(recipe, n=n, v=v, dtype=dt, seed=seed, device=DEV)
        _check_against_handle_and_oracle(w)


def test_static_entry_allocates_nothing():
    w = synth.make_recipe("ctx", n=700, v=8192, dtype=synth.BF16, seed=25, device=DEV)
    out = torch.zeros(ctypes.sizeof(_lib.Result), dtype=torch.uint8, device=DEV)
    _static_call(w.base, w.quant, w.token_ids, out)  # warm-up: per-device set-up, kernel loading
    torch.cuda.synchronize(DEV)
    free0, _ = torch.cuda.mem_get_info(DEV)
    torch0 = torch.cuda.memory_allocated(DEV)
    reserved0 = torch.cuda.memory_reserved(DEV)
    for _ in range(3):
        _static_call(w.base, w.quant, w.token_ids, out)
    torch.cuda.synchronize(DEV)
    free1, _ = torch.cuda.mem_get_info(DEV)
    assert free1 == free0
    assert torch.cuda.memory_allocated(DEV) == torch0
    assert torch.cuda.memory_reserved(DEV) == reserved0


def test_static_entry_rejects_more_rows_than_its_scratch():
    lib = _lib.load()
    p = torch.zeros(16, dtype=torch.float32, device=DEV)
    out = torch.zeros(ctypes.sizeof(_lib.Result), dtype=torch.uint8, device=DEV)
    st = lib.kld_stats_run_static(ctypes.c_void_p(p.data_ptr()), ctypes.c_void_p(p.data_ptr()),
                                  None, _lib.KLD_STATIC_MAX_ROWS + 1, 1, _lib.KLD_F32,
                                  ctypes.c_void_p(out.data_ptr()), None)
    assert st == _lib.KLD_ERR_CAPACITY
