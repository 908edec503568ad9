"""ctypes declarations of the C ABI in ``include/kld_stats.h``.

Argument marshalling only: every step of the statistic runs in the CUDA
kernels of ``libkld_stats.so``. Loading fails loudly when the library is
missing; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

KLD_OK = 0
KLD_ERR_INVALID_ARG = 1
KLD_ERR_DTYPE = 2
KLD_ERR_OOM = 3
KLD_ERR_CUDA = 4
KLD_ERR_NONFINITE = 5
KLD_ERR_BAD_TOKEN = 6
KLD_ERR_TIMEOUT = 7
KLD_ERR_NO_DEVICE = 8
KLD_ERR_NOT_READY = 9
KLD_ERR_CAPACITY = 10
KLD_STATIC_MAX_ROWS = 65536

KLD_F32, KLD_BF16, KLD_F16 = 0, 1, 2
KLD_PARTIAL_BYTES = 64
KLD_MAX_TOPK = 1024

ROW_NONFINITE = 1 << 0
ROW_EMPTY = 1 << 1
ROW_INF_KL = 1 << 2
ROW_BAD_TOKEN = 1 << 3
ROW_INF_NLL = 1 << 4
ROW_INF_NLL_BASE = 1 << 5


class Row(ctypes.Structure):
    _fields_ = [
        ("kld", ctypes.c_double),
        ("nll", ctypes.c_double),
        ("nll_base", ctypes.c_double),
        ("argmax_base", ctypes.c_int32),
        ("argmax_quant", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
        ("dp", ctypes.c_float),
    ]


class Result(ctypes.Structure):
    _fields_ = [
        ("n_rows", ctypes.c_int64),
        ("n_valid", ctypes.c_int64),
        ("mean_kld", ctypes.c_double),
        ("median_kld", ctypes.c_double),
        ("p90_kld", ctypes.c_double),
        ("p99_kld", ctypes.c_double),
        ("max_kld", ctypes.c_double),
        ("top1_agree", ctypes.c_int64),
        ("top1_agree_pct", ctypes.c_double),
        ("has_nll", ctypes.c_int32),
        ("reserved0", ctypes.c_int32),
        ("n_nll", ctypes.c_int64),
        ("mean_nll", ctypes.c_double),
        ("ppl", ctypes.c_double),
        ("n_flagged", ctypes.c_int64),
        ("flags_or", ctypes.c_uint32),
        ("device_error", ctypes.c_uint32),
        ("mean_nll_base", ctypes.c_double),
        ("ppl_base", ctypes.c_double),
        ("ln_ppl_ratio", ctypes.c_double),
        ("mean_dp", ctypes.c_double),
        ("rms_dp", ctypes.c_double),
    ]


class Plan(ctypes.Structure):
    _fields_ = [
        ("variant", ctypes.c_int32),
        ("grid", ctypes.c_int32),
        ("ctas_per_row", ctypes.c_int32),
        ("threads", ctypes.c_int32),
        ("smem_bytes", ctypes.c_int32),
        ("stage_bytes", ctypes.c_int32),
        ("stages", ctypes.c_int32),
        ("cluster_ctas", ctypes.c_int32),
        ("whole_rounds", ctypes.c_int32),
        ("tail_rows", ctypes.c_int32),
        ("tail_ctas", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


assert ctypes.sizeof(Row) == 40
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int
_ST = ctypes.c_int

# name -> (restype, argtypes); the same set the header declares.
SIGNATURES = {
    "kld_abi_version": (_I32, []),
    "kld_status_string": (ctypes.c_char_p, [_ST]),
    "kld_last_cuda_error": (ctypes.c_char_p, []),
    "kld_stats_create": (_ST, [ctypes.POINTER(_P), _I64, _I32]),
    "kld_stats_destroy": (None, [_P]),
    "kld_stats_run": (_ST, [_P, _P, _P, _P, _I64, _I64, _I32, _P]),
    "kld_stats_result": (_ST, [_P, ctypes.POINTER(Result)]),
    "kld_stats_rows": (_ST, [_P, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P),
                             ctypes.POINTER(_P)]),
    "kld_stats_records": (_ST, [_P, ctypes.POINTER(_P), ctypes.POINTER(_I64)]),
    "kld_stats_run_rows": (_ST, [_P, _P, _P, _P, _I64, _I64, _I32, _P, _P]),
    "kld_stats_reduce": (_ST, [_P, _P, _I64, _I32, _P]),
    "kld_stats_run_host": (_ST, [_P, _P, _P, _P, _I64, _I64, _I32, _P]),
    "kld_stats_run_rows_host": (_ST, [_P, _P, _P, _P, _I64, _I64, _I32, _P, _P]),
    "kld_stats_set_timing": (_ST, [_P, _I32]),
    "kld_stats_set_split": (_ST, [_P, _I32]),
    "kld_stats_run_grad": (_ST, [_P, _P, _P, _P, _I64, _I64, _I32, _P, _I32, ctypes.c_double, _P]),
    "kld_stats_second_pass_timing": (_ST, [_P, ctypes.POINTER(ctypes.c_float)]),
    "kld_stats_topk_exact_rows": (_ST, [_P, ctypes.POINTER(ctypes.c_int64)]),
    "kld_stats_read_probe": (_ST, [_P, _P, _P, _I64, _P]),
    "kld_selftest_bounded_wait": (_ST, [_I32, ctypes.c_uint64, _I32, ctypes.POINTER(ctypes.c_uint64)]),
    "kld_stats_run_topk": (_ST, [_P, _P, _P, _P, _I64, _I64, _I32, _I32, _P, _P, _P, _P, _P]),
    "kld_stats_run_partials": (_ST, [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _I32, _P, _P]),
    "kld_stats_merge_partials": (_ST, [_P, _P, _I32, _I64, _P, _I64, _P]),
    "kld_stats_timing": (_ST, [_P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]),
    "kld_plan": (_ST, [_I64, _I64, _I32, _I32, ctypes.POINTER(Plan)]),
    "kld_stats_run_static": (_ST, [_P, _P, _P, _I64, _I64, _I32, _P, _P]),
}

_lock = threading.Lock()
_lib = None


def lib_path() -> str:
    return _build.LIB


def load(auto_build: bool = True):
    """Load ``libkld_stats.so`` (building it first when it is missing or stale
    and ``auto_build`` is set). Raises if it cannot be loaded."""
    global _lib
    with _lock:
        if _lib is None:
            if auto_build and _build.needs_build():
                _build.build()
            if not os.path.exists(_build.LIB):
                raise RuntimeError(f"{_build.LIB} is missing: run `python -m logit_kl_divergence_b200.build`")
            lib = ctypes.CDLL(_build.LIB)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


class KLDError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        msg = lib.kld_status_string(status).decode()
        if status in (KLD_ERR_CUDA, KLD_ERR_OOM, KLD_ERR_NO_DEVICE):
            detail = lib.kld_last_cuda_error().decode()
            if detail:
                msg += f" ({detail})"
        super().__init__(f"{where}: {msg}")
        self.status = status


def check(status: int, where: str) -> int:
    if status != KLD_OK:
        raise KLDError(status, where)
    return status
