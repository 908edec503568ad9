"""Plain fp64 CPU oracle for the logit KL-divergence statistic.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``. The product library never imports
it, and it imports nothing from the product package.

The arithmetic lives in ``kld_oracle.cpp`` (plain C++, fp64, two passes per
row, ``std::sort`` percentiles); this module compiles it with ``g++`` and
marshals numpy arrays through ctypes. Sources for each step are cited in the
C++ file: "Qwen3.6 27B Quantization Benchmark" (sections "Understand KLD and
Same Top P" and "Raw benchmark data") and the "Mistral-Small-4-119B-2603
GSQ-RCO IQ3_S GGUF" card ("How it was made", step 5: KL(BF16 || quantized)
over the full vocabulary; "Quality": the perplexity ratio and the points of
probability given to the correct token).

Parity of every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, invariants, brute force and library routines.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kld_oracle.cpp")
_HDR = os.path.join(_HERE, "kld_oracle.h")
_LIB = os.path.join(_HERE, "_build", "libkld_oracle.so")

F32, BF16, F16 = 0, 1, 2

ROW_NONFINITE = 1 << 0
ROW_EMPTY = 1 << 1
ROW_INF_KL = 1 << 2
ROW_BAD_TOKEN = 1 << 3
ROW_INF_NLL = 1 << 4
ROW_INF_NLLB = 1 << 5


class _Result(ctypes.Structure):
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
        ("_pad", ctypes.c_int32),
        ("n_nll", ctypes.c_int64),
        ("mean_nll", ctypes.c_double),
        ("ppl", ctypes.c_double),
        ("n_flagged", ctypes.c_int64),
        ("flags_or", ctypes.c_uint32),
        ("_pad2", ctypes.c_uint32),
        ("mean_nll_base", ctypes.c_double),
        ("ppl_base", ctypes.c_double),
        ("ln_ppl_ratio", ctypes.c_double),
        ("mean_dp", ctypes.c_double),
        ("rms_dp", ctypes.c_double),
    ]


_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/libkld_oracle.so``.

    Plain ``-O2`` without fast-math, so NaN/inf semantics stay IEEE.
    """
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.run(
            ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
             "-fno-fast-math", "-o", tmp, _SRC],
            check=True,
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # KLD_ORACLE_LIB points the binding at another build of this file
            # (the mutation tests load deliberately broken copies this way).
            path = os.environ.get("KLD_ORACLE_LIB") or build()
            lib = ctypes.CDLL(path)
            lib.oracle_rows.restype = ctypes.c_int
            lib.oracle_rows.argtypes = [
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ]
            lib.oracle_reduce.restype = ctypes.c_int
            lib.oracle_reduce.argtypes = [
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_int64, ctypes.c_int, ctypes.POINTER(_Result),
            ]
            lib.oracle_grad.restype = ctypes.c_int
            lib.oracle_grad.argtypes = [
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                ctypes.c_int, ctypes.c_double, ctypes.c_void_p,
            ]
            lib.oracle_topk.restype = ctypes.c_int
            lib.oracle_topk.argtypes = [
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_void_p, ctypes.c_void_p,
            ]
            lib.oracle_percentile_sorted.restype = ctypes.c_double
            lib.oracle_percentile_sorted.argtypes = [
                ctypes.c_void_p, ctypes.c_int64, ctypes.c_double,
            ]
            _lib = lib
    return _lib


def _as_logits(x, dtype: int) -> np.ndarray:
    """Accept numpy arrays or CPU torch tensors; bf16/f16 as raw uint16 bits."""
    if hasattr(x, "detach"):  # torch tensor
        import torch

        t = x.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16 or t.dtype == torch.float16:
            t = t.view(torch.int16)
        x = t.numpy()
    x = np.ascontiguousarray(x)
    if dtype == F32:
        if x.dtype != np.float32:
            raise TypeError("F32 logits must be float32")
    else:
        if x.dtype.itemsize != 2:
            raise TypeError("BF16/F16 logits must be 2-byte raw bits")
        x = x.view(np.uint16)
    if x.ndim != 2:
        raise ValueError("logits must be [N, V]")
    return x


def rows(base, quant, token_ids=None, dtype: int = F32, nthreads: int = 1) -> dict:
    """Per-row KL, NLL under quant and base, argmaxes and flags (numpy arrays
    of length N)."""
    lib = _load()
    b = _as_logits(base, dtype)
    q = _as_logits(quant, dtype)
    if b.shape != q.shape:
        raise ValueError("base and quant shapes differ")
    N, V = b.shape
    tok = None
    if token_ids is not None:
        if hasattr(token_ids, "detach"):
            token_ids = token_ids.detach().cpu().numpy()
        tok = np.ascontiguousarray(token_ids, dtype=np.int32).reshape(-1)
        if tok.shape[0] != N:
            raise ValueError("token_ids must have N entries")
    out = {
        "kld": np.empty(N, np.float64),
        "nll": np.empty(N, np.float64),
        "nll_base": np.empty(N, np.float64),
        "amax_b": np.empty(N, np.int32),
        "amax_q": np.empty(N, np.int32),
        "flags": np.empty(N, np.uint32),
    }
    rc = lib.oracle_rows(
        b.ctypes.data, q.ctypes.data, None if tok is None else tok.ctypes.data,
        N, V, dtype,
        out["kld"].ctypes.data, out["nll"].ctypes.data, out["nll_base"].ctypes.data,
        out["amax_b"].ctypes.data, out["amax_q"].ctypes.data,
        out["flags"].ctypes.data, int(nthreads),
    )
    if rc != 0:
        raise ValueError("oracle_rows rejected its arguments")
    return out


def reduce(r: dict, has_nll: bool) -> dict:
    """Summary statistics from the per-row arrays of :func:`rows`."""
    lib = _load()
    N = r["kld"].shape[0]
    kld = np.ascontiguousarray(r["kld"], np.float64)
    nll = np.ascontiguousarray(r["nll"], np.float64)
    nllb = np.ascontiguousarray(r.get("nll_base", np.full(N, np.nan)), np.float64)
    ab = np.ascontiguousarray(r["amax_b"], np.int32)
    aq = np.ascontiguousarray(r["amax_q"], np.int32)
    fl = np.ascontiguousarray(r["flags"], np.uint32)
    res = _Result()
    rc = lib.oracle_reduce(kld.ctypes.data, nll.ctypes.data, nllb.ctypes.data, ab.ctypes.data,
                           aq.ctypes.data, fl.ctypes.data, N, int(bool(has_nll)),
                           ctypes.byref(res))
    if rc != 0:
        raise ValueError("oracle_reduce rejected its arguments")
    return {name: getattr(res, name) for name, _ in _Result._fields_
            if not name.startswith("_")}


def run(base, quant, token_ids=None, dtype: int = F32, nthreads: int = 1):
    """Per-row arrays and summary statistics for one [N, V] pair."""
    r = rows(base, quant, token_ids, dtype, nthreads)
    return r, reduce(r, token_ids is not None)


def grad(base, quant, dtype: int = F32, scale: float = 1.0) -> np.ndarray:
    """[N, V] float64 gradient of KL(P_base || P_quant) with respect to the
    quant logits: scale * (softmax(q) - softmax(b)); zero on excluded rows."""
    lib = _load()
    b = _as_logits(base, dtype)
    q = _as_logits(quant, dtype)
    if b.shape != q.shape:
        raise ValueError("base and quant shapes differ")
    N, V = b.shape
    out = np.empty((N, V), np.float64)
    if lib.oracle_grad(b.ctypes.data, q.ctypes.data, N, V, dtype, float(scale), out.ctypes.data) != 0:
        raise ValueError("oracle_grad rejected its arguments")
    return out


def topk(base, quant, k: int = 128, dtype: int = F32) -> dict:
    """Top-k compression of each base row and the KL of the quant row against
    it: idx [N, k] int32, logp [N, k] and rest [N] (log P_base), kl_topk [N]."""
    lib = _load()
    b = _as_logits(base, dtype)
    q = _as_logits(quant, dtype)
    if b.shape != q.shape:
        raise ValueError("base and quant shapes differ")
    N, V = b.shape
    out = {"idx": np.empty((N, k), np.int32), "logp": np.empty((N, k), np.float64),
           "rest": np.empty(N, np.float64), "kl_topk": np.empty(N, np.float64)}
    rc = lib.oracle_topk(b.ctypes.data, q.ctypes.data, N, V, dtype, int(k), out["idx"].ctypes.data,
                         out["logp"].ctypes.data, out["rest"].ctypes.data, out["kl_topk"].ctypes.data)
    if rc != 0:
        raise ValueError("oracle_topk rejected its arguments")
    return out


def percentile_sorted(x, p: float) -> float:
    """Type-7 percentile of an ascending float64 array (as the oracle uses)."""
    lib = _load()
    a = np.ascontiguousarray(x, np.float64)
    return lib.oracle_percentile_sorted(a.ctypes.data, a.shape[0], float(p))
