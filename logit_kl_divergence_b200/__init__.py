"""KL-divergence statistics of quantized vs. base logits on B200 (sm_100a).

Thin Python binding over the C ABI of ``libkld_stats.so`` (``include/
kld_stats.h``). PyTorch supplies device memory and streams; all arithmetic
runs in the library's CUDA kernels.

    >>> from logit_kl_divergence_b200 import KLDStats
    >>> st = KLDStats(max_rows=8192)
    >>> st.run(base_logits, quant_logits, next_token_ids)   # async on the stream
    >>> res = st.result()    # mean/median/p90/p99/max KLD, top-1 agreement, PPL
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (KLD_BF16, KLD_F16, KLD_F32, ROW_BAD_TOKEN, ROW_EMPTY,  # noqa: F401
                   ROW_INF_KL, ROW_INF_NLL, ROW_INF_NLL_BASE, ROW_NONFINITE, KLDError)

__all__ = ["KLDStats", "kld_stats", "run_static", "result_from_bytes", "plan", "dtype_code",
           "ROW_RECORD_BYTES", "selftest_bounded_wait"]

ROW_RECORD_BYTES = 40
PARTIAL_BYTES = 64

_DTYPES = {torch.float32: KLD_F32, torch.bfloat16: KLD_BF16, torch.float16: KLD_F16}

# statuses that still come with valid statistics of the remaining rows
_SOFT = (_lib.KLD_OK, _lib.KLD_ERR_NONFINITE, _lib.KLD_ERR_BAD_TOKEN)


def dtype_code(t: torch.Tensor) -> int:
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported logit dtype {t.dtype}") from None


def _stream_ptr(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_pair(base: torch.Tensor, quant: torch.Tensor, token_ids, on_device: bool):
    if base.dim() != 2 or base.shape != quant.shape:
        raise ValueError("base and quant must be [N, V] tensors of the same shape")
    if base.dtype != quant.dtype:
        raise TypeError("base and quant must share a dtype")
    if not (base.is_contiguous() and quant.is_contiguous()):
        raise ValueError("base and quant must be contiguous")
    if on_device and not (base.is_cuda and quant.is_cuda):
        raise ValueError("base and quant must be CUDA tensors")
    if token_ids is not None:
        if token_ids.dtype != torch.int32 or token_ids.dim() != 1 or token_ids.shape[0] != base.shape[0]:
            raise ValueError("token_ids must be an int32 [N] tensor")
        if not token_ids.is_contiguous():
            raise ValueError("token_ids must be contiguous")
        if on_device and token_ids.device != base.device:
            raise ValueError("token_ids must be on the logits' device")


def rows_view(records: torch.Tensor) -> dict:
    """Field views of a [N, 40] uint8 tensor of row records (kld_row_t)."""
    r = records.view(torch.uint8).reshape(-1, ROW_RECORD_BYTES)
    f64 = r[:, :24].contiguous().view(torch.float64)
    i32 = r[:, 24:36].contiguous().view(torch.int32)
    f32 = r[:, 36:40].contiguous().view(torch.float32)
    return {"kld": f64[:, 0], "nll": f64[:, 1], "nll_base": f64[:, 2], "amax_b": i32[:, 0],
            "amax_q": i32[:, 1], "flags": i32[:, 2], "dp": f32[:, 0]}


class KLDStats:
    """One handle of the library: workspace for up to ``max_rows`` rows on one
    device. Not thread-safe; use one per concurrent stream."""

    def __init__(self, max_rows: int, device=None):
        self._lib = _lib.load()
        if device is None:
            device = torch.cuda.current_device()
        self.device = torch.device("cuda", torch.device(device).index if not isinstance(device, int) else device)
        self.max_rows = int(max_rows)
        h = ctypes.c_void_p()
        _lib.check(self._lib.kld_stats_create(ctypes.byref(h), self.max_rows, self.device.index),
                   "kld_stats_create")
        self._h = h
        self._has_nll = False

    def close(self):
        if getattr(self, "_h", None):
            self._lib.kld_stats_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # ------------------------------------------------------------ calls
    def run(self, base: torch.Tensor, quant: torch.Tensor, token_ids: torch.Tensor | None = None,
            stream=None) -> None:
        _check_pair(base, quant, token_ids, True)
        st = self._lib.kld_stats_run(self._h, _ptr(base), _ptr(quant), _ptr(token_ids),
                                     base.shape[0], base.shape[1], dtype_code(base),
                                     ctypes.c_void_p(_stream_ptr(stream, base.device)))
        _lib.check(st, "kld_stats_run")

    def run_grad(self, base: torch.Tensor, quant: torch.Tensor, token_ids: torch.Tensor | None = None,
                 out: torch.Tensor | None = None, scale: float = 1.0, grad_dtype=None,
                 stream=None) -> torch.Tensor:
        """The statistic (read it with :meth:`result`) plus the gradient of
        KL(P_base || P_quant) with respect to the quant logits,
        ``scale * (softmax(quant) - softmax(base))`` per row (zero on excluded
        rows), written to ``out`` (allocated as ``grad_dtype``, default the
        logits' dtype, when None). Asynchronous on the stream."""
        _check_pair(base, quant, token_ids, True)
        if out is None:
            out = torch.empty(base.shape, dtype=grad_dtype or base.dtype, device=base.device)
        if out.shape != base.shape or not out.is_contiguous() or out.device != base.device:
            raise ValueError("out must be a contiguous [N, V] tensor on the logits' device")
        st = self._lib.kld_stats_run_grad(self._h, _ptr(base), _ptr(quant), _ptr(token_ids),
                                          base.shape[0], base.shape[1], dtype_code(base), _ptr(out),
                                          dtype_code(out), float(scale),
                                          ctypes.c_void_p(_stream_ptr(stream, base.device)))
        _lib.check(st, "kld_stats_run_grad")
        return out

    def run_topk(self, base: torch.Tensor, quant: torch.Tensor, token_ids: torch.Tensor | None = None,
                 k: int = 128, stream=None) -> dict:
        """The statistic (read it with :meth:`result`) plus the top-k
        compression of each base row and the KL of the quant row against it:
        ``idx`` [N, k] int32, ``logp`` [N, k] float32 (log P_base), ``rest``
        [N] float32 (log of the mass outside the top k) and ``kl_topk`` [N]
        float64, CUDA tensors filled asynchronously on the stream."""
        _check_pair(base, quant, token_ids, True)
        n = base.shape[0]
        out = {"idx": torch.empty((n, k), dtype=torch.int32, device=base.device),
               "logp": torch.empty((n, k), dtype=torch.float32, device=base.device),
               "rest": torch.empty(n, dtype=torch.float32, device=base.device),
               "kl_topk": torch.empty(n, dtype=torch.float64, device=base.device)}
        st = self._lib.kld_stats_run_topk(self._h, _ptr(base), _ptr(quant), _ptr(token_ids), n,
                                          base.shape[1], dtype_code(base), int(k), _ptr(out["idx"]),
                                          _ptr(out["logp"]), _ptr(out["rest"]), _ptr(out["kl_topk"]),
                                          ctypes.c_void_p(_stream_ptr(stream, base.device)))
        _lib.check(st, "kld_stats_run_topk")
        return out

    def topk_exact_rows(self) -> int:
        """Rows of the last run_topk that took the exact path instead of the
        threshold's fast path (waits for that run)."""
        n = ctypes.c_int64()
        _lib.check(self._lib.kld_stats_topk_exact_rows(self._h, ctypes.byref(n)),
                   "kld_stats_topk_exact_rows")
        return n.value

    def second_pass_timing(self) -> float:
        """Milliseconds of the second pass of the last run_grad (the gradient
        pass) or run_topk (the top-k pass, with its threshold kernel when the
        row pass scanned); timing enabled."""
        ms = ctypes.c_float()
        _lib.check(self._lib.kld_stats_second_pass_timing(self._h, ctypes.byref(ms)),
                   "kld_stats_second_pass_timing")
        return ms.value

    def read_probe(self, a: torch.Tensor, b: torch.Tensor, stream=None) -> None:
        """Read-bandwidth probe: stream both (contiguous, same-size) device
        tensors from HBM into shared memory as the row pass does, computing
        nothing; time it with CUDA events on the stream."""
        if not (a.is_cuda and b.is_cuda and a.is_contiguous() and b.is_contiguous()):
            raise ValueError("a and b must be contiguous CUDA tensors")
        nbytes = a.numel() * a.element_size()
        if b.numel() * b.element_size() != nbytes:
            raise ValueError("a and b must have the same size in bytes")
        st = self._lib.kld_stats_read_probe(self._h, _ptr(a), _ptr(b), nbytes,
                                            ctypes.c_void_p(_stream_ptr(stream, a.device)))
        _lib.check(st, "kld_stats_read_probe")

    def run_partials(self, base: torch.Tensor, quant: torch.Tensor, token_ids: torch.Tensor | None,
                     col_offset: int, v_total: int, out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
        """This GPU's vocabulary slice (columns [col_offset, col_offset + V) of
        a V_total-wide vocabulary): one 64-byte partial per row, returned as
        (or written to) an [N, 64] uint8 CUDA tensor."""
        _check_pair(base, quant, token_ids, True)
        n = base.shape[0]
        if out is None:
            out = torch.empty((n, PARTIAL_BYTES), dtype=torch.uint8, device=base.device)
        if out.dtype != torch.uint8 or out.numel() < n * PARTIAL_BYTES or not out.is_contiguous():
            raise ValueError("out must be a contiguous uint8 tensor of N*64 bytes")
        st = self._lib.kld_stats_run_partials(self._h, _ptr(base), _ptr(quant), _ptr(token_ids), n,
                                              base.shape[1], int(col_offset), int(v_total),
                                              dtype_code(base), _ptr(out),
                                              ctypes.c_void_p(_stream_ptr(stream, base.device)))
        _lib.check(st, "kld_stats_run_partials")
        return out

    def merge_partials(self, parts: torch.Tensor, token_ids: torch.Tensor | None, v_total: int,
                       stream=None) -> None:
        """Merge [G, N, 64] (or [G*N, 64]) slice partials, in slice order,
        into this handle's records and reduce them (read with :meth:`result`)."""
        if parts.dtype != torch.uint8 or not parts.is_cuda or not parts.is_contiguous():
            raise ValueError("parts must be a contiguous uint8 CUDA tensor")
        p = parts.reshape(-1, PARTIAL_BYTES)
        if token_ids is not None:
            n = token_ids.shape[0]
        elif parts.dim() == 3:
            n = parts.shape[1]
        else:
            raise ValueError("give [G, N, 64] parts or the token ids")
        if p.shape[0] % n:
            raise ValueError("parts must hold G * N partials")
        st = self._lib.kld_stats_merge_partials(self._h, _ptr(p), p.shape[0] // n, n, _ptr(token_ids),
                                                int(v_total),
                                                ctypes.c_void_p(_stream_ptr(stream, parts.device)))
        _lib.check(st, "kld_stats_merge_partials")

    def run_host(self, base: torch.Tensor, quant: torch.Tensor, token_ids: torch.Tensor | None = None,
                 stream=None) -> None:
        """Same as :meth:`run` for host (preferably pinned) CPU tensors."""
        _check_pair(base, quant, token_ids, False)
        if base.is_cuda:
            raise ValueError("run_host takes CPU tensors")
        st = self._lib.kld_stats_run_host(self._h, _ptr(base), _ptr(quant), _ptr(token_ids),
                                          base.shape[0], base.shape[1], dtype_code(base),
                                          ctypes.c_void_p(_stream_ptr(stream, self.device)))
        _lib.check(st, "kld_stats_run_host")

    def run_rows_host(self, base: torch.Tensor, quant: torch.Tensor, token_ids: torch.Tensor | None = None,
                      out: torch.Tensor | None = None, stream=None):
        """Row pass only, for host (preferably pinned) CPU tensors: chunked
        copies overlapped with the row pass; records go to ``out`` ([N, 40]
        uint8 on the device) or to the handle's workspace."""
        _check_pair(base, quant, token_ids, False)
        if base.is_cuda:
            raise ValueError("run_rows_host takes CPU tensors")
        if out is not None and (out.dtype != torch.uint8 or not out.is_cuda
                                or out.numel() < base.shape[0] * ROW_RECORD_BYTES):
            raise ValueError("out must be a CUDA uint8 tensor of N*40 bytes")
        st = self._lib.kld_stats_run_rows_host(self._h, _ptr(base), _ptr(quant), _ptr(token_ids),
                                               base.shape[0], base.shape[1], dtype_code(base), _ptr(out),
                                               ctypes.c_void_p(_stream_ptr(stream, self.device)))
        _lib.check(st, "kld_stats_run_rows_host")
        return out

    def run_rows(self, base, quant, token_ids=None, out: torch.Tensor | None = None, stream=None):
        """Row pass only; records go to ``out`` ([N, 40] uint8 on the device)
        or to the handle's workspace."""
        _check_pair(base, quant, token_ids, True)
        if out is not None and (out.dtype != torch.uint8 or out.numel() < base.shape[0] * ROW_RECORD_BYTES):
            raise ValueError("out must be a uint8 tensor of N*40 bytes")
        st = self._lib.kld_stats_run_rows(self._h, _ptr(base), _ptr(quant), _ptr(token_ids),
                                          base.shape[0], base.shape[1], dtype_code(base), _ptr(out),
                                          ctypes.c_void_p(_stream_ptr(stream, base.device)))
        _lib.check(st, "kld_stats_run_rows")
        return out

    def reduce(self, records: torch.Tensor | None, n_rows: int, has_nll: bool, stream=None) -> None:
        """Reduction over ``n_rows`` records (a device uint8 tensor, or None for
        the handle's workspace)."""
        st = self._lib.kld_stats_reduce(self._h, _ptr(records), int(n_rows), int(bool(has_nll)),
                                        ctypes.c_void_p(_stream_ptr(stream, self.device)))
        _lib.check(st, "kld_stats_reduce")

    def result(self, raise_on_soft: bool = False) -> dict:
        """Wait for the last run and return its statistics as a dict. Rows that
        were excluded (``status`` != 0) do not raise unless asked to."""
        res = _lib.Result()
        st = self._lib.kld_stats_result(self._h, ctypes.byref(res))
        if st not in _SOFT or (raise_on_soft and st != _lib.KLD_OK):
            _lib.check(st, "kld_stats_result")
        out = {name: getattr(res, name) for name, _ in _lib.Result._fields_
               if not name.startswith("reserved")}
        out["status"] = st
        return out

    def records(self) -> torch.Tensor:
        """Copy of the last run's per-row records as a [N, 40] uint8 CUDA
        tensor (see :func:`rows_view`), ordered after the run on the current
        stream (kld_stats_records)."""
        p = ctypes.c_void_p()
        n = ctypes.c_int64()
        _lib.check(self._lib.kld_stats_records(self._h, ctypes.byref(p), ctypes.byref(n)),
                   "kld_stats_records")
        nbytes = n.value * ROW_RECORD_BYTES
        if nbytes == 0:
            return torch.empty((0, ROW_RECORD_BYTES), dtype=torch.uint8, device=self.device)
        view = torch.as_tensor(_DeviceBytes(p.value, nbytes), device=self.device)
        return view.view(n.value, ROW_RECORD_BYTES).clone()

    def rows(self, stream=None) -> dict:
        """Per-row results of the last run as four CUDA tensors of N values
        (kld_stats_rows): ``kld`` and ``nll`` float64, ``amax_b`` and
        ``amax_q`` int32. Copies of the handle's arrays, taken after the
        library's per-field kernel on the run's stream."""
        ptrs = [ctypes.c_void_p() for _ in range(4)]
        _lib.check(self._lib.kld_stats_rows(self._h, *(ctypes.byref(p) for p in ptrs)),
                   "kld_stats_rows")
        n = ctypes.c_int64()
        dummy = ctypes.c_void_p()
        _lib.check(self._lib.kld_stats_records(self._h, ctypes.byref(dummy), ctypes.byref(n)),
                   "kld_stats_records")
        # the per-field kernel runs on the run's stream; order the copies after it
        torch.cuda.synchronize(self.device)
        out = {}
        for name, p, (dt, size) in zip(("kld", "nll", "amax_b", "amax_q"), ptrs,
                                       ((torch.float64, 8), (torch.float64, 8),
                                        (torch.int32, 4), (torch.int32, 4))):
            view = torch.as_tensor(_DeviceBytes(p.value, n.value * size), device=self.device)
            out[name] = view.view(dt).clone()
        return out

    def set_split(self, cluster_ctas: int) -> None:
        """Few-row launch shape: -1 never split rows, 0 default, 1 plain
        CTAs, 2/4/8 thread-block clusters of up to that many CTAs."""
        _lib.check(self._lib.kld_stats_set_split(self._h, int(cluster_ctas)), "kld_stats_set_split")

    def set_timing(self, enable: bool) -> None:
        _lib.check(self._lib.kld_stats_set_timing(self._h, int(bool(enable))), "kld_stats_set_timing")

    def timing(self) -> tuple[float, float]:
        a, b = ctypes.c_float(), ctypes.c_float()
        _lib.check(self._lib.kld_stats_timing(self._h, ctypes.byref(a), ctypes.byref(b)), "kld_stats_timing")
        return a.value, b.value

    def plan(self, n_rows: int, vocab: int, dtype: int) -> dict:
        return plan(n_rows, vocab, dtype, torch.cuda.get_device_properties(self.device).multi_processor_count)


def run_static(base: torch.Tensor, quant: torch.Tensor, token_ids: torch.Tensor | None,
               result_out: torch.Tensor, stream=None) -> None:
    """kld_stats_run_static: the whole statistic with no allocation, written
    asynchronously into ``result_out`` (a device uint8 tensor of at least
    ``sizeof(kld_result_t)`` bytes, 8-byte aligned; decode with
    :func:`result_from_bytes`)."""
    _check_pair(base, quant, token_ids, True)
    if result_out.dtype != torch.uint8 or result_out.numel() < ctypes.sizeof(_lib.Result) or not result_out.is_cuda:
        raise ValueError("result_out must be a CUDA uint8 tensor of sizeof(kld_result_t) bytes")
    lib = _lib.load()
    st = lib.kld_stats_run_static(_ptr(base), _ptr(quant), _ptr(token_ids), base.shape[0], base.shape[1],
                                  dtype_code(base), _ptr(result_out),
                                  ctypes.c_void_p(_stream_ptr(stream, base.device)))
    _lib.check(st, "kld_stats_run_static")


def result_from_bytes(buf: torch.Tensor) -> dict:
    """Statistics from a kld_result_t held in a uint8 tensor (copied to host)."""
    res = _lib.Result.from_buffer_copy(bytes(buf[:ctypes.sizeof(_lib.Result)].cpu().numpy()))
    return {name: getattr(res, name) for name, _ in _lib.Result._fields_ if not name.startswith("reserved")}


def plan(n_rows: int, vocab: int, dtype: int, sm_count: int) -> dict:
    lib = _lib.load()
    p = _lib.Plan()
    _lib.check(lib.kld_plan(int(n_rows), int(vocab), int(dtype), int(sm_count), ctypes.byref(p)), "kld_plan")
    return {name: getattr(p, name) for name, _ in _lib.Plan._fields_}


def selftest_bounded_wait(device: int = 0, limit_ns: int = 2_000_000, use_abort: bool = False) -> tuple[int, int]:
    """Run the library's bounded-wait self-test on ``device``: a kernel waits
    on a barrier nothing completes and must give up after ``limit_ns`` (or on
    its abort flag). Returns ``(status, waited_ns)``; the expected status is
    ``KLD_ERR_TIMEOUT``. Any other failure raises."""
    lib = _lib.load()
    waited = ctypes.c_uint64(0)
    st = lib.kld_selftest_bounded_wait(int(device), int(limit_ns), int(bool(use_abort)), ctypes.byref(waited))
    if st not in (_lib.KLD_OK, _lib.KLD_ERR_TIMEOUT):
        _lib.check(st, "kld_selftest_bounded_wait")
    return st, waited.value


class _DeviceBytes:
    """Zero-copy view of library-owned device memory for torch.as_tensor."""

    def __init__(self, ptr: int, nbytes: int):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1",
                                         "data": (ptr, False), "version": 3}


def kld_stats(base: torch.Tensor, quant: torch.Tensor, token_ids: torch.Tensor | None = None) -> dict:
    """One-shot convenience: statistics of one [N, V] pair on the current stream."""
    with KLDStats(base.shape[0], base.device) as st:
        st.run(base, quant, token_ids)
        return st.result()
