"""The C-ABI library loads, exports what include/kld_stats.h declares, agrees
with the header on struct layouts, and rejects bad arguments before touching
a GPU. Runs without a GPU: no compute call is made."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from logit_kl_divergence_b200 import _lib, build, plan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kld_stats.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kld_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_every_declared_function_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"binding misses {n}"
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (kld_\w+)", out))
    assert set(names) <= exported
    assert exported <= set(names), f"undeclared exports: {exported - set(names)}"


def test_library_is_built_for_sm100a_only():
    assert build.ARCH_FLAGS == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_struct_layouts_match_header():
    src = r'''
#include <stdio.h>
#include <stddef.h>
#include "kld_stats.h"
int main(void) {
  printf("%zu %zu %zu\n", sizeof(kld_row_t), sizeof(kld_result_t), sizeof(kld_plan_t));
  printf("%zu %zu %zu %zu %zu %zu\n", offsetof(kld_result_t, top1_agree), offsetof(kld_result_t, has_nll),
         offsetof(kld_result_t, ppl), offsetof(kld_result_t, device_error),
         offsetof(kld_result_t, mean_nll_base), offsetof(kld_result_t, rms_dp));
  printf("%zu %zu %zu\n", offsetof(kld_row_t, argmax_base), offsetof(kld_row_t, flags),
         offsetof(kld_row_t, nll_base));
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        lines = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    sizes = [int(x) for x in lines[0].split()]
    assert sizes == [ctypes.sizeof(_lib.Row), ctypes.sizeof(_lib.Result), ctypes.sizeof(_lib.Plan)]
    offs = [int(x) for x in lines[1].split()]
    assert offs == [_lib.Result.top1_agree.offset, _lib.Result.has_nll.offset,
                    _lib.Result.ppl.offset, _lib.Result.device_error.offset,
                    _lib.Result.mean_nll_base.offset, _lib.Result.rms_dp.offset]
    roffs = [int(x) for x in lines[2].split()]
    assert roffs == [_lib.Row.argmax_base.offset, _lib.Row.flags.offset, _lib.Row.nll_base.offset]


def test_abi_version_and_status_strings(lib):
    assert lib.kld_abi_version() == 4
    for s in range(0, 10):
        assert lib.kld_status_string(s)
    assert lib.kld_status_string(12345) == b"unknown status"


def test_arguments_rejected_before_any_gpu_work(lib):
    h = ctypes.c_void_p()
    assert lib.kld_stats_create(None, 10, 0) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_stats_create(ctypes.byref(h), 0, 0) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_stats_create(ctypes.byref(h), 10, -1) == _lib.KLD_ERR_INVALID_ARG
    p = ctypes.c_void_p(1 << 20)
    assert lib.kld_stats_run(None, p, p, None, 1, 1, 0, None) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_stats_result(None, None) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_stats_reduce(None, None, 1, 0, None) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_stats_run_host(None, p, p, None, 1, 1, 0, None) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_stats_set_timing(None, 1) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_stats_read_probe(None, p, p, 1 << 20, None) == _lib.KLD_ERR_INVALID_ARG
    d, n = ctypes.c_void_p(), ctypes.c_int64()
    assert lib.kld_stats_rows(None, ctypes.byref(d), None, None, None) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_stats_records(None, ctypes.byref(d), ctypes.byref(n)) == _lib.KLD_ERR_INVALID_ARG
    ms = ctypes.c_float()
    assert lib.kld_stats_second_pass_timing(None, ctypes.byref(ms)) == _lib.KLD_ERR_INVALID_ARG
    w = ctypes.c_uint64()
    assert lib.kld_selftest_bounded_wait(-1, 10**6, 0, ctypes.byref(w)) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_selftest_bounded_wait(0, 999, 0, ctypes.byref(w)) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_selftest_bounded_wait(0, 10**10 + 1, 0, ctypes.byref(w)) == _lib.KLD_ERR_INVALID_ARG
    lib.kld_stats_destroy(None)  # no-op


def test_header_declarations_link_and_reject_a_null_handle():
    # A C caller compiled against include/kld_stats.h, linked to the library:
    # the per-field row accessor of the boundary takes exactly the declared
    # arguments (four output arrays), and its checks run before any CUDA call.
    src = r'''
#include <stdio.h>
#include "kld_stats.h"
int main(void) {
  const double* kld = 0; const double* nll = 0;
  const int32_t* amax_b = 0; const int32_t* amax_q = 0;
  const kld_row_t* rec = 0; int64_t n = 0; float ms = 0.f;
  printf("%d %d %d %d\n", (int)kld_stats_rows(0, &kld, &nll, &amax_b, &amax_q),
         (int)kld_stats_records(0, &rec, &n), (int)kld_stats_second_pass_timing(0, &ms),
         kld_abi_version());
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(src)
        libdir = os.path.dirname(build.LIB)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe, build.LIB,
                        f"-Wl,-rpath,{libdir}"], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()
    assert [int(x) for x in out] == [_lib.KLD_ERR_INVALID_ARG] * 3 + [4]


def test_create_without_gpu_reports_no_device(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    assert lib.kld_stats_create(ctypes.byref(h), 16, 0) == _lib.KLD_ERR_NO_DEVICE
    assert not h.value
    assert lib.kld_last_cuda_error()


def _tail_ranges(n, v, sms, p):
    """Items of every CTA under plan p, recomputed from the plan's fields:
    whole rows round robin, then balanced ranges of the tail's chunks."""
    nchv = -(-v // 512)
    items = {b: [] for b in range(p["grid"])}
    for b in range(p["grid"]):
        for j in range(p["whole_rounds"]):
            r = b + j * p["grid"]
            if r < n:
                items[b].append((r, 0, nchv))
    R, Gt = p["tail_rows"], p["tail_ctas"]
    if R:
        Tc = R * nchv
        for b in range(Gt):
            c0, c1 = Tc * b // Gt, Tc * (b + 1) // Gt
            for rt in range(c0 // nchv, (c1 - 1) // nchv + 1):
                lo, hi = max(c0, rt * nchv) - rt * nchv, min(c1, (rt + 1) * nchv) - rt * nchv
                items[b].append((p["whole_rounds"] * p["grid"] + rt, lo, hi))
    return items


def test_plan_host_logic():
    p = plan(8192, 151936, _lib.KLD_F32, 148)
    # many whole rounds: the last partial wave takes whole rows too
    assert (p["variant"], p["grid"], p["whole_rounds"], p["tail_rows"]) == (0, 148, 56, 0)
    assert p["threads"] % 32 == 0 and p["smem_bytes"] <= 227 * 1024
    # two whole rounds, then 4 rows split over the SMs
    p = plan(300, 151936, _lib.KLD_BF16, 148)
    assert (p["variant"], p["whole_rounds"], p["tail_rows"]) == (2, 2, 4)
    # three whole rounds: whole rows
    p = plan(3 * 148 + 5, 151936, _lib.KLD_F32, 148)
    assert (p["variant"], p["whole_rounds"], p["tail_rows"]) == (0, 4, 0)
    p = plan(148 * 4, 151936, _lib.KLD_F32, 148)
    assert (p["variant"], p["whole_rounds"], p["tail_rows"]) == (0, 4, 0)
    # one row more than a wave: that row over as many CTAs as keep >= 10 chunks each
    p = plan(149, 151936, _lib.KLD_F32, 148)
    assert (p["variant"], p["whole_rounds"], p["tail_rows"], p["tail_ctas"]) == (2, 1, 1, 29)
    # few rows: every row split into row-aligned parts, one per CTA
    p = plan(1, 262144, _lib.KLD_F32, 148)
    assert (p["variant"], p["whole_rounds"], p["tail_rows"], p["grid"], p["ctas_per_row"]) == (2, 0, 1, 32, 32)
    p = plan(16, 262144, _lib.KLD_F32, 148)
    assert (p["grid"], p["ctas_per_row"]) == (144, 9)
    # between half a wave and a wave, and a large last wave: whole rows
    assert plan(100, 151936, _lib.KLD_F32, 148)["variant"] == 0
    p = plan(1000, 151936, _lib.KLD_F32, 148)
    assert (p["variant"], p["whole_rounds"], p["grid"]) == (0, 7, 148)
    for sms in (1, 8, 132, 148):
        for n in list(range(1, 320)) + [1000, 8192, 8193, 32768]:
            for v in (1, 7, 512, 513, 4096, 70001, 151936):
                p = plan(n, v, _lib.KLD_F32, sms)
                assert p["cluster_ctas"] == 1 and p["variant"] in (0, 2) and p["grid"] <= sms
                if p["tail_rows"]:
                    # a split last wave of at most sms/2 rows after at most two
                    # whole rounds (all rows below one wave: row-aligned parts)
                    assert p["variant"] == 2 and 2 * p["tail_rows"] <= sms
                    assert p["whole_rounds"] == n // sms <= 2 and p["tail_rows"] == n % sms
                    assert p["tail_rows"] <= p["tail_ctas"] <= p["grid"]
                    if p["whole_rounds"] == 0:
                        assert p["tail_ctas"] % n == 0 and p["ctas_per_row"] == p["tail_ctas"] // n
                else:
                    # whole rows round robin over grid CTAs
                    assert p["variant"] == 0 and p["whole_rounds"] * p["grid"] >= n
                    assert (p["whole_rounds"] - 1) * p["grid"] < n
                if n > 300 and v > 4096:
                    continue  # the item check below is exhaustive for the small cases
                items = _tail_ranges(n, v, sms, p)
                nchv = -(-v // 512)
                seen = {}
                for b, its in items.items():
                    assert len(its) <= p["whole_rounds"] + 2
                    for r, lo, hi in its:
                        seen.setdefault(r, []).append((lo, hi, b))
                assert sorted(seen) == list(range(n))  # every row, once per part
                for r, parts in seen.items():
                    parts.sort()
                    assert parts[0][0] == 0 and parts[-1][1] == nchv
                    assert all(parts[i][1] == parts[i + 1][0] for i in range(len(parts) - 1))
                    assert len(parts) <= 32 and len(parts) <= max(1, p["ctas_per_row"])
    lib = _lib.load()
    out = _lib.Plan()
    assert lib.kld_plan(0, 10, 0, 148, ctypes.byref(out)) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_plan(1, 0, 0, 148, ctypes.byref(out)) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_plan(1, 1 << 31, 0, 148, ctypes.byref(out)) == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_plan(1, 10, 7, 148, ctypes.byref(out)) == _lib.KLD_ERR_DTYPE
    assert lib.kld_plan(1, 10, 0, 0, ctypes.byref(out)) == _lib.KLD_ERR_INVALID_ARG


def test_product_code_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "logit_kl_divergence_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".h", ".cuh")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "kld_oracle" not in text, f
