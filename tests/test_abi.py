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
    assert lib.kld_abi_version() == 3
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
    assert [int(x) for x in out] == [_lib.KLD_ERR_INVALID_ARG] * 3 + [3]


def test_create_without_gpu_reports_no_device(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    assert lib.kld_stats_create(ctypes.byref(h), 16, 0) == _lib.KLD_ERR_NO_DEVICE
    assert not h.value
    assert lib.kld_last_cuda_error()


def test_plan_host_logic():
    p = plan(8192, 151936, _lib.KLD_F32, 148)
    assert p["grid"] == 148 and p["threads"] % 32 == 0
    assert p["smem_bytes"] <= 227 * 1024
    # few rows: split into as many parts (<= 32 per row) as fit in one wave
    p = plan(1, 151936, _lib.KLD_F32, 148)
    assert (p["variant"], p["cluster_ctas"], p["ctas_per_row"], p["grid"]) == (1, 1, 32, 32)
    p = plan(5, 1000, _lib.KLD_BF16, 148)
    assert (p["variant"], p["cluster_ctas"], p["ctas_per_row"], p["grid"]) == (1, 1, 29, 145)
    p = plan(74, 1000, _lib.KLD_F16, 148)
    assert (p["cluster_ctas"], p["ctas_per_row"], p["grid"]) == (1, 2, 148)
    p = plan(75, 1000, _lib.KLD_F32, 148)
    assert (p["variant"], p["cluster_ctas"], p["ctas_per_row"], p["grid"]) == (0, 1, 1, 75)
    for sms in (1, 8, 132, 148):
        for n in range(1, 300):
            p = plan(n, 4096, _lib.KLD_F32, sms)
            g, per = p["cluster_ctas"], p["ctas_per_row"]
            assert g in (1, 2, 4, 8) and per % g == 0 and per // g <= 32
            if p["variant"] == 0:
                assert per == 1 and g == 1 and p["grid"] == min(n, sms)
            else:
                assert 2 * n <= sms and p["grid"] == n * per <= sms and per >= 2
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
