"""The C-ABI library loads without a GPU and exports every function that include/dg.h
declares; host-side helpers that need no device behave as documented."""
import ctypes
import subprocess
import threading

import pytest

from moe_grouped_gemm_sm_b200 import _lib, build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_header_declares_the_boundary():
    names = set(_lib.declared_functions())
    assert {"dg_fp8_gemm_nt", "dg_m_grouped_fp8_gemm_nt_contiguous", "dg_m_grouped_fp8_gemm_nt_masked",
            "dg_transform_sf", "dg_cast_fp8_per_token", "dg_cast_fp8_per_block", "dg_sf_ld",
            "dg_get_device_error", "dg_status_string"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in _lib.declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(_lib.declared_functions()) <= exported
    # only the ABI is exported (no C++ or CUDA runtime symbols leak out)
    assert all(s.startswith("dg_") or s.startswith("_init") or s.startswith("_fini") for s in exported), \
        sorted(s for s in exported if not s.startswith("dg_"))[:10]


def test_host_only_helpers(lib):
    assert [_lib.dg_sf_ld(x) for x in (0, 1, 4, 5, 4093)] == [0, 4, 4, 8, 4096]
    for code, name in _lib.STATUS.items():
        assert _lib.dg_status_string(code) == name


def test_last_call_reporting_starts_empty(lib):
    """dg_last_kernel / dg_last_launch_count are per thread: a thread that made no GEMM call
    sees the empty name and a count of 0."""
    seen = {}

    def probe():
        seen["name"] = _lib.dg_last_kernel()
        seen["launches"] = _lib.dg_last_launch_count()
    t = threading.Thread(target=probe)
    t.start()
    t.join()
    assert seen == {"name": "", "launches": 0}


def test_newer_entry_points_reject_bad_arguments_without_a_device(lib):
    P = 16
    ks = (ctypes.c_int * 2)(128, 256)
    bad_ks = (ctypes.c_int * 2)(128, 100)
    kg = lib.dg_k_grouped_fp8_gemm_tn_contiguous
    assert kg(P, P, P, P, None, P, ks, P, 2, 64, 136, None) == _lib.DG_ERR_INVALID_ARG      # N % 16
    assert kg(P, P, P, P, None, P, ks, P, 2, 72, 128, None) == _lib.DG_ERR_INVALID_ARG      # M % 16
    assert kg(P, P, P, P, None, P, bad_ks, P, 2, 64, 128, None) == _lib.DG_ERR_INVALID_ARG  # K group % 128
    assert kg(P, P, P, P, None, P, ks, P, 0, 64, 128, None) == _lib.DG_ERR_INVALID_ARG      # G = 0
    assert kg(P, P, P, P, None, P, ks, P, 512, 64, 128, None) == _lib.DG_ERR_INVALID_ARG    # G > 511
    assert kg(P, P, P, P, None, P + 4, ks, P, 2, 64, 128, None) == _lib.DG_ERR_ALIGNMENT
    assert kg(P, P, P, P, None, P, ks, P, 2, 0, 128, None) == _lib.DG_OK                     # empty
    assert lib.dg_fp8_gemm_nt_ue8m0(P, P, P, P, None, P, 64, 136, 128, None) == _lib.DG_ERR_INVALID_ARG
    assert lib.dg_fp8_gemm_nt_ue8m0(P, P, P, P, None, P, 0, 128, 128, None) == _lib.DG_OK
    assert lib.dg_fp8_gemm_nn(P, P, P, P, None, P, 64, 136, 128, None) == _lib.DG_ERR_INVALID_ARG   # B MN-major: N % 16
    assert lib.dg_fp8_gemm_tn(P, P, P, P, None, P, 72, 128, 128, None) == _lib.DG_ERR_INVALID_ARG   # A MN-major: M % 16
    assert lib.dg_fp8_gemm_tt(P, P, P, P, None, P, 72, 136, 128, None) == _lib.DG_ERR_INVALID_ARG
    assert lib.dg_fp8_gemm_tt(P, P, P, P, None, P, 0, 128, 128, None) == _lib.DG_OK
    assert lib.dg_fp8_gemm_nt_noalloc(P, P, P, P, None, P, 64, 128, 100, None) == _lib.DG_ERR_INVALID_ARG


def test_argument_errors_need_no_device(lib):
    # rejected before any device query: NULL tensors, K not a multiple of 128, N % 8 != 0
    P = 16
    assert lib.dg_fp8_gemm_nt(None, P, P, P, None, P, 64, 128, 128, None) == _lib.DG_ERR_INVALID_ARG
    assert lib.dg_fp8_gemm_nt(P, P, P, P, None, P, 64, 128, 100, None) == _lib.DG_ERR_INVALID_ARG
    assert lib.dg_fp8_gemm_nt(P, P, P, P, None, P, 64, 12, 128, None) == _lib.DG_ERR_INVALID_ARG
    assert lib.dg_fp8_gemm_nt(P, P, P, P, None, P, -1, 128, 128, None) == _lib.DG_ERR_INVALID_ARG
    assert lib.dg_fp8_gemm_nt(P + 1, P, P, P, None, P, 64, 128, 128, None) == _lib.DG_ERR_ALIGNMENT
    assert lib.dg_fp8_gemm_nt(P, P, P, P, None, P, 0, 128, 128, None) == _lib.DG_OK       # empty
    assert lib.dg_m_grouped_fp8_gemm_nt_contiguous(P, P, P, P, None, P, P, 100, 128, 128, 2, None) \
        == _lib.DG_ERR_INVALID_ARG                                                             # M_sum % 128
    assert lib.dg_m_grouped_fp8_gemm_nt_contiguous(P, P, P, P, None, P, None, 128, 128, 128, 2, None) \
        == _lib.DG_ERR_INVALID_ARG                                                             # no layout
    assert lib.dg_m_grouped_fp8_gemm_nt_masked(P, P, P, P, None, P, P, 64, 0, 256, 128, 128, None) \
        == _lib.DG_ERR_INVALID_ARG                                                             # G = 0
    assert lib.dg_m_grouped_fp8_gemm_nt_masked(P, P, P, P, None, P, None, 64, 2, 256, 128, 128, None) \
        == _lib.DG_ERR_INVALID_ARG                                                             # no masked_m
    assert lib.dg_cast_fp8_per_token(P, P, P, 1, 4, 130, None) == _lib.DG_ERR_INVALID_ARG
    assert lib.dg_cast_fp8_per_block(P, P, P, 1, 4, 100, None) == _lib.DG_ERR_INVALID_ARG
    assert lib.dg_transform_sf(None, P, 1, 4, 4, None) == _lib.DG_ERR_INVALID_ARG


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        _lib.load()
