"""The C-ABI library loads and exports every function include/svq.h declares;
host-side validation (no GPU needed) returns the documented status codes."""
import ctypes
import subprocess

import pytest

import bit_spherical_vector_b200 as svq


def test_library_loads_and_exports_every_declared_symbol():
    names = svq.header_functions()
    assert "svq_repack" in names and "svq_linear_gemv" in names
    L = svq.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, f"declared but not exported: {missing}"
    out = subprocess.run(["nm", "-D", "--defined-only", svq.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(names) <= exported
    # nothing else leaks out of the library with the svq_ prefix
    assert {n for n in exported if n.startswith("svq_")} == set(names)


def test_pure_host_queries():
    assert svq.lib().svq_version() >= 100
    assert svq.svq_packed_bytes(1024, 1024) == 1024 * 1024 * 9 // 32
    assert svq.svq_packed_bytes(2560, 9728) == 2560 * 9728 * 9 // 32
    assert svq.svq_packed_bytes(1024, 1000) == 0          # K % 128 != 0: no device layout
    assert svq.svq_packed_bytes(6, 128) == 0              # N % 4 != 0
    assert svq.svq_canonical_bytes(3, 40) == 3 * 12       # 5 codes * 18 bits = 90 bits -> 12 bytes
    for s in range(6):
        assert svq.status_string(s)
    assert "unknown" in svq.status_string(99)


def test_validation_without_gpu():
    L = svq.lib()
    nullp = ctypes.c_void_p(0)
    dummy = ctypes.c_void_p(0x1000)          # never dereferenced: validation fails first
    assert L.svq_repack(nullp, 128, 128, 8, dummy, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert L.svq_repack(dummy, 128, 100, 8, dummy, nullp) == svq.SVQ_ERR_UNSUPPORTED_SHAPE
    assert L.svq_repack(dummy, 128, 128, 11, dummy, nullp) == svq.SVQ_ERR_UNSUPPORTED_SHAPE
    assert L.svq_repack(dummy, 128, 128, 0, dummy, nullp) == svq.SVQ_ERR_UNSUPPORTED_SHAPE
    assert L.svq_repack(dummy, 128, 128, 8, ctypes.c_void_p(0x1008), nullp) == svq.SVQ_ERR_INVALID_ARG
    m = svq.svq_matrix(128, 128, 8, 0, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000)
    bad = svq.svq_matrix(128, 136, 8, 0, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000)
    n = ctypes.c_size_t(0)
    assert L.svq_linear_gemv_workspace_size(ctypes.byref(bad), 1, ctypes.byref(n)) == svq.SVQ_ERR_UNSUPPORTED_SHAPE
    assert L.svq_linear_gemv_workspace_size(ctypes.byref(m), 0, ctypes.byref(n)) == svq.SVQ_ERR_INVALID_ARG
    assert L.svq_linear_gemv_workspace_size(ctypes.byref(m), 17, ctypes.byref(n)) == svq.SVQ_ERR_INVALID_ARG
    unaligned = svq.svq_matrix(128, 128, 8, 0, 0x1008, 0x2000, 0x3000, 0x4000, 0x5000)
    assert L.svq_dequantize(ctypes.byref(unaligned), svq.SVQ_F16, dummy, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert L.svq_dequantize(ctypes.byref(m), svq.SVQ_F32, dummy, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert L.svq_linear_gemv(ctypes.byref(m), nullp, 1, dummy, svq.SVQ_F32, nullp, 0, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert L.svq_linear_gemv(ctypes.byref(m), dummy, 1, dummy, svq.SVQ_BF16, nullp, 0, nullp) == svq.SVQ_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(svq, "_lib", None)
    monkeypatch.setattr(svq, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        svq.lib()
