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
    assert svq.svq_packed_bytes(1024, 1000) == 1024 * 1024 * 9 // 32   # K padded to 1024 columns
    assert svq.svq_packed_bytes(6, 128) == 8 * 128 * 9 // 32            # N padded to 8 rows
    assert svq.svq_packed_bytes(1024, 1004) == 0          # K % 8 != 0: not an SVQ shape
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
    bad = svq.svq_matrix(128, 132, 8, 0, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000)      # K % 8 != 0
    n = ctypes.c_size_t(0)
    assert L.svq_linear_gemv_workspace_size(ctypes.byref(bad), 1, ctypes.byref(n)) == svq.SVQ_ERR_UNSUPPORTED_SHAPE
    assert L.svq_linear_gemv_workspace_size(ctypes.byref(m), 0, ctypes.byref(n)) == svq.SVQ_ERR_INVALID_ARG
    assert L.svq_linear_gemv_workspace_size(ctypes.byref(m), 17, ctypes.byref(n)) == svq.SVQ_ERR_INVALID_ARG
    unaligned = svq.svq_matrix(128, 128, 8, 0, 0x1008, 0x2000, 0x3000, 0x4000, 0x5000)
    assert L.svq_dequantize(ctypes.byref(unaligned), svq.SVQ_F16, dummy, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert L.svq_dequantize(ctypes.byref(m), svq.SVQ_F32, dummy, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert L.svq_linear_gemv(ctypes.byref(m), nullp, 1, dummy, svq.SVQ_F32, nullp, 0, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert L.svq_linear_gemv(ctypes.byref(m), dummy, 1, dummy, svq.SVQ_BF16, nullp, 0, nullp) == svq.SVQ_ERR_INVALID_ARG
    # host-buffer grouped call: every check runs before anything is enqueued
    mats = (svq.svq_matrix * 1)(m)
    hc = L.svq_linear_gemv_batched_host
    assert hc(mats, 1, nullp, dummy, 1, dummy, dummy, svq.SVQ_F32, nullp, 0, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert hc(mats, 0, dummy, dummy, 1, dummy, dummy, svq.SVQ_F32, nullp, 0, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert hc(mats, 1, dummy, dummy, 0, dummy, dummy, svq.SVQ_F32, nullp, 0, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert hc(mats, 1, dummy, dummy, 1, dummy, dummy, svq.SVQ_BF16, nullp, 0, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert hc(mats, 1, dummy, ctypes.c_void_p(0x1001), 1, dummy, dummy, svq.SVQ_F32, nullp, 0,
              nullp) == svq.SVQ_ERR_INVALID_ARG
    badm = (svq.svq_matrix * 1)(bad)
    assert hc(badm, 1, dummy, dummy, 1, dummy, dummy, svq.SVQ_F32, nullp, 0, nullp) == svq.SVQ_ERR_UNSUPPORTED_SHAPE


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(svq, "_lib", None)
    monkeypatch.setattr(svq, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        svq.lib()


def test_header_compiles_as_c_and_links(tmp_path):
    """include/svq.h is plain C (C99, warnings as errors); a C program links against libsvq.so and calls the
    host-only entry points."""
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "use_svq.c"
    src.write_text(
        '#include <stdio.h>\n#include "svq.h"\n'
        "int main(void) {\n"
        "  svq_matrix m = {128, 128, 8, 0, 0, 0, 0, 0, 0, 0};\n"
        "  size_t n = 0;\n"
        "  int st = svq_linear_gemv_workspace_size(&m, 1, &n);\n"
        '  printf("%zu %zu %d %s\\n", svq_packed_bytes(1024, 1024), svq_canonical_bytes(3, 40), st,\n'
        "         svq_status_string(SVQ_ERR_WORKSPACE));\n"
        "  return 0;\n}\n")
    exe = tmp_path / "use_svq"
    libdir = os.path.dirname(svq.LIB_PATH)
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"),
                         str(src), "-L", libdir, "-lsvq", "-Wl,-rpath," + libdir, "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, run.stderr
    packed, canon, st, msg = run.stdout.split(" ", 3)
    assert int(packed) == 1024 * 1024 * 9 // 32 and int(canon) == 36
    assert int(st) == svq.SVQ_ERR_INVALID_ARG          # NULL weight pointers are refused on the host
    assert msg.strip()


def test_stored_order_and_producer_validation_without_gpu():
    """Checks that return before any CUDA call: perm NULL is accepted by the matrix check, the GEMM then
    wants a 16-byte aligned x; producers refuse bad counts, shapes and alignments, and M = 0 is a no-op."""
    L = svq.lib()
    nullp = ctypes.c_void_p(0)
    m = svq.svq_matrix(128, 128, 8, 0, 0x1000, 0x2000, 0x3000, 0x4000, 0)     # perm NULL
    x_unaligned = ctypes.c_void_p(0x6002)
    assert L.svq_linear_gemm(ctypes.byref(m), x_unaligned, svq.SVQ_BF16, 16, ctypes.c_void_p(0x7000),
                             svq.SVQ_F32, nullp, 0, nullp) == svq.SVQ_ERR_INVALID_ARG
    badperm = svq.svq_matrix(128, 128, 8, 0, 0x1000, 0x2000, 0x3000, 0x4000, 0x5002)
    assert L.svq_dequantize(ctypes.byref(badperm), svq.SVQ_F16, ctypes.c_void_p(0x7000), nullp) == \
        svq.SVQ_ERR_INVALID_ARG
    P = ctypes.c_void_p
    outs = (P * 2)(0x8000, 0x9000)
    perms = (P * 2)(0, 0)
    h, gamma = P(0x1000), P(0x2000)
    f = L.svq_rmsnorm_permute
    assert f(h, svq.SVQ_F16, gamma, 1e-6, 1, 64, perms, outs, 0, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert f(h, svq.SVQ_F16, gamma, 1e-6, 1, 64, perms, outs, 9, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert f(h, svq.SVQ_F32, gamma, 1e-6, 1, 64, perms, outs, 2, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert f(h, svq.SVQ_F16, gamma, -1.0, 1, 64, perms, outs, 2, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert f(h, svq.SVQ_F16, gamma, 1e-6, 1, 60, perms, outs, 2, nullp) == svq.SVQ_ERR_UNSUPPORTED_SHAPE
    assert f(P(0x1002), svq.SVQ_F16, gamma, 1e-6, 1, 64, perms, outs, 2, nullp) == svq.SVQ_ERR_INVALID_ARG
    assert f(h, svq.SVQ_F16, gamma, 1e-6, 0, 64, perms, outs, 2, nullp) == svq.SVQ_OK
    g = L.svq_swiglu_permute
    assert g(P(0x1000), P(0x2000), 1, 12, nullp, P(0x3000), nullp) == svq.SVQ_ERR_UNSUPPORTED_SHAPE
    assert g(P(0x1000), P(0x2004), 1, 16, nullp, P(0x3000), nullp) == svq.SVQ_ERR_INVALID_ARG
    assert g(P(0x1000), P(0x2000), 1, 16, P(0x4002), P(0x3000), nullp) == svq.SVQ_ERR_INVALID_ARG
    assert g(nullp, nullp, 0, 16, nullp, nullp, nullp) == svq.SVQ_OK
