"""svq_linear_gemv_noalloc: the GEMV entry point for callers that cannot
allocate device memory (its split-K scratch is a fixed array inside the
library instead of a caller workspace).  Checked through the C ABI against
svq_linear_gemv on two calls in a row, so that scratch contents left by the
first call cannot spoil the second.  This file is collected last; its tests
pass alone in a fresh process and after the rest of the suite."""
import ctypes

import numpy as np
import pytest

import synth
from tests.gpu_util import need_gpu, torch, x_f16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu
TOL = 1e-3
LIMIT = 1 << 20


def _noalloc(desc, x_ptr, M, y_ptr):
    return svq.lib().svq_linear_gemv_noalloc(ctypes.byref(desc), ctypes.c_void_p(x_ptr), M,
                                             ctypes.c_void_p(y_ptr), svq.SVQ_F32,
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("N,K,M,b_d", [(2560, 9728, 1, 8), (1024, 2560, 3, 7), (9728, 2560, 2, 6)])
def test_noalloc_matches_workspace_entry_two_calls(N, K, M, b_d):
    need_gpu()
    m = synth.make_matrix(99, N + M, N, K, b_d)
    W = svq.SvqWeight.from_synth(m)
    nb = svq.svq_linear_gemv_workspace_size(W, M)
    assert 0 < nb <= LIMIT                     # split-K scratch is used, and fits the fixed array
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    wq = torch.empty((N, K), dtype=torch.float16, device="cuda")
    svq.svq_dequantize(W, wq)
    perm = torch.from_numpy(m.perm.astype(np.int64)).cuda()
    for call in range(2):
        x = x_f16(synth.make_x(99, 10 * call + M, M, K))
        ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
        svq.svq_linear_gemv(W, x, ref, ws)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(W.desc, x.data_ptr(), M, y.data_ptr()) == svq.SVQ_OK
        torch.cuda.synchronize()
        den = x[:, perm].float().abs() @ wq.float().abs().t()     # sum_j |W[n][j]| |x[m][perm[j]]|
        assert bool(((y - ref).abs() <= TOL * den).all())
        assert torch.equal(y, ref)             # same kernel and plan: in fact identical


def test_noalloc_rejects_scratch_beyond_limit():
    """A shape whose split-K scratch exceeds the fixed 1 MiB (32768 x 2560, 8 rows: 256 row tiles,
    most of them shared by two or three CTAs) is refused before anything is enqueued (the
    pointers below are never dereferenced)."""
    need_gpu()
    desc = svq.svq_matrix(32768, 2560, 8, 0, 0x10000, 0x20000, 0x30000, 0x40000, 0x50000)
    n = ctypes.c_size_t(0)
    assert svq.lib().svq_linear_gemv_workspace_size(ctypes.byref(desc), 8, ctypes.byref(n)) == svq.SVQ_OK
    assert n.value > LIMIT
    assert _noalloc(desc, 0x60000, 8, 0x70000) == svq.SVQ_ERR_WORKSPACE


def _ptr_y(y):
    return svq.SVQ_F16 if y.dtype == torch.float16 else svq.SVQ_F32


@pytest.mark.parametrize("stored", [False, True])
def test_noalloc_against_oracle_m12_fp16_out(stored):
    """9728 x 2560, M = 12 (two passes of 8 and 4 tokens), fp16 output, against the oracle; with
    stored=True the matrix is called with perm NULL and x already in stored column order."""
    need_gpu()
    import oracle
    N, K, M, b_d = 9728, 2560, 12, 7
    m = synth.make_matrix(98, 12, N, K, b_d)
    W = svq.SvqWeight.from_synth(m)
    x_bits = synth.make_x(98, 13, M, K)
    x = x_f16(x_bits)
    if stored:
        W = W.without_perm()
        x = x[:, torch.from_numpy(m.perm.astype(np.int64)).cuda()].contiguous()
    nb = svq.svq_linear_gemv_workspace_size(W, M)
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    rc = svq.lib().svq_linear_gemv_noalloc(ctypes.byref(W.desc), ctypes.c_void_p(x.data_ptr()), M,
                                           ctypes.c_void_p(y.data_ptr()), _ptr_y(y),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if nb > LIMIT:
        assert rc == svq.SVQ_ERR_WORKSPACE
        return
    assert rc == svq.SVQ_OK
    torch.cuda.synchronize()
    y_ref, den = oracle.linear(m, x_bits)
    got = y.float().cpu().numpy().astype(np.float64)
    # fp16 output: add the output rounding (half an ulp of |y_ref|, 2^-11 relative) to the bound
    assert np.all(np.abs(got - y_ref) <= TOL * den + np.abs(y_ref) * 2.0 ** -11)
