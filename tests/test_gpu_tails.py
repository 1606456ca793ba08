"""Shape tails: N not a multiple of 4, K a multiple of 8 but not of 128.

The device layout stores such matrices padded (Np = 4 ceil(N/4) rows, Kp = 128
ceil(K/128) columns, zero codes); kernels read activation columns >= K as zero
and write no row >= N.  Checked against the oracle on the unpadded matrix:
repack/unpack and dequantize bit-exact, GEMV within 1e-3 and GEMM within 1e-2
of sum_j |W[n][j]| |x[m][perm[j]]|, with and without permutation, with radius
tables, grouped with aligned shapes.  The MoE kernel refuses ragged shapes."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import need_gpu, rel_err, torch, u16, x_bf16, x_f16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu

SHAPES = [(6, 8), (130, 200), (1, 1000), (257, 136), (1030, 1032), (4098, 2568)]


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("b_d", [7, 9])
def test_format_roundtrip_and_dequant(N, K, b_d):
    m = synth.make_matrix(120, N + K + b_d, N, K, b_d)
    W = svq.SvqWeight.from_synth(m)
    G = K // 8
    sg = torch.empty((N, G), dtype=torch.uint8, device="cuda")
    ix = torch.empty((N, G), dtype=torch.int16, device="cuda")
    cd = torch.empty((N, G), dtype=torch.int16, device="cuda")
    svq.svq_unpack_fields(W.packed, N, K, b_d, sg, ix, cd)
    torch.cuda.synchronize()
    s, i, c = oracle.unpack(N, K, b_d, m.canonical)
    assert np.array_equal(sg.cpu().numpy(), s) and np.array_equal(u16(ix), i) and np.array_equal(u16(cd), c)
    out = torch.empty((N, K), dtype=torch.float16, device="cuda")
    svq.svq_dequantize(W, out)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out), oracle.dequant(m, "f16"))


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("M", [1, 3, 9])
def test_gemv_every_output(N, K, M):
    m = synth.make_matrix(121, N * 7 + K, N, K, 8)
    x = synth.make_x(121, M, M, K)
    W = svq.SvqWeight.from_synth(m)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(svq.svq_linear_gemv_workspace_size(W, M), 256), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    svq.svq_linear_gemv(W, x_f16(x), y, ws)
    torch.cuda.synchronize()
    y_ref, den = oracle.linear(m, x)
    assert rel_err(y.cpu().numpy(), y_ref, den) <= 1e-3
    # the same matrix called with x already in stored order (perm NULL)
    xs = x_f16(np.ascontiguousarray(x[:, m.perm]))
    y2 = torch.empty_like(y)
    svq.svq_linear_gemv(W.without_perm(), xs, y2, ws)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


def test_gemv_tail_with_radius_tables_and_grouped():
    """A ragged matrix with a radius table, and a grouped call mixing ragged and aligned shapes."""
    m = synth.make_matrix(122, 0, 130, 200, 7)
    m.lut = synth.make_lut(122, 0, 130, 7)
    x = synth.make_x(122, 0, 2, 200)
    W = svq.SvqWeight.from_synth(m)
    y = torch.empty((2, 130), dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    svq.svq_linear_gemv(W, x_f16(x), y, ws)
    torch.cuda.synchronize()
    y_ref, den = oracle.linear(m, x)
    assert rel_err(y.cpu().numpy(), y_ref, den) <= 1e-3
    shapes = [(1030, 1032, 7), (1024, 1024, 8), (6, 8, 9)]
    mats = [synth.make_matrix(123, i, N, K, b) for i, (N, K, b) in enumerate(shapes)]
    xs = [synth.make_x(123, 10 + i, 1, K) for i, (N, K, b) in enumerate(shapes)]
    Ws = [svq.SvqWeight.from_synth(mm) for mm in mats]
    ys = [torch.empty((1, N), dtype=torch.float32, device="cuda") for N, _, _ in shapes]
    wsb = torch.empty(max(svq.svq_linear_gemv_batched_workspace_size(Ws, 1), 256), dtype=torch.uint8,
                      device="cuda")
    svq.svq_workspace_init(wsb)
    svq.svq_linear_gemv_batched(Ws, [x_f16(v) for v in xs], ys, wsb)
    torch.cuda.synchronize()
    for mm, v, yy in zip(mats, xs, ys):
        y_ref, den = oracle.linear(mm, v)
        assert rel_err(yy.cpu().numpy(), y_ref, den) <= 1e-3


@pytest.mark.parametrize("N,K,M", [(6, 8, 3), (130, 200, 100), (1030, 1032, 1100), (257, 136, 40)])
@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
def test_gemm_every_output(N, K, M, y_dtype):
    m = synth.make_matrix(124, N + M, N, K, 8)
    x = synth.make_x(124, M, M, K, dtype="bf16")
    W = svq.SvqWeight.from_synth(m)
    y = torch.empty((M, N), dtype=y_dtype, device="cuda")
    ws = torch.empty(max(svq.svq_linear_gemm_workspace_size(W, M), 256), dtype=torch.uint8, device="cuda")
    svq.svq_linear_gemm(W, x_bf16(x), y, ws)
    torch.cuda.synchronize()
    assert svq.svq_get_device_status() == svq.SVQ_OK
    y_ref, den = oracle.linear(m, x, "bf16")
    tol = 1e-2 + (2.0 ** -8 if y_dtype == torch.bfloat16 else 0.0)
    assert rel_err(y.float().cpu().numpy(), y_ref, den) <= tol


def test_moe_refuses_ragged_shapes():
    m = synth.make_matrix(125, 0, 130, 256, 8)
    W = svq.SvqWeight.from_synth(m)
    tab = svq.descriptor_table([W])
    items = svq.item_table(torch.zeros(1, dtype=torch.int32, device="cuda"),
                           torch.zeros(1, dtype=torch.int32, device="cuda"),
                           torch.zeros(1, dtype=torch.int32, device="cuda"), torch.ones(1, device="cuda"))
    x = x_f16(synth.make_x(125, 0, 1, 256))
    y = torch.empty((1, 130), dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(svq.SvqError) as e:
        svq.svq_moe_grouped_gemv(tab, 1, 130, 256, 8, items, 1, 1, x, svq.SVQ_X_F16, y, 1, False, ws)
    assert e.value.status == svq.SVQ_ERR_UNSUPPORTED_SHAPE
