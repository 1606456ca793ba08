"""GPU parity of the per-row radius table (svq_matrix.radius_lut: r = lut[n][code],
2^b_r fp16 levels per row, b_r <= 4) against the oracle's table form.

Bars as for the affine radius: dequantized weights bit-exact; GEMV within 1e-3
and GEMM within 1e-2 of sum_j |W[n][j]| |x[m][perm[j]]|; the encoder's codes
bit-exact.  Matrices with a table are refused where they are not taken (the MoE
kernel reports them through the status word; b_r > 4 and groups mixing both
forms are refused at the call)."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import need_gpu, rel_err, torch, u16, x_bf16, x_f16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def _lut_matrix(config, N, K, b_d):
    m = synth.make_matrix(config, b_d, N, K, b_d)
    m.lut = synth.make_lut(config, b_d, N, b_d)
    return m


def _gemv(W, x_bits):
    M = x_bits.shape[0]
    y = torch.empty((M, W.N), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(svq.svq_linear_gemv_workspace_size(W, M), 1), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    svq.svq_linear_gemv(W, x_f16(x_bits), y, ws)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("b_d", [6, 7, 8, 9, 10])
@pytest.mark.parametrize("N", [256, 132])
def test_dequantize_bit_exact(b_d, N):
    m = _lut_matrix(110, N, 384, b_d)
    W = svq.SvqWeight.from_synth(m)
    for kind, dt in (("f16", torch.float16), ("bf16", torch.bfloat16)):
        out = torch.empty((m.N, m.K), dtype=dt, device="cuda")
        svq.svq_dequantize(W, out)
        torch.cuda.synchronize()
        assert np.array_equal(u16(out), oracle.dequant(m, kind))


@pytest.mark.parametrize("b_d", [6, 8, 9])
@pytest.mark.parametrize("N,K", [(1024, 1152), (132, 256), (4100, 2560)])
@pytest.mark.parametrize("M", [1, 2, 5, 9])
def test_gemv_every_output(b_d, N, K, M):
    m = _lut_matrix(111, N, K, b_d)
    x = synth.make_x(111, b_d, M, K)
    y = _gemv(svq.SvqWeight.from_synth(m), x)
    y_ref, den = oracle.linear(m, x)
    assert rel_err(y, y_ref, den) <= 1e-3


def test_grouped_decoder_layer_with_tables():
    """The seven decoder-layer linears, each with a radius table, in one grouped launch (batch 1)."""
    layer = synth.qwen3_4b_layer(0)
    mats = []
    for i, (m, _) in enumerate(layer):
        m.lut = synth.make_lut(112, i, m.N, m.b_d)
        mats.append(m)
    Ws = [svq.SvqWeight.from_synth(m) for m in mats]
    xs = [x_f16(x) for _, x in layer]
    ys = [torch.empty((1, m.N), dtype=torch.float32, device="cuda") for m in mats]
    ws = torch.empty(max(svq.svq_linear_gemv_batched_workspace_size(Ws, 1), 1), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    svq.svq_linear_gemv_batched(Ws, xs, ys, ws)
    torch.cuda.synchronize()
    for (m, x), y in zip(zip(mats, [x for _, x in layer]), ys):
        y_ref, den = oracle.linear(m, x)
        assert rel_err(y.cpu().numpy(), y_ref, den) <= 1e-3


def test_group_mixing_both_forms_refused():
    a = svq.SvqWeight.from_synth(_lut_matrix(113, 256, 256, 7))
    b = svq.SvqWeight.from_synth(synth.make_matrix(113, 1, 256, 256, 7))
    xs = [x_f16(synth.make_x(113, i, 1, 256)) for i in range(2)]
    ys = [torch.empty((1, 256), dtype=torch.float32, device="cuda") for _ in range(2)]
    ws = torch.empty(1 << 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(svq.SvqError) as e:
        svq.svq_linear_gemv_batched([a, b], xs, ys, ws)
    assert e.value.status == svq.SVQ_ERR_INVALID_ARG


def test_table_needs_at_most_16_levels():
    m = synth.make_matrix(114, 0, 256, 256, 5)
    m.lut = synth.make_lut(114, 0, 256, 5)                  # 32 levels
    W = svq.SvqWeight.from_synth(m)
    y = torch.empty((1, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(svq.SvqError) as e:
        svq.svq_linear_gemv(W, x_f16(synth.make_x(114, 0, 1, 256)), y, torch.empty(1 << 16, dtype=torch.uint8,
                                                                                  device="cuda"))
    assert e.value.status == svq.SVQ_ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("M", [100, 1100])
def test_gemm_with_tables(M):
    """On-chip decode (100 tokens) and the pre-decoded plan (1100 tokens) with radius tables."""
    m = _lut_matrix(115, 1028, 512, 8)
    x = synth.make_x(115, M, M, 512, dtype="bf16")
    W = svq.SvqWeight.from_synth(m)
    y = torch.empty((M, m.N), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(svq.svq_linear_gemm_workspace_size(W, M), 256), dtype=torch.uint8, device="cuda")
    svq.svq_linear_gemm(W, x_bf16(x), y, ws)
    torch.cuda.synchronize()
    assert svq.svq_get_device_status() == svq.SVQ_OK
    y_ref, den = oracle.linear(m, x, "bf16")
    assert rel_err(y.cpu().numpy(), y_ref, den) <= 1e-2


@pytest.mark.parametrize("b_d", [6, 7, 9])
def test_encoder_with_tables_bit_exact(b_d):
    N, K = 12, 328
    m = _lut_matrix(116, N, K, b_d)
    Ws = oracle.decode_exact(m)
    rng = np.random.default_rng(116)
    Ws = Ws * (1.0 + 0.03 * rng.standard_normal(Ws.shape))
    W = np.empty_like(Ws)
    W[:, m.perm] = Ws
    W = W.astype(np.float32)
    wts = rng.lognormal(0.0, 1.0, K).astype(np.float32)
    canon = torch.zeros((N, oracle.row_bytes(K)), dtype=torch.uint8, device="cuda")
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    dev16 = lambda a: dev(np.ascontiguousarray(a, np.uint16).view(np.int16))
    svq.svq_encode(dev(W), b_d, dev(m.perm.astype(np.int32)), dev(wts), dev16(m.codebook), None, None, canon,
                   lut=dev16(m.lut))
    torch.cuda.synchronize()
    Wst = np.ascontiguousarray(W.astype(np.float64)[:, m.perm])
    ws = np.ascontiguousarray(wts.astype(np.float64)[m.perm])
    s, i, c = oracle.encode(N, K, b_d, Wst, m.codebook, None, None, ws, lut=m.lut)
    assert np.array_equal(canon.cpu().numpy(), oracle.pack(N, K, b_d, s, i, c))


def test_moe_reports_a_matrix_with_a_table():
    m = _lut_matrix(117, 256, 256, 8)
    W = svq.SvqWeight.from_synth(m)
    tab = svq.descriptor_table([W])
    x = x_f16(synth.make_x(117, 0, 1, 256))
    items = svq.item_table(torch.zeros(1, dtype=torch.int32, device="cuda"),
                           torch.zeros(1, dtype=torch.int32, device="cuda"),
                           torch.zeros(1, dtype=torch.int32, device="cuda"), torch.ones(1, device="cuda"))
    y = torch.full((1, 256), 5.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(svq.svq_moe_grouped_gemv_workspace_size(1, 1, 256, False), 256), dtype=torch.uint8,
                     device="cuda")
    assert svq.svq_get_device_status() == svq.SVQ_OK
    svq.svq_moe_grouped_gemv(tab, 1, 256, 256, 8, items, 1, 1, x, svq.SVQ_X_F16, y, 1, False, ws)
    torch.cuda.synchronize()
    assert svq.svq_get_device_status() == svq.SVQ_ERR_INVALID_ARG
    assert np.all(y.cpu().numpy() == 0.0)                    # the refused matrix decodes as zeros
