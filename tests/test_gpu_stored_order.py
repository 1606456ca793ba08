"""x supplied in stored column order (descriptor perm NULL).

A decoder layer's producer can write its output already permuted, so the
layer skips the gather ("SAGE", Figure 6: the permutation exists only to
group the input channels of each tile).  The kernels read the same x values
in the same order either way, so every path must give bit-identical results:
  y(W, perm, x) == y(W with perm NULL, x[:, perm])
and the parity of the permuted path against the oracle carries over."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import need_gpu, rel_err, torch, x_bf16, x_f16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu


def _gemv(W, x_bits):
    M = x_bits.shape[0]
    y = torch.empty((M, W.N), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(svq.svq_linear_gemv_workspace_size(W, M), 1), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    svq.svq_linear_gemv(W, x_f16(x_bits), y, ws)
    torch.cuda.synchronize()
    return y


def _gemm(W, x):
    M = x.shape[0]
    y = torch.empty((M, W.N), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(svq.svq_linear_gemm_workspace_size(W, M), 256), dtype=torch.uint8, device="cuda")
    svq.svq_linear_gemm(W, x, y, ws)
    torch.cuda.synchronize()
    assert svq.svq_get_device_status() == svq.SVQ_OK
    return y


@pytest.mark.parametrize("N,K,b_d,M", [(132, 256, 3, 1), (388, 640, 8, 3), (2560, 9728, 8, 1),
                                       (1024, 2560, 10, 8), (640, 2560, 6, 16)])
def test_gemv_null_perm_bit_exact(N, K, b_d, M):
    need_gpu()
    m = synth.make_matrix(90, b_d, N, K, b_d)
    x = synth.make_x(90, b_d, M, K)
    W = svq.SvqWeight.from_synth(m)
    y1 = _gemv(W, x)
    y2 = _gemv(W.without_perm(), np.ascontiguousarray(x[:, m.perm]))
    assert torch.equal(y1, y2)
    y_ref, den = oracle.linear(m, x)
    assert rel_err(y2.cpu().numpy(), y_ref, den) <= 1e-3


def test_gemv_batched_mixed_null_and_permuted():
    """One grouped launch over matrices with and without perm."""
    need_gpu()
    shapes = [(4096, 2560, 8), (1024, 2560, 7), (2560, 4096, 8), (388, 640, 5)]
    ms = [synth.make_matrix(91, i, N, K, b) for i, (N, K, b) in enumerate(shapes)]
    Ws = [svq.SvqWeight.from_synth(m) for m in ms]
    Wn = [W.without_perm() if i % 2 == 0 else W for i, W in enumerate(Ws)]
    M = 2
    xs_bits = [synth.make_x(91, i, M, m.K) for i, m in enumerate(ms)]
    xs = [x_f16(x) for x in xs_bits]
    xs_n = [x_f16(np.ascontiguousarray(x[:, m.perm])) if i % 2 == 0 else x_f16(x)
            for i, (x, m) in enumerate(zip(xs_bits, ms))]

    def run(mats, xin):
        ys = [torch.empty((M, m.N), dtype=torch.float32, device="cuda") for m in ms]
        ws = torch.empty(max(svq.svq_linear_gemv_batched_workspace_size(mats, M), 1), dtype=torch.uint8,
                         device="cuda")
        svq.svq_workspace_init(ws)
        svq.svq_linear_gemv_batched(mats, xin, ys, ws)
        torch.cuda.synchronize()
        return ys

    for a, b in zip(run(Ws, xs), run(Wn, xs_n)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("N,K,M", [(256, 1024, 64), (1028, 2048, 300), (2560, 1024, 1)])
def test_gemm_null_perm_bit_exact(N, K, M):
    need_gpu()
    m = synth.make_matrix(92, M, N, K, 8)
    x = synth.make_x(92, M, M, K, dtype="bf16")
    W = svq.SvqWeight.from_synth(m)
    y1 = _gemm(W, x_bf16(x))
    y2 = _gemm(W.without_perm(), x_bf16(np.ascontiguousarray(x[:, m.perm])))
    assert torch.equal(y1, y2)
    y_ref, den = oracle.linear(m, x, "bf16")
    assert rel_err(y2.cpu().numpy(), y_ref, den) <= 1e-2


def test_gemm_null_perm_needs_16_byte_aligned_x():
    """With perm NULL the tensor-map load reads x directly: a 2-byte-aligned x is refused before any launch."""
    need_gpu()
    m = synth.make_matrix(93, 0, 256, 1024, 8)
    W = svq.SvqWeight.from_synth(m).without_perm()
    buf = torch.zeros(16 * 1024 + 8, dtype=torch.bfloat16, device="cuda")
    x = buf[1:1 + 16 * 1024].view(16, 1024)
    y = torch.empty((16, 256), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(svq.svq_linear_gemm_workspace_size(W, 16), 256), dtype=torch.uint8, device="cuda")
    with pytest.raises(svq.SvqError) as e:
        svq.svq_linear_gemm(W, x, y, ws)
    assert e.value.status == svq.SVQ_ERR_INVALID_ARG


def test_moe_null_perm_bit_exact():
    """Grouped MoE GEMV over matrices without perm equals the same matrices with the identity permutation."""
    need_gpu()
    E, N, K, T = 8, 768, 2048, 5
    ms = [synth.make_matrix(94, e, N, K, 8, identity_perm=True) for e in range(E)]
    Ws = [svq.SvqWeight.from_synth(m) for m in ms]
    rng = np.random.default_rng(94)
    mat = torch.from_numpy(rng.integers(0, E, 3 * T).astype(np.int32)).cuda()
    xrow = torch.arange(3 * T, device="cuda", dtype=torch.int32) // 3
    orow = torch.arange(3 * T, device="cuda", dtype=torch.int32)
    items = svq.item_table(mat, xrow, orow, torch.ones(3 * T, device="cuda"))
    x = x_f16(synth.make_x(94, 0, T, K))
    max_per = int(torch.bincount(mat.long(), minlength=E).max())

    def run(mats):
        tab = svq.descriptor_table(mats)
        y = torch.empty((3 * T, N), dtype=torch.float32, device="cuda")
        ws = torch.empty(max(svq.svq_moe_grouped_gemv_workspace_size(E, 3 * T, N, False), 1),
                         dtype=torch.uint8, device="cuda")
        svq.svq_moe_grouped_gemv(tab, E, N, K, 8, items, 3 * T, max_per, x, svq.SVQ_X_F16, y, 3 * T, False, ws)
        torch.cuda.synchronize()
        assert svq.svq_get_device_status() == svq.SVQ_OK
        return y

    assert torch.equal(run(Ws), run([W.without_perm() for W in Ws]))
