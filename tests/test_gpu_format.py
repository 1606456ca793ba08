"""GPU parity of the integer path: repack -> field unpack and the dense
dequantisation are bit-exact against the CPU oracle (integer work: exact;
fp16/bf16 exports: exact bit patterns, including -0 and subnormals)."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import need_gpu, torch, u16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu

SHAPES = [(4, 128), (128, 128), (132, 256), (260, 384), (1024, 1024), (512, 9728)]


def _fields_gpu(W):
    G = W.K // 8
    s = torch.empty((W.N, G), dtype=torch.uint8, device="cuda")
    i = torch.empty((W.N, G), dtype=torch.int16, device="cuda")
    c = torch.empty((W.N, G), dtype=torch.int16, device="cuda")
    svq.svq_unpack_fields(W.packed, W.N, W.K, W.b_d, s, i, c)
    torch.cuda.synchronize()
    return s.cpu().numpy(), u16(i), u16(c)


@pytest.mark.parametrize("b_d", range(1, 11))
@pytest.mark.parametrize("N,K", SHAPES)
def test_repack_unpack_bit_exact(N, K, b_d):
    need_gpu()
    m = synth.make_matrix(50, 100 * b_d + N % 97, N, K, b_d)
    W = svq.SvqWeight.from_synth(m)
    assert W.packed.numel() == N * K * 9 // 32
    s, i, c = _fields_gpu(W)
    rs, ri, rc = oracle.unpack(N, K, b_d, m.canonical)
    assert np.array_equal(s, rs)
    assert np.array_equal(i, ri)
    assert np.array_equal(c, rc)


@pytest.mark.parametrize("b_d", range(1, 11))
@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("kind", ["f16", "bf16"])
def test_dequantize_bit_exact(N, K, b_d, kind):
    need_gpu()
    m = synth.make_matrix(51, 100 * b_d + N % 97, N, K, b_d)
    W = svq.SvqWeight.from_synth(m)
    out = torch.empty((N, K), dtype=torch.float16 if kind == "f16" else torch.bfloat16, device="cuda")
    svq.svq_dequantize(W, out)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out), oracle.dequant(m, kind))


def test_dequantize_negative_zero_and_subnormals():
    """A codebook with zero and tiny components: -0 and fp16 subnormals must match bit for bit."""
    need_gpu()
    N, K, b_d = 8, 128, 4
    m = synth.make_matrix(52, 0, N, K, b_d)
    cb = m.codebook.view(np.float16).copy()
    cb[0] = 0
    cb[1] = np.array([2.0 ** -20, 2.0 ** -24, 0, 1, 0, 2.0 ** -15, 0, 0], np.float16)
    cb[2, :4] = 0
    m.codebook = cb.view(np.uint16)
    W = svq.SvqWeight.from_synth(m)
    out = torch.empty((N, K), dtype=torch.float16, device="cuda")
    svq.svq_dequantize(W, out)
    torch.cuda.synchronize()
    want = oracle.dequant(m, "f16")
    assert np.array_equal(u16(out), want)
    assert (want == 0x8000).any() and ((want & 0x7C00) == 0).any()


@pytest.mark.parametrize("name,N,K,b_d", [(n, N, K, b) for (n, N, K), b in
                                         zip(synth.QWEN3_4B_SHAPES, synth.QWEN3_4B_SPLITS)])
def test_repack_full_size_decoder_layer(name, N, K, b_d):
    """Full-size decoder-layer matrices: every field of every subvector survives the repack."""
    need_gpu()
    m = synth.make_matrix(1, 7, N, K, b_d)
    W = svq.SvqWeight.from_synth(m)
    s, i, c = _fields_gpu(W)
    rs, ri, rc = oracle.unpack(N, K, b_d, m.canonical)
    assert np.array_equal(s, rs) and np.array_equal(i, ri) and np.array_equal(c, rc)
