"""Stress cases of the GEMV's accumulation precision (fp32 sums of fp16 products).

The method's decode reconstructs each weight as radius x (sign x codeword entry)
("SAGE", arXiv 2610.14745, Figure 2 caption); a row of the product sums K such
terms.  Two adversarial inputs, each checked element by element against the
fp64 oracle with the GEMV's bound |y - y_ref| <= 1e-3 * sum_j |W[n][j]| |x_j|:

* coherent accumulation: every sign bit positive (codewords are non-negative)
  and x > 0, so no term cancels and the bound is a relative bound on y itself,
  over the longest input of the decoder layer (K = 9728);
* large activations: |x| = 3e4 with coherent signs, where one subvector's dot
  product (up to sqrt(8) * 3e4) exceeds the fp16 range -- any fp16
  intermediate sum would overflow.
Both run with full 128-row tiles (tensor-core decode) and with a partial last
tile (N % 128 = 4; the per-lane decode)."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import need_gpu, rel_err, torch, x_f16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _coherent_matrix(N, K, b_d, seed):
    """A synthetic matrix with every sign bit cleared (all weights >= 0)."""
    m = synth.make_matrix(seed, 0, N, K, b_d)
    signs, idx, code = oracle.unpack(N, K, b_d, m.canonical)
    m.canonical = oracle.pack(N, K, b_d, np.zeros_like(signs), idx, code)
    return m


def _gemv(m, x_bits):
    W = svq.SvqWeight.from_synth(m)
    M = x_bits.shape[0]
    y = torch.empty((M, m.N), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(svq.svq_linear_gemv_workspace_size(W, M), 1), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    svq.svq_linear_gemv(W, x_f16(x_bits), y, ws)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("N", [256, 132])
@pytest.mark.parametrize("M", [1, 2])
def test_coherent_signs_positive_x_long_rows(N, M):
    need_gpu()
    K = 9728
    m = _coherent_matrix(N, K, 7, 70)
    x = np.abs(synth.make_x(70, 1, M, K).view(np.float16)).astype(np.float16).view(np.uint16)
    y = _gemv(m, x)
    y_ref, den = oracle.linear(m, x)
    assert np.all(y_ref > 0) and np.allclose(den, y_ref)      # no cancellation: the bound is relative
    assert np.all(np.isfinite(y))
    assert rel_err(y, y_ref, den) <= TOL


@pytest.mark.parametrize("N", [256, 132])
def test_activations_at_3e4(N):
    need_gpu()
    K = 2560
    m = _coherent_matrix(N, K, 8, 71)
    rng = np.random.default_rng(71)
    # |x| = 3e4 everywhere; the first row all positive (coherent), the second with random signs
    x = np.full((2, K), 3e4)
    x[1] *= rng.choice([-1.0, 1.0], K)
    x = x.astype(np.float16).view(np.uint16)
    y = _gemv(m, x)
    y_ref, den = oracle.linear(m, x)
    assert np.all(np.isfinite(y))
    assert np.abs(y_ref[0]).max() > 65504.0                    # beyond the fp16 range
    assert rel_err(y, y_ref, den) <= TOL
