"""GPU parity of the tcgen05 prefill GEMM against the CPU oracle.

Bar: max |y - y_ref| / sum_j |W[n][j]| |x[m][perm[j]]| <= 1e-2 (weights rounded to
bf16 -- or fp16 for fp16 activations -- fp32 accumulation in tensor memory).
Small shapes are checked on every output; the full prefill shapes on a seeded
sample of token rows that the oracle computes one by one."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import need_gpu, rel_err, torch, u16, x_bf16, x_f16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu
TOL = 1e-2


def _gemm(W, x_bits, kind="bf16", y_dtype=torch.float32):
    M = x_bits.shape[0]
    x = x_bf16(x_bits) if kind == "bf16" else x_f16(x_bits)
    y = torch.empty((M, W.N), dtype=y_dtype, device="cuda")
    nb = svq.svq_linear_gemm_workspace_size(W, M)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    svq.svq_linear_gemm(W, x, y, ws)
    torch.cuda.synchronize()
    assert svq.svq_get_device_status() == svq.SVQ_OK
    return y, ws, x


@pytest.mark.parametrize("N,K,M", [(128, 128, 16), (256, 512, 100), (132, 384, 37), (1024, 1024, 256),
                                   (1028, 2048, 300), (512, 1024, 513), (384, 4096, 64), (2560, 1024, 1)])
@pytest.mark.parametrize("b_d", [6, 8, 9])
def test_gemm_small_shapes_every_output(N, K, M, b_d):
    need_gpu()
    m = synth.make_matrix(70, N + M + b_d, N, K, b_d)
    x = synth.make_x(70, N + M + b_d, M, K, dtype="bf16")
    W = svq.SvqWeight.from_synth(m)
    y, _, _ = _gemm(W, x)
    y_ref, den = oracle.linear(m, x, "bf16")
    assert rel_err(y.cpu().numpy(), y_ref, den) <= TOL


@pytest.mark.parametrize("b_d", [1, 2, 3, 4, 5, 7, 10])
def test_gemm_every_split(b_d):
    need_gpu()
    m = synth.make_matrix(71, b_d, 256, 640, b_d)
    x = synth.make_x(71, b_d, 48, 640, dtype="bf16")
    W = svq.SvqWeight.from_synth(m)
    y, _, _ = _gemm(W, x)
    y_ref, den = oracle.linear(m, x, "bf16")
    assert rel_err(y.cpu().numpy(), y_ref, den) <= TOL


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16])
def test_gemm_fp16_small_batch(M):
    """The tensor-core path for small fp16 batches (the GEMV/GEMM crossover), W rounded to fp16."""
    need_gpu()
    m = synth.make_matrix(72, M, 1024, 2048, 7)
    x = synth.make_x(72, M, M, 2048)
    W = svq.SvqWeight.from_synth(m)
    y, _, _ = _gemm(W, x, kind="f16")
    y_ref, den = oracle.linear(m, x)
    assert rel_err(y.cpu().numpy(), y_ref, den) <= TOL


def test_gemm_matches_cublas_on_dequantized_weights():
    """y == matmul(x[:, perm], dequantize(W)^T) (cuBLAS on the exported bf16 weights)."""
    need_gpu()
    m = synth.make_matrix(73, 0, 1024, 2048, 8)
    x = synth.make_x(73, 0, 512, 2048, dtype="bf16")
    W = svq.SvqWeight.from_synth(m)
    y, _, xd = _gemm(W, x)
    wq = torch.empty((m.N, m.K), dtype=torch.bfloat16, device="cuda")
    svq.svq_dequantize(W, wq)
    perm = torch.from_numpy(m.perm.astype(np.int64)).cuda()
    ref = torch.matmul(xd[:, perm].float(), wq.float().t())
    _, den = oracle.linear(m, x, "bf16")
    # same bf16 weights and activations, fp32 accumulation in both: only summation order differs
    assert rel_err(y.cpu().numpy(), ref.cpu().numpy().astype(np.float64), den) <= 1e-4


def test_gemm_bf16_output_and_reproducible():
    need_gpu()
    m = synth.make_matrix(74, 0, 2560, 9728, 8)
    x = synth.make_x(74, 0, 300, 9728, dtype="bf16")
    W = svq.SvqWeight.from_synth(m)
    y1, ws, xd = _gemm(W, x, y_dtype=torch.bfloat16)
    y2 = torch.empty_like(y1)
    svq.svq_linear_gemm(W, xd, y2, ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    rows = np.random.default_rng(0).choice(300, 24, replace=False)
    y_ref, den = oracle.linear(m, np.ascontiguousarray(x[rows]), "bf16")
    assert rel_err(y1.float().cpu().numpy()[rows], y_ref, den) <= TOL + 2.0 ** -8


@pytest.mark.parametrize("which,M", [(0, 512), (0, 2048), (1, 512), (1, 2048)])
def test_prefill_full_size_sampled(which, M):
    """Qwen3-4B gate/up (2560 -> 9728) and down (9728 -> 2560), (8,2), bf16 activations:
    the launch the benchmark times, checked on 32 seeded token rows."""
    need_gpu()
    m = synth.prefill_mats()[which]
    x = synth.prefill_x(M, m.K, which)
    W = svq.SvqWeight.from_synth(m)
    y, _, _ = _gemm(W, x)
    rows = np.random.default_rng(M + which).choice(M, 32, replace=False)
    y_ref, den = oracle.linear(m, np.ascontiguousarray(x[rows]), "bf16")
    assert rel_err(y.cpu().numpy()[rows], y_ref, den) <= TOL


def test_gemm_metamorphic_permutation():
    need_gpu()
    m = synth.make_matrix(75, 0, 256, 1024, 8)
    mid = synth.make_matrix(75, 0, 256, 1024, 8, identity_perm=True)
    x = synth.make_x(75, 0, 64, 1024, dtype="bf16")
    y1, _, _ = _gemm(svq.SvqWeight.from_synth(m), x)
    y2, _, _ = _gemm(svq.SvqWeight.from_synth(mid), np.ascontiguousarray(x[:, m.perm]))
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("x_dtype", ["bf16", "f16"])
def test_gemm_pre_decoded_plan_matches_decoded_tiles(x_dtype):
    """Two or more token tiles switch the GEMM to weights decoded once into the workspace and loaded
    by TMA; one tile decodes on chip.  Both place the same 16-bit weights in the MMA (the export
    reading), so the first 128 tokens of a 1100-token call (pre-decoded, 256-token tiles) and of a
    200-token call (pre-decoded, 128-token tiles) equal a 128-token call (on-chip decode) bit for bit
    (K = 512: no K split in any of them), and every output is within the bound of the oracle.
    N = 1028 ends in a 4-row tile (rows past N read as zeros by the TMA box)."""
    need_gpu()
    N, K = 1028, 512
    m = synth.make_matrix(76, 1 if x_dtype == "f16" else 0, N, K, 7)
    x = synth.make_x(76, 2, 1100, K, dtype=x_dtype)
    W = svq.SvqWeight.from_synth(m)
    yb, _, _ = _gemm(W, x, kind=x_dtype)
    y200, _, _ = _gemm(W, np.ascontiguousarray(x[:200]), kind=x_dtype)
    y128, _, _ = _gemm(W, np.ascontiguousarray(x[:128]), kind=x_dtype)
    assert torch.equal(yb[:128], y128)
    assert torch.equal(y200[:128], y128)
    y_ref200, den200 = oracle.linear(m, np.ascontiguousarray(x[:200]), x_dtype)
    assert rel_err(y200.cpu().numpy(), y_ref200, den200) <= TOL
    y_ref, den = oracle.linear(m, x, x_dtype)
    assert rel_err(yb.cpu().numpy(), y_ref, den) <= TOL


@pytest.mark.parametrize("N,K,M,kind,y_dtype", [
    (4100, 4096, 1300, "bf16", torch.float32),    # pre-decoded tiles: 33 x 6 = 198 tiles, the last 50 split
    (4100, 4096, 1300, "f16", torch.bfloat16),
    (20478, 2048, 128, "bf16", torch.float32),    # on-chip decode, one token tile: 160 row tiles, the last 12 split
    (4100, 1024, 2300, "bf16", torch.float32),    # pre-decoded 256-row tiles: 17 x 9 = 153 tiles, the last 5 split
    (4100, 1024, 2300, "f16", torch.bfloat16),
])
def test_gemm_split_last_round(N, K, M, kind, y_dtype):
    """On a 148-SM part these shapes have more tiles than SMs and a last, partial round; its tiles are
    split along K into slices that spread over all SMs, and a second kernel sums their fp32 partials in
    slice order (ragged N: the last row tile holds 4 or 126 rows).  The 2300-token shape runs the
    pre-decoded kernel with 256-row tiles.  Checked on token rows that fall in split tiles and in whole
    tiles, every output row n."""
    need_gpu()
    m = synth.make_matrix(77, N + M, N, K, 8)
    x = synth.make_x(77, N + M, M, K, dtype=kind)
    W = svq.SvqWeight.from_synth(m)
    y, _, _ = _gemm(W, x, kind=kind, y_dtype=y_dtype)
    rng = np.random.default_rng(N + M)
    if M > 256:
        lo = M - 256 - M % 256                      # the last two token tiles hold the split tiles
        rows = np.concatenate([rng.choice(np.arange(lo, M), 12, replace=False),
                               rng.choice(lo, 8, replace=False)])
    else:
        rows = rng.choice(M, 16, replace=False)
    y_ref, den = oracle.linear(m, np.ascontiguousarray(x[rows]), kind)
    tol = TOL + (2.0 ** -8 if y_dtype == torch.bfloat16 else 0.0)
    assert rel_err(y.float().cpu().numpy()[rows], y_ref, den) <= tol
