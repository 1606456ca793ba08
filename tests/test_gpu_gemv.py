"""GPU parity of the fused decode-and-multiply GEMV against the CPU oracle.

Bar: max |y - y_ref| / sum_j |W[n][j]| |x[m][perm[j]]| <= 1e-3 (fp32 accumulate
across subvectors), on every output for sizes the oracle finishes quickly, and
at the full decoder-layer and 8192 x 8192 sizes on every output as well (the
fp64 oracle handles them in seconds).  Also: permutation metamorphic test,
run-to-run bit reproducibility, fp16 outputs, the grouped launch."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import need_gpu, rel_err, torch, u16, x_f16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _run(W, x_bits, y_dtype=torch.float32):
    M = x_bits.shape[0]
    x = x_f16(x_bits)
    y = torch.empty((M, W.N), dtype=y_dtype, device="cuda")
    nb = svq.svq_linear_gemv_workspace_size(W, M)
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    svq.svq_linear_gemv(W, x, y, ws)
    torch.cuda.synchronize()
    return y, ws


def test_single_layer_1024():
    need_gpu()
    m, x = synth.single_layer_1024()
    W = svq.SvqWeight.from_synth(m)
    y, _ = _run(W, x)
    y_ref, den = oracle.linear(m, x)
    assert rel_err(y.cpu().numpy(), y_ref, den) <= TOL


@pytest.mark.parametrize("b_d", range(1, 11))
@pytest.mark.parametrize("N,K", [(4, 128), (132, 256), (388, 640), (1024, 1152)])
def test_gemv_every_split_and_ragged_tiles(N, K, b_d):
    need_gpu()
    m = synth.make_matrix(60, 10 * b_d + N % 7, N, K, b_d)
    x = synth.make_x(60, 10 * b_d + N % 7, 1, K)
    W = svq.SvqWeight.from_synth(m)
    y, _ = _run(W, x)
    y_ref, den = oracle.linear(m, x)
    assert rel_err(y.cpu().numpy(), y_ref, den) <= TOL


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 16])
def test_gemv_small_batches(M):
    need_gpu()
    m = synth.make_matrix(61, M, 640, 2560, 7)
    x = synth.make_x(61, M, M, 2560)
    W = svq.SvqWeight.from_synth(m)
    y, _ = _run(W, x)
    y_ref, den = oracle.linear(m, x)
    assert rel_err(y.cpu().numpy(), y_ref, den) <= TOL


def test_gemv_fp16_output():
    need_gpu()
    m = synth.make_matrix(62, 0, 512, 1024, 8)
    x = synth.make_x(62, 0, 2, 1024)
    W = svq.SvqWeight.from_synth(m)
    y, _ = _run(W, x, torch.float16)
    y_ref, den = oracle.linear(m, x)
    # fp16 output adds one rounding of y (relative 2^-11 of |y| <= den)
    assert rel_err(y.float().cpu().numpy(), y_ref, den) <= TOL + 2.0 ** -11


def test_permutation_metamorphic_bit_exact():
    """y(W, perm, x) == y(W, identity, x[perm]) bit for bit (same data order in the kernel)."""
    need_gpu()
    m = synth.make_matrix(63, 0, 256, 1024, 8)
    x = synth.make_x(63, 0, 1, 1024)
    W = svq.SvqWeight.from_synth(m)
    mid = synth.make_matrix(63, 0, 256, 1024, 8, identity_perm=True)
    Wid = svq.SvqWeight.from_synth(mid)
    y1, _ = _run(W, x)
    y2, _ = _run(Wid, np.ascontiguousarray(x[:, m.perm]))
    assert torch.equal(y1, y2)


def test_reproducible_and_workspace_reusable():
    """Split-K partials are reduced in a fixed order: repeated calls on one workspace agree bit for bit,
    and the completion counters are left at zero."""
    need_gpu()
    m = synth.make_matrix(64, 0, 2560, 9728, 8)
    x = synth.make_x(64, 0, 1, 9728)
    W = svq.SvqWeight.from_synth(m)
    y1, ws = _run(W, x)
    xd = x_f16(x)
    ys = []
    for _ in range(3):
        y = torch.empty_like(y1)
        svq.svq_linear_gemv(W, xd, y, ws)
        ys.append(y)
    torch.cuda.synchronize()
    for y in ys:
        assert torch.equal(y, y1)
    y_ref, den = oracle.linear(m, x)
    assert rel_err(y1.cpu().numpy(), y_ref, den) <= TOL


def test_workspace_too_small_rejected():
    need_gpu()
    m = synth.make_matrix(65, 0, 2560, 9728, 8)
    W = svq.SvqWeight.from_synth(m)
    nb = svq.svq_linear_gemv_workspace_size(W, 1)
    assert nb > 0
    x = torch.zeros((1, 9728), dtype=torch.float16, device="cuda")
    y = torch.empty((1, 2560), dtype=torch.float32, device="cuda")
    ws = torch.zeros(nb - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(svq.SvqError) as e:
        svq.svq_linear_gemv(W, x, y, ws)
    assert e.value.status == svq.SVQ_ERR_WORKSPACE


@pytest.mark.parametrize("M", [1, 3])
def test_grouped_ragged_tiles_inside_long_ranges(M):
    """Two matrices of different b_d in one grouped call, one with a 4-row last tile: CTA and warp
    ranges cross tile boundaries and end inside the ragged tile."""
    need_gpu()
    shapes = [(4100, 2560, 7), (388, 1152, 9)]
    mats = [synth.make_matrix(66, i, N, K, b_d) for i, (N, K, b_d) in enumerate(shapes)]
    xs = [synth.make_x(66, 10 + i, M, K) for i, (N, K, b_d) in enumerate(shapes)]
    Ws = [svq.SvqWeight.from_synth(m) for m in mats]
    nb = svq.svq_linear_gemv_batched_workspace_size(Ws, M)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    ys = [torch.empty((M, m.N), dtype=torch.float32, device="cuda") for m in mats]
    svq.svq_linear_gemv_batched(Ws, [x_f16(x) for x in xs], ys, ws)
    torch.cuda.synchronize()
    for m, x, y in zip(mats, xs, ys):
        y_ref, den = oracle.linear(m, x)
        assert rel_err(y.cpu().numpy(), y_ref, den) <= TOL


def test_decoder_layer_grouped_full_size():
    """The seven linears of a Qwen3-4B-shaped decoder layer (batch 1) in one grouped launch,
    every output checked against the oracle."""
    need_gpu()
    layer = synth.qwen3_4b_layer(0)
    Ws = [svq.SvqWeight.from_synth(m) for m, _ in layer]
    xs = [x_f16(x) for _, x in layer]
    ys = [torch.empty((1, m.N), dtype=torch.float32, device="cuda") for m, _ in layer]
    nb = svq.svq_linear_gemv_batched_workspace_size(Ws, 1)
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    svq.svq_linear_gemv_batched(Ws, xs, ys, ws)
    torch.cuda.synchronize()
    for (m, x), y in zip(layer, ys):
        y_ref, den = oracle.linear(m, x)
        assert rel_err(y.cpu().numpy(), y_ref, den) <= TOL, m.name
    # the prepared-call form of the same launch gives the same bits
    ys2 = [torch.empty_like(y) for y in ys]
    svq.GemvBatchCall(Ws, xs, ys2, ws)()
    torch.cuda.synchronize()
    for y, y2 in zip(ys, ys2):
        assert torch.equal(y, y2)
    # the grouped launch equals the per-matrix launches
    for (m, x), W, y in zip(layer, Ws, ys):
        y1, _ = _run(W, x)
        assert rel_err(y1.cpu().numpy(), y.cpu().numpy().astype(np.float64), oracle.linear(m, x)[1]) <= 1e-6


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16])
def test_square_8192_sweep(M):
    need_gpu()
    m = synth.square_8192()
    x = synth.square_8192_x(M)
    W = svq.SvqWeight.from_synth(m)
    y, _ = _run(W, x)
    y_ref, den = oracle.linear(m, x)
    assert rel_err(y.cpu().numpy(), y_ref, den) <= TOL


def test_lm_head_sized_matrix_sampled_rows():
    """A vocabulary-sized matrix (151936 x 2560, b_d 8, 109 MB of codes): every CTA range spans
    ten row tiles, most of them whole.  Sampled 4-row groups against the oracle."""
    need_gpu()
    N, K = 151936, 2560
    m = synth.make_matrix(67, 0, N, K, 8)
    x = synth.make_x(67, 0, 1, K)
    W = svq.SvqWeight.from_synth(m)
    y, _ = _run(W, x)
    y = y.cpu().numpy()
    rng = np.random.default_rng(3)
    for r0 in list(rng.choice(N // 4, 24, replace=False) * 4) + [0, N - 4]:
        sub = synth.SvqMatrix(4, K, 8, np.ascontiguousarray(m.canonical[r0:r0 + 4]), m.codebook,
                              np.ascontiguousarray(m.scale[r0:r0 + 4]), np.ascontiguousarray(m.offset[r0:r0 + 4]),
                              m.perm)
        y_ref, den = oracle.linear(sub, x)
        assert rel_err(y[:, r0:r0 + 4], y_ref, den) <= TOL


@pytest.mark.parametrize("M", [1, 2, 5])
@pytest.mark.parametrize("N", [9728, 9660])
def test_grouped_two_permuted_gate_shaped_matrices(N, M):
    """Two N x 2560 matrices with permutations and different b_d in one grouped call, CTA ranges
    spanning more than one row tile (N = 9660 adds a 60-row last tile).  Every output against the
    oracle."""
    need_gpu()
    K = 2560
    mats = [synth.make_matrix(68, i + N % 7, N, K, 7 + i) for i in range(2)]
    xs = [synth.make_x(68, 20 + i, M, K) for i in range(2)]
    Ws = [svq.SvqWeight.from_synth(m) for m in mats]
    nb = svq.svq_linear_gemv_batched_workspace_size(Ws, M)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    ys = [torch.empty((M, N), dtype=torch.float32, device="cuda") for _ in mats]
    svq.svq_linear_gemv_batched(Ws, [x_f16(x) for x in xs], ys, ws)
    torch.cuda.synchronize()
    for m, x, y in zip(mats, xs, ys):
        y_ref, den = oracle.linear(m, x)
        assert rel_err(y.cpu().numpy(), y_ref, den) <= TOL


@pytest.mark.parametrize("M", [1, 3])
@pytest.mark.parametrize("y_dtype", [torch.float32, torch.float16])
def test_batched_host_call_matches_device_call(M, y_dtype):
    """svq_linear_gemv_batched_host (pinned host x -> device copy, grouped launch, device -> pinned
    host y copy in one call) on the seven decoder-layer linears: the host results equal the
    device-buffer call bit for bit, and are within the bound of the oracle."""
    need_gpu()
    layer = synth.qwen3_4b_layer(0)
    Ws = [svq.SvqWeight.from_synth(m) for m, _ in layer]
    xs_np = [synth.make_x(90, i, M, m.K) for i, (m, _) in enumerate(layer)]
    xs = [x_f16(x) for x in xs_np]
    ys = [torch.empty((M, m.N), dtype=y_dtype, device="cuda") for m, _ in layer]
    nb = svq.svq_linear_gemv_batched_workspace_size(Ws, M)
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    svq.svq_linear_gemv_batched(Ws, xs, ys, ws)
    x_host = torch.cat([x.reshape(-1) for x in xs]).cpu().pin_memory()
    x_dev = torch.empty_like(x_host, device="cuda")
    n_out = sum(M * m.N for m, _ in layer)
    y_host = torch.full((n_out,), float("nan"), dtype=y_dtype).pin_memory()
    y_dev = torch.empty(n_out, dtype=y_dtype, device="cuda")
    call = svq.GemvBatchHostCall(Ws, M, x_host, x_dev, y_host, y_dev, ws)
    call()
    call()                                        # twice: the workspace counters come back to zero
    torch.cuda.synchronize()
    assert torch.equal(y_host, torch.cat([y.reshape(-1) for y in ys]).cpu())
    off = 0
    for (m, _), x in zip(layer, xs_np):
        y_ref, den = oracle.linear(m, x)
        got = y_host[off:off + M * m.N].reshape(M, m.N).float().numpy()
        tol = TOL + (2.0 ** -11 if y_dtype == torch.float16 else 0.0)
        assert rel_err(got, y_ref, den) <= tol, m.name
        off += M * m.N
