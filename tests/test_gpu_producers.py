"""GPU parity of the decoder-layer producers (RMS normalisation and the
SiLU-gated product, written in a consumer's stored column order) against the
oracle, and of the producer -> SVQ layer chain.

Bar: every output within 1 fp16 unit in the last place of the oracle's fp64
value rounded once (the kernels compute in fp32, whose error is far below half
an fp16 ulp, so only values next to an fp16 rounding boundary can land on the
neighbouring code), and at most 1% of the outputs (or 3, for short rows) off by
that one unit.  A producer written in stored order followed by a perm-NULL
layer must equal the natural-order producer followed by the permuted layer bit
for bit."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import need_gpu, torch, u16, x_bf16, x_f16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu
EPS = float(np.float32(1e-6))


def _ulp(a, b):
    def ordered(v):
        v = v.astype(np.int64)
        return np.where(v & 0x8000, -(v & 0x7FFF), v)
    return np.abs(ordered(a) - ordered(b))


def _check_ulp(got, want):
    d = _ulp(got, want)
    assert d.max() <= 1
    assert (d > 0).sum() <= max(3, 0.01 * d.size)


def _dev_h(bits, kind):
    return x_f16(bits) if kind == "f16" else x_bf16(bits)


def _gamma(rng, K):
    return rng.uniform(0.25, 2.0, K).astype(np.float16).view(np.uint16)


def _perm_dev(p):
    return None if p is None else torch.from_numpy(np.ascontiguousarray(p, np.int32)).cuda()


@pytest.mark.parametrize("M,K,kind", [(1, 2560, "f16"), (3, 4096, "bf16"), (16, 2560, "f16"), (2, 136, "f16"),
                                      (5, 9728, "bf16"), (1, 2056, "f16")])
def test_rmsnorm_permute_against_oracle(M, K, kind):
    need_gpu()
    rng = np.random.default_rng(K + M)
    h = synth.make_x(95, K % 97, M, K, dtype=kind, energies=True)
    gamma = _gamma(rng, K)
    perms = [rng.permutation(K), None, rng.permutation(K)]
    outs = [torch.empty((M, K), dtype=torch.float16, device="cuda") for _ in perms]
    svq.svq_rmsnorm_permute(_dev_h(h, kind), x_f16(gamma), EPS, [_perm_dev(p) for p in perms], outs)
    torch.cuda.synchronize()
    want = oracle.rmsnorm_permute(h, kind, gamma, EPS, perms)
    for o, w in zip(outs, want):
        _check_ulp(u16(o), w)


def test_rmsnorm_permute_zero_row_and_eps():
    """An all-zero row gives zeros (eps keeps the scale finite); a constant row gives gamma * c / sqrt(c^2 + eps)."""
    need_gpu()
    K = 512
    h = np.zeros((2, K), np.float16)
    h[1] = 1.0
    gamma = _gamma(np.random.default_rng(7), K)
    out = torch.empty((2, K), dtype=torch.float16, device="cuda")
    svq.svq_rmsnorm_permute(x_f16(h.view(np.uint16)), x_f16(gamma), 3.0, [None], [out])
    torch.cuda.synchronize()
    got = u16(out)
    assert np.all(got[0] == 0)
    _check_ulp(got, oracle.rmsnorm_permute(h.view(np.uint16), "f16", gamma, 3.0, [None])[0])


def test_rmsnorm_permute_reproducible():
    need_gpu()
    rng = np.random.default_rng(8)
    K, M = 2560, 4
    h = x_f16(synth.make_x(96, 0, M, K, energies=True))
    gamma = x_f16(_gamma(rng, K))
    p = _perm_dev(rng.permutation(K))
    a = torch.empty((M, K), dtype=torch.float16, device="cuda")
    b = torch.empty_like(a)
    svq.svq_rmsnorm_permute(h, gamma, EPS, [p], [a])
    svq.svq_rmsnorm_permute(h, gamma, EPS, [p], [b])
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("M", [1, 4])
def test_norm_then_qkv_gemv_stored_order_bit_exact(M):
    """norm (natural) -> grouped q|k|v GEMV with perms  ==  norm (stored order) -> q|k|v GEMV with perm NULL,
    issued back to back on one stream (programmatic dependent launches)."""
    need_gpu()
    layer = synth.qwen3_4b_layer(0)
    mats = [layer[i][0] for i in range(3)]
    Ws = [svq.SvqWeight.from_synth(m) for m in mats]
    K = mats[0].K
    rng = np.random.default_rng(9)
    h = x_f16(synth.make_x(97, 0, M, K, energies=True))
    gamma = x_f16(_gamma(rng, K))
    ys_a = [torch.empty((M, m.N), dtype=torch.float32, device="cuda") for m in mats]
    ys_b = [torch.empty_like(y) for y in ys_a]
    ws = torch.empty(max(svq.svq_linear_gemv_batched_workspace_size(Ws, M), 1), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    xn = torch.empty((M, K), dtype=torch.float16, device="cuda")
    svq.svq_rmsnorm_permute(h, gamma, EPS, [None], [xn])
    svq.svq_linear_gemv_batched(Ws, [xn] * 3, ys_a, ws)
    xs = [torch.empty((M, K), dtype=torch.float16, device="cuda") for _ in mats]
    svq.svq_rmsnorm_permute(h, gamma, EPS, [W.perm for W in Ws], xs)
    svq.svq_linear_gemv_batched([W.without_perm() for W in Ws], xs, ys_b, ws)
    torch.cuda.synchronize()
    for a, b in zip(ys_a, ys_b):
        assert torch.equal(a, b)
    # and the chain against the oracle: layer on the oracle's normalised input
    xo = oracle.rmsnorm_permute(synth.make_x(97, 0, M, K, energies=True), "f16", u16(gamma), EPS, [None])[0]
    _check_ulp(u16(xn), xo)


@pytest.mark.parametrize("M,I,with_perm", [(1, 9728, True), (4, 768, True), (3, 136, False), (16, 9728, False)])
def test_swiglu_permute_against_oracle(M, I, with_perm):
    need_gpu()
    rng = np.random.default_rng(I + M)
    g = (rng.standard_normal((M, I)) * 3).astype(np.float32)
    u = (rng.standard_normal((M, I)) * 2).astype(np.float32)
    g[0, :6] = [0.0, 30.0, -30.0, -200.0, 1e-30, -1e-30]
    p = rng.permutation(I) if with_perm else None
    x = torch.empty((M, I), dtype=torch.float16, device="cuda")
    svq.svq_swiglu_permute(torch.from_numpy(g).cuda(), torch.from_numpy(u).cuda(), _perm_dev(p), x)
    torch.cuda.synchronize()
    _check_ulp(u16(x), oracle.swiglu_permute(g, u, p))


def test_swiglu_then_down_gemv_stored_order_bit_exact():
    need_gpu()
    down = synth.qwen3_4b_layer(0)[6][0]
    W = svq.SvqWeight.from_synth(down)
    M, I = 2, down.K
    rng = np.random.default_rng(10)
    g = torch.from_numpy((rng.standard_normal((M, I)) * 3).astype(np.float32)).cuda()
    u = torch.from_numpy(rng.standard_normal((M, I)).astype(np.float32)).cuda()
    ws = torch.empty(max(svq.svq_linear_gemv_workspace_size(W, M), 1), dtype=torch.uint8, device="cuda")
    svq.svq_workspace_init(ws)
    xa = torch.empty((M, I), dtype=torch.float16, device="cuda")
    xb = torch.empty_like(xa)
    ya = torch.empty((M, down.N), dtype=torch.float32, device="cuda")
    yb = torch.empty_like(ya)
    svq.svq_swiglu_permute(g, u, None, xa)
    svq.svq_linear_gemv(W, xa, ya, ws)
    svq.svq_swiglu_permute(g, u, W.perm, xb)
    svq.svq_linear_gemv(W.without_perm(), xb, yb, ws)
    torch.cuda.synchronize()
    assert torch.equal(ya, yb)


def test_swiglu_permute_matches_moe_fused_input():
    """The MoE kernel's fused SiLU-gated input and this producer evaluate the same expression: an MoE call on
    [gate | up] rows equals an MoE call on the producer's fp16 output, bit for bit."""
    need_gpu()
    E, N, I, T = 2, 256, 768, 3
    ms = [synth.make_matrix(98, e, N, I, 8) for e in range(E)]
    Ws = [svq.SvqWeight.from_synth(m) for m in ms]
    rng = np.random.default_rng(11)
    g = torch.from_numpy((rng.standard_normal((T, I)) * 3).astype(np.float32)).cuda()
    u = torch.from_numpy(rng.standard_normal((T, I)).astype(np.float32)).cuda()
    gu = torch.cat([g, u], 1).contiguous()
    x = torch.empty((T, I), dtype=torch.float16, device="cuda")
    svq.svq_swiglu_permute(g, u, None, x)
    mat = torch.tensor([0, 1, 0, 1, 1, 0], dtype=torch.int32, device="cuda")
    xrow = torch.tensor([0, 0, 1, 1, 2, 2], dtype=torch.int32, device="cuda")
    orow = torch.arange(6, dtype=torch.int32, device="cuda")
    items = svq.item_table(mat, xrow, orow, torch.ones(6, device="cuda"))
    tab = svq.descriptor_table(Ws)

    def run(xin, mode):
        y = torch.empty((6, N), dtype=torch.float32, device="cuda")
        ws = torch.empty(max(svq.svq_moe_grouped_gemv_workspace_size(E, 6, N, False), 1), dtype=torch.uint8,
                         device="cuda")
        svq.svq_moe_grouped_gemv(tab, E, N, I, 8, items, 6, 3, xin, mode, y, 6, False, ws)
        torch.cuda.synchronize()
        assert svq.svq_get_device_status() == svq.SVQ_OK
        return y

    assert torch.equal(run(gu, svq.SVQ_X_SWIGLU_F32), run(x, svq.SVQ_X_F16))


def test_producer_argument_errors():
    """Refused on the host before any launch."""
    need_gpu()
    K = 64
    h = torch.zeros((2, K), dtype=torch.float16, device="cuda")
    gamma = torch.ones(K, dtype=torch.float16, device="cuda")
    out = torch.empty((2, K), dtype=torch.float16, device="cuda")
    buf = torch.empty(2 * K + 8, dtype=torch.float16, device="cuda")
    bad = buf[1:1 + 2 * K].view(2, K)                       # 2-byte aligned only
    cases = [
        (lambda: svq.svq_rmsnorm_permute(h, gamma, EPS, [None] * 9, [out] * 9), svq.SVQ_ERR_INVALID_ARG),
        (lambda: svq.svq_rmsnorm_permute(h, gamma, EPS, [None], [bad]), svq.SVQ_ERR_INVALID_ARG),
        (lambda: svq.svq_rmsnorm_permute(h, gamma, float("nan"), [None], [out]), svq.SVQ_ERR_INVALID_ARG),
        (lambda: svq.svq_rmsnorm_permute(h[:, :12].contiguous(), gamma, EPS, [None], [out]),
         svq.SVQ_ERR_UNSUPPORTED_SHAPE),
    ]
    for call, status in cases:
        with pytest.raises(svq.SvqError) as e:
            call()
        assert e.value.status == status
    g = torch.zeros((2, 12), dtype=torch.float32, device="cuda")
    with pytest.raises(svq.SvqError) as e:
        svq.svq_swiglu_permute(g, g, None, out)
    assert e.value.status == svq.SVQ_ERR_UNSUPPORTED_SHAPE
    # M = 0 is accepted and launches nothing
    svq.svq_rmsnorm_permute(h[:0], gamma, EPS, [None], [out[:0]])
    svq.svq_swiglu_permute(g[:0, :8], g[:0, :8], None, out[:0])
