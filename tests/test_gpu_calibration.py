"""GPU calibration side (ESG, radius grid, encoder, ABS) against the CPU oracle.

Bar: bit-exact for every integer result -- the ESG permutation, the canonical
code stream (signs, direction indices, radius codes), the radius grid's fp16
bit patterns and the chosen split; fp64 energies bit-exact (same operations in
the same order); per-row and total weighted errors within 1e-12 relative (the
GPU sums in a different fixed order than numpy's pairwise sum).  Readings:
"SAGE" (arXiv 2610.14745), abstract, Figure 2 caption and Figure 4(a)."""
import numpy as np
import pytest

import oracle
from oracle import calibration as cal
import synth
from tests.gpu_util import need_gpu, torch, u16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.cuda() if dtype is None else t.to(dtype).cuda()


def _dev16(a):
    return _dev(np.ascontiguousarray(a, np.uint16).view(np.int16))


def _weights_like(N, K, b_d, seed, noise=0.02):
    """fp32 weights near an SVQ matrix (its exact decode in natural order plus relative noise), the
    matrix's permutation, and positive fp32 fitting weights."""
    m = synth.make_matrix(seed, b_d, N, K, b_d)
    Ws = oracle.decode_exact(m)
    rng = np.random.default_rng(seed)
    Ws = Ws * (1.0 + noise * rng.standard_normal(Ws.shape))
    W = np.empty_like(Ws)
    W[:, m.perm] = Ws
    wts = rng.lognormal(0.0, 1.0, K).astype(np.float32)
    return W.astype(np.float32), m, wts


def _gpu_encode(W, b_d, perm, wts, codebook, scale, offset):
    N, K = W.shape
    canon = torch.zeros((N, oracle.row_bytes(K)), dtype=torch.uint8, device="cuda")
    row_err = torch.empty(N, dtype=torch.float64, device="cuda")
    svq.svq_encode(_dev(W), b_d, None if perm is None else _dev(perm.astype(np.int32)),
                   None if wts is None else _dev(wts), _dev16(codebook), _dev16(scale), _dev16(offset), canon, row_err)
    torch.cuda.synchronize()
    return canon.cpu().numpy(), row_err.cpu().numpy()


def _oracle_encode(W, b_d, perm, wts, codebook, scale, offset):
    """Canonical stream and per-row weighted error the oracle gives for the same fp32 inputs."""
    N, K = W.shape
    p = np.arange(K) if perm is None else perm.astype(np.int64)
    Ws = np.ascontiguousarray(W.astype(np.float64)[:, p])
    ws = np.ones(K) if wts is None else np.ascontiguousarray(wts.astype(np.float64)[p])
    signs, idx, code = oracle.encode(N, K, b_d, Ws, codebook, scale, offset, None if wts is None else ws)
    canon = oracle.pack(N, K, b_d, signs, idx, code)
    m = synth.SvqMatrix(N, K, b_d, canon, np.asarray(codebook, np.uint16), np.asarray(scale, np.uint16),
                        np.asarray(offset, np.uint16), p.astype(np.int32))
    W_hat = oracle.decode_exact(m)
    row_err = (ws[None, :] * (Ws - W_hat) ** 2).sum(axis=1)
    return canon, row_err


def _check_encode(W, b_d, perm, wts, codebook, scale, offset):
    got, gerr = _gpu_encode(W, b_d, perm, wts, codebook, scale, offset)
    want, werr = _oracle_encode(W, b_d, perm, wts, codebook, scale, offset)
    assert np.array_equal(got, want)
    assert np.allclose(gerr, werr, rtol=1e-12, atol=0.0)


@pytest.mark.parametrize("b_d", range(1, 11))
def test_encode_bit_exact_every_split(b_d):
    """N = 12, K = 328 (41 subvectors: a full chunk of 32 and a ragged one), random permutation and
    fitting weights, the oracle's radius grid of the stored-order rows."""
    N, K = 12, 328
    W, m, wts = _weights_like(N, K, b_d, 80)
    sc, of = cal.radius_grid(W.astype(np.float64)[:, m.perm], b_d)
    _check_encode(W, b_d, m.perm, wts, m.codebook, sc, of)
    _check_encode(W, b_d, None, None, m.codebook, sc, of)          # no permutation, unit weights


def test_encode_degenerate_cases():
    """Ties decided by the rule (lowest direction, then lowest code): scale 0 (every code gives the
    same radius), duplicated codewords, all-zero subvectors, zero fitting weights, a negative scale,
    a single subvector per row."""
    N, K, b_d = 8, 64, 6
    W, m, wts = _weights_like(N, K, b_d, 81)
    W[1, :] = 0.0                                                   # all-zero row
    W[2, m.perm[8:16]] = 0.0                                         # one all-zero subvector
    wts[:5] = 0.0                                                   # channels with zero weight
    cb = m.codebook.copy()
    cb[5] = cb[3]                                                   # duplicated codewords
    cb[40] = cb[3]
    sc, of = cal.radius_grid(W.astype(np.float64)[:, m.perm], b_d)
    sc = sc.copy()
    sc[3] = 0                                                       # scale +0: one radius for all codes
    sc[4] = 0x8000                                                  # scale -0
    sc[5] = np.float16(-0.01).view(np.uint16)                       # decreasing radius levels
    _check_encode(W, b_d, m.perm, wts, cb, sc, of)
    W1, m1, w1 = _weights_like(3, 8, 7, 82)
    s1, o1 = cal.radius_grid(W1.astype(np.float64)[:, m1.perm], 7)
    _check_encode(W1, 7, m1.perm, w1, m1.codebook, s1, o1)


def test_encode_full_size_sampled_rows():
    """9728 x 2560 (the gate projection's shape), b_d 7 with weights: every row encoded on the GPU;
    24 sampled rows (and the first and last) against the oracle."""
    N, K, b_d = 9728, 2560, 7
    W, m, wts = _weights_like(N, K, b_d, 83)
    sc, of = cal.radius_grid(W.astype(np.float64)[:, m.perm], b_d)
    got, gerr = _gpu_encode(W, b_d, m.perm, wts, m.codebook, sc, of)
    rows = sorted(set(np.random.default_rng(83).choice(N, 24, replace=False).tolist() + [0, N - 1]))
    want, werr = _oracle_encode(W[rows], b_d, m.perm, wts, m.codebook, sc[rows], of[rows])
    assert np.array_equal(got[rows], want)
    assert np.allclose(gerr[rows], werr, rtol=1e-12, atol=0.0)


def test_radius_grid_bit_exact():
    N, K = 64, 256
    W, m, _ = _weights_like(N, K, 8, 84)
    # crafted rows (one nonzero element per subvector, so each norm is that element exactly):
    # row 0: smallest norm 1 + 2^-11, halfway between two fp16 values (rounds to the even one, 1.0);
    # row 1: smallest norm 3e-6 (an fp16 subnormal) and a largest of 7e4; row 2: every norm beyond
    # the fp16 range (offset overflows to infinity)
    for row, lo, hi in ((0, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11), (1, 3e-6, 7e4), (2, 7e4, 7e4)):
        W[row, :] = 0.0
        W[row, m.perm[0::8]] = lo
        W[row, m.perm[8]] = hi
    for b_d in (6, 8, 10):
        for perm in (m.perm, None):
            p = np.arange(K) if perm is None else perm
            sc, of = cal.radius_grid(W.astype(np.float64)[:, p], b_d)
            gs = torch.empty(N, dtype=torch.int16, device="cuda")
            go = torch.empty(N, dtype=torch.int16, device="cuda")
            svq.svq_radius_grid(_dev(W), None if perm is None else _dev(perm.astype(np.int32)), b_d, gs, go)
            torch.cuda.synchronize()
            assert np.array_equal(u16(gs), sc) and np.array_equal(u16(go), of)


@pytest.mark.parametrize("K,T", [(16, 1), (2560, 64), (9728, 16)])
def test_esg_bit_exact(K, T):
    rng = np.random.default_rng(K + T)
    if K == 16:
        # the hand-worked example of the oracle pins: energies x^2 with one calibration row
        e = np.array([5, 1, 9, 3, 7, 2, 8, 6, 0.5, 4, 10, 11, 12, 13, 14, 15], np.float64)
        x = np.sqrt(e).astype(np.float32)[None, :]
    else:
        x = (rng.standard_normal((T, K)) * rng.lognormal(0.0, 1.0, K)[None, :]).astype(np.float32)
        x[:, 7] = x[:, 3]                                           # equal energies: lower index first
        x[:, 100] = x[:, 3]
    energy = torch.empty(K, dtype=torch.float64, device="cuda")
    perm = torch.empty(K, dtype=torch.int32, device="cuda")
    wts = torch.empty(K, dtype=torch.float32, device="cuda")
    for gamma in (1.0, 0.5):
        svq.svq_esg(_dev(x), gamma, energy, perm, wts)
        torch.cuda.synchronize()
        e_ref = cal.channel_energy(x.astype(np.float64))
        assert np.array_equal(energy.cpu().numpy(), e_ref)
        assert np.array_equal(perm.cpu().numpy(), cal.esg_perm(e_ref))
        w_ref = cal.esg_weights(e_ref, gamma)
        w = wts.cpu().numpy().astype(np.float64)
        # fp32 rounding of an fp64 power accurate to 2 ulp: within one fp32 ulp of the reference
        assert np.all(np.abs(w - w_ref) <= 2.0 ** -23 * np.abs(w_ref))
    if K == 16:
        assert perm.cpu().numpy().tolist() == [15, 13, 11, 2, 4, 0, 3, 1, 14, 12, 10, 6, 7, 9, 5, 8]


def test_abs_select_matches_oracle():
    """Four candidate splits (b_d 6..9), each with its codebook and the radius grid of the stored-order
    rows: the GPU's totals and choice against the oracle's ABS; then a matrix built from split 7's
    codes, which that split reproduces exactly (total 0)."""
    N, K = 48, 256
    W, m, wts = _weights_like(N, K, 7, 85, noise=0.05)
    cands, errs = [], []
    for b in (6, 7, 8, 9):
        mb = synth.make_matrix(85, 100 + b, N, K, b)
        sc, of = cal.radius_grid(W.astype(np.float64)[:, m.perm], b)
        cands.append((b, mb.codebook, sc, of))
    row_err = torch.empty((4, N), dtype=torch.float64, device="cuda")
    for k, (b, cb, sc, of) in enumerate(cands):
        canon = torch.zeros((N, oracle.row_bytes(K)), dtype=torch.uint8, device="cuda")
        svq.svq_encode(_dev(W), b, _dev(m.perm.astype(np.int32)), _dev(wts), _dev16(cb), _dev16(sc), _dev16(of),
                       canon, row_err[k])
    totals = torch.empty(4, dtype=torch.float64, device="cuda")
    best = torch.empty(1, dtype=torch.int32, device="cuda")
    svq.svq_abs_select(row_err, totals, best)
    torch.cuda.synchronize()
    ref_best, ref_errs = cal.abs_select(W.astype(np.float64), m.perm, wts.astype(np.float64), cands)
    assert int(best.item()) == ref_best
    assert np.allclose(totals.cpu().numpy(), ref_errs, rtol=1e-12, atol=0.0)
    # exact reproduction under split 7: radius 1 everywhere (scale 0, offset 1.0), so the decoded
    # weights are signed fp16 codebook entries, exact in fp32
    m.scale[:] = 0
    m.offset[:] = 0x3C00
    Wx = np.empty((N, K))
    Wx[:, m.perm] = oracle.decode_exact(m)
    Wx32 = Wx.astype(np.float32)
    assert np.array_equal(Wx32.astype(np.float64), Wx)
    cands_x = [(b, synth.make_matrix(85, 100 + b, N, K, b).codebook, m.scale, m.offset) for b in (6, 8)]
    cands_x.insert(1, (7, m.codebook, m.scale, m.offset))
    for k, (b, cb, sc, of) in enumerate(cands_x):
        canon = torch.zeros((N, oracle.row_bytes(K)), dtype=torch.uint8, device="cuda")
        svq.svq_encode(_dev(Wx32), b, _dev(m.perm.astype(np.int32)), _dev(wts), _dev16(cb), _dev16(sc),
                       _dev16(of), canon, row_err[k])
    svq.svq_abs_select(row_err[:3], totals, best)
    torch.cuda.synchronize()
    assert int(best.item()) == 1 and totals[1].item() == 0.0


def test_calibration_argument_checks():
    need_gpu()
    W = torch.zeros((4, 12), dtype=torch.float32, device="cuda")  # K not a multiple of 8
    canon = torch.zeros((4, 4), dtype=torch.uint8, device="cuda")
    z16 = torch.zeros(16, dtype=torch.int16, device="cuda")
    with pytest.raises(svq.SvqError) as e:
        svq.svq_encode(W, 7, None, None, z16, z16, z16, canon)
    assert e.value.status == svq.SVQ_ERR_UNSUPPORTED_SHAPE
    re = torch.zeros((65, 4), dtype=torch.float64, device="cuda")  # more than 64 candidates
    with pytest.raises(svq.SvqError) as e:
        svq.svq_abs_select(re, None, torch.zeros(1, dtype=torch.int32, device="cuda"))
    assert e.value.status == svq.SVQ_ERR_INVALID_ARG
