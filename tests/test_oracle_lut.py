"""Pins of the oracle's per-row radius table (the quantized radius as a table of
fitted levels: "SAGE", arXiv 2610.14745, Figure 2 caption gives a quantized
radius per subvector and the pages optimise its levels; a per-row table of
2^b_r fp16 levels is the plainest form of fitted levels).  With a table,
r(n, code) = fp32(lut[n][code]) replaces fma(scale_n, code, offset_n).

Pinned against: the affine form (a table holding exactly the affine levels
decodes identically), a closed form (constant codebook, integer levels, exact
sums), the norm invariant, and the brute-force encoder's round trip."""
import math

import numpy as np
import pytest

import oracle
import synth


def _affine_exact_matrix(b_d, N=16, K=256):
    """A matrix whose affine levels are exact in fp16 (scale 2^-6, offset 0.5: r = 0.5 + code/64),
    and the table holding those same levels."""
    m = synth.make_matrix(93, b_d, N, K, b_d)
    m.scale = np.full(N, 0x2400, np.uint16)                 # 2^-6
    m.offset = np.full(N, 0x3800, np.uint16)                # 0.5
    nr = 1 << (10 - b_d)
    levels = 0.5 + np.arange(nr) / 64.0
    lut = np.tile(levels.astype(np.float16).view(np.uint16), (N, 1))
    assert np.array_equal(lut.view(np.float16).astype(np.float64)[0], levels)   # exact in fp16
    return m, lut


@pytest.mark.parametrize("b_d", [6, 7, 8, 9, 10])
def test_table_of_affine_levels_decodes_identically(b_d):
    m, lut = _affine_exact_matrix(b_d)
    W_aff = oracle.decode_exact(m)
    d_aff = oracle.dequant(m, "f16"), oracle.dequant(m, "bf16")
    x = synth.make_x(93, b_d, 2, m.K)
    y_aff, _ = oracle.linear(m, x)
    m.lut = lut
    assert np.array_equal(oracle.decode_exact(m), W_aff)
    assert np.array_equal(oracle.dequant(m, "f16"), d_aff[0])
    assert np.array_equal(oracle.dequant(m, "bf16"), d_aff[1])
    assert np.array_equal(oracle.linear(m, x)[0], y_aff)


def test_closed_form_constant_codebook_integer_levels():
    """Every codeword (1,...,1)/sqrt(8) in fp16 (0x35A8 = 0.353515625), levels lut[n][c] = n + c + 1:
    W[n][8g+i] = +-(n + code + 1) * 0.353515625, so y = 0.353515625 * sum_j (+-level) x[perm[j]]
    (exact sum via math.fsum)."""
    N, K, b_d = 6, 128, 7
    m = synth.make_matrix(94, 0, N, K, b_d)
    m.codebook = np.full((1 << b_d, 8), 0x35A8, np.uint16)
    nr = 1 << (10 - b_d)
    m.lut = (np.arange(N)[:, None] + np.arange(nr)[None, :] + 1.0).astype(np.float16).view(np.uint16)
    x = synth.make_x(94, 0, 1, K)
    y, den = oracle.linear(m, x)
    s, _, c = oracle.unpack(N, K, b_d, m.canonical)
    xf = x.view(np.float16).astype(np.float64)[0]
    cw = 0.353515625
    for n in range(N):
        terms = []
        for g in range(K // 8):
            lv = n + int(c[n, g]) + 1
            for i in range(8):
                sg = -1.0 if (s[n, g] >> i) & 1 else 1.0
                terms.append(sg * lv * cw * xf[m.perm[8 * g + i]])
        exact = math.fsum(terms)
        assert y[0, n] == pytest.approx(exact, rel=1e-12, abs=1e-12 * den[0, n])
        assert den[0, n] == pytest.approx(math.fsum(abs(t) for t in terms), rel=1e-12)


@pytest.mark.parametrize("b_d", [6, 8])
def test_subvector_norm_is_the_table_level(b_d):
    m = synth.make_matrix(95, b_d, 24, 512, b_d)
    m.lut = synth.make_lut(95, b_d, m.N, b_d)
    W = oracle.decode_exact(m)
    _, i, c = oracle.unpack(m.N, m.K, b_d, m.canonical)
    cb = m.codebook.view(np.float16).astype(np.float64)
    norms = np.sqrt((W.reshape(m.N, -1, 8) ** 2).sum(-1))
    lv = m.lut.view(np.float16).astype(np.float64)[np.arange(m.N)[:, None], c.astype(np.int64)]
    cn = np.sqrt((cb[i.astype(np.int64)] ** 2).sum(-1))
    assert np.allclose(norms, lv * cn, rtol=1e-12, atol=0)


@pytest.mark.parametrize("b_d", [5, 7, 9])
def test_encode_decode_roundtrip_with_table(b_d):
    """Decoded weights of random codes re-encode, under the same table, to the same codes (distinct
    codewords and distinct, increasing levels per row make them unique)."""
    N, K = 6, 48
    r = np.random.default_rng(96 + b_d)
    cb = np.abs(r.standard_normal((1 << b_d, 8)))
    cb = (cb / np.linalg.norm(cb, axis=1, keepdims=True)).astype(np.float16)
    assert len({row.tobytes() for row in cb}) == len(cb)
    lut = synth.make_lut(96, b_d, N, b_d)
    assert np.all(np.diff(lut.view(np.float16).astype(np.float64), axis=1) > 0)
    G = K // 8
    s = r.integers(0, 256, (N, G)).astype(np.uint8)
    i = r.integers(0, 1 << b_d, (N, G)).astype(np.uint16)
    c = r.integers(0, 1 << (10 - b_d), (N, G)).astype(np.uint16)
    m = synth.SvqMatrix(N, K, b_d, oracle.pack(N, K, b_d, s, i, c), cb.view(np.uint16),
                        np.zeros(N, np.uint16), np.zeros(N, np.uint16), np.arange(K, dtype=np.int32), lut=lut)
    W = oracle.decode_exact(m)
    s2, i2, c2 = oracle.encode(N, K, b_d, W, m.codebook, None, None, lut=lut)
    assert np.array_equal(i2, i) and np.array_equal(c2, c)
