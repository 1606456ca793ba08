"""Pins that tie the CPU oracle to what the pages and the mathematics fix.

Sources ("SAGE: Pushing 2-Bit Vector-Quantized LLMs toward Real-World Usability"):
  Figure 2 caption -- signs, a direction index and a quantized radius per
  8-weight subvector, 18 bits per eight weights, a per-matrix direction/radius
  bit split; Figure 6 caption -- eight reordered activations per subvector;
  Figures 1 and 5 -- weights reconstructed on demand (y = W x).

Each test is chosen so that a plausible slip in the oracle (bit order, field
order, sign meaning, radius formula, permutation direction, a dropped term)
fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth


def _golden(golden_dir):
    with open(os.path.join(golden_dir, "canonical_2x16.json")) as f:
        return json.load(f)


def _golden_matrix(g):
    N, K, b_d = g["N"], g["K"], g["b_d"]
    canon = np.array([list(bytes.fromhex(h)) for h in g["canonical_hex"]], np.uint8)
    cb = np.tile(np.array(g["codebook_rows"]["default"], np.float16), (1 << b_d, 1))
    for k, row in g["codebook_rows"].items():
        if k != "default":
            cb[int(k)] = np.array(row, np.float16)
    return synth.SvqMatrix(N, K, b_d, canon, cb.view(np.uint16),
                           np.array(g["scale"], np.float16).view(np.uint16),
                           np.array(g["offset"], np.float16).view(np.uint16),
                           np.array(g["perm"], np.int32))


# ----------------------------------------------------------------------------- P1
@pytest.mark.parametrize("K", [8, 16, 24, 32, 64, 768, 1024, 2048, 2560, 4096, 9728, 8192])
def test_p1_eighteen_bits_per_eight_weights(K):
    """Figure 2: 18 bits per eight weights -> ceil(18 K / 64) bytes per row; 9K/32 when K % 32 == 0."""
    assert oracle.row_bytes(K) == -(-18 * K // 64)
    if K % 32 == 0:
        assert oracle.row_bytes(K) * 32 == 9 * K
    N = 3
    G = K // 8
    r = np.random.default_rng(K)
    canon = oracle.pack(N, K, 8, r.integers(0, 256, (N, G)), r.integers(0, 256, (N, G)),
                        r.integers(0, 4, (N, G)))
    assert canon.shape == (N, oracle.row_bytes(K))


# ----------------------------------------------------------------------------- P2
def test_p2_golden_stream_unpacks_to_hand_fields(golden_dir):
    g = _golden(golden_dir)
    m = _golden_matrix(g)
    s, i, c = oracle.unpack(m.N, m.K, m.b_d, m.canonical)
    assert s.tolist() == g["fields"]["signs"]
    assert i.tolist() == g["fields"]["idx"]
    assert c.tolist() == g["fields"]["code"]


def test_p2_golden_fields_pack_to_hand_stream(golden_dir):
    g = _golden(golden_dir)
    f = g["fields"]
    canon = oracle.pack(g["N"], g["K"], g["b_d"], f["signs"], f["idx"], f["code"])
    assert [bytes(row).hex().upper() for row in canon] == g["canonical_hex"]


@pytest.mark.parametrize("b_d", range(1, 11))
@pytest.mark.parametrize("K", [8, 16, 40, 128, 264])
def test_p2_pack_unpack_roundtrip(b_d, K):
    N, G = 5, K // 8
    r = np.random.default_rng(1000 * b_d + K)
    s = r.integers(0, 256, (N, G)).astype(np.uint8)
    i = r.integers(0, 1 << b_d, (N, G)).astype(np.uint16)
    c = r.integers(0, 1 << (10 - b_d), (N, G)).astype(np.uint16)
    canon = oracle.pack(N, K, b_d, s, i, c)
    s2, i2, c2 = oracle.unpack(N, K, b_d, canon)
    assert np.array_equal(s, s2) and np.array_equal(i, i2) and np.array_equal(c, c2)
    # pad bits are written as zero and ignored on read
    pad = canon.shape[1] * 8 - 18 * G
    if pad:
        assert np.all(canon[:, -1] >> (8 - pad) == 0)
        dirty = canon.copy()
        dirty[:, -1] |= np.uint8((0xFF << (8 - pad)) & 0xFF)
        s3, i3, c3 = oracle.unpack(N, K, b_d, dirty)
        assert np.array_equal(s, s3) and np.array_equal(i, i3) and np.array_equal(c, c3)


def test_p2_field_out_of_range_rejected():
    with pytest.raises(ValueError):
        oracle.pack(1, 8, 6, [[0]], [[64]], [[0]])
    with pytest.raises(ValueError):
        oracle.pack(1, 8, 6, [[0]], [[0]], [[16]])


# ----------------------------------------------------------------------------- golden decode and layer
def test_golden_radius_decode_and_layer(golden_dir):
    g = _golden(golden_dir)
    m = _golden_matrix(g)
    for n in range(m.N):
        for gg in range(m.K // 8):
            code = g["fields"]["code"][n][gg]
            assert oracle.radius(int(m.scale[n]), int(m.offset[n]), code) == g["radius"][n][gg]
    W = oracle.decode_exact(m)
    want = np.array(g["W"], np.float64)
    assert np.array_equal(W, want)
    assert np.array_equal(np.signbit(W), np.signbit(want))          # -0.0 where a zero entry has sign 1
    w16 = oracle.dequant(m, "f16")
    assert [[f"{v:04X}" for v in row] for row in w16] == g["W_f16_hex"]
    x = np.array(g["x"], np.float16).view(np.uint16).reshape(1, -1)
    y, den = oracle.linear(m, x)
    assert y[0].tolist() == g["y"] and den[0].tolist() == g["den"]


# ----------------------------------------------------------------------------- P4 (oracle side)
@pytest.mark.parametrize("b_d", [6, 7, 8, 9])
def test_p4_dequant_is_rounded_binary32_product(b_d):
    """fp16 / bf16 export == RNE of the binary32 product r * c (numpy float32 multiply,
    numpy / torch casts), sign applied after rounding."""
    import torch
    m = synth.make_matrix(90, b_d, 16, 256, b_d)
    s, i, c = oracle.unpack(m.N, m.K, m.b_d, m.canonical)
    sc = m.scale.view(np.float16).astype(np.float32)
    off = m.offset.view(np.float16).astype(np.float32)
    r = np.array([[oracle.radius(int(m.scale[n]), int(m.offset[n]), int(c[n, g]))
                   for g in range(m.K // 8)] for n in range(m.N)], np.float32)
    # the radius: scale * code is exact in binary32 (11-bit by <= 9-bit), so one rounding
    assert np.array_equal(r, (sc[:, None] * c.astype(np.float32)) + off[:, None])
    cb = m.codebook.view(np.float16).astype(np.float32)
    prod = r[:, :, None] * cb[i.astype(np.int64)]                     # [N][G][8] float32
    sign = ((s[:, :, None] >> np.arange(8, dtype=np.uint8)) & 1).astype(bool)
    want16 = prod.astype(np.float16).view(np.uint16) ^ (sign.astype(np.uint16) << 15)
    assert np.array_equal(oracle.dequant(m, "f16"), want16.reshape(m.N, m.K))
    tb = torch.from_numpy(prod.reshape(-1)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    wantbf = tb.reshape(sign.shape) ^ (sign.astype(np.uint16) << 15)
    assert np.array_equal(oracle.dequant(m, "bf16"), wantbf.reshape(m.N, m.K))


def test_p4_subnormal_and_negative_zero():
    """A codebook with tiny and zero components exports fp16 subnormals and -0."""
    K, N, b_d = 16, 2, 2
    cb = np.zeros((4, 8), np.float16)
    cb[1] = np.array([2.0 ** -20, 2.0 ** -24, 0, 1, 0, 0, 0, 0], np.float16)
    s = np.array([[0xFF, 0x00], [0x01, 0xFE]], np.uint8)
    i = np.array([[1, 1], [0, 1]], np.uint16)
    c = np.zeros((2, 2), np.uint16)
    canon = oracle.pack(N, K, b_d, s, i, c)
    m = synth.SvqMatrix(N, K, b_d, canon, cb.view(np.uint16),
                        np.zeros(2, np.float16).view(np.uint16),
                        np.array([1.0, 0.5], np.float16).view(np.uint16), np.arange(K, dtype=np.int32))
    w = oracle.dequant(m, "f16")
    assert w[0, 0] == 0x8000 | 0x0010          # -(2^-20) is fp16 subnormal 16 * 2^-24
    assert w[0, 1] == 0x8001                   # -(2^-24)
    assert w[0, 2] == 0x8000                   # -0
    assert w[0, 8] == 0x0010 and w[0, 10] == 0x0000
    assert w[1, 8] == 0x0008                   # 0.5 * 2^-20 = 8 * 2^-24
    assert w[1, 9] == 0x8000                   # -(0.5 * 2^-24): the tie rounds to even (0), sign -> -0
    assert w[1, 0] == 0x8000                   # zero codeword with sign 1
    assert w[1, 11] == 0xB800                  # -(0.5 * 1)


# ----------------------------------------------------------------------------- P5
@pytest.mark.parametrize("b_d", [6, 7, 8, 9])
def test_p5_subvector_norm_is_radius_and_signs_follow_bits(b_d):
    m = synth.make_matrix(91, b_d, 32, 512, b_d)
    W = oracle.decode_exact(m)
    s, i, c = oracle.unpack(m.N, m.K, m.b_d, m.canonical)
    cb = m.codebook.view(np.float16).astype(np.float64)
    G = m.K // 8
    Wv = W.reshape(m.N, G, 8)
    norms = np.sqrt((Wv ** 2).sum(-1))
    sc = m.scale.view(np.float16).astype(np.float64)
    off = m.offset.view(np.float16).astype(np.float64)
    r = off[:, None] + sc[:, None] * c                      # exact in fp64
    cn = np.sqrt((cb[i.astype(np.int64)] ** 2).sum(-1))
    assert np.allclose(norms, r * cn, rtol=1e-12, atol=0)
    assert np.all(np.abs(cn - 1.0) <= 8 * 2.0 ** -11)       # unit codewords up to fp16 rounding
    bits = ((s[:, :, None] >> np.arange(8, dtype=np.uint8)) & 1).astype(bool)
    assert np.array_equal(np.signbit(Wv), bits)


# ----------------------------------------------------------------------------- P6
@pytest.mark.parametrize("b_d", range(1, 11))
def test_p6_bruteforce_encode_decode_roundtrip(b_d):
    """Decoded weights of random codes re-encode (nearest codeword) to the same decode."""
    N, K = 6, 48
    r = np.random.default_rng(77 + b_d)
    cb = np.abs(r.standard_normal((1 << b_d, 8)))
    cb = (cb / np.linalg.norm(cb, axis=1, keepdims=True)).astype(np.float16)
    # distinct radius levels and distinct codebook rows make the codes unique as well
    assert len({row.tobytes() for row in cb}) == len(cb)
    scale = r.uniform(0.05, 0.3, N).astype(np.float16)
    offset = r.uniform(0.5, 1.5, N).astype(np.float16)
    G = K // 8
    s = r.integers(0, 256, (N, G)).astype(np.uint8)
    i = r.integers(0, 1 << b_d, (N, G)).astype(np.uint16)
    c = r.integers(0, 1 << (10 - b_d), (N, G)).astype(np.uint16)
    canon = oracle.pack(N, K, b_d, s, i, c)
    m = synth.SvqMatrix(N, K, b_d, canon, cb.view(np.uint16), scale.view(np.uint16),
                        offset.view(np.uint16), np.arange(K, dtype=np.int32))
    W = oracle.decode_exact(m)
    s2, i2, c2 = oracle.encode(N, K, b_d, W, m.codebook, m.scale, m.offset)
    m2 = synth.SvqMatrix(N, K, b_d, oracle.pack(N, K, b_d, s2, i2, c2), m.codebook, m.scale,
                         m.offset, m.perm)
    assert np.array_equal(oracle.decode_exact(m2), W)
    assert np.array_equal(i2, i) and np.array_equal(c2, c)
    nz = W.reshape(N, G, 8) != 0
    bits = ((s[:, :, None] >> np.arange(8, dtype=np.uint8)) & 1).astype(bool)
    bits2 = ((s2[:, :, None] >> np.arange(8, dtype=np.uint8)) & 1).astype(bool)
    assert np.array_equal(bits[nz], bits2[nz])


def test_p6_energy_weights_change_the_choice():
    """The weighted fit: a heavy weight on one channel pulls the chosen codeword towards it."""
    cb = np.array([[1, 0, 0, 0, 0, 0, 0, 0], [0.6, 0.8, 0, 0, 0, 0, 0, 0]], np.float16)
    w = np.array([[0.9, 0.45, 0, 0, 0, 0, 0, 0]], np.float64)
    sc = np.array([0.0], np.float16).view(np.uint16)
    off = np.array([1.0], np.float16).view(np.uint16)
    _, i_plain, _ = oracle.encode(1, 8, 1, w, cb.view(np.uint16), sc, off)
    _, i_heavy, _ = oracle.encode(1, 8, 1, w, cb.view(np.uint16), sc, off,
                                  energy=np.array([100, 1, 1, 1, 1, 1, 1, 1], np.float64))
    # unweighted the two rows are within 1e-3 of each other; a weight of 100 on channel 0
    # makes row 0 (which matches channel 0 better) win clearly.
    e0 = (0.9 - 1) ** 2 + 0.45 ** 2
    e1 = (0.9 - float(cb[1, 0])) ** 2 + (0.45 - float(cb[1, 1])) ** 2
    assert i_plain[0, 0] == (0 if e0 <= e1 else 1)
    assert i_heavy[0, 0] == 0


# ----------------------------------------------------------------------------- P7
@pytest.mark.parametrize("K", [64, 1024])
def test_p7_closed_form_constant_codebook(K):
    """Every codebook row (1,...,1)/sqrt(8) in fp16 (0x35A8) and b_r = 0: W = +-offset * 0.353515625,
    so y = offset * 0.353515625 * sum_j (+-1) x[perm[j]] (exact sum via math.fsum)."""
    N, b_d = 8, 10
    m = synth.make_matrix(92, K, N, K, b_d)
    m.codebook = np.full((1 << b_d, 8), 0x35A8, np.uint16)
    x = synth.make_x(92, K, 1, K)
    y, den = oracle.linear(m, x)
    s, _, _ = oracle.unpack(N, K, b_d, m.canonical)
    sign = np.where(((s[:, :, None] >> np.arange(8, dtype=np.uint8)) & 1).astype(bool), -1, 1).reshape(N, K)
    xf = x.view(np.float16).astype(np.float64)[0]
    c = 0.353515625
    for n in range(N):
        off = float(m.offset.view(np.float16)[n])
        exact = off * c * math.fsum(float(sign[n, j]) * xf[m.perm[j]] for j in range(K))
        assert y[0, n] == pytest.approx(exact, rel=1e-12, abs=1e-12 * den[0, n])
        assert den[0, n] == pytest.approx(off * c * math.fsum(abs(v) for v in xf), rel=1e-12)


# ----------------------------------------------------------------------------- P8 / P9 (oracle side)
def test_p8_permutation_metamorphic():
    """y(W, perm, x) == y(W, identity, x[perm])."""
    m = synth.make_matrix(93, 0, 16, 256, 7)
    x = synth.make_x(93, 0, 3, 256)
    y1, _ = oracle.linear(m, x)
    mid = synth.SvqMatrix(m.N, m.K, m.b_d, m.canonical, m.codebook, m.scale, m.offset,
                          np.arange(m.K, dtype=np.int32))
    y2, _ = oracle.linear(mid, np.ascontiguousarray(x[:, m.perm]))
    assert np.array_equal(y1, y2)


def test_p9_linear_matches_library_matmul():
    """The oracle's loop == numpy matmul on the oracle's decoded weights and x[:, perm]."""
    m = synth.make_matrix(94, 0, 64, 512, 8)
    x = synth.make_x(94, 0, 4, 512)
    y, den = oracle.linear(m, x)
    W = oracle.decode_exact(m)
    xf = x.view(np.float16).astype(np.float64)[:, m.perm]
    assert np.allclose(y, xf @ W.T, rtol=0, atol=1e-12 * den.max())
    assert np.allclose(den, np.abs(xf) @ np.abs(W).T, rtol=1e-12)
    xb = synth.make_x(94, 1, 2, 512, dtype="bf16")
    yb, _ = oracle.linear(m, xb, "bf16")
    xbf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)[:, m.perm]
    assert np.allclose(yb, xbf @ W.T, rtol=0, atol=1e-12 * np.abs(xbf).sum())


# ----------------------------------------------------------------------------- generator properties
def test_generator_codebook_and_stream_properties():
    m = synth.make_matrix(95, 0, 12, 40, 9)
    cb = m.codebook.view(np.float16).astype(np.float64)
    assert np.all((m.codebook & 0x8000) == 0)
    assert np.all(np.abs(np.linalg.norm(cb, axis=1) - 1) <= 8 * 2.0 ** -11)
    pad = m.canonical.shape[1] * 8 - 18 * (m.K // 8)
    assert pad == 6 and np.all(m.canonical[:, -1] >> (8 - pad) == 0)
    assert sorted(m.perm.tolist()) == list(range(m.K))
    # the same seed gives the same matrix; another seed a different one
    m2 = synth.make_matrix(95, 0, 12, 40, 9)
    assert np.array_equal(m.canonical, m2.canonical) and np.array_equal(m.perm, m2.perm)
    m3 = synth.make_matrix(95, 1, 12, 40, 9)
    assert not np.array_equal(m.canonical, m3.canonical)


def test_generator_bf16_activations_are_rne():
    import torch
    xb = synth.make_x(96, 0, 3, 64, dtype="bf16")
    z = synth.rng(96, 0, synth.F_X).standard_normal((3, 64)).astype(np.float32)
    ref = torch.from_numpy(z).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(xb, ref)


def test_routing_topk_and_renormalisation():
    ids, w = synth.moe_routing(16)
    assert ids.shape == (16, 8) and np.allclose(w.sum(1), 1, atol=1e-6)
    assert all(len(set(r)) == 8 for r in ids.tolist())
    assert np.all(np.diff(w, axis=1) <= 0)                     # sorted by weight
