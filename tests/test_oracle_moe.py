"""Pin of the oracle's MoE composition (oracle.moe_ffn), the checker of the
grouped-expert parity tests.

The pages evaluate SVQ on a mixture-of-experts model (Qwen3-30B-A3B, SAGE
abstract) and every expert matrix is an SVQ matrix as in the Figure 2 caption.
Here every codebook row is (1,...,1)/sqrt(8) rounded to fp16 (0x35A8) and
b_r = 0, so each weight is +-offset_n * 0.353515625 exactly and every layer
output is an exact signed sum (math.fsum).  The combine is then written out by
hand: out[t] = sum_k w[t,k] * down_{e(t,k)}(h[t,k]) and
den[t] = sum_k |w[t,k]| * sum_j |W_down[n][j]| |h[t,k][perm[j]]|.  A slip in the
composition -- a routing weight applied twice or not at all, den built from
signed weights, the wrong expert's matrix, the gate and up outputs swapped --
fails one of the assertions below.
"""
import math

import numpy as np
import pytest

import oracle
import synth

C = 0.353515625                                  # fp16 0x35A8


def _const_matrix(config, mid, N, K):
    m = synth.make_matrix(config, mid, N, K, 10)
    m.codebook = np.full((1 << 10, 8), 0x35A8, np.uint16)
    # offsets with few mantissa bits, so that offset * C and every partial sum are exact in fp64
    r = np.random.default_rng(1000 + mid)
    m.offset = r.choice([0.5, 0.625, 0.75, 1.0, 1.25, 1.5], N).astype(np.float16).view(np.uint16)
    return m


def _signs(m):
    s, _, _ = oracle.unpack(m.N, m.K, m.b_d, m.canonical)
    bits = (s[:, :, None] >> np.arange(8, dtype=np.uint8)) & 1
    return np.where(bits.astype(bool), -1.0, 1.0).reshape(m.N, m.K)


def _closed_form(m, xf):
    """y[n] = sum_j (+-offset_n C) x[perm[j]] and den[n] = sum_j offset_n C |x[perm[j]]|."""
    sg = _signs(m)
    off = m.offset.view(np.float16).astype(np.float64)
    y = np.array([off[n] * C * math.fsum(sg[n, j] * xf[m.perm[j]] for j in range(m.K)) for n in range(m.N)])
    den = np.array([off[n] * C * math.fsum(abs(xf[m.perm[j]]) for j in range(m.K)) for n in range(m.N)])
    return y, den


def _experts(n=2, H=32, I=16):
    return [(_const_matrix(95, 3 * e, I, H), _const_matrix(95, 3 * e + 1, I, H), _const_matrix(95, 3 * e + 2, H, I))
            for e in range(n)]


def _small_int_fp16(r, shape, lo=-4, hi=5):
    return r.integers(lo, hi, shape).astype(np.float16).view(np.uint16)


@pytest.mark.parametrize("ids,w", [([[1, 0]], [[0.625, 0.375]]), ([[0, 1]], [[0.75, -0.25]])])
def test_moe_ffn_closed_form_with_given_h(ids, w):
    """Two experts, one token, hand-set routing weights, the down layer fed given fp16 h."""
    experts = _experts()
    r = np.random.default_rng(7)
    x = _small_int_fp16(r, (1, 32))
    h = _small_int_fp16(r, (1, 2, 16))
    ids = np.array(ids, np.int32)
    w = np.array(w, np.float32)
    gate_y, up_y, out, den = oracle.moe_ffn(experts, x, ids, w, h_bits=h)
    xf = x.view(np.float16).astype(np.float64)[0]
    exp_out = [[] for _ in range(32)]
    exp_den = [[] for _ in range(32)]
    for k in range(2):
        g, u, d = experts[int(ids[0, k])]
        gy, _ = _closed_form(g, xf)
        uy, _ = _closed_form(u, xf)
        assert np.array_equal(gate_y[0, k], gy)          # gate output of the selected expert, exact
        assert np.array_equal(up_y[0, k], uy)
        hf = h[0, k].view(np.float16).astype(np.float64)
        dy, dden = _closed_form(d, hf)
        for n in range(32):
            exp_out[n].append(float(w[0, k]) * dy[n])
            exp_den[n].append(abs(float(w[0, k])) * dden[n])
    for n in range(32):
        assert out[0, n] == pytest.approx(math.fsum(exp_out[n]), rel=1e-12, abs=1e-12)
        assert den[0, n] == pytest.approx(math.fsum(exp_den[n]), rel=1e-12, abs=1e-12)
    # the two experts' down matrices differ, so swapping them changes the result
    d0, _ = _closed_form(experts[0][2], h[0, 0].view(np.float16).astype(np.float64))
    d1, _ = _closed_form(experts[1][2], h[0, 0].view(np.float16).astype(np.float64))
    assert not np.array_equal(d0, d1)


def test_moe_ffn_own_h_is_silu_gate_times_up_in_fp16():
    """Without given h the down layer takes fp16(silu(gate) * up); checked here against scipy's
    logistic (silu(v) = v * expit(v)), an independent route to the same value."""
    from scipy.special import expit
    experts = _experts()
    r = np.random.default_rng(8)
    x = _small_int_fp16(r, (1, 32), -2, 3)
    ids = np.array([[1, 0]], np.int32)
    w = np.array([[0.5, 0.5]], np.float32)
    gate_y, up_y, out, den = oracle.moe_ffn(experts, x, ids, w)
    for k in range(2):
        h = gate_y[0, k] * expit(gate_y[0, k]) * up_y[0, k]
        hb = h.astype(np.float32).astype(np.float16).view(np.uint16)
        d = experts[int(ids[0, k])][2]
        dy, dden = _closed_form(d, hb.view(np.float16).astype(np.float64))
        _, _, out_k, den_k = oracle.moe_ffn(experts, x, ids[:, k:k + 1], np.ones((1, 1), np.float32),
                                            h_bits=hb.reshape(1, 1, -1))
        np.testing.assert_allclose(out_k[0], dy, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(den_k[0], dden, rtol=1e-12, atol=1e-12)
    # and the combined output is the weighted sum of the two
    parts = []
    for k in range(2):
        h = gate_y[0, k] * expit(gate_y[0, k]) * up_y[0, k]
        hb = h.astype(np.float32).astype(np.float16)
        dy, _ = _closed_form(experts[int(ids[0, k])][2], hb.astype(np.float64))
        parts.append(0.5 * dy)
    np.testing.assert_allclose(out[0], parts[0] + parts[1], rtol=1e-12, atol=1e-12)
