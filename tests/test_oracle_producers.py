"""Pins of the oracle's decoder-layer producers (RMS normalisation and the
SiLU-gated product, each written in a consumer's stored column order) and of
its one-step binary64 -> binary16 rounding.  Every expected value below is a
closed form, an exact special case, or an independent library routine."""
import math

import numpy as np
import pytest

import oracle


def _h(vals):
    return np.asarray(vals, np.float16).view(np.uint16)


def test_f64_to_h_matches_c_conversion_on_binary32_inputs():
    """On binary32 inputs one rounding step is the C oracle's conversion; includes every fp16 tie point
    between 1 and 2 and random values over the whole range (overflow, subnormals)."""
    rng = np.random.default_rng(1)
    ties = (1.0 + (np.arange(1024) + 0.5) * 2.0 ** -10).astype(np.float32)
    rnd = (rng.standard_normal(20000) * np.exp(rng.uniform(-25, 12, 20000))).astype(np.float32)
    v = np.concatenate([ties, -ties, rnd, np.float32([0.0, -0.0, 65504.0, 65520.0, 1e-8, -6e-8])])
    assert np.array_equal(oracle.f64_to_h_rne(v.astype(np.float64)), oracle.f2h_rne(v))


@pytest.mark.parametrize("v,bits", [(1 + 2 ** -11 + 2 ** -40, 0x3C01),   # above the tie: up (f32 first would give 0x3C00)
                                    (1 + 2 ** -11, 0x3C00),              # tie: to even
                                    (1 + 3 * 2 ** -11, 0x3C02),          # tie: to even (up)
                                    (-(1 + 2 ** -11 - 2 ** -40), 0xBC00)])
def test_f64_to_h_single_rounding(v, bits):
    assert int(oracle.f64_to_h_rne(v)) == bits


def test_rmsnorm_constant_rows_give_gamma():
    """A constant row c has RMS |c|: with eps 0 the output is sign(c) * gamma exactly, row by row."""
    K = 64
    gamma = _h(np.linspace(-2, 3, K))
    h = _h(np.stack([np.full(K, 0.75), np.full(K, -3.0), np.full(K, 1024.0)]))
    x = oracle.rmsnorm(h, "f16", gamma, 0.0)
    g = oracle.h2f(gamma).astype(np.float64)
    assert np.array_equal(x, np.stack([g, -g, g]))


def test_rmsnorm_eps_closed_form():
    """Row of ones, eps 3: 1 / sqrt(1 + 3) = 1/2."""
    K = 40
    x = oracle.rmsnorm(_h(np.ones((1, K))), "f16", _h(np.ones(K)), 3.0)
    assert np.array_equal(x, np.full((1, K), 0.5))


def test_rmsnorm_is_scale_invariant_and_unit_rms():
    rng = np.random.default_rng(2)
    K = 2560
    h = _h(rng.standard_normal((3, K)))
    h4 = _h(oracle.h2f(h).reshape(h.shape) * 4.0)      # exact: a power of two
    one = _h(np.ones(K))
    x = oracle.rmsnorm(h, "f16", one, 0.0)
    assert np.array_equal(x, oracle.rmsnorm(h4, "f16", one, 0.0))
    assert np.allclose(np.mean(x * x, axis=1), 1.0, rtol=1e-12)


def test_rmsnorm_bf16_input():
    """bf16 input: a row with two values +-b has RMS |b| (eps 0)."""
    b = np.float32(1.5)
    bits = np.array([[np.float32(b).view(np.uint32) >> 16, np.float32(-b).view(np.uint32) >> 16]], np.uint16)
    x = oracle.rmsnorm(bits, "bf16", _h([2.0, 5.0]), 0.0)
    assert np.array_equal(x, np.array([[2.0, -5.0]]))


def test_rmsnorm_permute_gathers_input_and_gamma_by_the_consumer_permutation():
    """Row of ones, eps 0: x_g[j] = gamma[p_g[j]] exactly, for each consumer's own permutation."""
    K = 32
    rng = np.random.default_rng(3)
    gamma_f = np.arange(1, K + 1) * 0.25
    p1, p2 = rng.permutation(K), rng.permutation(K)
    outs = oracle.rmsnorm_permute(_h(np.ones((2, K))), "f16", _h(gamma_f), 0.0, [p1, None, p2])
    assert np.array_equal(outs[0], np.tile(_h(gamma_f[p1]), (2, 1)))
    assert np.array_equal(outs[1], np.tile(_h(gamma_f), (2, 1)))
    assert np.array_equal(outs[2], np.tile(_h(gamma_f[p2]), (2, 1)))


def test_rmsnorm_permute_gathers_per_element_not_per_row():
    """h varies along the row: the permuted output is the natural one with its columns permuted."""
    rng = np.random.default_rng(4)
    K = 256
    h = _h(rng.standard_normal((2, K)))
    gamma = _h(rng.uniform(0.5, 2.0, K))
    p = rng.permutation(K)
    nat, per = oracle.rmsnorm_permute(h, "f16", gamma, 1e-6, [None, p])
    assert np.array_equal(per, nat[:, p])
    assert not np.array_equal(per, nat)


def test_swiglu_against_the_logistic_function():
    """silu(v) = v * logistic(v); scipy's expit is an independent logistic."""
    scipy_special = pytest.importorskip("scipy.special")
    rng = np.random.default_rng(5)
    g = (rng.standard_normal((4, 500)) * 4).astype(np.float32)
    u = rng.standard_normal((4, 500)).astype(np.float32)
    a = oracle.swiglu(g, u)
    b = g.astype(np.float64) * scipy_special.expit(g.astype(np.float64)) * u.astype(np.float64)
    assert np.allclose(a, b, rtol=1e-13, atol=0)


def test_swiglu_odd_part_identity():
    """silu(v) - silu(-v) = v for every v (logistic(v) + logistic(-v) = 1)."""
    v = np.linspace(-20, 20, 1001)
    one = np.ones_like(v)
    assert np.allclose(oracle.swiglu(v, one) - oracle.swiglu(-v, one), v, rtol=0, atol=1e-13)


@pytest.mark.parametrize("g,u,bits", [(0.0, 1.0, 0x0000), (30.0, 1.0, 0x4F80), (30.0, -2.0, 0xD380),
                                      (-30.0, 1.0, 0x8000), (-30.0, -1.0, 0x0000), (-200.0, 3.0, 0x8000)])
def test_swiglu_permute_special_values(g, u, bits):
    """0 -> 0; large v -> v (silu(30) = 30 to within 1e-11); very negative v -> signed zero."""
    out = oracle.swiglu_permute(np.array([[g]], np.float32), np.array([[u]], np.float32), None)
    assert int(out[0, 0]) == bits


def test_swiglu_permute_order():
    rng = np.random.default_rng(6)
    g = rng.standard_normal((2, 64)).astype(np.float32)
    u = rng.standard_normal((2, 64)).astype(np.float32)
    p = rng.permutation(64)
    nat = oracle.swiglu_permute(g, u, None)
    assert np.array_equal(oracle.swiglu_permute(g, u, p), nat[:, p])
    assert np.array_equal(nat, oracle.f64_to_h_rne(oracle.swiglu(g, u)))
