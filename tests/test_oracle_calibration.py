"""Pins of the calibration-side oracle: channel energies, the Energy-Stratified
Grouping permutation, the radius grid and the Adaptive Bit Split choice.
Expected values are worked by hand from the definitions, closed forms, or
matrices built so that one split reproduces them exactly."""
import numpy as np
import pytest

import oracle
from oracle import calibration as cal
import synth


def test_channel_energy_closed_form():
    assert np.array_equal(cal.channel_energy([[1.0, 2.0], [3.0, -4.0]]), np.array([5.0, 10.0]))


def test_esg_perm_worked_example():
    """K = 16: order by energy (highest first) = 15 14 13 12 11 10 2 6 4 7 0 9 3 5 1 8; tiers of two;
    subvector 0 takes the first channel of each tier, subvector 1 the second."""
    e = [5, 1, 9, 3, 7, 2, 8, 6, 0.5, 4, 10, 11, 12, 13, 14, 15]
    want = [15, 13, 11, 2, 4, 0, 3, 1,
            14, 12, 10, 6, 7, 9, 5, 8]
    assert cal.esg_perm(e).tolist() == want


def test_esg_perm_equal_energies_closed_form():
    """All energies equal: order = 0..K-1, so perm[8g + t] = t * K/8 + g."""
    K = 64
    G = K // 8
    want = [t * G + g for g in range(G) for t in range(8)]
    assert cal.esg_perm(np.ones(K)).tolist() == want


def test_esg_perm_is_a_permutation_with_one_channel_per_tier():
    rng = np.random.default_rng(20)
    K = 2560
    e = rng.lognormal(0.0, 1.0, K)
    p = cal.esg_perm(e)
    assert sorted(p.tolist()) == list(range(K))
    # tier of a channel = how many channels have a strictly higher energy, divided by K/8 (energies distinct)
    higher = np.array([(e > e[k]).sum() for k in range(K)])
    tiers = (higher // (K // 8))[p].reshape(-1, 8)
    assert np.array_equal(tiers, np.tile(np.arange(8), (K // 8, 1)))
    # energies fall along each subvector and, within a tier, along the subvectors
    ev = e[p].reshape(-1, 8)
    assert np.all(np.diff(ev, axis=1) < 0)
    assert np.all(np.diff(ev, axis=0) < 0)


def test_esg_perm_invariant_under_monotone_maps():
    rng = np.random.default_rng(21)
    e = rng.lognormal(0.0, 1.0, 256)
    p = cal.esg_perm(e)
    for gamma in (0.25, 0.5, 2.0):
        assert np.array_equal(cal.esg_perm(cal.esg_weights(e, gamma)), p)
    assert np.array_equal(cal.esg_perm(3.0 * e), p)


def test_radius_grid_closed_form():
    """Row with subvector norms 1, 2.5 and 4 at b_d 8 (3 levels apart): offset 1, scale 1."""
    W = np.zeros((1, 24))
    W[0, 0] = 1.0
    W[0, 8:10] = [1.5, 2.0]
    W[0, 16] = -4.0
    sc, of = cal.radius_grid(W, 8)
    assert int(sc[0]) == 0x3C00 and int(of[0]) == 0x3C00


def _natural(m):
    """Exact weights of a synthetic matrix in natural column order, and its permutation."""
    Ws = oracle.decode_exact(m)
    W = np.empty_like(Ws)
    W[:, m.perm] = Ws
    return W


def test_abs_picks_the_split_that_reproduces_the_matrix():
    N, K = 6, 64
    mats = {b: synth.make_matrix(99, b, N, K, b) for b in (6, 7, 8, 9)}
    W = _natural(mats[7])
    cands = [(b, mats[b].codebook, mats[b].scale, mats[b].offset) for b in (6, 7, 8, 9)]
    weights = np.random.default_rng(22).uniform(0.5, 2.0, K)
    best, errors = cal.abs_select(W, mats[7].perm, weights, cands)
    assert best == 1 and errors[1] == 0.0
    assert min(errors[0], errors[2], errors[3]) > 0.0


def test_abs_weighting_decides_between_splits():
    """First half of the columns exact under split 6, second half under split 8: the split whose exact
    half carries the weight wins."""
    N, K = 4, 128
    m6 = synth.make_matrix(98, 6, N, K, 6, identity_perm=True)
    m8 = synth.make_matrix(98, 8, N, K, 8, identity_perm=True)
    m8.scale, m8.offset = m6.scale, m6.offset         # shared radius grid keeps both halves exact
    W6, W8 = oracle.decode_exact(m6), oracle.decode_exact(m8)
    W = np.concatenate([W6[:, :K // 2], W8[:, K // 2:]], axis=1)
    perm = np.arange(K, dtype=np.int32)
    cands = [(6, m6.codebook, m6.scale, m6.offset), (8, m8.codebook, m8.scale, m8.offset)]
    first = np.where(np.arange(K) < K // 2, 1.0, 0.0)
    # preconditions: each split is exact on its half and not on the other
    assert cal.split_error(W, perm, first, *cands[0])[0] == 0.0
    assert cal.split_error(W, perm, 1.0 - first, *cands[1])[0] == 0.0
    assert cal.split_error(W, perm, first, *cands[1])[0] > 0.0
    assert cal.split_error(W, perm, 1.0 - first, *cands[0])[0] > 0.0
    heavy_first = np.where(np.arange(K) < K // 2, 1e6, 1e-6)
    assert cal.abs_select(W, perm, heavy_first, cands)[0] == 0
    assert cal.abs_select(W, perm, heavy_first[::-1].copy(), cands)[0] == 1


def test_abs_error_scales_with_the_weights_and_single_candidate():
    N, K = 3, 64
    m = synth.make_matrix(97, 0, N, K, 8)
    W = _natural(m) + np.random.default_rng(23).normal(0, 0.01, (N, K))
    c6 = synth.make_matrix(97, 1, N, K, 6)
    cands = [(8, m.codebook, m.scale, m.offset), (6, c6.codebook, c6.scale, c6.offset)]
    w = np.random.default_rng(24).uniform(0.5, 2.0, K)
    b1, e1 = cal.abs_select(W, m.perm, w, cands)
    b3, e3 = cal.abs_select(W, m.perm, 3.0 * w, cands)
    assert b1 == b3
    assert np.allclose(np.array(e3), 3.0 * np.array(e1), rtol=1e-12)
    assert cal.abs_select(W, m.perm, w, cands[1:])[0] == 0


def test_first_candidate_wins_a_tie():
    N, K = 2, 32
    m = synth.make_matrix(96, 0, N, K, 7)
    W = _natural(m)
    c = (7, m.codebook, m.scale, m.offset)
    best, errors = cal.abs_select(W, m.perm, np.ones(K), [c, c])
    assert best == 0 and errors[0] == errors[1] == 0.0


@pytest.mark.parametrize("gamma", [0.5, 1.0])
def test_esg_pipeline_on_calibration_activations(gamma):
    """Energies from activations, weights e^gamma, permutation from the energies, ABS over four splits:
    the output is a valid permutation and a split index with finite, non-negative errors."""
    rng = np.random.default_rng(25)
    K, N = 64, 4
    x_cal = rng.standard_normal((32, K)) * rng.lognormal(0.0, 1.0, K)
    e = cal.channel_energy(x_cal)
    p = cal.esg_perm(e)
    W = rng.standard_normal((N, K)) * 0.05
    Ws = W[:, p]
    cands = []
    for b in (6, 7, 8, 9):
        sc, of = cal.radius_grid(Ws, b)
        cands.append((b, synth.make_codebook(synth.rng(95, b, 0), b), sc, of))
    best, errors = cal.abs_select(W, p, cal.esg_weights(e, gamma), cands)
    assert 0 <= best < 4 and all(np.isfinite(errors)) and min(errors) >= 0.0
    assert errors[best] == min(errors)
