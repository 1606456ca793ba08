"""CPU oracle of the calibration side of SAGE: Energy-Stratified Grouping (ESG)
and Adaptive Bit Split (ABS).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle``.

"SAGE" (arXiv 2610.14745), abstract and Figure 2 caption: ESG uses calibration
activations to put channels of different energy tiers into each subvector and
weights the fit by activation energy; Figure 4(a): the energy enters through
an exponent gamma; ABS encodes a matrix under each candidate direction/radius
split of the 18-bit budget and keeps the split with the lowest
activation-weighted reconstruction error.  The pages give no formulas; the
readings taken here (each the plainest one the captions support):

* channel energy e_k = mean over calibration rows of x[t][k]^2, fitting weight
  e_k ** gamma;
* tiers: channels sorted by energy, highest first (equal energies: lower
  channel index first), cut into 8 tiers of K/8 consecutive channels; the g-th
  channel of every tier goes to subvector g, tier t at position t:
  perm[8g + t] = order[t * K/8 + g];
* ABS error: sum over rows and stored columns j of w[perm[j]] * (W[n][perm[j]]
  - What[n][j])^2, What decoded exactly (fp64) from the codes the weighted
  brute-force encoder picks; the first candidate wins a tie;
* radius grid (an input to ABS, not fixed by the pages, which optimise the
  radius levels blockwise): uniform between the smallest and largest subvector
  norm of each row, scale and offset rounded to fp16;
* sums whose order the pages leave open (channel energies over calibration
  rows, a subvector's squared norm over its elements) run in ascending index
  order in fp64, one rounding per operation.
"""
from __future__ import annotations

from types import SimpleNamespace

import numpy as np

from . import decode_exact, encode, f64_to_h_rne, h2f, pack


def channel_energy(x_cal) -> np.ndarray:
    """e_k = (1/T) sum_t x[t][k]^2 in fp64 for calibration activations x_cal [T][K] (float values).

    The sum runs over t in ascending order, one rounding per addition, then one
    division by T: a fixed order, so that another implementation can reproduce
    the value exactly."""
    x = np.asarray(x_cal, np.float64)
    T = x.shape[0]
    s = x[0] * x[0]
    for t in range(1, T):
        s = s + x[t] * x[t]
    return s / float(T)


def esg_weights(energy, gamma: float) -> np.ndarray:
    """Fitting weight of each input channel: energy ** gamma."""
    return np.asarray(energy, np.float64) ** float(gamma)


def esg_perm(energy) -> np.ndarray:
    """ESG permutation [K] (int32): subvector g takes the g-th channel of each of the 8 energy tiers."""
    e = np.asarray(energy, np.float64)
    K = e.shape[0]
    assert K % 8 == 0
    G = K // 8
    order = sorted(range(K), key=lambda k: (-e[k], k))
    perm = np.empty(K, np.int32)
    for g in range(G):
        for t in range(8):
            perm[8 * g + t] = order[t * G + g]
    return perm


def radius_grid(W_stored, b_d: int):
    """Per-row uniform radius grid over the row's subvector norms: fp16 (scale, offset) bit patterns [N]."""
    W = np.asarray(W_stored, np.float64)
    N, K = W.shape
    sub = W.reshape(N, K // 8, 8)
    # squared norm summed over the eight elements in element order (fixed order, see channel_energy)
    sq = sub[:, :, 0] * sub[:, :, 0]
    for i in range(1, 8):
        sq = sq + sub[:, :, i] * sub[:, :, i]
    norms = np.sqrt(sq)
    lo, hi = norms.min(axis=1), norms.max(axis=1)
    levels = (1 << (10 - b_d)) - 1
    scale = (hi - lo) / levels if levels > 0 else np.zeros(N)
    return f64_to_h_rne(scale), f64_to_h_rne(lo)


def split_error(W_nat, perm, weights, b_d: int, codebook, scale, offset):
    """Activation-weighted reconstruction error of W under one split, and the codes the encoder picked.

    W_nat [N][K] in natural column order; codebook/scale/offset fp16 bit patterns."""
    W_nat = np.asarray(W_nat, np.float64)
    perm = np.asarray(perm, np.int64)
    N, K = W_nat.shape
    Ws = np.ascontiguousarray(W_nat[:, perm])
    ws = np.ascontiguousarray(np.asarray(weights, np.float64)[perm])
    signs, idx, code = encode(N, K, b_d, Ws, codebook, scale, offset, ws)
    m = SimpleNamespace(N=N, K=K, b_d=b_d, canonical=pack(N, K, b_d, signs, idx, code),
                        codebook=np.asarray(codebook, np.uint16), scale=np.asarray(scale, np.uint16),
                        offset=np.asarray(offset, np.uint16), perm=perm.astype(np.int32))
    W_hat = decode_exact(m)
    err = float(np.sum(ws[None, :] * (Ws - W_hat) ** 2))
    return err, (signs, idx, code)


def abs_select(W_nat, perm, weights, candidates):
    """ABS: the candidate split with the lowest weighted error (first one on ties).

    candidates: list of (b_d, codebook, scale, offset).  Returns (index, errors)."""
    errors = [split_error(W_nat, perm, weights, b_d, cb, sc, of)[0] for b_d, cb, sc, of in candidates]
    best = 0
    for i, e in enumerate(errors):
        if e < errors[best]:
            best = i
    return best, errors


def codebook_values(codebook) -> np.ndarray:
    """fp16 codebook bit patterns [2^b_d][8] as fp64 values."""
    cb = np.asarray(codebook, np.uint16)
    return h2f(cb).astype(np.float64).reshape(cb.shape)
