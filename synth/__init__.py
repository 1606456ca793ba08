"""Seeded synthetic inputs for the SVQ layer workloads.

This module is shared by the tests, the benchmark and the smoke check.  It
holds no decoding or matrix arithmetic of the method: it only draws random
inputs of the right shapes and distributions (with numpy's PCG64) and returns
them as plain arrays.

Recipe (every stream is ``Generator(PCG64(SeedSequence([config, matrix, field])))``):
  field 0  codebook: 2^b_d x 8 draws of |N(0,1)|, each row divided by its L2
           norm in fp64, then rounded to fp16.
  field 1  canonical code stream: uniform random bytes, N rows of
           ceil(18*(K/8)/8) bytes, pad bits at the end of a row cleared.  Every
           field of an 18-bit code word spans its full bit range, so uniform
           bytes give independent Bernoulli(1/2) signs, uniform direction
           indices and uniform radius codes.
  field 4  per-row radius offset ~ U(0.5, 1.5), rounded to fp16.
  field 5  per-row radius scale  ~ U(0.05, 0.3), rounded to fp16.
  field 6  input-channel permutation: a uniform random permutation of 0..K-1.
  field 7  activations: N(0,1) rounded to fp16 (or bf16 for the prefill case).
  field 8  per-channel energies ~ LogNormal(0, 1) (the decoder-layer case
           multiplies the N(0,1) draws by them before rounding).
  field 9  router logits ~ N(0,1) (MoE case).
  field 10 per-matrix bit split choice (MoE case): a fair coin between
           (b_d, b_r) = (7, 3) and (8, 2).
  field 11 per-row radius look-up tables: 0.5 + cumulative sums of 2^b_r
           draws of U(1, 2) / 2^b_r per row (increasing levels), rounded to fp16.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

F_CODEBOOK, F_CODES, F_OFFSET, F_SCALE, F_PERM, F_X, F_ENERGY, F_ROUTER, F_SPLIT, F_LUT = 0, 1, 4, 5, 6, 7, 8, 9, 10, 11


def rng(config: int, matrix: int, fld: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([config, matrix, fld])))


def canonical_row_bytes(K: int) -> int:
    """Bytes per row of the canonical stream: 18 bits per 8 weights, rounded up to a byte."""
    return ((K // 8) * 18 + 7) // 8


@dataclass
class SvqMatrix:
    """One SVQ matrix W[N][K] in the canonical (interchange) format.

    canonical: uint8 [N][row_bytes]   18-bit codes, little-endian bit stream per row
    codebook:  uint16 [2^b_d][8]      fp16 bit patterns of non-negative unit vectors
    scale:     uint16 [N]             fp16 radius scale per row
    offset:    uint16 [N]             fp16 radius offset per row
    perm:      int32 [K]              stored column j multiplies x[perm[j]]
    lut:       uint16 [N][2^b_r] or None   fp16 radius level of each code, per row
                                           (replaces scale/offset when present)
    """
    N: int
    K: int
    b_d: int
    canonical: np.ndarray
    codebook: np.ndarray
    scale: np.ndarray
    offset: np.ndarray
    perm: np.ndarray
    name: str = ""
    meta: dict = field(default_factory=dict)
    lut: np.ndarray | None = None

    @property
    def b_r(self) -> int:
        return 10 - self.b_d


def make_codebook(r: np.random.Generator, b_d: int) -> np.ndarray:
    z = np.abs(r.standard_normal((1 << b_d, 8)))
    z = z / np.sqrt((z * z).sum(axis=1, keepdims=True))
    return z.astype(np.float16).view(np.uint16)


def make_codes(r: np.random.Generator, N: int, K: int) -> np.ndarray:
    rb = canonical_row_bytes(K)
    codes = r.integers(0, 256, size=(N, rb), dtype=np.uint8)
    pad = rb * 8 - (K // 8) * 18
    if pad:
        codes[:, -1] &= np.uint8(0xFF >> pad)
    return codes


def make_matrix(config: int, matrix: int, N: int, K: int, b_d: int, name: str = "",
                identity_perm: bool = False) -> SvqMatrix:
    assert K % 8 == 0 and 1 <= b_d <= 10
    cb = make_codebook(rng(config, matrix, F_CODEBOOK), b_d)
    codes = make_codes(rng(config, matrix, F_CODES), N, K)
    offset = rng(config, matrix, F_OFFSET).uniform(0.5, 1.5, N).astype(np.float16).view(np.uint16)
    scale = rng(config, matrix, F_SCALE).uniform(0.05, 0.3, N).astype(np.float16).view(np.uint16)
    if identity_perm:
        perm = np.arange(K, dtype=np.int32)
    else:
        perm = rng(config, matrix, F_PERM).permutation(K).astype(np.int32)
    return SvqMatrix(N, K, b_d, codes, cb, scale, offset, perm, name)


def make_lut(config: int, matrix: int, N: int, b_d: int) -> np.ndarray:
    """Per-row radius levels [N][2^b_r] as fp16 bit patterns: 0.5 plus cumulative sums of U(1, 2) / 2^b_r
    draws, so each row's levels increase (by at least 2^-b_r: distinct in fp16 for b_r <= 8) over about
    [0.5, 2]."""
    nr = 1 << (10 - b_d)
    lv = 0.5 + np.cumsum(rng(config, matrix, F_LUT).uniform(1.0, 2.0, (N, nr)), axis=1) / nr
    return lv.astype(np.float16).view(np.uint16)


def make_x(config: int, matrix: int, M: int, K: int, dtype: str = "f16",
           energies: bool = False) -> np.ndarray:
    """Activations [M][K] as 16-bit patterns (fp16 or bf16)."""
    z = rng(config, matrix, F_X).standard_normal((M, K))
    if energies:
        e = rng(config, matrix, F_ENERGY).lognormal(0.0, 1.0, K)
        z = z * e[None, :]
    if dtype == "f16":
        return z.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        # bfloat16 by round-to-nearest-even of the binary32 value (numpy has no bf16).
        f = z.astype(np.float32).view(np.uint32).astype(np.uint64)
        bias = np.uint64(0x7FFF) + ((f >> np.uint64(16)) & np.uint64(1))
        return ((f + bias) >> np.uint64(16)).astype(np.uint16)
    raise ValueError(dtype)


# --------------------------------------------------------------------------- workloads
# (b_d, b_r) cycle of the decoder-layer case, in the order q, k, v, o, gate, up, down.
QWEN3_4B_SPLITS = [6, 7, 8, 9, 6, 7, 8]
QWEN3_4B_SHAPES = [("q", 4096, 2560), ("k", 1024, 2560), ("v", 1024, 2560), ("o", 2560, 4096),
                   ("gate", 9728, 2560), ("up", 9728, 2560), ("down", 2560, 9728)]


def single_layer_1024():
    """K = N = 1024, (b_d, b_r) = (8, 2), one fp16 N(0,1) input vector."""
    m = make_matrix(0, 0, 1024, 1024, 8, name="layer1024")
    x = make_x(0, 0, 1, 1024)
    return m, x


def qwen3_4b_layer(layer: int = 0):
    """The seven linears of a Qwen3-4B-shaped decoder layer at batch 1.

    `layer` selects an independent copy (different seeds) so that a benchmark
    can rotate through more weight bytes than the L2 cache holds.  Returns a
    list of (SvqMatrix, x[1][K]) with x scaled by log-normal channel energies."""
    out = []
    for i, ((name, N, K), b_d) in enumerate(zip(QWEN3_4B_SHAPES, QWEN3_4B_SPLITS)):
        mid = 1000 * layer + i
        m = make_matrix(1, mid, N, K, b_d, name=name)
        x = make_x(1, mid, 1, K, energies=True)
        out.append((m, x))
    return out


def square_8192():
    """One 8192 x 8192 matrix with (b_d, b_r) = (7, 3)."""
    return make_matrix(2, 0, 8192, 8192, 7, name="sq8192")


def square_8192_x(M: int) -> np.ndarray:
    return make_x(2, 100 + M, M, 8192)


def prefill_mats():
    """Qwen3-4B gate/up (2560 -> 9728) and down (9728 -> 2560) with (8, 2)."""
    return [make_matrix(3, 0, 9728, 2560, 8, name="gate_up"),
            make_matrix(3, 1, 2560, 9728, 8, name="down")]


def prefill_x(M: int, K: int, which: int) -> np.ndarray:
    return make_x(3, 100 * which + M, M, K, dtype="bf16")


MOE_HIDDEN, MOE_EXPERTS, MOE_INTER, MOE_TOPK = 2048, 128, 768, 8


def moe_experts(n_experts: int = MOE_EXPERTS):
    """Per expert (gate 2048->768, up 2048->768, down 768->2048), each with its own
    codebook and a seeded split from {(7,3), (8,2)}."""
    experts = []
    for e in range(n_experts):
        trip = []
        for j, (N, K) in enumerate([(MOE_INTER, MOE_HIDDEN), (MOE_INTER, MOE_HIDDEN),
                                    (MOE_HIDDEN, MOE_INTER)]):
            mid = 3 * e + j
            b_d = 7 if rng(4, mid, F_SPLIT).integers(0, 2) == 0 else 8
            trip.append(make_matrix(4, mid, N, K, b_d, name=f"e{e}.{'gate up down'.split()[j]}"))
        experts.append(tuple(trip))
    return experts


def moe_routing(T: int, n_experts: int = MOE_EXPERTS, topk: int = MOE_TOPK):
    """Router: softmax over N(0,1) logits, top-k (ties to the lower expert id),
    weights renormalised over the selected k.  Returns (ids int32 [T][k], w fp32 [T][k])."""
    logits = rng(4, 10000 + T, F_ROUTER).standard_normal((T, n_experts))
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)
    ids = np.empty((T, topk), np.int32)
    w = np.empty((T, topk), np.float32)
    for t in range(T):
        order = sorted(range(n_experts), key=lambda e: (-p[t, e], e))[:topk]
        ids[t] = order
        sel = p[t, order]
        w[t] = (sel / sel.sum()).astype(np.float32)
    return ids, w


def moe_x(T: int) -> np.ndarray:
    return make_x(4, 20000 + T, T, MOE_HIDDEN)
