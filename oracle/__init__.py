"""CPU oracle for the SVQ fused decode-and-multiply layer.

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The library under
``bit_spherical_vector_b200`` never imports this package, and this package
never imports the library: they share nothing but the seeded input generators
in ``synth``.

The arithmetic lives in ``svqref.cpp`` (plain C++, fp64 loops, IEEE fp16/bf16
conversions written from the definitions).  This module compiles it with g++
on first use and wraps it with numpy-friendly functions.  The MoE composition
(routing weights, SiLU gate, weighted combine) is written here in numpy fp64
on top of the C linear layer, and so are the decoder-layer producers (RMS
normalisation and the SiLU-gated product written in a consumer's stored column
order).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svqref.cpp")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libsvqref.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library (g++, OpenMP, no contraction)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", _SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_int64
        lib.svqref_h2f.argtypes = [ctypes.c_uint16]
        lib.svqref_h2f.restype = ctypes.c_float
        lib.svqref_bf2f.argtypes = [ctypes.c_uint16]
        lib.svqref_bf2f.restype = ctypes.c_float
        lib.svqref_f2h_rne.argtypes = [ctypes.c_float]
        lib.svqref_f2h_rne.restype = ctypes.c_uint16
        lib.svqref_f2bf_rne.argtypes = [ctypes.c_float]
        lib.svqref_f2bf_rne.restype = ctypes.c_uint16
        for name in ("svqref_f2h_rne_array", "svqref_f2bf_rne_array", "svqref_h2f_array"):
            getattr(lib, name).argtypes = [P, P, i64]
            getattr(lib, name).restype = None
        lib.svqref_row_bytes.argtypes = [i32]
        lib.svqref_row_bytes.restype = i64
        lib.svqref_pack.argtypes = [i32, i32, i32, P, P, P, P]
        lib.svqref_pack.restype = i32
        lib.svqref_unpack.argtypes = [i32, i32, i32, P, P, P, P]
        lib.svqref_unpack.restype = None
        lib.svqref_radius.argtypes = [ctypes.c_uint16, ctypes.c_uint16, ctypes.c_uint32]
        lib.svqref_radius.restype = ctypes.c_float
        lib.svqref_decode_exact.argtypes = [i32, i32, i32, P, P, P, P, P, P]
        lib.svqref_decode_exact.restype = None
        lib.svqref_dequant.argtypes = [i32, i32, i32, P, P, P, P, P, i32, P]
        lib.svqref_dequant.restype = None
        lib.svqref_linear.argtypes = [i32, i32, i32, P, P, P, P, P, P, P, i32, i32, P, P]
        lib.svqref_linear.restype = None
        lib.svqref_encode.argtypes = [i32, i32, i32, P, P, P, P, P, P, P, P, P]
        lib.svqref_encode.restype = None
        lib.svqref_num_threads.argtypes = []
        lib.svqref_num_threads.restype = i32
        lib.svqref_set_threads.argtypes = [i32]
        lib.svqref_set_threads.restype = None
        _lib = lib
        return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------- conversions
def h2f(bits) -> np.ndarray:
    bits = _c(bits, np.uint16).reshape(-1)
    out = np.empty(bits.shape, np.float32)
    _load().svqref_h2f_array(_ptr(bits), _ptr(out), bits.size)
    return out


def f2h_rne(x) -> np.ndarray:
    x = _c(x, np.float32).reshape(-1)
    out = np.empty(x.shape, np.uint16)
    _load().svqref_f2h_rne_array(_ptr(x), _ptr(out), x.size)
    return out


def f2bf_rne(x) -> np.ndarray:
    x = _c(x, np.float32).reshape(-1)
    out = np.empty(x.shape, np.uint16)
    _load().svqref_f2bf_rne_array(_ptr(x), _ptr(out), x.size)
    return out


def bf2f_scalar(b: int) -> float:
    return float(_load().svqref_bf2f(int(b)))


def radius(scale_bits: int, offset_bits: int, code: int) -> float:
    return float(_load().svqref_radius(int(scale_bits), int(offset_bits), int(code)))


# --------------------------------------------------------------------------- format
def row_bytes(K: int) -> int:
    return int(_load().svqref_row_bytes(int(K)))


def pack(N, K, b_d, signs, idx, code) -> np.ndarray:
    signs = _c(signs, np.uint8)
    idx = _c(idx, np.uint16)
    code = _c(code, np.uint16)
    out = np.empty((N, row_bytes(K)), np.uint8)
    rc = _load().svqref_pack(N, K, b_d, _ptr(signs), _ptr(idx), _ptr(code), _ptr(out))
    if rc != 0:
        raise ValueError("field out of range for the bit split")
    return out


def unpack(N, K, b_d, canon):
    canon = _c(canon, np.uint8)
    G = K // 8
    signs = np.empty((N, G), np.uint8)
    idx = np.empty((N, G), np.uint16)
    code = np.empty((N, G), np.uint16)
    _load().svqref_unpack(N, K, b_d, _ptr(canon), _ptr(signs), _ptr(idx), _ptr(code))
    return signs, idx, code


# --------------------------------------------------------------------------- decode
def _radius_arrays(m):
    """(scale, offset, lut) contiguous arrays of an SvqMatrix-like object: a per-row level table when it
    has one (m.lut [N][2^b_r] fp16 bits) and no affine pair, else the affine pair and no table.  The
    caller keeps the arrays alive across the C call."""
    lut = getattr(m, "lut", None)
    if lut is not None:
        lut = _c(lut, np.uint16)
        assert lut.shape == (m.N, 1 << (10 - m.b_d))
        return None, None, lut
    return _c(m.scale, np.uint16), _c(m.offset, np.uint16), None


def _optr(a):
    return None if a is None else _ptr(a)


def decode_exact(m) -> np.ndarray:
    """Exact fp64 weights [N][K] (stored column order) of an SvqMatrix-like object."""
    W = np.empty((m.N, m.K), np.float64)
    sc, of, lt = _radius_arrays(m)
    _load().svqref_decode_exact(m.N, m.K, m.b_d, _ptr(_c(m.canonical, np.uint8)),
                                _ptr(_c(m.codebook, np.uint16)), _optr(sc), _optr(of), _optr(lt), _ptr(W))
    return W


def dequant(m, kind: str = "f16") -> np.ndarray:
    """Bit patterns [N][K] of the exported fp16 ('f16') or bf16 ('bf16') weights."""
    out = np.empty((m.N, m.K), np.uint16)
    sc, of, lt = _radius_arrays(m)
    _load().svqref_dequant(m.N, m.K, m.b_d, _ptr(_c(m.canonical, np.uint8)),
                           _ptr(_c(m.codebook, np.uint16)), _optr(sc), _optr(of), _optr(lt),
                           0 if kind == "f16" else 1, _ptr(out))
    return out


def linear(m, x_bits, x_kind: str = "f16"):
    """y[M][N] = W x[perm] and den[M][N] = |W| |x[perm]|, both fp64.

    x_bits: [M][K] 16-bit patterns (fp16 or bf16 per x_kind)."""
    x_bits = _c(x_bits, np.uint16)
    if x_bits.ndim == 1:
        x_bits = x_bits.reshape(1, -1)
    M = x_bits.shape[0]
    assert x_bits.shape[1] == m.K
    y = np.empty((M, m.N), np.float64)
    den = np.empty((M, m.N), np.float64)
    sc, of, lt = _radius_arrays(m)
    _load().svqref_linear(m.N, m.K, m.b_d, _ptr(_c(m.canonical, np.uint8)),
                          _ptr(_c(m.codebook, np.uint16)), _optr(sc), _optr(of), _optr(lt),
                          _ptr(_c(m.perm, np.int32)),
                          _ptr(x_bits), 0 if x_kind == "f16" else 1, M, _ptr(y), _ptr(den))
    return y, den


def encode(N, K, b_d, W, codebook, scale, offset, energy=None, lut=None):
    """Brute-force nearest-codeword encoder; returns (signs, idx, code) [N][K/8].  The radius levels of
    row n are fma(scale[n], code, offset[n]), or lut[n][code] when a per-row table is given."""
    W = _c(W, np.float64)
    G = K // 8
    signs = np.empty((N, G), np.uint8)
    idx = np.empty((N, G), np.uint16)
    code = np.empty((N, G), np.uint16)
    e = None if energy is None else _c(energy, np.float64)
    lt = None if lut is None else _c(lut, np.uint16)
    _load().svqref_encode(N, K, b_d, _ptr(W), _ptr(_c(codebook, np.uint16)),
                          None if lt is not None else _ptr(_c(scale, np.uint16)),
                          None if lt is not None else _ptr(_c(offset, np.uint16)),
                          None if lt is None else _ptr(lt),
                          None if e is None else _ptr(e), _ptr(signs), _ptr(idx), _ptr(code))
    return signs, idx, code


def num_threads() -> int:
    return int(_load().svqref_num_threads())


def set_threads(n: int) -> None:
    """Threads used by the C++ oracle's parallel loops (timing only; results are independent of it)."""
    _load().svqref_set_threads(int(n))


# --------------------------------------------------------------------------- MoE
def silu(v: np.ndarray) -> np.ndarray:
    v = np.asarray(v, np.float64)
    return v / (1.0 + np.exp(-v))


def moe_ffn(experts, x_bits, topk_ids, topk_w, h_bits=None):
    """Reference MoE feed-forward: for token t,
        out[t] = sum_k w[t,k] * down_e( silu(gate_e x_t) * up_e x_t ),  e = topk_ids[t,k].

    experts: list of (gate, up, down) SvqMatrix-like triples.
    If h_bits ([T][k][I] fp16 bit patterns) is given, the down projection takes
    those activations instead of the oracle's own fp64 h (this isolates the
    down-projection layer from the activation's rounding).
    Returns (gate_y [T,k,I], up_y [T,k,I], out [T,H], out_den [T,H])."""
    x_bits = _c(x_bits, np.uint16)
    T, k = topk_ids.shape
    g0 = experts[0][0]
    inter, hidden = g0.N, experts[0][2].N
    gate_y = np.zeros((T, k, inter))
    up_y = np.zeros((T, k, inter))
    out = np.zeros((T, hidden))
    den = np.zeros((T, hidden))
    for t in range(T):
        for s in range(k):
            e = int(topk_ids[t, s])
            gate, up, down = experts[e]
            gy, _ = linear(gate, x_bits[t:t + 1])
            uy, _ = linear(up, x_bits[t:t + 1])
            gate_y[t, s] = gy[0]
            up_y[t, s] = uy[0]
            if h_bits is None:
                h = silu(gy[0]) * uy[0]
                # The down layer consumes fp16 activations.
                hb = f2h_rne(h.astype(np.float32))
            else:
                hb = _c(h_bits[t, s], np.uint16)
            dy, dden = linear(down, hb.reshape(1, -1))
            out[t] += float(topk_w[t, s]) * dy[0]
            den[t] += abs(float(topk_w[t, s])) * dden[0]
    return gate_y, up_y, out, den


# --------------------------------------------------------------------------- decoder-layer producers
# The pages only say that each subvector multiplies eight reordered
# activations ("SAGE", Figure 6 caption).  A decoder layer can have the kernel
# that produces a linear layer's input write it in that layer's stored column
# order; these are the two producers of a Qwen3-style decoder layer (the models
# the pages evaluate), written out from their definitions.
def f64_to_h_rne(v) -> np.ndarray:
    """binary64 -> binary16 bit patterns, one round-to-nearest-even step (numpy's conversion;
    pinned against the C conversion on binary32 inputs and on double-rounding cases)."""
    with np.errstate(over="ignore"):           # overflow to +-inf is the defined result
        return np.asarray(v, np.float64).astype(np.float16).view(np.uint16)


def act_to_f64(bits, kind: str = "f16") -> np.ndarray:
    """fp16 or bf16 bit patterns -> fp64 (exact)."""
    bits = _c(bits, np.uint16)
    if kind == "f16":
        return h2f(bits).astype(np.float64).reshape(bits.shape)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rmsnorm(h_bits, h_kind, gamma_bits, eps: float) -> np.ndarray:
    """RMS normalisation of each row, fp64 before any rounding:
        x[m][k] = h[m][k] * gamma[k] / sqrt( (1/K) sum_k' h[m][k']^2 + eps )."""
    h = act_to_f64(h_bits, h_kind)
    g = act_to_f64(gamma_bits, "f16")
    ms = np.mean(h * h, axis=1, keepdims=True)
    return h * g / np.sqrt(ms + float(eps))


def rmsnorm_permute(h_bits, h_kind, gamma_bits, eps: float, perms):
    """The normalised rows written for each consumer in its stored column order,
    x_g[m][j] = RNE_fp16(rmsnorm(h)[m][p_g[j]]); p_g None = natural order.
    Returns a list of fp16 bit arrays [M][K]."""
    xn = rmsnorm(h_bits, h_kind, gamma_bits, eps)
    return [f64_to_h_rne(xn if p is None else xn[:, np.asarray(p, np.int64)]) for p in perms]


def swiglu(gate, up) -> np.ndarray:
    """silu(gate) * up in fp64 (gate/up: the fp32 outputs of the gate and up projections)."""
    return silu(np.asarray(gate, np.float64)) * np.asarray(up, np.float64)


def swiglu_permute(gate, up, perm) -> np.ndarray:
    """x[m][j] = RNE_fp16(silu(gate[m][p[j]]) * up[m][p[j]]), p None = natural order (fp16 bits)."""
    a = swiglu(gate, up)
    return f64_to_h_rne(a if perm is None else a[:, np.asarray(perm, np.int64)])
