"""Python binding of libsvq (include/svq.h): argument marshalling only.

Every entry point takes torch CUDA tensors (device memory) and the current
torch stream, passes raw pointers to the C ABI and raises SvqError on a
non-zero status.  All computation happens in the CUDA kernels of libsvq.so;
there is no CPU or PyTorch fallback.  If the library is missing the import of
the binding functions fails loudly (call ``compile_library()`` or
``python -m bit_spherical_vector_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "lib", "libsvq.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "svq.h")

SVQ_OK, SVQ_ERR_INVALID_ARG, SVQ_ERR_UNSUPPORTED_SHAPE, SVQ_ERR_WORKSPACE, SVQ_ERR_CUDA, SVQ_ERR_TIMEOUT = range(6)
SVQ_F16, SVQ_BF16, SVQ_F32 = 1, 2, 3


class SvqError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: status {status} ({status_string(status)})")
        self.status = status


class svq_matrix(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("b_d", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("packed", ctypes.c_void_p), ("codebook", ctypes.c_void_p),
                ("radius_scale", ctypes.c_void_p), ("radius_offset", ctypes.c_void_p),
                ("perm", ctypes.c_void_p), ("radius_lut", ctypes.c_void_p)]


_lib = None


def compile_library(force: bool = False) -> str:
    """Compile libsvq.so in-tree (see bit_spherical_vector_b200/build.py)."""
    import importlib
    return importlib.import_module(__name__ + ".build").build(force=force)


def lib():
    """The loaded libsvq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libsvq.so not found at {LIB_PATH}; build it with "
                          "`python -m bit_spherical_vector_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    MP = ctypes.POINTER(svq_matrix)
    sig = {
        "svq_status_string": ([I], ctypes.c_char_p),
        "svq_version": ([], I),
        "svq_packed_bytes": ([I, I], SZ),
        "svq_canonical_bytes": ([I, I], SZ),
        "svq_repack": ([P, I, I, I, P, P], I),
        "svq_unpack_fields": ([P, I, I, I, P, P, P, P], I),
        "svq_dequantize": ([MP, I, P, P], I),
        "svq_linear_gemv_workspace_size": ([MP, I, ctypes.POINTER(SZ)], I),
        "svq_workspace_init": ([P, SZ, P], I),
        "svq_linear_gemv": ([MP, P, I, P, I, P, SZ, P], I),
        "svq_linear_gemv_batched_workspace_size": ([MP, I, I, ctypes.POINTER(SZ)], I),
        "svq_linear_gemv_batched": ([MP, I, ctypes.POINTER(P), I, ctypes.POINTER(P), I, P, SZ, P], I),
        "svq_linear_gemv_batched_host": ([MP, I, P, P, I, P, P, I, P, SZ, P], I),
        "svq_linear_gemv_noalloc": ([MP, P, I, P, I, P], I),
        "svq_linear_gemm_workspace_size": ([MP, I, ctypes.POINTER(SZ)], I),
        "svq_linear_gemm": ([MP, P, I, I, P, I, P, SZ, P], I),
        "svq_moe_grouped_gemv_workspace_size": ([I, I, I, I, ctypes.POINTER(SZ)], I),
        "svq_debug_set_wait_polls": ([ctypes.c_uint], ctypes.c_uint),
        "svq_moe_grouped_gemv": ([P, I, I, I, I, P, I, I, P, I, I, P, I, I, P, SZ, P], I),
        "svq_rmsnorm_permute": ([P, I, P, ctypes.c_float, I, I, ctypes.POINTER(P), ctypes.POINTER(P), I, P], I),
        "svq_swiglu_permute": ([P, P, I, I, P, P, P], I),
        "svq_get_device_status": ([P], I),
        "svq_esg": ([P, I, I, ctypes.c_double, P, P, P, P], I),
        "svq_radius_grid": ([P, I, I, P, I, P, P, P], I),
        "svq_encode": ([P, I, I, I, P, P, P, P, P, P, P, P, P], I),
        "svq_abs_select": ([P, I, I, P, P, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def status_string(status: int) -> str:
    try:
        return lib().svq_status_string(int(status)).decode()
    except ImportError:
        return "library not loaded"


def _check(status: int, what: str):
    if status != SVQ_OK:
        raise SvqError(status, what)


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _dtype_code(dtype) -> int:
    import torch
    return {torch.float16: SVQ_F16, torch.bfloat16: SVQ_BF16, torch.float32: SVQ_F32}[dtype]


# ----------------------------------------------------------------------------- format
def svq_packed_bytes(N: int, K: int) -> int:
    return int(lib().svq_packed_bytes(N, K))


def svq_canonical_bytes(N: int, K: int) -> int:
    return int(lib().svq_canonical_bytes(N, K))


def svq_repack(canonical, N: int, K: int, b_d: int, packed_out, stream=None):
    _check(lib().svq_repack(_ptr(canonical), N, K, b_d, _ptr(packed_out), _stream(stream)), "svq_repack")


def svq_unpack_fields(packed, N: int, K: int, b_d: int, signs, idx, code, stream=None):
    _check(lib().svq_unpack_fields(_ptr(packed), N, K, b_d, _ptr(signs), _ptr(idx), _ptr(code),
                                   _stream(stream)), "svq_unpack_fields")


class SvqWeight:
    """Device-resident SVQ matrix (packed codes, codebook, radius params, perm, optional per-row radius
    table) and its C descriptor.  Built from canonical host arrays by ``from_canonical``.  ``perm``
    None means x is supplied already in the stored column order; ``lut`` (fp16 [N][2^b_r]) replaces the
    affine radius when given."""

    def __init__(self, N, K, b_d, packed, codebook, scale, offset, perm, lut=None):
        self.N, self.K, self.b_d = N, K, b_d
        self.packed, self.codebook, self.scale, self.offset, self.perm = packed, codebook, scale, offset, perm
        self.lut = lut
        ptr = lambda t: 0 if t is None else t.data_ptr()
        self.desc = svq_matrix(N, K, b_d, 0, packed.data_ptr(), codebook.data_ptr(), ptr(scale), ptr(offset),
                               ptr(perm), ptr(lut))

    def without_perm(self):
        """The same device arrays with perm NULL: its calls take x in stored column order."""
        return SvqWeight(self.N, self.K, self.b_d, self.packed, self.codebook, self.scale, self.offset, None,
                         self.lut)

    @classmethod
    def from_canonical(cls, N, K, b_d, canonical, codebook, scale, offset, perm, device="cuda", stream=None,
                       lut=None):
        """canonical/codebook/scale/offset/perm/lut: numpy arrays (uint8 / uint16 bit patterns / int32)."""
        import numpy as np
        import torch
        dev = torch.device(device)
        canon_d = torch.from_numpy(np.ascontiguousarray(canonical, np.uint8)).to(dev)
        packed = torch.empty(svq_packed_bytes(N, K), dtype=torch.uint8, device=dev)
        svq_repack(canon_d, N, K, b_d, packed, stream)
        to16 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).to(dev)
        w = cls(N, K, b_d, packed, to16(codebook), to16(scale), to16(offset),
                torch.from_numpy(np.ascontiguousarray(perm, np.int32)).to(dev),
                None if lut is None else to16(lut))
        w._canon_d = canon_d   # keep alive until the repack has run
        return w

    @classmethod
    def from_synth(cls, m, device="cuda", stream=None):
        return cls.from_canonical(m.N, m.K, m.b_d, m.canonical, m.codebook, m.scale, m.offset, m.perm,
                                  device, stream, getattr(m, "lut", None))


def svq_dequantize(W: SvqWeight, out, stream=None):
    _check(lib().svq_dequantize(ctypes.byref(W.desc), _dtype_code(out.dtype), _ptr(out), _stream(stream)),
           "svq_dequantize")


def svq_linear_gemv_workspace_size(W: SvqWeight, M: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().svq_linear_gemv_workspace_size(ctypes.byref(W.desc), M, ctypes.byref(n)),
           "svq_linear_gemv_workspace_size")
    return int(n.value)


def svq_linear_gemv_batched_workspace_size(Ws, M: int) -> int:
    arr = (svq_matrix * len(Ws))(*[w.desc for w in Ws])
    n = ctypes.c_size_t(0)
    _check(lib().svq_linear_gemv_batched_workspace_size(arr, len(Ws), M, ctypes.byref(n)),
           "svq_linear_gemv_batched_workspace_size")
    return int(n.value)


def svq_workspace_init(ws, stream=None):
    if ws is None or ws.numel() == 0:
        return
    _check(lib().svq_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "svq_workspace_init")


def svq_linear_gemv(W: SvqWeight, x, y, ws=None, stream=None):
    """y[M][N] = W x[M][K]^T with x fp16; y fp16 or fp32."""
    M = x.shape[0]
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().svq_linear_gemv(ctypes.byref(W.desc), _ptr(x), M, _ptr(y), _dtype_code(y.dtype), _ptr(ws), nb,
                                 _stream(stream)), "svq_linear_gemv")


def svq_linear_gemv_batched(Ws, xs, ys, ws=None, stream=None):
    n = len(Ws)
    arr = (svq_matrix * n)(*[w.desc for w in Ws])
    xp = (ctypes.c_void_p * n)(*[x.data_ptr() for x in xs])
    yp = (ctypes.c_void_p * n)(*[y.data_ptr() for y in ys])
    M = xs[0].shape[0]
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().svq_linear_gemv_batched(arr, n, xp, M, yp, _dtype_code(ys[0].dtype), _ptr(ws), nb,
                                         _stream(stream)), "svq_linear_gemv_batched")


class GemvBatchCall:
    """svq_linear_gemv_batched with its arguments marshalled once, for loops that call
    the same layers on the same buffers (one decode step after another)."""

    def __init__(self, Ws, xs, ys, ws=None):
        n = len(Ws)
        self._keep = (list(Ws), list(xs), list(ys), ws)           # the buffers must outlive the calls
        self._args = ((svq_matrix * n)(*[w.desc for w in Ws]), n,
                      (ctypes.c_void_p * n)(*[x.data_ptr() for x in xs]), xs[0].shape[0],
                      (ctypes.c_void_p * n)(*[y.data_ptr() for y in ys]), _dtype_code(ys[0].dtype), _ptr(ws),
                      0 if ws is None else ws.numel() * ws.element_size())
        self._fn = lib().svq_linear_gemv_batched

    def __call__(self, stream=None):
        _check(self._fn(*self._args, _stream(stream)), "svq_linear_gemv_batched")


class GemvBatchHostCall:
    """svq_linear_gemv_batched_host with its arguments marshalled once: each call copies the step's
    inputs x_host (pinned, the inputs back to back) into x_dev, runs the grouped launch and copies
    y_dev (the outputs back to back) into y_host (pinned), all enqueued on the stream."""

    def __init__(self, Ws, M, x_host, x_dev, y_host, y_dev, ws=None):
        n = len(Ws)
        self._keep = (list(Ws), x_host, x_dev, y_host, y_dev, ws)  # the buffers must outlive the calls
        self._args = ((svq_matrix * n)(*[w.desc for w in Ws]), n, _ptr(x_host), _ptr(x_dev), M,
                      _ptr(y_host), _ptr(y_dev), _dtype_code(y_dev.dtype), _ptr(ws),
                      0 if ws is None else ws.numel() * ws.element_size())
        self._fn = lib().svq_linear_gemv_batched_host

    def __call__(self, stream=None):
        _check(self._fn(*self._args, _stream(stream)), "svq_linear_gemv_batched_host")


def svq_linear_gemv_noalloc(W: SvqWeight, x, y, stream=None):
    """svq_linear_gemv with the library's fixed internal scratch (no workspace argument)."""
    M = x.shape[0]
    _check(lib().svq_linear_gemv_noalloc(ctypes.byref(W.desc), _ptr(x), M, _ptr(y), _dtype_code(y.dtype),
                                         _stream(stream)), "svq_linear_gemv_noalloc")


def svq_linear_gemm_workspace_size(W: SvqWeight, M: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().svq_linear_gemm_workspace_size(ctypes.byref(W.desc), M, ctypes.byref(n)),
           "svq_linear_gemm_workspace_size")
    return int(n.value)


def svq_linear_gemm(W: SvqWeight, x, y, ws, stream=None):
    """y[M][N] = W x[M][K]^T on the tensor cores; x bf16 or fp16, y fp32 or bf16."""
    M = x.shape[0]
    nb = ws.numel() * ws.element_size()
    _check(lib().svq_linear_gemm(ctypes.byref(W.desc), _ptr(x), _dtype_code(x.dtype), M, _ptr(y),
                                 _dtype_code(y.dtype), _ptr(ws), nb, _stream(stream)), "svq_linear_gemm")


class svq_group_item(ctypes.Structure):
    _fields_ = [("matrix", ctypes.c_int32), ("x_row", ctypes.c_int32), ("out_row", ctypes.c_int32),
                ("out_scale", ctypes.c_float)]


SVQ_X_F16, SVQ_X_SWIGLU_F32 = 0, 1


def descriptor_table(Ws, device="cuda"):
    """Device array of svq_matrix descriptors (the layout the MoE kernel reads)."""
    import numpy as np
    import torch
    arr = (svq_matrix * len(Ws))(*[w.desc for w in Ws])
    raw = np.frombuffer(bytes(arr), dtype=np.uint8).copy()
    return torch.from_numpy(raw).to(device)


def item_table(matrix, x_row, out_row, out_scale):
    """Device array of svq_group_item from four equal-length device tensors (int32, int32, int32, float32)."""
    import torch
    t = torch.stack([matrix.to(torch.int32), x_row.to(torch.int32), out_row.to(torch.int32),
                     out_scale.to(torch.float32).view(torch.int32)], dim=1).contiguous()
    return t


def svq_moe_grouped_gemv_workspace_size(n_mats: int, n_items: int, N: int, accumulate: bool) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().svq_moe_grouped_gemv_workspace_size(n_mats, n_items, N, int(accumulate), ctypes.byref(n)),
           "svq_moe_grouped_gemv_workspace_size")
    return int(n.value)


def svq_moe_grouped_gemv(mats_dev, n_mats, N, K, max_b_d, items_dev, n_items, max_items_per_matrix, x, x_mode,
                         y, n_out_rows, accumulate, ws, stream=None):
    n_x_rows = int(x.shape[0])                 # items' x_row must lie below (checked on the device)
    _check(lib().svq_moe_grouped_gemv(_ptr(mats_dev), n_mats, N, K, max_b_d, _ptr(items_dev), n_items,
                                      max_items_per_matrix, _ptr(x), x_mode, n_x_rows, _ptr(y), n_out_rows,
                                      int(accumulate), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "svq_moe_grouped_gemv")


# ----------------------------------------------------------------------------- decoder-layer producers
def svq_rmsnorm_permute(h, gamma, eps: float, perms, outs, stream=None):
    """outs[g][m][j] = fp16(rmsnorm(h)[m][perms[g][j]]) (perms[g] None: natural order).
    h: [M][K] fp16/bf16, gamma: fp16 [K], outs: list of fp16 [M][K]."""
    n = len(outs)
    M, K = h.shape
    pp = (ctypes.c_void_p * n)(*[0 if p is None else p.data_ptr() for p in perms])
    op = (ctypes.c_void_p * n)(*[o.data_ptr() for o in outs])
    _check(lib().svq_rmsnorm_permute(_ptr(h), _dtype_code(h.dtype), _ptr(gamma), float(eps), M, K, pp, op, n,
                                     _stream(stream)), "svq_rmsnorm_permute")


def svq_swiglu_permute(gate, up, perm, x, stream=None):
    """x[m][j] = fp16(silu(gate[m][s]) * up[m][s]), s = perm[j] (perm None: s = j); gate/up fp32 [M][I]."""
    M, I = gate.shape
    _check(lib().svq_swiglu_permute(_ptr(gate), _ptr(up), M, I, _ptr(perm), _ptr(x), _stream(stream)),
           "svq_swiglu_permute")


# ------------------------------------------------------------------ calibration (ESG, radius grid, encoder, ABS)
def svq_esg(x_cal, gamma, energy, perm, weights=None, stream=None):
    """Channel energies (fp64 [K]), the ESG permutation (int32 [K]) and fitting weights e^gamma (fp32 [K] or None)
    from calibration activations x_cal (fp32 [T][K])."""
    T, K = x_cal.shape
    _check(lib().svq_esg(_ptr(x_cal), T, K, float(gamma), _ptr(energy), _ptr(perm), _ptr(weights), _stream(stream)),
           "svq_esg")


def svq_radius_grid(W, perm, b_d, scale, offset, stream=None):
    """Per-row uniform radius grid (fp16 bit patterns scale/offset [N], as int16/uint16 tensors) of W (fp32 [N][K])."""
    N, K = W.shape
    _check(lib().svq_radius_grid(_ptr(W), N, K, _ptr(perm), int(b_d), _ptr(scale), _ptr(offset), _stream(stream)),
           "svq_radius_grid")


def svq_encode(W, b_d, perm, weights, codebook, scale, offset, canonical, row_err=None, stream=None, lut=None):
    """Activation-weighted SVQ encoding of W (fp32 [N][K], natural column order) into the canonical stream
    (uint8 [N][row_bytes]); row_err (fp64 [N]) receives each row's weighted reconstruction error.  lut
    (fp16 [N][2^b_r]) gives per-row radius levels in place of scale/offset."""
    N, K = W.shape
    _check(lib().svq_encode(_ptr(W), N, K, int(b_d), _ptr(perm), _ptr(weights), _ptr(codebook), _ptr(scale),
                            _ptr(offset), _ptr(lut), _ptr(canonical), _ptr(row_err), _stream(stream)), "svq_encode")


def svq_abs_select(row_err, totals, best, stream=None):
    """ABS: totals[k] = sum of row_err[k] (fp64 [n_cand][N]) and best[0] = the first least total (int32)."""
    n_cand, N = row_err.shape
    _check(lib().svq_abs_select(_ptr(row_err), n_cand, N, _ptr(totals), _ptr(best), _stream(stream)),
           "svq_abs_select")


def svq_get_device_status(stream=None) -> int:
    return int(lib().svq_get_device_status(_stream(stream)))


def svq_debug_set_wait_polls(polls: int) -> int:
    """Poll bound of the GEMM's bounded waits for later launches (tests); returns the previous bound."""
    return int(lib().svq_debug_set_wait_polls(int(polls)))


def header_functions() -> list[str]:
    """Names of the functions declared in include/svq.h."""
    import re
    with open(HEADER) as f:
        src = f.read()
    return sorted(set(re.findall(r"SVQ_API\s+[\w\s\*]+?\b(svq_\w+)\s*\(", src)))
