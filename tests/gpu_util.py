"""Helpers shared by the GPU tests (device transfers and the error metric)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def to_dev_u16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).cuda()


def x_f16(bits):
    return to_dev_u16(bits).view(torch.float16)


def x_bf16(bits):
    return to_dev_u16(bits).view(torch.bfloat16)


def u16(t) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def rel_err(y, y_ref, den):
    """max over entries of |y - y_ref| / den, where den = sum_j |W[n][j]| |x[m][perm[j]]|."""
    y = np.asarray(y, np.float64)
    d = np.where(den > 0, den, 1.0)
    r = np.abs(y - y_ref) / d
    r = np.where(den > 0, r, np.where(np.abs(y) <= 1e-30, 0.0, np.inf))
    return float(r.max())
