"""Helpers for the GPU tests: move the generator's bit patterns to the device."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def dev_bits(bits: np.ndarray, dtype=None):
    """uint16 patterns -> CUDA tensor (int16 view, or bf16/f16 when dtype is given)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t if dtype is None else t.view(dtype)


def padded(rows: int, cols: int, ld: int, dtype, fill):
    """A [rows, ld] buffer filled with `fill`; the [:, :cols] view is the operand."""
    buf = torch.full((rows, ld), fill, dtype=dtype, device="cuda")
    return buf, buf[:, :cols]


def host(t) -> np.ndarray:
    torch.cuda.synchronize()
    return t.detach().cpu().numpy()
