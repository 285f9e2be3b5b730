"""Shared helpers of the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch

import oracle

Q40, KSB = oracle.FMT_Q4_0, oracle.FMT_KSB


def x_for_oracle(x: torch.Tensor):
    """Activation tensor -> (numpy array, oracle element code)."""
    x = x.detach().cpu().contiguous()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view(np.uint16), oracle.BF16
    if x.dtype == torch.float16:
        return x.numpy(), oracle.F16
    return x.float().numpy(), oracle.F32


def out_ulp(v: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """One unit in the last place of |v| in the output type (0 for fp32)."""
    if dtype == torch.float32:
        return np.zeros_like(v)
    mant = 10 if dtype == torch.float16 else 7
    tiny = 2.0 ** -24 if dtype == torch.float16 else 2.0 ** -133
    e = np.floor(np.log2(np.maximum(np.abs(v), tiny)))
    return np.maximum(2.0 ** (e - mant), tiny)


def assert_product_close(y_gpu: torch.Tensor, Y: np.ndarray, bound: np.ndarray, rel: float = 1e-4):
    """|y - Y| <= rel * sum|w||x| + one ulp of the output type, element by element."""
    y = y_gpu.detach().float().cpu().numpy().astype(np.float64)
    assert y.shape == Y.shape, (y.shape, Y.shape)
    assert np.all(np.isfinite(y))
    err = np.abs(y - Y)
    allow = rel * bound + out_ulp(np.maximum(np.abs(Y), np.abs(y)), y_gpu.dtype)
    bad = err > allow
    if bad.any():
        i = np.unravel_index(np.argmax(err / np.maximum(allow, 1e-300)), err.shape)
        raise AssertionError(
            f"{int(bad.sum())} of {bad.size} outputs out of tolerance; worst at {i}: "
            f"gpu {y[i]!r} ref {Y[i]!r} err {err[i]:.3e} allowed {allow[i]:.3e}")
    return float((err / np.maximum(bound, 1e-300)).max())
