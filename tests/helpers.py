"""Shared test helpers: moving seeded inputs around and the acceptance check.

The acceptance rule for floating-point outputs: every element is finite and
|y - y_ref| <= 2e-3 * sum_k |x_k * w_k| + 1e-5, with y_ref and the bound from
the fp64 oracle.  Integer / byte outputs must match exactly.
"""
import numpy as np
import torch

RTOL = 2e-3
ATOL = 1e-5


def np_inputs(x, codes, scales):
    """torch CPU tensors -> numpy arrays the oracle takes (fp16 as uint16 bits)."""
    return (x.contiguous().view(torch.int16).numpy().view(np.uint16),
            codes.contiguous().numpy(),
            scales.contiguous().view(torch.int16).numpy().view(np.uint16))


def f16_to_f64(t):
    return t.detach().float().cpu().double().numpy()


def check_close(y_gpu, y_ref, bound, what=""):
    y = f16_to_f64(y_gpu).reshape(np.shape(y_ref))
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    err = np.abs(y - y_ref)
    tol = RTOL * bound + ATOL
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; "
                             f"worst at {i}: got {y[i]!r} want {y_ref[i]!r} bound {bound[i]!r}")
    return float((err / tol).max()) if err.size else 0.0
