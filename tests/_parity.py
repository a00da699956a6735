"""Shared helpers of the GPU parity tests: the error bound of the layer's
outputs and small marshalling utilities (no arithmetic of the method)."""
import numpy as np

import oracle

E4 = oracle.e4m3_table()
E5 = oracle.e5m2_table()


def linear_bound(ref: np.ndarray, K: int, a_hat: np.ndarray, w_hat: np.ndarray) -> np.ndarray:
    """The layer's stated tolerance on an FP32-accumulated, 16-bit-rounded
    output:  |y - ref| <= 2^-8 |ref| + 1e-4 sqrt(K) * A_m * W_n,
    with A_m = max_k |a[m,k]| and W_n = max_k |w[n,k]| taken over the
    (dequantised) operands of row m and column n."""
    return 2.0 ** -8 * np.abs(ref) + 1e-4 * np.sqrt(K) * a_hat[:, None] * w_hat[None, :]


def fp8_row_max(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """max_k |dec_e4m3(code[r,k]) * scale[r]| per row."""
    return np.abs(E4[codes]).max(axis=1) * scales.astype(np.float64)


def assert_within(y: np.ndarray, ref: np.ndarray, bound: np.ndarray, what: str):
    y = y.astype(np.float64)
    assert np.all(np.isfinite(y)), f"{what}: non-finite outputs"
    err = np.abs(y - ref)
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside the bound; first at {tuple(i)}: "
                             f"y={y[tuple(i)]!r} ref={ref[tuple(i)]!r} err={err[tuple(i)]:.3e} "
                             f"bound={bound[tuple(i)]:.3e}")
    return float((err / np.maximum(bound, 1e-300)).max())
