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


def e4m3_half_step(t: np.ndarray) -> np.ndarray:
    """Half the spacing of E4M3 values around |t| (subnormal spacing 2^-9,
    normal 2^(e-3) in the binade [2^e, 2^(e+1)), e >= -6)."""
    a = np.abs(t)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return 0.5 * np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (e - 3))


def assert_valid_codes(q: np.ndarray, s: np.ndarray, y64: np.ndarray, what: str, min_exact: float = 0.995):
    """Codes q [R,C] with scales s [R] are a valid per-token E4M3
    quantisation of the binary64 values y64 (which the kernel evaluates in
    binary32, in its own order): the scale agrees with fl32(amax / 448) of
    y64 to 2^-18 relative; every code decodes to a nearest E4M3 value of
    t = y64 / s, or to the other neighbour where t lies within
    2^-14 |t| + 2^-12 of a rounding midpoint (the binary32 evaluation error,
    relative and, after LayerNorm's mean subtraction, absolute; a quarter of
    the smallest half step at most), saturating beyond 448; and at least
    min_exact of the codes equal the encoding of fl32(t)."""
    s = s.astype(np.float64)
    amax = np.abs(y64).max(axis=1)
    s_ref = (amax.astype(np.float32) / np.float32(448.0)).astype(np.float64)
    s_ref[s_ref == 0] = 1.0
    rel = np.abs(s / s_ref - 1.0)
    assert rel.max() <= 2.0 ** -18, f"{what}: scale off by {rel.max():.3e} relative"
    t = y64 / s[:, None]
    d = E4[q]
    sat = np.abs(t) > 448.0
    assert np.all(np.abs(d[sat]) == 448.0) and np.all(np.sign(d[sat]) == np.sign(t[sat])), f"{what}: saturation"
    ok = np.abs(d - t) <= e4m3_half_step(t) + 2.0 ** -14 * np.abs(t) + 2.0 ** -12
    ok |= sat
    assert ok.all(), (f"{what}: {int((~ok).sum())} codes are not a nearest E4M3 value; first at "
                      f"{tuple(np.argwhere(~ok)[0])}")
    ref = oracle.e4m3_encode_array(t.astype(np.float32))
    exact = float((ref == q).mean())
    assert exact >= min_exact, f"{what}: only {exact:.4f} of the codes equal the oracle's"
    return exact
