"""Pins of the oracle's per-row quantisation, FP8 linear and NestedFP
functions against invariants, closed forms, library routines and brute force
(CPU only)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic

E4 = oracle.e4m3_table()
E5 = oracle.e5m2_table()


def _half_ulp_e4m3(v):
    """Half the spacing of E4M3 values at magnitude |v| (binary64)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return 0.5 * 2.0 ** (e - 3)


# ------------------------------------------------------------------ quantize
@pytest.mark.parametrize("recipe", ["normal_outl_1pct_x20", "student_t4_unit", "student_t3"])
def test_quantize_invariants(recipe):
    g = np.random.default_rng(11)
    x = synthetic.activations(recipe, 24, 301, g)
    q, s = oracle.quantize_rows(x)
    amax = np.abs(x).max(axis=1)
    # scale is the binary32 quotient amax / 448 (numpy binary32 division as witness)
    np.testing.assert_array_equal(s, (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32))
    for r in range(x.shape[0]):
        k = int(np.argmax(np.abs(x[r])))
        assert q[r, k] & 0x7F == 0x7E, "the amax element must land on 448"
        deq = E4[q[r]] * float(s[r])
        err = np.abs(deq - x[r].astype(np.float64))
        bound = _half_ulp_e4m3(x[r].astype(np.float64) / float(s[r])) * float(s[r])
        assert np.all(err <= bound * (1 + 1e-6) + 1e-30)
        # sign is kept for every element, including those that round to zero
        np.testing.assert_array_equal(q[r] >> 7, np.signbit(x[r]).astype(np.uint8))


def test_quantize_matches_library_cast_of_scaled_values():
    """Codes equal torch's float32 division followed by its float8_e4m3fn cast
    (in range, since |x / s| <= 448 up to rounding of the division)."""
    g = np.random.default_rng(3)
    x = synthetic.activations("normal_outl_0p5pct_x30", 9, 1000, g)
    q, s = oracle.quantize_rows(x)
    xt = torch.from_numpy(x)
    scaled = xt / torch.from_numpy(s)[:, None]
    assert float(scaled.abs().max()) <= 448.0 * (1 + 2 ** -20)
    lib = scaled.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(q, lib)


def test_quantize_power_of_two_scale_invariance():
    g = np.random.default_rng(5)
    x = synthetic.activations("student_t3", 6, 257, g)
    q1, s1 = oracle.quantize_rows(x)
    for p in (-20, -3, 1, 7):
        q2, s2 = oracle.quantize_rows((x * np.float32(2.0 ** p)).astype(np.float32))
        np.testing.assert_array_equal(q1, q2)
        np.testing.assert_array_equal(s2, (s1 * np.float32(2.0 ** p)).astype(np.float32))


def test_quantize_zero_row_and_signed_zero():
    x = np.zeros((3, 16), dtype=np.float32)
    x[1, 3] = -0.0
    x[2] = -0.0
    q, s = oracle.quantize_rows(x)
    np.testing.assert_array_equal(s, np.ones(3, dtype=np.float32))
    assert q[0].tolist() == [0] * 16
    assert q[1, 3] == 0x80 and q[1, 2] == 0x00
    assert q[2].tolist() == [0x80] * 16


def test_quantize_static_mode_saturates():
    x = np.array([[1.0, -1.0, 900.0, -2000.0, 448.0, 0.001]], dtype=np.float32)
    q, s = oracle.quantize_rows(x, scales=np.array([1.0], dtype=np.float32))
    assert s[0] == 1.0
    assert q[0].tolist() == [0x38, 0xB8, 0x7E, 0xFE, 0x7E, oracle.e4m3_encode(0.001)]
    assert oracle.e4m3_encode(0.001) == 0x00 + round(0.001 * 512)  # subnormal grid


def test_quantize_rejects_nonfinite():
    x = np.ones((2, 4), dtype=np.float32)
    x[1, 2] = np.inf
    with pytest.raises(oracle.OracleError):
        oracle.quantize_rows(x)


def test_quantize_f16_equals_f32_of_widened_values():
    g = np.random.default_rng(9)
    x16 = synthetic.activations("normal_f16", 5, 129, g)
    q16, s16 = oracle.quantize_rows(x16)
    q32, s32 = oracle.quantize_rows(x16.astype(np.float32))
    np.testing.assert_array_equal(q16, q32)
    np.testing.assert_array_equal(s16, s32)


# ------------------------------------------------------------------ FP8 linear
def _rand_codes(g, shape):
    c = g.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38          # no NaN codes
    return c


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 5, 7), (16, 9, 64), (7, 33, 40)])
def test_fp8_linear_brute_force_vs_numpy(M, N, K):
    g = np.random.default_rng(M * 100 + N)
    aq, wq = _rand_codes(g, (M, K)), _rand_codes(g, (N, K))
    sa = g.uniform(0.01, 2.0, M).astype(np.float32)
    sw = g.uniform(0.001, 0.1, N).astype(np.float32)
    ref = oracle.fp8_linear(aq, sa, wq, sw)
    lib = (E4[aq] @ E4[wq].T) * sa.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :]
    np.testing.assert_allclose(ref, lib, rtol=1e-13, atol=0)


def test_fp8_linear_one_hot_weights_reproduce_dequantised_activations():
    g = np.random.default_rng(2)
    M, K = 4, 48
    aq = _rand_codes(g, (M, K))
    sa = np.array([0.5, 2.0, 0.125, 1.0], dtype=np.float32)
    wq = np.zeros((K, K), dtype=np.uint8)
    wq[np.arange(K), np.arange(K)] = 0x38      # identity in E4M3 (1.0)
    sw = np.ones(K, dtype=np.float32)
    ref = oracle.fp8_linear(aq, sa, wq, sw)
    np.testing.assert_array_equal(ref, E4[aq] * sa.astype(np.float64)[:, None])


def test_fp8_linear_permuted_one_hot_checks_index_roles():
    """W = a permutation: ref[m, n] picks A[m, perm[n]], scaled by sw[n]."""
    g = np.random.default_rng(4)
    M, K = 3, 20
    aq = _rand_codes(g, (M, K))
    perm = g.permutation(K)
    wq = np.zeros((K, K), dtype=np.uint8)
    wq[np.arange(K), perm] = 0x40               # 2.0
    sa = np.float32([1.0, 0.25, 4.0])
    sw = (2.0 ** g.integers(-4, 4, K)).astype(np.float32)
    ref = oracle.fp8_linear(aq, sa, wq, sw)
    expect = E4[aq][:, perm] * 2.0 * sa[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    np.testing.assert_array_equal(ref, expect)


# ------------------------------------------------------------------ NestedFP
def test_nestedfp_split_rebuild_all_65536_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    hi, lo = oracle.nestedfp_split(bits)
    rebuilt = (hi.astype(np.uint16) << 8) | lo.astype(np.uint16)
    np.testing.assert_array_equal(rebuilt, bits)
    for b in (0x0000, 0x3C00, 0x7BFF, 0x8001, 0xFC00, 0x7E00, 0x1234, 0xABCD):
        assert oracle.nestedfp_rebuild(b >> 8, b & 0xFF) == b


def test_upper_byte_is_e5m2_of_truncated_fp16():
    """For every binary16 pattern except NaNs whose payload sits only in the low
    byte, decoding the upper byte as E5M2 equals the binary16 value with its
    low 8 bits cleared (numpy's float16 decode as witness)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    hi, _ = oracle.nestedfp_split(bits)
    trunc = (bits & 0xFF00).view(np.float16).astype(np.float64)
    e5 = E5[hi]
    low_only_nan = ((bits & 0x7C00) == 0x7C00) & ((bits & 0x0300) == 0) & ((bits & 0x00FF) != 0)
    keep = ~low_only_nan
    np.testing.assert_array_equal(np.isnan(e5[keep]), np.isnan(trunc[keep]))
    fin = keep & ~np.isnan(trunc)
    np.testing.assert_array_equal(e5[fin], trunc[fin])
    assert low_only_nan.sum() == 2 * 255


@pytest.mark.parametrize("M,N,K", [(1, 3, 8), (5, 7, 33), (16, 12, 64)])
def test_nestedfp_fp16_linear_vs_numpy(M, N, K):
    g = np.random.default_rng(K)
    x16 = synthetic.activations("normal_f16", M, K, g)
    w16 = synthetic.weights_f16(N, K, 0.02, g)
    hi, lo = oracle.nestedfp_split(w16)
    ref = oracle.nestedfp_linear_fp16(x16, hi, lo)
    lib = x16.astype(np.float64) @ w16.astype(np.float64).T
    np.testing.assert_allclose(ref, lib, rtol=1e-13, atol=1e-300)


@pytest.mark.parametrize("M,N,K", [(1, 3, 8), (5, 7, 33), (16, 12, 64)])
def test_nestedfp_fp8_linear_vs_numpy(M, N, K):
    g = np.random.default_rng(K + 1)
    x16 = synthetic.activations("normal_f16", M, K, g)
    w16 = synthetic.weights_f16(N, K, 0.02, g)
    hi, _ = oracle.nestedfp_split(w16)
    ref, aq, sa = oracle.nestedfp_linear_fp8(x16, hi)
    q2, s2 = oracle.quantize_rows(x16)
    np.testing.assert_array_equal(aq, q2)
    np.testing.assert_array_equal(sa, s2)
    wtrunc = (w16.view(np.uint16) & 0xFF00).view(np.float16).astype(np.float64)
    lib = (E4[aq] * sa.astype(np.float64)[:, None]) @ wtrunc.T
    np.testing.assert_allclose(ref, lib, rtol=1e-12, atol=1e-300)


def test_fp8_linear_full_pipeline_error_vs_exact_product():
    """End-to-end property: quantise x and w with the oracle, contract, and the
    result approximates the exact fp64 product of the unquantised operands to
    within the two E4M3 rounding errors (relative 2^-4 each per element)."""
    g = np.random.default_rng(8)
    x = synthetic.activations("normal_outl_1pct_x20", 8, 256, g)
    w = synthetic.weights_f16(32, 256, 0.02, g)
    aq, sa = oracle.quantize_rows(x)
    wq, sw = oracle.quantize_rows(w)
    ref = oracle.fp8_linear(aq, sa, wq, sw)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    bound = (np.abs(x).astype(np.float64) @ np.abs(w).astype(np.float64).T) * (2 * 2.0 ** -4 + 2.0 ** -8) \
        + 256 * (2.0 ** -10) * (sa[:, None] * np.abs(w).max() + sw[None, :] * np.abs(x).max())
    assert np.all(np.abs(ref - exact) <= bound)
    assert math.isfinite(float(np.abs(ref).max()))
