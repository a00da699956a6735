"""Pins of the oracle's normalisation and gated activation (the steps fused
ahead of the activation quantisation: LayerNorm with the QKV projection's
input, "7B on an RTX 4060 with FP8" computation-graph §2.1; the SiLU gate
ahead of the down projection).  Closed forms and invariants of the textbook
definitions: LayerNorm y = (x - mean)/sqrt(var + eps)*gamma + beta with the
biased variance; RMSNorm y = x/sqrt(mean(x^2) + eps)*gamma; h = g/(1 +
exp(-g))*u."""
import math

import numpy as np

import oracle

F32 = np.float32


def test_rmsnorm_closed_forms():
    one = np.ones(8, F32)
    y = oracle.norm_rows(np.array([[3.0] * 8, [-2.0] * 8, [1, -1] * 4], F32), one, None, 0.0)
    np.testing.assert_array_equal(y, [[1.0] * 8, [-1.0] * 8, [1, -1] * 4])
    # with eps: c / sqrt(c^2 + eps)
    y = oracle.norm_rows(np.array([[2.0] * 4], F32), np.ones(4, F32), None, 5.0)
    assert np.allclose(y, 2.0 / 3.0, rtol=0, atol=1e-15)
    # no mean subtraction: [5,7,5,7] -> x / sqrt(37)
    y = oracle.norm_rows(np.array([[5, 7, 5, 7]], F32), np.ones(4, F32), None, 0.0)
    assert np.allclose(y, np.array([5, 7, 5, 7]) / math.sqrt(37.0), rtol=1e-15)


def test_rmsnorm_invariants():
    g = np.random.default_rng(1)
    x = g.standard_normal((5, 96)).astype(F32)
    gamma = g.uniform(0.5, 2, 96).astype(F32)
    y1 = oracle.norm_rows(x, np.ones(96, F32), None, 0.0)
    assert np.allclose((y1 ** 2).mean(axis=1), 1.0, rtol=1e-12)                 # unit RMS
    assert np.allclose(oracle.norm_rows(x * F32(8), np.ones(96, F32), None, 0.0), y1, rtol=1e-12)   # scale-free
    assert np.allclose(oracle.norm_rows(x, gamma, None, 0.0), y1 * gamma.astype(np.float64), rtol=1e-12)
    assert np.all(np.sign(y1) == np.sign(x))


def test_layernorm_closed_forms_and_invariants():
    # two alternating values: mean midway, biased variance ((a-b)/2)^2 -> +-1
    y = oracle.norm_rows(np.array([[5, 7, 5, 7]], F32), np.ones(4, F32), np.zeros(4, F32), 0.0)
    np.testing.assert_array_equal(y, [[-1, 1, -1, 1]])
    g = np.random.default_rng(2)
    # on a 2^-8 grid below 2^6, so that x + 64 is exact in binary32
    x = (np.round((g.standard_normal((4, 128)) * 3 + 10) * 256) / 256).astype(F32)
    one, zero = np.ones(128, F32), np.zeros(128, F32)
    y = oracle.norm_rows(x, one, zero, 0.0)
    assert np.allclose(y.mean(axis=1), 0.0, atol=1e-12)
    assert np.allclose(y.var(axis=1), 1.0, rtol=1e-12)
    assert np.allclose(oracle.norm_rows(x + F32(64), one, zero, 0.0), y, atol=1e-9)   # shift-free
    beta = g.standard_normal(128).astype(F32)
    assert np.allclose(oracle.norm_rows(x, one, beta, 0.0), y + beta.astype(np.float64), atol=1e-12)


def test_silu_mul_closed_forms():
    x = np.array([0.0, math.log(3.0), 40.0, -40.0, 2.5, -2.5])
    h = oracle.silu_mul(x, np.ones_like(x))
    assert h[0] == 0.0
    assert abs(h[1] - 0.75 * math.log(3.0)) < 1e-15
    assert abs(h[2] - 40.0) < 1e-15 and abs(h[3]) < 1e-15
    assert abs((h[4] - h[5]) - 2.5) < 1e-15                    # silu(x) - silu(-x) = x
    u = np.array([3.0, -2.0, 0.5, 7.0, 0.0, -1.0])
    np.testing.assert_allclose(oracle.silu_mul(x, u), h * u, rtol=1e-15, atol=0)


def test_norms_and_gate_equal_the_library_routines():
    """torch's binary64 layer_norm, rms_norm and silu on the same (widened)
    inputs: pins eps placement in both norms with gamma and beta applied."""
    import torch
    import torch.nn.functional as F
    g = np.random.default_rng(3)
    x = (g.standard_normal((6, 80)) * 2 + 0.5).astype(F32)
    x[0] *= F32(1e-3)                                          # a row where eps matters
    gamma = g.uniform(0.5, 2, 80).astype(F32)
    beta = g.standard_normal(80).astype(F32)
    xt, gt, bt = (torch.from_numpy(a.astype(np.float64)) for a in (x, gamma, beta))
    for eps in (1e-5, 1e-6, 0.25):
        np.testing.assert_allclose(oracle.norm_rows(x, gamma, beta, eps),
                                   F.layer_norm(xt, (80,), gt, bt, eps).numpy(), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(oracle.norm_rows(x, gamma, None, eps),
                                   F.rms_norm(xt, (80,), gt, eps).numpy(), rtol=1e-12, atol=1e-13)
    gg = g.standard_normal(200) * 6
    uu = g.standard_normal(200)
    np.testing.assert_allclose(oracle.silu_mul(gg, uu), (F.silu(torch.from_numpy(gg)) * torch.from_numpy(uu)).numpy(),
                               rtol=1e-14, atol=1e-300)
