"""GPU parity of the per-tensor scaling variants against the oracle:
MINMAX calibration amax ("C++ and FP8" §5.1), static per-tensor
quantisation, and delayed scaling over an amax history ("7B on an RTX 4060
with FP8" §6.1).  Codes, scales and the window of recorded amaxes are
bit-exact; downstream GEMMs stay within the layer's bound."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from _parity import assert_within, fp8_row_max, linear_bound

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _to(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _strided(x, pad):
    M, K = x.shape
    big = np.zeros((M, K + pad), dtype=x.dtype)
    big[:, :K] = x
    return _to(big)[:, :K]


@pytest.mark.parametrize("dt,pad", [(np.float32, 0), (np.float16, 8), (np.float32, 4)])
def test_calibration_amax_and_static_per_tensor(dt, pad):
    g = np.random.default_rng(11)
    batches = [(synthetic.activations("normal_outl_0p5pct_x30", r, 1040, g) * g.uniform(0.2, 3)).astype(dt)
               for r in (1, 7, 33, 300)]
    amax_t = None
    a_ref = 0.0
    for b in batches:
        amax_t = pg.fp8_amax_accumulate(_strided(b, pad) if pad else _to(b), amax_t)
        a_ref = oracle.amax_accumulate(b, a_ref)
    torch.cuda.synchronize()
    assert amax_t.item() == np.float32(a_ref)
    x = batches[2]
    q, s = pg.fp8_quantize_tensor(_strided(x, pad) if pad else _to(x), amax_t)
    torch.cuda.synchronize()
    q0, s0 = oracle.quantize_tensor(x, a_ref)
    np.testing.assert_array_equal(q.cpu().numpy(), q0)
    assert np.all(s.cpu().numpy() == s0)
    assert pg.device_status() == pg.OK


def test_amax_ignores_nan_and_accumulates_from_a_given_start():
    x = np.ones((4, 64), np.float32)
    x[1, 3] = np.nan
    x[2, 5] = -7.0
    a = pg.fp8_amax_accumulate(_to(x))
    assert a.item() == 7.0
    a = pg.fp8_amax_accumulate(_to(x), torch.tensor([9.5], device=DEV))
    assert a.item() == 9.5


@pytest.mark.parametrize("H,steps,rows,cols,dt", [(3, 12, 5, 528, np.float32), (16, 40, 300, 272, np.float32),
                                                   (1024, 1030, 2, 64, np.float16), (1, 6, 1, 4096, np.float32)])
def test_delayed_scaling_matches_the_oracle_step_by_step(H, steps, rows, cols, dt):
    g = np.random.default_rng(H * 1000 + steps)
    d_gpu = pg.DelayedScaling(H, initial_scale=0.02, device=DEV)
    d_ref = oracle.DelayedScaling(H, initial_scale=0.02)
    # amaxes rise then fall, so the window's maximum is evicted repeatedly
    mags = np.concatenate([np.linspace(0.5, 40, steps // 2), np.linspace(40, 0.1, steps - steps // 2)])
    check_every = 1 if steps <= 64 else 97
    for t in range(steps):
        x = (g.standard_normal((rows, cols)) * mags[t]).astype(dt)
        q, s = d_gpu.step(_to(x))
        q0, s0 = d_ref.step(x)
        if t % check_every == 0 or t == steps - 1:
            torch.cuda.synchronize()
            np.testing.assert_array_equal(q.cpu().numpy(), q0, err_msg=f"step {t}")
            assert np.all(s.cpu().numpy() == s0), f"step {t}"
            np.testing.assert_array_equal(d_gpu.window(), d_ref.history, err_msg=f"step {t}")
    assert pg.device_status() == pg.OK


def test_delayed_codes_feed_the_gemm():
    """Delayed per-tensor codes and scales go into the FP8 linear as they
    are; the result stays within the layer's bound of the oracle."""
    g = np.random.default_rng(21)
    M, K, N = 8, 2048, 1536
    w = synthetic.weights_f16(N, K, 0.02, g)
    wq, sw = pg.fp8_quantize_rows(_to(w))
    wq0, sw0 = oracle.quantize_rows(w)
    d_gpu = pg.DelayedScaling(1024, device=DEV)
    d_ref = oracle.DelayedScaling(1024)
    for t in range(3):
        x = synthetic.activations("normal_outl_0p5pct_x30", M, K, g)
        aq, sa = d_gpu.step(_to(x))
        aq0, sa0 = d_ref.step(x)
        y = pg.fp8_linear(aq, sa, wq, sw)
        torch.cuda.synchronize()
        ref = oracle.fp8_linear(aq0, np.full(M, sa0, np.float32), wq0, sw0)
        bound = linear_bound(ref, K, fp8_row_max(aq0, np.full(M, sa0, np.float32)), fp8_row_max(wq0, sw0))
        assert_within(y.float().cpu().numpy(), ref, bound, f"delayed step {t}")


def test_overlapped_launches_match_plain_ones():
    """Per-tensor quantisation launched with FLAG_OVERLAP_PREVIOUS between
    overlapped GEMMs reads its inputs only after the previous kernel has
    completed: same codes, scales, recorded amaxes and outputs as plain
    launches."""
    g = np.random.default_rng(33)
    M, K, N = 4, 1024, 1024
    ws_ = [pg.fp8_quantize_rows(_to(synthetic.weights_f16(N, K, 0.02, g))) for _ in range(3)]
    xs = [(g.standard_normal((M, K)) * (i + 1)).astype(np.float32) for i in range(6)]
    s = torch.cuda.Stream()
    results = []
    for flags in (0, pg.FLAG_OVERLAP_PREVIOUS):
        with torch.cuda.stream(s):
            d = pg.DelayedScaling(16, device=DEV, stream=s)
            amax = pg.fp8_amax_accumulate(_to(xs[0]), stream=s)
            outs = []
            x = _to(xs[0])
            for t, xn in enumerate(xs):
                wq, sw = ws_[t % 3]
                aq, sa = d.step(x, flags=flags, stream=s)
                y = pg.fp8_linear(aq, sa, wq, sw, flags=flags, stream=s)
                aq2, sa2 = pg.fp8_quantize_tensor(x, amax, flags=flags, stream=s)
                y2 = pg.fp8_linear(aq2, sa2, wq, sw, flags=flags, stream=s)
                outs.append((aq, sa, y, aq2, y2))
                x = (y.float() * 0.5 + _to(xn)).contiguous()     # next input depends on this output
        s.synchronize()
        assert pg.device_status() == pg.OK
        results.append(([tuple(t.cpu().numpy().copy() if t.dtype != torch.bfloat16 else
                               t.view(torch.int16).cpu().numpy() for t in o) for o in outs], d.window().tolist()))
    (a, ca), (b, cb) = results
    assert ca == cb
    for i, (ta, tb) in enumerate(zip(a, b)):
        for u, v in zip(ta, tb):
            np.testing.assert_array_equal(u, v, err_msg=f"step {i}")
