"""Pins of the oracle's per-tensor scaling variants (MINMAX calibration,
"C++ and FP8" §5.1; delayed scaling over an amax history, "7B on an RTX 4060
with FP8" §6.1) against closed forms and against the per-row quantiser
already pinned elsewhere.  Readings: amax = max |x| over the tensor; scale =
fl32(amax / 448), 1 when 0; a delayed step quantises with the scale carried
from the previous step, then records its amax in a ring of H and carries
fl32(max(history) / 448)."""
import numpy as np
import pytest

import oracle

F32 = np.float32


def _s(a):
    """fl32(a / 448) in numpy binary32, 1 when 0."""
    s = F32(a) / F32(448.0)
    return F32(1.0) if s == 0 else s


def test_amax_is_the_largest_magnitude_and_accumulates_over_batches():
    g = np.random.default_rng(3)
    batches = [g.standard_normal((r, 96)).astype(F32) * F32(10 ** g.uniform(-3, 3)) for r in (1, 5, 17)]
    a = 0.0
    for b in batches:
        assert oracle.amax_accumulate(b) == np.max(np.abs(b))
        a = oracle.amax_accumulate(b, a)
    assert a == max(np.max(np.abs(b)) for b in batches)
    assert oracle.amax_accumulate(np.zeros((3, 16), F32)) == 0.0
    assert oracle.amax_accumulate(np.array([[-3.5, 2.0]], F32)) == 3.5          # sign dropped
    assert oracle.amax_accumulate(np.array([[1.0, 2.0]], np.float16), 2.5) == 2.5
    with pytest.raises(oracle.OracleError):
        oracle.amax_accumulate(np.array([[1.0, np.nan]], F32))


def test_static_per_tensor_reduces_to_the_row_quantiser():
    g = np.random.default_rng(4)
    x = (g.standard_normal((7, 160)) * 3).astype(F32)
    amax = float(np.max(np.abs(x)))
    q, s = oracle.quantize_tensor(x, amax)
    assert s == _s(amax)
    q_rows, _ = oracle.quantize_rows(x, np.full(7, s, F32))        # static rows, one broadcast scale
    np.testing.assert_array_equal(q, q_rows)
    # one row: per-tensor == dynamic per-row
    q1, s1 = oracle.quantize_tensor(x[2:3], float(np.max(np.abs(x[2]))))
    qd, sd = oracle.quantize_rows(x[2:3])
    np.testing.assert_array_equal(q1, qd)
    assert s1 == sd[0]
    # the amax element lands on +-448 (0x7E / 0xFE); a calibrated amax below
    # the data's saturates the excess
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert q[i] in (0x7E, 0xFE)
    qs, _ = oracle.quantize_tensor(x, amax / 4)
    big = np.abs(x) > 448 * float(_s(amax / 4)) * 1.0001
    assert big.any() and np.all((qs[big] & 0x7F) == 0x7E)
    # zero amax: scale 1
    assert oracle.quantize_tensor(np.zeros((2, 16), F32), 0.0)[1] == 1.0


def test_delayed_scale_sequence_closed_form_window():
    d = oracle.DelayedScaling(3, initial_scale=0.5)
    amaxes = [5.0, 1.0, 2.0, 3.0, 0.5, 0.25, 0.125]
    used, carried = [], []
    for a in amaxes:
        _, s = d.step(np.array([[a, -a / 2], [0.0, a / 4]], F32))
        used.append(s)
        carried.append(d.scale)
    # carried after step t = max of the last 3 amaxes / 448
    expect = [_s(max(amaxes[max(0, t - 2):t + 1])) for t in range(len(amaxes))]
    assert carried == expect
    # each step uses the previous carried scale, the first the initial one
    assert used == [F32(0.5)] + expect[:-1]
    assert d.pos == len(amaxes) % 3


def test_delayed_history_of_one_is_the_previous_amax_and_codes_reduce_to_rows():
    g = np.random.default_rng(5)
    d = oracle.DelayedScaling(1)
    prev = None
    for t in range(5):
        x = (g.standard_normal((3, 48)) * (t + 1)).astype(F32)
        q, s = d.step(x)
        assert s == (F32(1.0) if prev is None else _s(prev))
        q_rows, _ = oracle.quantize_rows(x, np.full(3, s, F32))
        np.testing.assert_array_equal(q, q_rows)
        prev = float(np.max(np.abs(x)))
        assert d.scale == _s(prev)


def test_delayed_history_1024_evicts_the_oldest():
    H = 1024
    d = oracle.DelayedScaling(H)
    for i in range(H):                     # amaxes 1024, 1023, ..., 1
        d.step(np.array([[float(H - i)]], F32))
    assert d.scale == _s(1024.0) and d.pos == 0
    d.step(np.array([[0.5]], F32))         # evicts 1024: window max 1023
    assert d.scale == _s(1023.0) and d.pos == 1


def test_delayed_saturates_above_the_carried_range_and_zero_steps():
    d = oracle.DelayedScaling(4, initial_scale=0.01)
    x = np.array([[1.0, 4.48, 4.49, 100.0, -100.0, -2.0]], F32)
    q, s = d.step(x)
    assert s == F32(0.01)
    assert q[0, 1] == 0x7E and q[0, 3] == 0x7E and q[0, 4] == 0xFE and q[0, 2] == 0x7E
    e = oracle.DelayedScaling(4)
    e.step(np.zeros((2, 16), F32))
    assert e.scale == 1.0


def test_delayed_argument_errors():
    with pytest.raises(ValueError):
        oracle.DelayedScaling(0)
    d = oracle.DelayedScaling(2)
    with pytest.raises(oracle.OracleError):
        d.step(np.array([[np.inf, 1.0]], F32))
    with pytest.raises(oracle.OracleError):
        oracle.DelayedScaling(2, initial_scale=0.0).step(np.ones((1, 16), F32))
