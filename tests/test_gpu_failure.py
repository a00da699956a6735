"""Failure detection without a GPU fault: a device-side wait that can never
complete gives up after its bound, the kernel returns, the host reads
PGF8_ERR_TIMEOUT, and the context stays usable for the next call."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from _parity import assert_within, fp8_row_max, linear_bound

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    torch.cuda.set_device(0)
    assert pg.device_status() == pg.OK                     # nothing pending
    assert pg.lib.pgf8_selftest_bounded_wait(5_000_000, None) == pg.OK   # 5 ms bound
    assert pg.device_status() == pg.ERR_TIMEOUT            # reported once ...
    assert pg.device_status() == pg.OK                     # ... and cleared
    # the context is intact: a normal layer still matches the oracle
    g = np.random.default_rng(77)
    x = synthetic.activations("normal_outl_1pct_x20", 4, 256, g)
    w = synthetic.weights_f16(64, 256, 0.02, g)
    xt, wt = torch.from_numpy(x).cuda(), torch.from_numpy(w).cuda()
    wq, sw = pg.fp8_quantize_rows(wt)
    y = pg.fp8_linear_dynamic(xt, wq, sw)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    aq0, sa0 = oracle.quantize_rows(x)
    wq0, sw0 = oracle.quantize_rows(w)
    ref = oracle.fp8_linear(aq0, sa0, wq0, sw0)
    assert_within(y.float().cpu().numpy(), ref, linear_bound(ref, 256, fp8_row_max(aq0, sa0),
                                                             fp8_row_max(wq0, sw0)), "after timeout")


def test_selftest_rejects_bad_limits():
    assert pg.lib.pgf8_selftest_bounded_wait(10, None) == pg.ERR_INVALID_ARG
    assert pg.lib.pgf8_selftest_bounded_wait(10 ** 10, None) == pg.ERR_INVALID_ARG
