"""GPU parity of per-row E4M3 quantisation and the NestedFP split: codes,
scales and byte planes must equal the oracle's bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synthetic

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _gpu_quant(x: np.ndarray, scales=None, ldx=None):
    xt = torch.from_numpy(np.ascontiguousarray(x)).to(DEV)
    if ldx is not None:
        pad = torch.zeros((x.shape[0], ldx), dtype=xt.dtype, device=DEV)
        pad[:, :x.shape[1]] = xt
        xt = pad[:, :x.shape[1]]
    if scales is None:
        q, s = pg.fp8_quantize_rows(xt)
    else:
        s = torch.from_numpy(np.asarray(scales, dtype=np.float32)).to(DEV)
        q, s = pg.fp8_quantize_rows(xt, scales=s, mode=pg.SCALE_STATIC)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    return q.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 48), (16, 512), (17, 1008), (5, 4096), (2, 11008)])
@pytest.mark.parametrize("recipe", ["normal_outl_1pct_x20", "student_t4_unit", "student_t3", "normal_f16"])
def test_quantize_bit_exact(rows, cols, recipe):
    g = np.random.default_rng(rows * 7919 + cols)
    x = synthetic.activations(recipe, rows, cols, g)
    q, s = _gpu_quant(x)
    q0, s0 = oracle.quantize_rows(x)
    np.testing.assert_array_equal(s.view(np.uint32), s0.view(np.uint32))
    np.testing.assert_array_equal(q, q0)


def test_quantize_strided_rows():
    g = np.random.default_rng(1)
    x = synthetic.activations("student_t3", 7, 256, g)
    q, s = _gpu_quant(x, ldx=320)
    q0, s0 = oracle.quantize_rows(x)
    np.testing.assert_array_equal(q, q0)
    np.testing.assert_array_equal(s, s0)


def test_quantize_zero_rows_signed_zero_and_subnormals():
    x = np.zeros((4, 32), dtype=np.float32)
    x[1, 5] = -0.0
    x[2, :] = -0.0
    x[3, :] = np.float32(1e-30) * np.arange(32, dtype=np.float32)   # tiny values, amax normal
    x[3, 31] = 1.0                                                  # most codes underflow to 0 / subnormal
    q, s = _gpu_quant(x)
    q0, s0 = oracle.quantize_rows(x)
    np.testing.assert_array_equal(q, q0)
    np.testing.assert_array_equal(s, s0)
    assert s[0] == 1.0 and q[2].tolist() == [0x80] * 32


def test_quantize_subnormal_grid_and_ties():
    """Values placed on and between E4M3 subnormal / normal code points."""
    vals = np.array(sorted(set(np.abs(oracle.e4m3_table()[np.isfinite(oracle.e4m3_table())]))), dtype=np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    row = np.concatenate([vals.astype(np.float32), mids, -mids, np.nextafter(mids, np.float32(1))])
    row = row[: (row.size // 16) * 16]
    x = row[None, :].astype(np.float32)
    # static scale 1: the scaled values are the values themselves
    q, _ = _gpu_quant(x, scales=[1.0])
    q0, _ = oracle.quantize_rows(x, scales=np.float32([1.0]))
    np.testing.assert_array_equal(q, q0)


def test_quantize_static_saturation():
    g = np.random.default_rng(2)
    x = (synthetic.activations("student_t3", 6, 512, g) * 50).astype(np.float32)
    sc = np.float32([0.01, 0.1, 1.0, 0.5, 2.0, 1e-3])
    q, s = _gpu_quant(x, scales=sc)
    q0, _ = oracle.quantize_rows(x, scales=sc)
    np.testing.assert_array_equal(q, q0)
    assert (q & 0x7F == 0x7E).sum() > 100      # saturation really exercised


def test_quantize_no_rows_is_a_no_op():
    x = torch.zeros((0, 64), dtype=torch.float32, device=DEV)
    q = torch.zeros((0, 64), dtype=torch.uint8, device=DEV)
    s = torch.zeros((0,), dtype=torch.float32, device=DEV)
    pg.fp8_quantize_rows(x, q, s)
    torch.cuda.synchronize()


@pytest.mark.parametrize("wl,shape_idx,m_idx", [("prefill7b", 3, 2), ("llama70b", 3, 12)])
def test_quantize_full_size_activations(wl, shape_idx, m_idx):
    """Largest activation matrices of the workloads (e.g. 4096 x 28672), every
    row bit-exact."""
    x = synthetic.acts(wl, shape_idx, m_idx)
    q, s = _gpu_quant(x)
    q0, s0 = oracle.quantize_rows(x)
    np.testing.assert_array_equal(s, s0)
    np.testing.assert_array_equal(q, q0)


def test_quantize_full_size_weights_sampled_rows():
    """70B gate+up weights [57344, 8192] quantised per output channel on the GPU;
    256 sampled channels checked against the oracle bit for bit."""
    w = synthetic.weights("llama70b", 2)
    wt = torch.from_numpy(w).to(DEV)
    q, s = pg.fp8_quantize_rows(wt)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(0).choice(w.shape[0], 256, replace=False))
    q0, s0 = oracle.quantize_rows(w[rows])
    np.testing.assert_array_equal(s.cpu().numpy()[rows], s0)
    np.testing.assert_array_equal(q.cpu().numpy()[rows], q0)


def test_nestedfp_split_all_patterns_and_weights():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(256, 256)
    w = torch.from_numpy(bits.view(np.float16)).to(DEV)
    hi, lo = pg.nestedfp_split(w)
    h0, l0 = oracle.nestedfp_split(bits)
    np.testing.assert_array_equal(hi.cpu().numpy(), h0)
    np.testing.assert_array_equal(lo.cpu().numpy(), l0)
    w2 = synthetic.weights("nested7b", 1)
    hi2, lo2 = pg.nestedfp_split(torch.from_numpy(w2).to(DEV))
    h1, l1 = oracle.nestedfp_split(w2)
    np.testing.assert_array_equal(hi2.cpu().numpy(), h1)
    np.testing.assert_array_equal(lo2.cpu().numpy(), l1)
