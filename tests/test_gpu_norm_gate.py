"""GPU parity of the normalisation / gate fused with the per-token
quantisation (LayerNorm fused with the QKV projection's input, "7B on an
RTX 4060 with FP8" computation graph §2.1; RMSNorm for the Llama shapes; the
SiLU gate ahead of the down projection).  The values are binary32 in the
kernel and binary64 in the oracle, so codes are checked for validity
(nearest E4M3 under the kernel's scale, scale to 2^-18) and mostly equal."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from _parity import assert_valid_codes

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _to(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


@pytest.mark.parametrize("rows,cols,dt,layer", [(1, 4096, np.float32, False), (8, 4096, np.float32, True),
                                                (33, 1040, np.float16, False), (5, 8192, np.float16, True),
                                                (3, 16384, np.float32, False)])
def test_norm_quantize(rows, cols, dt, layer):
    g = np.random.default_rng(rows * 100 + cols)
    x = (synthetic.activations("normal_outl_0p5pct_x30", rows, cols, g) * 2 + (5 if layer else 0)).astype(dt)
    gamma = g.uniform(0.5, 2.0, cols).astype(np.float32)
    beta = g.standard_normal(cols).astype(np.float32) * 0.1 if layer else None
    eps = 1e-5
    q, s = pg.fp8_norm_quantize(_to(x), _to(gamma), None if beta is None else _to(beta), eps)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    y64 = oracle.norm_rows(x, gamma, beta, eps)
    assert_valid_codes(q.cpu().numpy(), s.cpu().numpy(), y64, f"{'LayerNorm' if layer else 'RMSNorm'} {rows}x{cols}")


def test_norm_quantize_rejects_long_rows_and_bad_eps():
    x = torch.zeros((2, 16400), device=DEV)
    gamma = torch.ones(16400, device=DEV)
    with pytest.raises(pg.Pgf8Error):
        pg.fp8_norm_quantize(x, gamma)
    with pytest.raises(pg.Pgf8Error):
        pg.fp8_norm_quantize(x[:, :4096].contiguous(), gamma[:4096].contiguous(), eps=-1.0)


@pytest.mark.parametrize("rows,inter,dtype", [(1, 11008, torch.bfloat16), (8, 11008, torch.bfloat16),
                                              (4, 28672, torch.bfloat16), (6, 1040, torch.float32)])
def test_silu_mul_quantize(rows, inter, dtype):
    g = torch.Generator().manual_seed(rows * 7 + inter)
    gu = (torch.randn((rows, 2 * inter), generator=g) * 3).to(dtype)
    q, s = pg.fp8_silu_mul_quantize(gu.to(DEV))
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    gu64 = gu.to(torch.float64).numpy()
    h64 = oracle.silu_mul(gu64[:, :inter], gu64[:, inter:])
    assert_valid_codes(q.cpu().numpy(), s.cpu().numpy(), h64, f"silu*up {rows}x{inter} {dtype}")


def test_decoder_mlp_chain_end_to_end():
    """RMSNorm+quantise -> gate+up GEMM -> SiLU gate+quantise -> down GEMM on
    the GPU against the same chain in binary64 without quantisation: the
    FP8 chain stays within a few percent (two E4M3 roundings of activations
    and weights)."""
    g = np.random.default_rng(99)
    M, H, I = 8, 1024, 2048
    x = synthetic.activations("normal_outl_0p5pct_x30", M, H, g)
    gamma = g.uniform(0.5, 1.5, H).astype(np.float32)
    w_gu = synthetic.weights_f16(2 * I, H, 0.02, g)
    w_dn = synthetic.weights_f16(H, I, 0.02, g)
    wq_gu, sw_gu = pg.fp8_quantize_rows(_to(w_gu))
    wq_dn, sw_dn = pg.fp8_quantize_rows(_to(w_dn))
    q1, s1 = pg.fp8_norm_quantize(_to(x), _to(gamma), None, 1e-6)
    gu = pg.fp8_linear(q1, s1, wq_gu, sw_gu)
    q2, s2 = pg.fp8_silu_mul_quantize(gu, flags=pg.FLAG_OVERLAP_PREVIOUS)
    y = pg.fp8_linear(q2, s2, wq_dn, sw_dn, flags=pg.FLAG_OVERLAP_PREVIOUS)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    n = oracle.norm_rows(x, gamma, None, 1e-6)
    gu64 = n @ w_gu.astype(np.float64).T
    h = oracle.silu_mul(gu64[:, :I], gu64[:, I:])
    ref = h @ w_dn.astype(np.float64).T
    err = np.linalg.norm(y.float().cpu().numpy() - ref) / np.linalg.norm(ref)
    assert err < 0.08, err
