"""GPU parity of the tensor-parallel building blocks ("C++ and FP8" §4.2,
§5.2) on one B200: R ranks of a layer split along K (or N) are run one
after another on the device, and the two collectives (all-reduce MAX of the
per-token amax, all-reduce SUM of the f32 partials) are taken by the test
between the steps.  Codes and scales of the split rows must equal the
oracle's per-token quantisation of the whole rows bit for bit; the rounded
sum must lie within |y - ref| <= 2^-8 |ref| + 1e-4 sqrt(K) A_m W_n of the
oracle's binary64 layer."""
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


@pytest.mark.parametrize("M,K,N,R", [(8, 4096, 1024, 2), (8, 4096, 1024, 4), (1, 2048, 528, 2),
                                     (100, 1024, 400, 2), (300, 2048, 528, 2), (512, 2048, 272, 4)])
def test_row_parallel_ranks_match_the_unsplit_layer(M, K, N, R):
    g = np.random.default_rng(M * 7 + K + N + R)
    x = synthetic.activations("student_t3", M, K, g)
    x[0, : K // R] = 0.0                          # rank 0's slice of row 0 is zero
    if M > 1:
        x[1] = 0.0                                # a zero row: scale 1, codes 0
    w = synthetic.weights_f16(N, K, 0.01, g)
    aq0, sa0 = oracle.quantize_rows(x)
    wq0, sw0 = oracle.quantize_rows(w)
    xt, wq, sw = _to(x), _to(wq0), _to(sw0)
    kb = K // R
    amax = None
    for r in range(R):                            # all-reduce MAX, taken here
        a = pg.fp8_row_amax(xt[:, r * kb:(r + 1) * kb].contiguous())
        amax = a if amax is None else torch.maximum(amax, a)
    assert np.array_equal(amax.cpu().numpy(), np.abs(x).max(axis=1).astype(np.float32))
    total = torch.zeros((M, N), dtype=torch.float32, device=DEV)
    codes = []
    for r in range(R):
        x_r = xt[:, r * kb:(r + 1) * kb].contiguous()
        q_r, s = pg.fp8_quantize_rows_amax(x_r, amax.clone())
        codes.append(q_r)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), sa0.view(np.uint32)), f"rank {r}: scales"
        total += pg.fp8_linear_partial(q_r, s, wq[:, r * kb:(r + 1) * kb].contiguous(), sw)   # all-reduce SUM
    y = pg.round_bf16(total)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    assert np.array_equal(torch.cat(codes, dim=1).cpu().numpy(), aq0), "codes differ from the unsplit rows'"
    ref = oracle.fp8_linear(aq0, sa0, wq0, sw0)
    bound = linear_bound(ref, K, fp8_row_max(aq0, sa0), fp8_row_max(wq0, sw0))
    assert_within(y.float().cpu().numpy(), ref, bound, f"row-parallel R={R} M={M} K={K} N={N}")
    # one rank's f32 partial against the oracle's binary64 partial of its slice
    p0 = pg.fp8_linear_partial(codes[0], _to(sa0), wq[:, :kb].contiguous(), sw)
    ref0 = oracle.fp8_linear(aq0[:, :kb], sa0, wq0[:, :kb], sw0)
    b0 = 2.0 ** -20 * np.abs(ref0) + 1e-4 * np.sqrt(kb) * fp8_row_max(aq0[:, :kb], sa0)[:, None] * \
        fp8_row_max(wq0[:, :kb], sw0)[None, :]
    assert_within(p0.cpu().numpy(), ref0, b0, "f32 partial")


@pytest.mark.parametrize("M,K,N,R", [(8, 2048, 1024, 4), (512, 1024, 512, 2)])
def test_column_parallel_blocks_match_the_unsplit_layer(M, K, N, R):
    g = np.random.default_rng(M + K + N)
    x = synthetic.activations("normal_outl_0p5pct_x30", M, K, g)
    w = synthetic.weights_f16(N, K, 0.02, g)
    aq0, sa0 = oracle.quantize_rows(x)
    wq0, sw0 = oracle.quantize_rows(w)
    ref = oracle.fp8_linear(aq0, sa0, wq0, sw0)
    bound = linear_bound(ref, K, fp8_row_max(aq0, sa0), fp8_row_max(wq0, sw0))
    xt, wq, sw = _to(x), _to(wq0), _to(sw0)
    nb = N // R
    blocks = [pg.fp8_linear_dynamic(xt, wq[r * nb:(r + 1) * nb].contiguous(), sw[r * nb:(r + 1) * nb].contiguous())
              for r in range(R)]
    y = torch.cat(blocks, dim=1)                  # all-gather, taken here
    torch.cuda.synchronize()
    assert_within(y.float().cpu().numpy(), ref, bound, f"column-parallel R={R}")


@pytest.mark.parametrize("K", [4096, 28672, 40960])
def test_quantize_from_amax_equals_dynamic_quantisation_and_round_bf16(K):
    """The row kernels (rows held in registers up to 16384 elements, the
    two-pass kernel beyond) in the amax-only and given-amax modes."""
    g = np.random.default_rng(5)
    x = synthetic.activations("student_t3", 40, K, g)
    x[3] = 0.0
    xt = _to(x)
    q_dyn, s_dyn = pg.fp8_quantize_rows(xt)
    q_am, s_am = pg.fp8_quantize_rows_amax(xt, pg.fp8_row_amax(xt))
    torch.cuda.synchronize()
    assert torch.equal(q_dyn, q_am) and torch.equal(s_dyn.view(torch.int32), s_am.view(torch.int32))
    q0, s0 = oracle.quantize_rows(x)
    assert np.array_equal(q_am.cpu().numpy(), q0)
    v = torch.from_numpy(g.standard_normal(4096 * 3).astype(np.float32) * 1e3).to(DEV)
    assert torch.equal(pg.round_bf16(v).view(torch.int16), v.to(torch.bfloat16).view(torch.int16))
