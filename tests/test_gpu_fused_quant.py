"""The skinny GEMM that quantises its activations itself (dynamic entry
points, M <= 32, each CTA's activation slice held in registers): per-token
scales from the amax over all of K ("7B on an RTX 4060 with FP8" §2.2,
§6.1), combined across the CTAs of a split-K cluster.
Against the two-kernel form (the default) the codes, scales and
outputs are bit-identical; against the oracle the codes and scales are
bit-exact and the outputs within the layer's bound."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from _parity import E5, assert_within, fp8_row_max, linear_bound

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _to(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy()


def _dynamic(xt, wq, sw, flags=0, **kw):
    M, K = xt.shape
    N = wq.shape[0]
    ws = torch.zeros(pg.fp8_linear_dynamic_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
    y = pg.fp8_linear_dynamic(xt, wq, sw, workspace=ws, flags=flags, **kw)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    aq, sa = pg.dynamic_workspace_views(ws, M, K)
    return y, aq.cpu().numpy(), sa.cpu().numpy()


def _strided(x, pad):
    """x as a row-strided device view (row stride K + pad elements)."""
    M, K = x.shape
    big = np.zeros((M, K + pad), dtype=x.dtype)
    big[:, :K] = x
    return _to(big)[:, :K]


CASES = [
    # M, N, K, x dtype, split_k, row padding
    (1, 4096, 4096, np.float32, 0, 0),
    (8, 1040, 4000, np.float32, 0, 0),      # ragged N (last tile 16 rows) and K (last k-block 32)
    (5, 528, 11008, np.float16, 3, 16),     # uneven K-slices, strided rows
    (16, 2048, 1024, np.float32, 8, 0),
    (17, 768, 2064, np.float16, 1, 8),      # BN 32, one K-slice, K tail of 16
    (32, 1024, 6144, np.float32, 2, 4),
    (3, 256, 16, np.float32, 0, 0),         # one k-block of 16 elements
    (1, 1024, 11008, np.float16, 8, 0),     # raw tiles of 1 row
    (2, 1040, 4000, np.float32, 0, 0),      # 2 rows, two raw slots
    (2, 512, 2048, np.float16, 2, 8),
    (4, 768, 4096, np.float16, 0, 0),       # 4 rows
    (4, 640, 1504, np.float32, 4, 0),
    # slices too long for the registers: the two-kernel form (same results)
    (1, 256, 16384, np.float32, 1, 0),
    (2, 384, 8192, np.float32, 1, 0),
    (4, 256, 8192, np.float16, 1, 16),
    # resident slice reusing weight stages, ragged last k-block
    (3, 256, 912, np.float32, 1, 0),
]


@pytest.mark.parametrize("M,N,K,dt,split,pad", CASES)
def test_fused_matches_separate_and_oracle(M, N, K, dt, split, pad):
    g = np.random.default_rng(M * 7919 + N * 31 + K)
    x = synthetic.activations("normal_outl_0p5pct_x30", M, K, g).astype(dt)
    w = synthetic.weights_f16(N, K, 0.02, g)
    xt = _strided(x, pad) if pad else _to(x)
    wq, sw = pg.fp8_quantize_rows(_to(w))
    # the fused kernel runs where each CTA's slice fits 128 threads' registers
    # (4 chunks of 16 f32, 8 of 16 f16 each), and only when asked for
    xdt = torch.float32 if dt == np.float32 else torch.float16
    fused, s_eff = pg.fp8_linear_dynamic_plan(M, N, K, xdt, split_k=split, flags=pg.FLAG_FUSED_QUANT)
    kb = (K + 127) // 128
    assert 1 <= s_eff <= min(8, kb)
    assert fused == (M * ((kb + s_eff - 1) // s_eff) * 8 <= 128 * (4 if dt == np.float32 else 8))
    assert pg.fp8_linear_dynamic_plan(M, N, K, xdt, split_k=split) == (False, s_eff)
    y_f, aq_f, sa_f = _dynamic(xt, wq, sw, flags=pg.FLAG_FUSED_QUANT, split_k=split)
    y_s, aq_s, sa_s = _dynamic(xt, wq, sw, split_k=split)
    np.testing.assert_array_equal(aq_f, aq_s)
    np.testing.assert_array_equal(sa_f, sa_s)
    np.testing.assert_array_equal(_bits(y_f), _bits(y_s))
    aq, sa = oracle.quantize_rows(x)
    np.testing.assert_array_equal(aq_f, aq)
    np.testing.assert_array_equal(sa_f, sa)
    wq_o, sw_o = oracle.quantize_rows(w)
    ref = oracle.fp8_linear(aq, sa, wq_o, sw_o)
    bound = linear_bound(ref, K, fp8_row_max(aq, sa), fp8_row_max(wq_o, sw_o))
    assert_within(y_f.float().cpu().numpy(), ref, bound, f"fused M{M} N{N} K{K}")


def test_fused_special_rows():
    """A zero row (scale 1, codes 0), a row with an infinity and one with a
    NaN take the same codes, scales and outputs as the separate quantisation
    kernel; the finite rows stay within the oracle's bound."""
    M, N, K = 6, 512, 1536
    g = np.random.default_rng(5)
    x = synthetic.activations("normal_outl_0p5pct_x30", M, K, g)
    w = synthetic.weights_f16(N, K, 0.02, g)
    x[1] = 0.0
    x[3, 700] = np.inf
    x[4, 5] = np.nan
    xt = _to(x)
    wq, sw = pg.fp8_quantize_rows(_to(w))
    for split in (0, 1, 4):
        y_f, aq_f, sa_f = _dynamic(xt, wq, sw, flags=pg.FLAG_FUSED_QUANT, split_k=split)
        y_s, aq_s, sa_s = _dynamic(xt, wq, sw, split_k=split)
        np.testing.assert_array_equal(aq_f, aq_s)
        np.testing.assert_array_equal(sa_f.view(np.uint32), sa_s.view(np.uint32))
        np.testing.assert_array_equal(_bits(y_f), _bits(y_s))
        assert sa_f[1] == 1.0 and not aq_f[1].any()
        fin = [0, 1, 2, 5]
        aq, sa = oracle.quantize_rows(x[fin])
        np.testing.assert_array_equal(aq_f[fin], aq)
        wq_o, sw_o = oracle.quantize_rows(w)
        ref = oracle.fp8_linear(aq, sa, wq_o, sw_o)
        bound = linear_bound(ref, K, fp8_row_max(aq, sa), fp8_row_max(wq_o, sw_o))
        assert_within(y_f.float().cpu().numpy()[fin], ref, bound, f"special rows split {split}")


def test_fused_tile_choice_and_fallbacks():
    """tile_n 16 / 32 use the fused kernel, tile_n 64 and the tiled path the
    two-kernel form; all agree with the oracle."""
    M, N, K = 12, 640, 2048
    g = np.random.default_rng(9)
    x = synthetic.activations("normal_outl_0p5pct_x30", M, K, g)
    w = synthetic.weights_f16(N, K, 0.02, g)
    xt = _to(x)
    wq, sw = pg.fp8_quantize_rows(_to(w))
    aq, sa = oracle.quantize_rows(x)
    wq_o, sw_o = oracle.quantize_rows(w)
    ref = oracle.fp8_linear(aq, sa, wq_o, sw_o)
    bound = linear_bound(ref, K, fp8_row_max(aq, sa), fp8_row_max(wq_o, sw_o))
    for kw in ({"tile_n": 16}, {"tile_n": 32}, {"tile_n": 64}, {"path": pg.PATH_TILED}, {"path": pg.PATH_STREAMK},
               {"path": pg.PATH_SKINNY, "split_k": 2}):
        y, aq_g, sa_g = _dynamic(xt, wq, sw, flags=pg.FLAG_FUSED_QUANT, **kw)
        np.testing.assert_array_equal(aq_g, aq)
        np.testing.assert_array_equal(sa_g, sa)
        assert_within(y.float().cpu().numpy(), ref, bound, str(kw))


def test_fused_chain_reads_previous_output():
    """Three chained layers, each quantising an f16 copy (made by torch on the
    same stream) of the previous layer's output.  With the overlap flag the
    fused kernel reads its activations only after the kernel that wrote them
    has completed: the chain gives the same bits with and without the flag
    and in the two-kernel form."""
    g = np.random.default_rng(17)
    M, K, N = 4, 2048, 2048
    x0 = synthetic.activations("normal_outl_0p5pct_x30", M, K, g).astype(np.float16)
    ws_w = [synthetic.weights_f16(N, K, 0.02, g) for _ in range(3)]
    wts = [pg.fp8_quantize_rows(_to(w)) for w in ws_w]
    s = torch.cuda.Stream()
    outs = {}
    for flags in (0, pg.FLAG_FUSED_QUANT, pg.FLAG_FUSED_QUANT | pg.FLAG_OVERLAP_PREVIOUS, pg.FLAG_OVERLAP_PREVIOUS):
        with torch.cuda.stream(s):
            x = _to(x0)
            seq = []
            for wq, sw in wts:
                ws = torch.zeros(pg.fp8_linear_dynamic_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
                y = pg.fp8_linear_dynamic(x, wq, sw, workspace=ws, flags=flags, stream=s)
                seq.append(y)
                x = (y.float() * 0.05).half()
        s.synchronize()
        assert pg.device_status() == pg.OK
        outs[flags] = [_bits(y) for y in seq]
    for flags, ys in outs.items():
        for a, b in zip(ys, outs[0]):
            np.testing.assert_array_equal(a, b, err_msg=f"flags {flags}")


def test_nested_fp8_mode_fused():
    """NestedFP FP8 mode (E4M3 activations x E5M2 hi plane) with M <= 32 runs
    the fused kernel: bit-identical to its two-kernel form (the quantisation,
    then the skinny kernel with the same split of K; the automatic choice
    without the flag runs the grouped kernel, whose partial sums are added in
    another order)."""
    M, N, K = 16, 1024, 4096
    g = np.random.default_rng(23)
    x = g.standard_normal((M, K), dtype=np.float32).astype(np.float16)
    w = synthetic.weights_f16(N, K, 0.02, g)
    hi, lo = pg.nestedfp_split(_to(w))
    xt = _to(x)
    fused, split = pg.fp8_linear_dynamic_plan(M, N, K, torch.float16, flags=pg.FLAG_FUSED_QUANT)
    assert fused
    y_f = pg.nestedfp_linear(xt, hi, None, mode=pg.NESTED_FP8, flags=pg.FLAG_FUSED_QUANT)
    y_s = pg.nestedfp_linear(xt, hi, None, mode=pg.NESTED_FP8, path=pg.PATH_SKINNY, split_k=split)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    np.testing.assert_array_equal(_bits(y_f), _bits(y_s))
    hi_o, _ = oracle.nestedfp_split(w)
    ref, aq, sa = oracle.nestedfp_linear_fp8(x, hi_o)
    bound = linear_bound(ref, K, fp8_row_max(aq, sa), np.abs(E5[hi_o]).max(axis=1))
    assert_within(y_f.float().cpu().numpy(), ref, bound, "nested fp8 fused")
