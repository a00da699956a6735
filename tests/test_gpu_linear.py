"""GPU parity of the FP8 linear layer (skinny and tiled kernels, split-K
clusters, ragged shapes) against the oracle, within the layer's stated bound:
|y - ref| <= 2^-8 |ref| + 1e-4 sqrt(K) A_m W_n."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from _parity import assert_within, fp8_row_max, linear_bound

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _oracle_case(x, w):
    aq, sa = oracle.quantize_rows(x)
    wq, sw = oracle.quantize_rows(w)
    ref = oracle.fp8_linear(aq, sa, wq, sw)
    bound = linear_bound(ref, x.shape[1], fp8_row_max(aq, sa), fp8_row_max(wq, sw))
    return aq, sa, wq, sw, ref, bound


def _to(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _run_linear(aq, sa, wq, sw, **kw):
    y = pg.fp8_linear(_to(aq), _to(sa), _to(wq), _to(sw), **kw)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    return y.float().cpu().numpy()


def test_small_workload_full_check():
    """16 x 512 x 512: every output, both kernel families."""
    x, w = synthetic.case("small", 0, 0)
    aq, sa, wq, sw, ref, bound = _oracle_case(x, w)
    for kw in ({}, {"path": pg.PATH_TILED}, {"path": pg.PATH_SKINNY, "split_k": 4}, {"path": pg.PATH_TILED_PAIR}):
        y = _run_linear(aq, sa, wq, sw, **kw)
        assert_within(y, ref, bound, f"small {kw}")


@pytest.mark.parametrize("M,N,K", [(256, 256, 128), (512, 768, 1024), (300, 528, 400), (1000, 1040, 2000),
                                   (2048, 4096, 4096), (4096, 12288, 256)])
def test_pair_kernel_against_oracle(M, N, K):
    """256 x 256 tiles on SM pairs: one or several tiles per pair (persistent
    loop), ragged M / N / K tails; large cases checked on sampled rows and
    columns (the oracle computes those one by one)."""
    g = np.random.default_rng(M + 7 * N + 13 * K)
    x = synthetic.activations("student_t4_unit", M, K, g)
    w = synthetic.weights_f16(N, K, 0.02, g)
    aq, sa = oracle.quantize_rows(x)
    wq, sw = oracle.quantize_rows(w)
    rng = np.random.default_rng(1)
    ms = np.arange(M) if M * N * K <= 2e9 else np.sort(rng.choice(M, 24, replace=False))
    ns = np.arange(N) if M * N * K <= 2e9 else np.sort(rng.choice(N, 256, replace=False))
    ref = oracle.fp8_linear(aq[ms], sa[ms], wq[ns], sw[ns])
    bound = linear_bound(ref, K, fp8_row_max(aq[ms], sa[ms]), fp8_row_max(wq[ns], sw[ns]))
    for tile_n in (0, 128, 192, 256):
        for _ in range(2):
            y = _run_linear(aq, sa, wq, sw, path=pg.PATH_TILED_PAIR, tile_n=tile_n)
            assert_within(y[np.ix_(ms, ns)], ref, bound, f"pair{tile_n} M{M} N{N} K{K}")


RAGGED = [  # M, N, K: several tiles plus ragged tails in every dimension
    (1, 16, 16), (3, 48, 144), (16, 272, 528), (17, 528, 1040), (64, 400, 272),
    (100, 144, 1008), (128, 256, 384), (129, 272, 528), (200, 528, 400), (300, 16, 160),
]


@pytest.mark.parametrize("M,N,K", RAGGED)
def test_ragged_shapes_all_paths(M, N, K):
    g = np.random.default_rng(M * 1000003 + N * 1009 + K)
    x = synthetic.activations("student_t3", M, K, g)
    w = synthetic.weights_f16(N, K, 0.02, g)
    aq, sa, wq, sw, ref, bound = _oracle_case(x, w)
    configs = [{"path": pg.PATH_TILED, "split_k": 1}, {"path": pg.PATH_TILED, "split_k": 3},
               {"path": pg.PATH_TILED, "tile_n": 256}, {"path": pg.PATH_TILED_PAIR}, {}]
    if M <= 128:
        configs += [{"path": pg.PATH_SKINNY, "split_k": 1}, {"path": pg.PATH_SKINNY, "split_k": 2},
                    {"path": pg.PATH_SKINNY, "split_k": 8}, {"path": pg.PATH_SKINNY, "tile_n": 128}]
    for kw in configs:
        y = _run_linear(aq, sa, wq, sw, **kw)
        assert_within(y, ref, bound, f"M{M} N{N} K{K} {kw}")


def test_split_k_is_deterministic():
    g = np.random.default_rng(5)
    x = synthetic.activations("normal_outl_0p5pct_x30", 8, 4096, g)
    w = synthetic.weights_f16(512, 4096, 0.02, g)
    aq, sa = oracle.quantize_rows(x)
    wq, sw = oracle.quantize_rows(w)
    ys = [_run_linear(aq, sa, wq, sw, path=pg.PATH_SKINNY, split_k=5) for _ in range(3)]
    for y in ys[1:]:
        np.testing.assert_array_equal(y, ys[0])


def test_outputs_untouched_outside_and_canaries():
    """The kernel writes exactly y[M, N]: guard zones around it keep their
    NaN poison and every element inside is overwritten."""
    M, N, K = 17, 272, 528
    g = np.random.default_rng(9)
    x = synthetic.activations("student_t4_unit", M, K, g)
    w = synthetic.weights_f16(N, K, 0.02, g)
    aq, sa, wq, sw, ref, bound = _oracle_case(x, w)
    guard = 4096
    for kw in ({"path": pg.PATH_SKINNY}, {"path": pg.PATH_SKINNY, "split_k": 3}, {"path": pg.PATH_TILED}):
        buf = torch.full((2 * guard + M * N,), float("nan"), dtype=torch.bfloat16, device=DEV)
        y = buf[guard:guard + M * N].view(M, N)
        pg.fp8_linear(_to(aq), _to(sa), _to(wq), _to(sw), y=y, **kw)
        torch.cuda.synchronize()
        b = buf.float().cpu().numpy()
        assert np.isnan(b[:guard]).all() and np.isnan(b[guard + M * N:]).all(), kw
        assert_within(b[guard:guard + M * N].reshape(M, N), ref, bound, str(kw))


def test_dynamic_entry_point_matches_two_step():
    """fp8_linear_dynamic (quantise + GEMM, chained) gives the oracle's codes
    in its workspace and the same outputs as the two separate calls."""
    x, w = synthetic.case("decode7b", 1, 2)          # O-proj, M = 8
    wt = _to(w)
    wq, sw = pg.fp8_quantize_rows(wt)
    xt = _to(x)
    ws = torch.zeros(pg.fp8_linear_dynamic_workspace_size(x.shape[0], w.shape[0], x.shape[1]),
                     dtype=torch.uint8, device=DEV)
    y = pg.fp8_linear_dynamic(xt, wq, sw, workspace=ws)
    torch.cuda.synchronize()
    aq_g, sa_g = pg.dynamic_workspace_views(ws, x.shape[0], x.shape[1])
    aq, sa = oracle.quantize_rows(x)
    np.testing.assert_array_equal(aq_g.cpu().numpy(), aq)
    np.testing.assert_array_equal(sa_g.cpu().numpy(), sa)
    y2 = pg.fp8_linear(aq_g, sa_g, wq, sw)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y.float().cpu().numpy(), y2.float().cpu().numpy())


def _full_size_case(wl, shape_idx, m_idx, n_cols=384, n_rows=16, seed=0):
    """Full-size layer on the GPU (quantise weights and activations there, run
    the dynamic entry point in its default launch configuration), checked on
    a sample of rows and columns the oracle computes one by one."""
    x = synthetic.acts(wl, shape_idx, m_idx)
    w = synthetic.weights(wl, shape_idx)
    M, K = x.shape
    N = w.shape[0]
    wt = _to(w)
    wq_g, sw_g = pg.fp8_quantize_rows(wt)
    y = pg.fp8_linear_dynamic(_to(x), wq_g, sw_g)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    rng = np.random.default_rng(seed)
    ns = np.sort(rng.choice(N, min(n_cols, N), replace=False))
    ms = np.sort(rng.choice(M, min(n_rows, M), replace=False))
    aq, sa = oracle.quantize_rows(x[ms])
    wq, sw = oracle.quantize_rows(w[ns])
    np.testing.assert_array_equal(wq_g.cpu().numpy()[ns], wq)
    np.testing.assert_array_equal(sw_g.cpu().numpy()[ns], sw)
    ref = oracle.fp8_linear(aq, sa, wq, sw)
    bound = linear_bound(ref, K, fp8_row_max(aq, sa), fp8_row_max(wq, sw))
    yg = y.float().cpu().numpy()[np.ix_(ms, ns)]
    assert np.isfinite(y.float().cpu().numpy()).all()
    return assert_within(yg, ref, bound, f"{wl} shape{shape_idx} M={M}")


@pytest.mark.parametrize("shape_idx", [0, 1, 2, 3])
@pytest.mark.parametrize("m_idx", [0, 1, 2])
def test_decode7b_full_size(shape_idx, m_idx):
    _full_size_case("decode7b", shape_idx, m_idx)


@pytest.mark.parametrize("shape_idx", [0, 1, 2, 3])
def test_prefill7b_full_size(shape_idx):
    _full_size_case("prefill7b", shape_idx, 2 if shape_idx != 2 else 0)


@pytest.mark.parametrize("shape_idx,m_idx", [(0, 0), (1, 4), (2, 7), (3, 9), (1, 12), (3, 5)])
def test_llama70b_full_size(shape_idx, m_idx):
    _full_size_case("llama70b", shape_idx, m_idx)


def test_dynamic_chain_with_overlap_flag_matches_unchained():
    """Back-to-back dynamic FP8 layers with FLAG_OVERLAP_PREVIOUS reusing one
    workspace (the next layer's quantisation overwrites codes the previous
    GEMM reads): results equal those of synchronised calls, bit for bit."""
    shapes = [(4096, 12288), (4096, 4096), (11008, 4096)]
    g = np.random.default_rng(21)
    Ws, Xs = [], []
    for K, N in shapes:
        wq, sw = pg.fp8_quantize_rows(_to(synthetic.weights_f16(N, K, 0.02, g)))
        Ws.append((wq, sw))
        Xs.append(_to(synthetic.activations("normal_outl_0p5pct_x30", 8, K, g)))
    ws = torch.zeros(max(pg.fp8_linear_dynamic_workspace_size(8, N, K) for K, N in shapes), dtype=torch.uint8,
                     device=DEV)
    torch.cuda.synchronize()

    def run(flags, sync):
        ys = []
        for (wq, sw), x in zip(Ws, Xs):
            ys.append(pg.fp8_linear_dynamic(x, wq, sw, workspace=ws, flags=flags))
            if sync:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return [y.float().cpu().numpy() for y in ys]

    ref = run(0, True)
    for _ in range(3):
        for a, b in zip(run(pg.FLAG_OVERLAP_PREVIOUS, False), ref):
            np.testing.assert_array_equal(a, b)
    assert pg.device_status() == pg.OK


STREAMK = [  # M <= 32; grids from 1 to 148 CTAs, tiles shared by up to 64 CTAs
    (1, 16, 16), (1, 128, 8192), (3, 272, 1040), (16, 528, 4096), (17, 400, 2000), (32, 4096, 512),
    (8, 12288, 4096), (5, 256, 11008),
]


@pytest.mark.parametrize("M,N,K", STREAMK)
def test_streamk_against_oracle_and_flags_cleared(M, N, K):
    g = np.random.default_rng(M * 7 + N * 13 + K)
    x = synthetic.activations("normal_outl_0p5pct_x30", M, K, g)
    w = synthetic.weights_f16(N, K, 0.02, g)
    aq, sa, wq, sw, ref, bound = _oracle_case(x, w)
    ws = torch.zeros(int(pg.lib.pgf8_fp8_linear_workspace_size(M, N, K)), dtype=torch.uint8, device=DEV)
    outs = []
    for _ in range(3):   # the flags must come back to zero for the next call
        y = _run_linear(aq, sa, wq, sw, workspace=ws, path=pg.PATH_STREAMK)
        assert ws[:1024].count_nonzero().item() == 0
        assert_within(y, ref, bound, f"stream-K M{M} N{N} K{K}")
        outs.append(y)
    for y in outs[1:]:
        np.testing.assert_array_equal(y, outs[0])


def test_dynamic_many_matches_single_calls():
    """pgf8_fp8_linear_dynamic_many runs the same kernels as one
    fp8_linear_dynamic call per layer: outputs bit-identical, and they stay
    within the bound of the oracle."""
    shapes = [(1, 4096, 12288), (4, 4096, 4096), (8, 11008, 4096), (300, 512, 1024)]
    g = np.random.default_rng(31)
    seq, singles, refs = [], [], []
    for M, K, N in shapes:
        x = synthetic.activations("normal_outl_0p5pct_x30", M, K, g)
        w = synthetic.weights_f16(N, K, 0.02, g)
        xt = _to(x)
        wq, sw = pg.fp8_quantize_rows(_to(w))
        y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
        ws = torch.zeros(pg.fp8_linear_dynamic_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
        seq.append((xt, wq, sw, y, ws))
        ws2 = torch.zeros_like(ws)
        singles.append(pg.fp8_linear_dynamic(xt, wq, sw, workspace=ws2))
        refs.append((x, w))
    pg.LayerSequence(seq).run()
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    for (xt, wq, sw, y, ws), y1, (x, w) in zip(seq, singles, refs):
        np.testing.assert_array_equal(y.float().cpu().numpy(), y1.float().cpu().numpy())
        aq, sa = oracle.quantize_rows(x[:8])
        wq0, sw0 = oracle.quantize_rows(w[:64])
        ref = oracle.fp8_linear(aq, sa, wq0, sw0)
        bound = linear_bound(ref, x.shape[1], fp8_row_max(aq, sa), fp8_row_max(wq0, sw0))
        assert_within(y.float().cpu().numpy()[:8, :64], ref, bound, f"many {x.shape}")


@pytest.mark.parametrize("M,N,K", [(300, 528, 400), (1000, 1040, 2000), (512, 10240, 1024), (2048, 4096, 4096),
                                   (4096, 12288, 256), (256, 8192, 8192)])
def test_pair_kernel_stream_k_region(M, N, K):
    """The pair kernel with its stream-K region (the last full round and the
    ragged tail of tiles split in k-block ranges over every pair, partial
    tiles summed through the workspace): within the bound against the oracle
    on sampled rows and columns, the same bits on a repeated call, the flag
    words left zero; the plain round-robin form (no room for the partials)
    within the bound as well."""
    g = np.random.default_rng(M + 3 * N + 5 * K)
    x = synthetic.activations("student_t3", M, K, g)
    w = synthetic.weights_f16(N, K, 0.01, g)
    aq, sa = oracle.quantize_rows(x)
    wq, sw = oracle.quantize_rows(w)
    rng = np.random.default_rng(2)
    big = M * N * K > 2e9
    ms = np.sort(rng.choice(M, 32, replace=False)) if big else np.arange(M)
    ns = np.sort(rng.choice(N, 384, replace=False)) if big else np.arange(N)
    ref = oracle.fp8_linear(aq[ms], sa[ms], wq[ns], sw[ns])
    bound = linear_bound(ref, K, fp8_row_max(aq[ms], sa[ms]), fp8_row_max(wq[ns], sw[ns]))
    ws = torch.zeros(pg.lib.pgf8_fp8_linear_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
    assert ws.numel() > 16 << 20
    A, SA, W, SW = _to(aq), _to(sa), _to(wq), _to(sw)
    y1 = pg.fp8_linear(A, SA, W, SW, workspace=ws, path=pg.PATH_TILED_PAIR, flags=pg.FLAG_STREAM_K_TAIL)
    y2 = pg.fp8_linear(A, SA, W, SW, workspace=ws, path=pg.PATH_TILED_PAIR, flags=pg.FLAG_STREAM_K_TAIL)
    y_rr = pg.fp8_linear(A, SA, W, SW, workspace=torch.zeros(1024, dtype=torch.uint8, device=DEV),
                         path=pg.PATH_TILED_PAIR)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert not ws[:1024].any(), "flag words not cleared"
    for name, y in (("stream-K", y1), ("round-robin", y_rr)):
        assert_within(y.float().cpu().numpy()[np.ix_(ms, ns)], ref, bound, f"pair {name} M{M} N{N} K{K}")
