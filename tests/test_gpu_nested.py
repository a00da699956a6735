"""GPU parity of the NestedFP linear layer in both modes against the oracle
(FP16 mode: weights rebuilt from (hi << 8) | lo; FP8 mode: hi read as E5M2,
activations per-token E4M3), within the layer's stated bound."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from _parity import E4, E5, assert_within, fp8_row_max, linear_bound

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _to(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _ref16(x16, hi, lo):
    ref = oracle.nestedfp_linear_fp16(x16, hi, lo)
    w = ((hi.astype(np.uint16) << 8) | lo.astype(np.uint16)).view(np.float16).astype(np.float64)
    a_hat = np.abs(x16.astype(np.float64)).max(axis=1)
    w_hat = np.abs(w).max(axis=1)
    return ref, linear_bound(ref, x16.shape[1], a_hat, w_hat)


def _ref8(x16, hi):
    ref, aq, sa = oracle.nestedfp_linear_fp8(x16, hi)
    w_hat = np.abs(E5[hi]).max(axis=1)
    return ref, linear_bound(ref, x16.shape[1], fp8_row_max(aq, sa), w_hat), aq, sa


def _run(x16, hi, lo, mode, **kw):
    y = pg.nestedfp_linear(_to(x16), _to(hi), _to(lo) if lo is not None else None, mode=mode, **kw)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    return y.float().cpu().numpy()


RAGGED = [(1, 16, 16), (5, 48, 144), (16, 272, 528), (17, 144, 1040), (128, 256, 256), (130, 272, 400),
          (200, 400, 1040), (256, 144, 272), (257, 528, 192)]


@pytest.mark.parametrize("M,N,K", RAGGED)
def test_nested_fp16_ragged(M, N, K):
    g = np.random.default_rng(M * 31 + N * 7 + K)
    x16 = synthetic.activations("normal_f16", M, K, g)
    w16 = synthetic.weights_f16(N, K, 0.02, g)
    hi, lo = oracle.nestedfp_split(w16)
    ref, bound = _ref16(x16, hi, lo)
    configs = [{}, {"path": pg.PATH_TILED}, {"path": pg.PATH_TILED, "split_k": 2},
               {"path": pg.PATH_TILED, "tile_n": 256},
               {"path": pg.PATH_TILED_PAIR}]   # {}: automatic (grouped kernel for M <= 256)
    if M <= 128:
        configs += [{"path": pg.PATH_SKINNY}, {"path": pg.PATH_SKINNY, "split_k": 3}]
    for kw in configs:
        assert_within(_run(x16, hi, lo, pg.NESTED_FP16, **kw), ref, bound, f"fp16 M{M} N{N} K{K} {kw}")


@pytest.mark.parametrize("M,N,K", RAGGED)
def test_nested_fp8_ragged(M, N, K):
    g = np.random.default_rng(M * 37 + N * 11 + K)
    x16 = synthetic.activations("normal_f16", M, K, g)
    w16 = synthetic.weights_f16(N, K, 0.02, g)
    hi, _ = oracle.nestedfp_split(w16)
    ref, bound, _, _ = _ref8(x16, hi)
    configs = [{}, {"path": pg.PATH_TILED}, {"path": pg.PATH_TILED, "split_k": 2}, {"path": pg.PATH_TILED_PAIR}]
    if M <= 128:
        configs += [{"path": pg.PATH_SKINNY}, {"path": pg.PATH_SKINNY, "split_k": 4}]
    for kw in configs:
        assert_within(_run(x16, hi, None, pg.NESTED_FP8, **kw), ref, bound, f"fp8 M{M} N{N} K{K} {kw}")


def test_nested_fp16_identity_weights():
    """W = identity (FP16 1.0 = 0x3C00 -> hi 0x3C, lo 0x00) plus a subnormal
    off-diagonal carried only by the lo plane: pins the hi/lo interleave and
    the swizzled layout of the rebuild (any mis-placed byte breaks the bound)."""
    K = 256
    g = np.random.default_rng(3)
    x16 = synthetic.activations("normal_f16", 40, K, g)
    w = np.zeros((K, K), dtype=np.float16)
    w[np.arange(K), np.arange(K)] = 1.0
    w[np.arange(K), (np.arange(K) + 1) % K] = np.float16(2.0 ** -20)   # exercises lo bits (subnormal)
    hi, lo = oracle.nestedfp_split(w)
    ref, bound = _ref16(x16, hi, lo)
    for kw in ({"path": pg.PATH_TILED}, {"path": pg.PATH_SKINNY}, {"path": pg.PATH_TILED_PAIR}):
        y = _run(x16, hi, lo, pg.NESTED_FP16, **kw)
        assert_within(y, ref, bound, str(kw))


@pytest.mark.parametrize("M,N,K", [(600, 784, 528), (2200, 2208, 272), (1030, 4096, 1040)])
def test_nested_fp16_pair_kernel(M, N, K):
    """FP16 mode on SM pairs: each CTA of a pair rebuilds its half of the
    256-row weight tile; the MMA reads both halves.  Cases: a few tiles per
    pair, more tiles than pairs (a second round), and enough tiles for the
    automatic choice to take the pair kernel; ragged M and N throughout."""
    g = np.random.default_rng(M + 3 * N + K)
    x16 = synthetic.activations("normal_f16", M, K, g)
    w16 = synthetic.weights_f16(N, K, 0.02, g)
    hi, lo = oracle.nestedfp_split(w16)
    ref, bound = _ref16(x16, hi, lo)
    first = _run(x16, hi, lo, pg.NESTED_FP16, path=pg.PATH_TILED_PAIR)
    assert_within(first, ref, bound, f"fp16 pair M{M} N{N} K{K}")
    again = _run(x16, hi, lo, pg.NESTED_FP16, path=pg.PATH_TILED_PAIR, flags=pg.FLAG_OVERLAP_PREVIOUS)
    np.testing.assert_array_equal(first, again)
    assert_within(_run(x16, hi, lo, pg.NESTED_FP16), ref, bound, f"fp16 auto M{M} N{N} K{K}")


@pytest.mark.parametrize("shape_idx", [0, 1])
@pytest.mark.parametrize("m_idx", [0, 1, 2, 3])
def test_nested7b_full_size_both_modes(shape_idx, m_idx):
    """Both modes on the same stored planes at the workload's sizes, checked
    on sampled rows and columns."""
    x16 = synthetic.acts("nested7b", shape_idx, m_idx)
    w16 = synthetic.weights("nested7b", shape_idx)
    M, K = x16.shape
    N = w16.shape[0]
    hi_g, lo_g = pg.nestedfp_split(_to(w16))
    xt = _to(x16)
    y16 = pg.nestedfp_linear(xt, hi_g, lo_g, mode=pg.NESTED_FP16)
    y8 = pg.nestedfp_linear(xt, hi_g, None, mode=pg.NESTED_FP8)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    rng = np.random.default_rng(1)
    ns = np.sort(rng.choice(N, 256, replace=False))
    ms = np.sort(rng.choice(M, min(M, 12), replace=False))
    hi, lo = oracle.nestedfp_split(w16[ns])
    np.testing.assert_array_equal(hi_g.cpu().numpy()[ns], hi)
    np.testing.assert_array_equal(lo_g.cpu().numpy()[ns], lo)
    ref, bound = _ref16(x16[ms], hi, lo)
    assert_within(y16.float().cpu().numpy()[np.ix_(ms, ns)], ref, bound, f"fp16 full M={M}")
    ref8, bound8, _, _ = _ref8(x16[ms], hi)
    assert_within(y8.float().cpu().numpy()[np.ix_(ms, ns)], ref8, bound8, f"fp8 full M={M}")


@pytest.mark.parametrize("mode", ["fp16", "fp8"])
def test_chained_layers_with_overlap_flag(mode):
    """Four NestedFP layers where each layer's input is the previous layer's
    output, enqueued back to back with FLAG_OVERLAP_PREVIOUS (each call may
    start while the previous layer is finishing).  The results must equal the
    same chain run with a synchronisation between layers, bit for bit: the
    overlap may only move weight loads earlier, never activation reads."""
    g = np.random.default_rng(11)
    M, D = 8, 1024
    m = pg.NESTED_FP16 if mode == "fp16" else pg.NESTED_FP8
    planes = []
    for _ in range(4):
        w = synthetic.weights_f16(D, D, 0.03, g)
        planes.append(pg.nestedfp_split(_to(w)))
    x0 = _to(synthetic.activations("normal_f16", M, D, g))
    torch.cuda.synchronize()

    def run(flags, sync):
        x = x0
        ys = []
        for hi, lo in planes:
            y = pg.nestedfp_linear(x, hi, lo if m == pg.NESTED_FP16 else None, mode=m, flags=flags)
            if sync:
                torch.cuda.synchronize()
            ys.append(y)
            x = y
        torch.cuda.synchronize()
        return [t.cpu().numpy() for t in ys]

    ref = run(0, True)
    for _ in range(3):
        got = run(pg.FLAG_OVERLAP_PREVIOUS, False)
        for a, b in zip(got, ref):
            np.testing.assert_array_equal(a.view(np.uint16), b.view(np.uint16))
    assert pg.device_status() == pg.OK


@pytest.mark.parametrize("M,N,K", [(1, 128, 4096), (16, 528, 1040), (30, 272, 2048)])
@pytest.mark.parametrize("mode", ["fp16", "fp8"])
def test_nested_streamk(M, N, K, mode):
    g = np.random.default_rng(M + N + K)
    x16 = synthetic.activations("normal_f16", M, K, g)
    w16 = synthetic.weights_f16(N, K, 0.02, g)
    hi, lo = oracle.nestedfp_split(w16)
    if mode == "fp16":
        ref, bound = _ref16(x16, hi, lo)
        m = pg.NESTED_FP16
    else:
        ref, bound, _, _ = _ref8(x16, hi)
        m = pg.NESTED_FP8
    ws = torch.zeros(pg.nestedfp_linear_workspace_size(M, N, K, m), dtype=torch.uint8, device=DEV)
    for _ in range(2):
        y = _run(x16, hi, lo if m == pg.NESTED_FP16 else None, m, workspace=ws, path=pg.PATH_STREAMK)
        assert_within(y, ref, bound, f"{mode} stream-K M{M} N{N} K{K}")


NESTED_GROUP = [(1, 528, 512), (16, 272, 1040), (17, 400, 144), (64, 1040, 528), (128, 256, 256),
                (130, 272, 400), (256, 144, 272), (300, 528, 192)]   # (M, N, K): every token class, one layer past it


@pytest.mark.parametrize("mode", ["fp16", "fp8"])
def test_nested_group_matches_the_oracle(mode):
    """pgf8_nestedfp_linear_group: layers of every token-tile class in one
    group (two grouped launches) and one past it, run twice: every layer
    within the bound of the oracle's, FP8 mode's codes and scales bit-exact,
    the second call bit-identical, the flags left zero."""
    m = pg.NESTED_FP16 if mode == "fp16" else pg.NESTED_FP8
    g = np.random.default_rng(41 if mode == "fp16" else 43)
    entries, host = [], []
    for (M, N, K) in NESTED_GROUP:
        x16 = synthetic.activations("normal_f16", M, K, g)
        w16 = synthetic.weights_f16(N, K, 0.02, g)
        hi, lo = oracle.nestedfp_split(w16)
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device=DEV)
        ws = None
        if m == pg.NESTED_FP8:
            ws = torch.zeros(pg.nestedfp_linear_workspace_size(M, N, K, m), dtype=torch.uint8, device=DEV)
        entries.append((_to(x16), _to(hi), _to(lo) if m == pg.NESTED_FP16 else None, y, ws))
        host.append((x16, hi, lo))
    grp = pg.NestedLayerGroup(entries, mode=m)
    grp.run()
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    first = [e[3].clone() for e in entries]
    for i, ((xt, _, _, y, ws), (x16, hi, lo)) in enumerate(zip(entries, host)):
        M, K = x16.shape
        if m == pg.NESTED_FP16:
            ref, bound = _ref16(x16, hi, lo)
        else:
            ref, bound, aq0, sa0 = _ref8(x16, hi)
            aq, sa = pg.dynamic_workspace_views(ws, M, K)
            assert np.array_equal(aq.cpu().numpy(), aq0), f"layer {i}: codes"
            assert np.array_equal(sa.cpu().numpy().view(np.uint32), sa0.view(np.uint32)), f"layer {i}: scales"
        assert_within(y.float().cpu().numpy(), ref, bound, f"{mode} group layer {i} (M={M})")
    for e in entries:
        e[3].fill_(float("nan"))
    grp.run(flags=pg.FLAG_OVERLAP_PREVIOUS)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    for i, (e, f) in enumerate(zip(entries, first)):
        assert torch.equal(e[3].view(torch.int16), f.view(torch.int16)), f"layer {i} differs on the second call"
    assert not grp.group_workspace[:1024].any(), "flag words not cleared"
