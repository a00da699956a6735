"""GPU parity of the grouped dynamic FP8 linear (pgf8_fp8_linear_dynamic_group):
every layer's codes and scales bit-exact against the oracle, every output
within the layer's stated bound |y - ref| <= 2^-8 |ref| + 1e-4 sqrt(K) A_m W_n
against the oracle's binary64 layer.  The cases cover every token-tile class
of the grouped kernel (M <= 16, 32, 64, 128, 256) in one group, layers past it
(M > 256, per-layer kernels), ragged N and K, groups small enough that one
weight tile is shared by several CTAs and large enough that a CTA walks
many tiles and crosses layer boundaries, and repeated calls (the flag words
must be left zero, and the results must repeat bit for bit)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from _parity import assert_within, fp8_row_max, linear_bound

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _make_group(shapes, seed, recipe="student_t3"):
    g = np.random.default_rng(seed)
    layers, host = [], []
    for (M, K, N) in shapes:
        x = synthetic.activations(recipe, M, K, g)
        w = synthetic.weights_f16(N, K, 0.02, g)
        wq, sw = pg.fp8_quantize_rows(torch.from_numpy(w).to(DEV))
        xt = torch.from_numpy(x).to(DEV)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        ws = torch.zeros(pg.fp8_linear_dynamic_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
        layers.append((xt, wq, sw, y, ws))
        host.append((x, w))
    return layers, host


def _check_layer(i, layer, x, w, ns=None):
    xt, wq_d, sw_d, y, ws = layer
    M, K = x.shape
    aq0, sa0 = oracle.quantize_rows(x)
    aq, sa = pg.dynamic_workspace_views(ws, M, K)
    assert np.array_equal(aq.cpu().numpy(), aq0), f"layer {i}: codes differ from the oracle"
    assert np.array_equal(sa.cpu().numpy().view(np.uint32), sa0.view(np.uint32)), f"layer {i}: scales"
    wsub = w if ns is None else w[ns]
    wq0, sw0 = oracle.quantize_rows(wsub)
    ref = oracle.fp8_linear(aq0, sa0, wq0, sw0)
    bound = linear_bound(ref, K, fp8_row_max(aq0, sa0), fp8_row_max(wq0, sw0))
    got = y.float().cpu().numpy()
    if ns is not None:
        got = got[:, ns]
    assert_within(got, ref, bound, f"group layer {i} (M={M} K={K} N={w.shape[0]})")


MIXED = [  # (M, K, N): all token classes, ragged N and K, one layer past the grouped kernel
    (1, 512, 528), (4, 272, 400), (8, 1040, 144), (16, 528, 1040), (17, 400, 272), (32, 1008, 656),
    (33, 144, 912), (64, 656, 528), (65, 272, 1296), (100, 528, 400), (128, 1024, 1024), (160, 400, 528),
    (256, 656, 272), (300, 400, 528),
]


def test_group_mixed_token_classes():
    layers, host = _make_group(MIXED, 11)
    grp = pg.LayerGroup(layers)
    grp.run()
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    first = [l[3].clone() for l in layers]
    for i, (layer, (x, w)) in enumerate(zip(layers, host)):
        _check_layer(i, layer, x, w)
    # the flags left by the first call are zero: the second call repeats it bit for bit
    for l in layers:
        l[3].fill_(float("nan"))
    grp.run()
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    for i, (l, f) in enumerate(zip(layers, first)):
        assert torch.equal(l[3].view(torch.int16), f.view(torch.int16)), f"layer {i} differs on the second call"
    assert not grp.group_workspace[:1024].any(), "flag words not cleared"


@pytest.mark.parametrize("shapes", [
    [(8, 4096, 512)],                       # 4 tiles x 32 k-blocks: tiles shared by many CTAs
    [(1, 16, 16), (2, 32, 16)],             # fewer units than SMs: one unit per CTA
    [(8, 11008, 256), (3, 128, 2048)],      # long K; short layer after it
])
def test_group_shared_tiles(shapes):
    layers, host = _make_group(shapes, 5 + len(shapes), recipe="normal_outl_0p5pct_x30")
    grp = pg.LayerGroup(layers)
    for _ in range(3):
        grp.run()
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    for i, (layer, (x, w)) in enumerate(zip(layers, host)):
        _check_layer(i, layer, x, w)
    assert not grp.group_workspace[:1024].any()


@pytest.mark.slow
def test_group_decode7b_full_size_sampled():
    """The decode7b step as one group (12 layers, 606 MB of weights at full
    size), checked on 384 sampled output channels of every layer."""
    wl = synthetic.WORKLOADS["decode7b"]
    layers, host = [], []
    for mi, M in enumerate(wl.ms):
        for si, (K, N, _) in enumerate(wl.shapes):
            x = synthetic.acts("decode7b", si, mi)
            w = synthetic.weights("decode7b", si, copy=mi)
            wq, sw = pg.fp8_quantize_rows(torch.from_numpy(w).to(DEV))
            y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
            ws = torch.zeros(pg.fp8_linear_dynamic_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
            layers.append((torch.from_numpy(x).to(DEV), wq, sw, y, ws))
            host.append((x, w))
    grp = pg.LayerGroup(layers)
    grp.run()
    grp.run()
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    rng = np.random.default_rng(3)
    for i, (layer, (x, w)) in enumerate(zip(layers, host)):
        ns = np.sort(rng.choice(w.shape[0], 384, replace=False))
        _check_layer(i, layer, x, w, ns)


def test_group_several_large_layers_after_a_producer():
    """Several layers past the grouped kernel: from the second one on, each
    layer's quantisation runs while the previous layer's GEMM computes.  The
    activations are written by a device kernel right before the call (the
    call's first launch overlaps it), and the last layer's activations are
    the ones written last: every layer must still see its final inputs."""
    shapes = [(4, 1024, 528), (200, 1024, 528), (260, 528, 1040), (300, 1008, 272), (33, 400, 144),
              (400, 656, 400)]
    layers, host = _make_group(shapes, 23)
    srcs = [torch.from_numpy(x).to(DEV) for (x, _) in host]
    for l in layers:
        l[0].zero_()
    grp = pg.LayerGroup(layers)
    stream = torch.cuda.current_stream()
    for _ in range(2):
        for l, s in zip(layers, srcs):
            l[0].copy_(s)                       # the producer kernels, in stream order
        grp.run(flags=pg.FLAG_OVERLAP_PREVIOUS, stream=stream)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    for i, (layer, (x, w)) in enumerate(zip(layers, host)):
        _check_layer(i, layer, x, w)


def _oracle_linear_threaded(aq, sa, wq, sw):
    """The oracle's binary64 layer, its output channels split over host
    threads (the oracle is a C library called through ctypes, which releases
    the interpreter lock; the arithmetic is unchanged)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    n = wq.shape[0]
    parts = [p for p in np.array_split(np.arange(n), os.cpu_count() or 1) if p.size]
    with ThreadPoolExecutor(len(parts)) as ex:
        outs = list(ex.map(lambda p: oracle.fp8_linear(aq, sa, wq[p[0]:p[-1] + 1], sw[p[0]:p[-1] + 1]), parts))
    return np.concatenate(outs, axis=1)


@pytest.mark.slow
def test_group_llama70b_streaming_layers_full_size_sampled():
    """The llama70b step's weight-streaming part at full size: the four 70B
    shapes at M = 1, 2, ..., 256 (36 layers, the benchmark's two grouped
    launches), codes and scales of every layer bit-exact, outputs of every
    token on 64 sampled output channels per layer within the bound."""
    wl = synthetic.WORKLOADS["llama70b"]
    ms = [m for m in wl.ms if m <= 256]
    weights = {}
    for si, (K, N, _) in enumerate(wl.shapes):
        w = synthetic.weights("llama70b", si)
        wq, sw = pg.fp8_quantize_rows(torch.from_numpy(w).to(DEV))
        weights[si] = (w, wq, sw)
    layers, host = [], []
    for mi, M in enumerate(ms):
        for si, (K, N, _) in enumerate(wl.shapes):
            x = synthetic.acts("llama70b", si, mi)
            w, wq, sw = weights[si]
            y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
            ws = torch.zeros(pg.fp8_linear_dynamic_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
            layers.append((torch.from_numpy(x).to(DEV), wq, sw, y, ws))
            host.append((x, si))
    grp = pg.LayerGroup(layers)
    grp.run()
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    rng = np.random.default_rng(4)
    wq0s = {}
    for i, (layer, (x, si)) in enumerate(zip(layers, host)):
        w = weights[si][0]
        if si not in wq0s:
            ns = np.sort(rng.choice(w.shape[0], 64, replace=False))
            wq0s[si] = (ns,) + oracle.quantize_rows(w[ns])
        ns, wq0, sw0 = wq0s[si]
        M, K = x.shape
        aq0, sa0 = oracle.quantize_rows(x)
        aq, sa = pg.dynamic_workspace_views(layer[4], M, K)
        assert np.array_equal(aq.cpu().numpy(), aq0), f"layer {i}: codes"
        assert np.array_equal(sa.cpu().numpy().view(np.uint32), sa0.view(np.uint32)), f"layer {i}: scales"
        ref = _oracle_linear_threaded(aq0, sa0, wq0, sw0)
        bound = linear_bound(ref, K, fp8_row_max(aq0, sa0), fp8_row_max(wq0, sw0))
        assert_within(layer[3].float().cpu().numpy()[:, ns], ref, bound, f"70B layer {i} (M={M}, shape {si})")


PAIR_GROUP = [(1, 512, 528), (100, 272, 400), (129, 1040, 144), (256, 656, 272), (300, 400, 528),
              (600, 1008, 784), (513, 144, 1040)]   # (M, K, N): ragged M, N and K; one-tile and many-tile layers


def test_fp8_linear_group_pre_quantised():
    """pgf8_fp8_linear_group: the codes and scales the oracle gives, several
    layers in one launch on SM pairs; every output within the layer's bound
    of the oracle's binary64 layer, and equal to a second call bit for bit."""
    g = np.random.default_rng(31)
    ops, host = [], []
    for (M, K, N) in PAIR_GROUP:
        x = synthetic.activations("student_t3", M, K, g)
        w = synthetic.weights_f16(N, K, 0.02, g)
        aq0, sa0 = oracle.quantize_rows(x)
        wq0, sw0 = oracle.quantize_rows(w)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)  # noqa: E731
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        ops.append((t(aq0), t(sa0), t(wq0), t(sw0), y))
        host.append((aq0, sa0, wq0, sw0))
    pg.fp8_linear_group(ops)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    first = [o[4].clone() for o in ops]
    for i, (o, (aq0, sa0, wq0, sw0)) in enumerate(zip(ops, host)):
        ref = oracle.fp8_linear(aq0, sa0, wq0, sw0)
        bound = linear_bound(ref, aq0.shape[1], fp8_row_max(aq0, sa0), fp8_row_max(wq0, sw0))
        assert_within(o[4].float().cpu().numpy(), ref, bound, f"pair-group layer {i}")
    pg.fp8_linear_group(ops, flags=pg.FLAG_OVERLAP_PREVIOUS)
    torch.cuda.synchronize()
    for i, (o, f) in enumerate(zip(ops, first)):
        assert torch.equal(o[4].view(torch.int16), f.view(torch.int16)), f"layer {i} differs on the second call"


def test_group_more_large_layers_than_one_launch_takes():
    """40 layers with M > 128 in one grouped call: two quantisation and
    tiled launches (32 layers per launch), each layer checked."""
    shapes = [(129 + 7 * i, 144 + 16 * (i % 5), 144 + 32 * (i % 3)) for i in range(40)]
    layers, host = _make_group(shapes, 37)
    grp = pg.LayerGroup(layers)
    grp.run()
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    for i, (layer, (x, w)) in enumerate(zip(layers, host)):
        _check_layer(i, layer, x, w)


@pytest.mark.slow
def test_group_llama70b_tiled_layers_full_size_sampled():
    """The llama70b step's tiled part at full size: the four 70B shapes at
    M = 256, 512, ..., 4096 (20 layers, one quantisation launch and one tiled
    launch on SM pairs), codes and scales bit-exact on 6 sampled rows of
    every layer, outputs of those rows on 64 sampled channels within the
    bound."""
    wl = synthetic.WORKLOADS["llama70b"]
    mis = [mi for mi, m in enumerate(wl.ms) if m >= 256]
    weights = {}
    for si, (K, N, _) in enumerate(wl.shapes):
        w = synthetic.weights("llama70b", si)
        wq, sw = pg.fp8_quantize_rows(torch.from_numpy(w).to(DEV))
        weights[si] = (w, wq, sw)
    layers, host = [], []
    for mi in mis:
        M = wl.ms[mi]
        for si, (K, N, _) in enumerate(wl.shapes):
            x = synthetic.acts("llama70b", si, mi)
            w, wq, sw = weights[si]
            y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
            ws = torch.zeros(pg.fp8_linear_dynamic_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
            layers.append((torch.from_numpy(x).to(DEV), wq, sw, y, ws))
            host.append((x, si))
    grp = pg.LayerGroup(layers)
    grp.run()
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    rng = np.random.default_rng(8)
    wq0s = {}
    for i, (layer, (x, si)) in enumerate(zip(layers, host)):
        w = weights[si][0]
        if si not in wq0s:
            ns = np.sort(rng.choice(w.shape[0], 64, replace=False))
            wq0s[si] = (ns,) + oracle.quantize_rows(w[ns])
        ns, wq0, sw0 = wq0s[si]
        M, K = x.shape
        ms = np.sort(rng.choice(M, 6, replace=False))
        aq0, sa0 = oracle.quantize_rows(x[ms])
        aq, sa = pg.dynamic_workspace_views(layer[4], M, K)
        assert np.array_equal(aq.cpu().numpy()[ms], aq0), f"layer {i}: codes"
        assert np.array_equal(sa.cpu().numpy()[ms].view(np.uint32), sa0.view(np.uint32)), f"layer {i}: scales"
        ref = oracle.fp8_linear(aq0, sa0, wq0, sw0)
        bound = linear_bound(ref, K, fp8_row_max(aq0, sa0), fp8_row_max(wq0, sw0))
        got = layer[3].float().cpu().numpy()[np.ix_(ms, ns)]
        assert_within(got, ref, bound, f"70B tiled layer {i} (M={M}, shape {si})")
