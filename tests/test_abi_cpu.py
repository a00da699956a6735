"""The C-ABI library builds, loads and exports every declared symbol, and its
host-side argument checks reject bad calls before anything touches a GPU
(CPU only: no call here reaches a CUDA runtime function)."""
import ctypes
import subprocess

import pytest

import precision_gemm_fp8_b200 as pg


def test_every_declared_symbol_is_exported():
    names = pg.header_symbols()
    assert len(names) >= 15
    for n in names:
        assert hasattr(pg.lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", pg.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing


def test_status_strings_and_version():
    for s in range(6):
        assert pg.lib.pgf8_status_str(s)
    assert pg.lib.pgf8_status_str(99) == b"unknown status"
    assert pg.version() >= 100


def test_workspace_sizes():
    # stream-K flags + partial slots for M <= 32, nothing above
    assert pg.lib.pgf8_fp8_linear_workspace_size(16, 512, 512) >= 1024 + 256 * 16 * 128 * 4
    assert pg.lib.pgf8_fp8_linear_workspace_size(32, 512, 512) >= 1024 + 256 * 32 * 128 * 4
    assert pg.lib.pgf8_fp8_linear_workspace_size(33, 512, 512) == 0
    for M in (3, 40):
        c0 = pg.lib.pgf8_fp8_linear_dynamic_codes_offset(M, 4096)
        off = pg.lib.pgf8_fp8_linear_dynamic_scales_offset(M, 4096)
        assert c0 >= 1024 and c0 % 256 == 0          # synchronisation words first, for every shape
        assert off % 256 == 0 and off >= c0 + M * 4096
        ws = pg.lib.pgf8_fp8_linear_dynamic_workspace_size(M, 4096, 4096)
        assert ws >= off + 4 * M and ws % 256 == 0
    # NestedFP FP16 mode up to 256 tokens: the grouped kernel's flags and partial slots
    assert pg.nestedfp_linear_workspace_size(64, 4096, 4096, pg.NESTED_FP16) == 1024 + 256 * 64 * 128 * 4
    assert pg.nestedfp_linear_workspace_size(300, 4096, 4096, pg.NESTED_FP16) == 0
    assert pg.nestedfp_linear_workspace_size(8, 4096, 4096, pg.NESTED_FP16) == \
        pg.lib.pgf8_fp8_linear_workspace_size(8, 4096, 4096)
    assert pg.nestedfp_linear_workspace_size(8, 4096, 4096, pg.NESTED_FP8) == \
        pg.lib.pgf8_fp8_linear_dynamic_workspace_size(8, 4096, 4096)


def test_last_cuda_error_starts_clear():
    e = ctypes.c_int(-1)
    assert pg.lib.pgf8_last_cuda_error(ctypes.byref(e)) == pg.OK
    assert e.value == 0
    assert pg.lib.pgf8_last_cuda_error(None) == pg.ERR_INVALID_ARG


A16 = 0x10000      # fake, 16-byte aligned addresses: argument checks fail before use
B16 = 0x20000
C16 = 0x30000
D16 = 0x40000
MIS = 0x10008      # 8-byte aligned only


@pytest.mark.parametrize("M,N,K,expect", [
    (0, 512, 512, pg.ERR_INVALID_ARG),      # M >= 1
    (16, 8, 512, pg.ERR_INVALID_ARG),       # N >= 16
    (16, 512, 8, pg.ERR_INVALID_ARG),       # K >= 16
    (16, 520, 512, pg.ERR_ALIGNMENT),       # N % 16
    (16, 512, 520, pg.ERR_ALIGNMENT),       # K % 16
])
def test_fp8_linear_rejects_bad_dims(M, N, K, expect):
    st = pg.lib.pgf8_fp8_linear(A16, B16, M, K, C16, D16, N, A16, None, 0, None)
    assert st == expect


def test_fp8_linear_rejects_null_and_misaligned():
    assert pg.lib.pgf8_fp8_linear(None, B16, 16, 512, C16, D16, 512, A16, None, 0, None) == pg.ERR_INVALID_ARG
    assert pg.lib.pgf8_fp8_linear(A16, B16, 16, 512, C16, D16, 512, None, None, 0, None) == pg.ERR_INVALID_ARG
    assert pg.lib.pgf8_fp8_linear(MIS, B16, 16, 512, C16, D16, 512, A16, None, 0, None) == pg.ERR_ALIGNMENT
    assert pg.lib.pgf8_fp8_linear(A16, B16, 16, 512, MIS, D16, 512, A16, None, 0, None) == pg.ERR_ALIGNMENT
    assert pg.lib.pgf8_fp8_linear(A16, B16 + 2, 16, 512, C16, D16, 512, A16, None, 0, None) == pg.ERR_ALIGNMENT


def test_fp8_linear_rejects_bad_options():
    bad = [pg.LinearOpts(7, 0, 0, 0), pg.LinearOpts(pg.PATH_SKINNY, 9, 0, 0),
           pg.LinearOpts(pg.PATH_SKINNY, 0, 48, 0), pg.LinearOpts(pg.PATH_TILED, 0, 64, 0),
           pg.LinearOpts(pg.PATH_SKINNY, 0, 16, 0)]
    Ms = [16, 16, 16, 16, 17]   # the last: tile_n 16 cannot hold 17 tokens
    for o, M in zip(bad, Ms):
        st = pg.lib.pgf8_fp8_linear_ex(A16, B16, M, 512, C16, D16, 512, A16, None, 0, ctypes.byref(o), None)
        assert st in (pg.ERR_INVALID_ARG, pg.ERR_UNSUPPORTED), (o.path, o.split_k, o.tile_n, st)
    big = pg.LinearOpts(pg.PATH_SKINNY, 0, 0, 0)
    assert pg.lib.pgf8_fp8_linear_ex(A16, B16, 129, 512, C16, D16, 512, A16, None, 0, ctypes.byref(big),
                                     None) == pg.ERR_UNSUPPORTED


def test_quantize_rejects_bad_args():
    q = pg.lib.pgf8_fp8_quantize_rows
    assert q(None, pg.F32, 4, 64, 64, B16, C16, 0, None) == pg.ERR_INVALID_ARG
    assert q(A16, pg.BF16, 4, 64, 64, B16, C16, 0, None) == pg.ERR_UNSUPPORTED
    assert q(A16, pg.F32, 4, 60, 64, B16, C16, 0, None) == pg.ERR_ALIGNMENT      # cols % 16
    assert q(A16, pg.F32, 4, 8, 64, B16, C16, 0, None) == pg.ERR_INVALID_ARG      # cols >= 16
    assert q(A16, pg.F32, 4, 64, 32, B16, C16, 0, None) == pg.ERR_INVALID_ARG    # ldx < cols
    assert q(A16, pg.F32, 4, 64, 66, B16, C16, 0, None) == pg.ERR_ALIGNMENT      # row stride not 16 B
    assert q(MIS, pg.F32, 4, 64, 64, B16, C16, 0, None) == pg.ERR_ALIGNMENT
    assert q(A16, pg.F32, 4, 64, 64, B16, C16 + 2, 0, None) == pg.ERR_ALIGNMENT
    assert q(A16, pg.F32, 4, 64, 64, B16, C16, 5, None) == pg.ERR_INVALID_ARG
    assert q(None, pg.F32, 0, 64, 64, None, None, 0, None) == pg.OK              # no rows: no-op


def test_dynamic_and_nested_reject_bad_args():
    d = pg.lib.pgf8_fp8_linear_dynamic
    small_ws = 16
    assert d(A16, pg.F32, 4, 512, 512, B16, C16, 512, D16, A16, small_ws, None, None) == pg.ERR_INVALID_ARG
    assert d(A16, pg.F32, 4, 512, 512, B16, C16, 512, D16, None, 1 << 20, None, None) == pg.ERR_INVALID_ARG
    n = pg.lib.pgf8_nestedfp_linear
    assert n(A16, 4, 512, B16, None, 512, pg.NESTED_FP16, D16, None, 0, None) == pg.ERR_INVALID_ARG
    assert n(A16, 4, 512, B16, C16, 512, 7, D16, None, 0, None) == pg.ERR_INVALID_ARG
    assert n(A16, 4, 512, B16, None, 512, pg.NESTED_FP8, D16, None, 0, None) == pg.ERR_INVALID_ARG
    # FP16 mode on SM pairs: 256-wide tiles only; refused before any device call
    pair128 = pg.LinearOpts(pg.PATH_TILED_PAIR, 0, 128, 0)
    assert pg.lib.pgf8_nestedfp_linear_ex(A16, 300, 512, B16, C16, 512, pg.NESTED_FP16, D16, None, 0,
                                          ctypes.byref(pair128), None) == pg.ERR_UNSUPPORTED
    s = pg.lib.pgf8_nestedfp_split
    assert s(None, 16, 16, B16, C16, None) == pg.ERR_INVALID_ARG
    assert s(A16, 3, 5, B16, C16, None) == pg.ERR_ALIGNMENT


def test_streamk_path_argument_checks():
    o = pg.LinearOpts(pg.PATH_STREAMK, 0, 0, 0)
    # no workspace: rejected before launch
    assert pg.lib.pgf8_fp8_linear_ex(A16, B16, 8, 512, C16, D16, 512, A16, None, 0, ctypes.byref(o),
                                     None) == pg.ERR_INVALID_ARG
    # workspace too small
    assert pg.lib.pgf8_fp8_linear_ex(A16, B16, 8, 512, C16, D16, 512, A16, D16, 4096, ctypes.byref(o),
                                     None) == pg.ERR_INVALID_ARG
    # M > 32 is not served by the stream-K kernel
    assert pg.lib.pgf8_fp8_linear_ex(A16, B16, 33, 512, C16, D16, 512, A16, D16, 1 << 24, ctypes.byref(o),
                                     None) == pg.ERR_UNSUPPORTED
    # misaligned workspace
    assert pg.lib.pgf8_fp8_linear_ex(A16, B16, 8, 512, C16, D16, 512, A16, D16 + 8, 1 << 24, ctypes.byref(o),
                                     None) == pg.ERR_ALIGNMENT


def test_dynamic_many_checks_every_layer_first():
    good = pg.Fp8Layer(A16, pg.F32, 0, 4, 512, 512, 512, B16, C16, D16, A16, 1 << 24)
    bad = pg.Fp8Layer(A16, pg.F32, 0, 4, 520, 520, 512, B16, C16, D16, A16, 1 << 24)   # K % 16
    arr = (pg.Fp8Layer * 3)(good, bad, good)
    # the invalid second layer is reported before anything (including layer 1) is enqueued
    assert pg.lib.pgf8_fp8_linear_dynamic_many(arr, 3, None, None) == pg.ERR_ALIGNMENT
    assert pg.lib.pgf8_fp8_linear_dynamic_many(None, 2, None, None) == pg.ERR_INVALID_ARG
    assert pg.lib.pgf8_fp8_linear_dynamic_many(None, 0, None, None) == pg.OK
    assert pg.lib.pgf8_fp8_linear_dynamic_many(arr, -1, None, None) == pg.ERR_INVALID_ARG


def test_dynamic_group_checks_layers_aliasing_and_workspace_first():
    """pgf8_fp8_linear_dynamic_group: every layer checked, independence (no
    output or workspace overlapping another layer's buffers) and the group
    workspace checked, all before anything is enqueued."""
    f = pg.lib.pgf8_fp8_linear_dynamic_group
    ws_need = pg.lib.pgf8_fp8_linear_group_workspace_size(4)
    assert ws_need == pg.lib.pgf8_fp8_linear_group_workspace_size(16) > 1024
    assert pg.lib.pgf8_fp8_linear_group_workspace_size(256) == pg.lib.pgf8_fp8_linear_group_workspace_size(4096)
    assert pg.lib.pgf8_fp8_linear_group_workspace_size(0) == 1024
    base = 1 << 32
    x0, x1, y0, y1, w0, w1 = (base + i * (1 << 26) for i in range(6))
    wsp0, wsp1, gws = base + 6 * (1 << 26), base + 7 * (1 << 26), base + 8 * (1 << 26)
    l0 = pg.Fp8Layer(x0, pg.F32, 0, 4, 512, 512, 512, base + 9 * (1 << 26), C16, y0, wsp0, 1 << 24)
    l1 = pg.Fp8Layer(x1, pg.F32, 0, 4, 512, 512, 512, base + 10 * (1 << 26), C16, y1, wsp1, 1 << 24)
    bad = pg.Fp8Layer(x1, pg.F32, 0, 4, 520, 520, 512, base + 10 * (1 << 26), C16, y1, wsp1, 1 << 24)   # K % 16
    arr = (pg.Fp8Layer * 2)(l0, bad)
    assert f(arr, 2, gws, ws_need, None, None) == pg.ERR_ALIGNMENT
    # layer 1 reads layer 0's output: not independent
    dep = pg.Fp8Layer(y0, pg.F32, 0, 4, 512, 512, 512, base + 10 * (1 << 26), C16, y1, wsp1, 1 << 24)
    assert f((pg.Fp8Layer * 2)(l0, dep), 2, gws, ws_need, None, None) == pg.ERR_INVALID_ARG
    # two layers sharing one workspace
    share = pg.Fp8Layer(x1, pg.F32, 0, 4, 512, 512, 512, base + 10 * (1 << 26), C16, y1, wsp0, 1 << 24)
    assert f((pg.Fp8Layer * 2)(l0, share), 2, gws, ws_need, None, None) == pg.ERR_INVALID_ARG
    ok2 = (pg.Fp8Layer * 2)(l0, l1)
    assert f(ok2, 2, None, 0, None, None) == pg.ERR_INVALID_ARG            # group workspace missing
    assert f(ok2, 2, gws, ws_need - 16, None, None) == pg.ERR_INVALID_ARG  # too small
    assert f(ok2, 2, gws + 8, ws_need, None, None) == pg.ERR_ALIGNMENT
    assert f(None, 2, gws, ws_need, None, None) == pg.ERR_INVALID_ARG
    assert f(None, 0, None, 0, None, None) == pg.OK


def test_fp8_linear_group_checks_first():
    """pgf8_fp8_linear_group: every layer's arguments and the outputs'
    independence checked before anything is enqueued; explicit kernel
    options refused."""
    f = pg.lib.pgf8_fp8_linear_group
    base = 1 << 34
    aq0, sa0, wq, sw, y0, y1, aq1, sa1 = (base + i * (1 << 26) for i in range(8))
    l0 = pg.Fp8GemmLayer(aq0, sa0, wq, sw, y0, 300, 512, 512)
    l1 = pg.Fp8GemmLayer(aq1, sa1, wq, sw, y1, 600, 512, 512)      # layers may share weights
    assert f(None, 0, None, None) == pg.OK
    assert f(None, 2, None, None) == pg.ERR_INVALID_ARG
    bad_k = pg.Fp8GemmLayer(aq1, sa1, wq, sw, y1, 600, 520, 512)
    assert f((pg.Fp8GemmLayer * 2)(l0, bad_k), 2, None, None) == pg.ERR_ALIGNMENT
    mis = pg.Fp8GemmLayer(aq1 + 8, sa1, wq, sw, y1, 600, 512, 512)
    assert f((pg.Fp8GemmLayer * 2)(l0, mis), 2, None, None) == pg.ERR_ALIGNMENT
    no_sw = pg.Fp8GemmLayer(aq1, sa1, wq, None, y1, 600, 512, 512)
    assert f((pg.Fp8GemmLayer * 2)(l0, no_sw), 2, None, None) == pg.ERR_INVALID_ARG
    same_y = pg.Fp8GemmLayer(aq1, sa1, wq, sw, y0, 600, 512, 512)
    assert f((pg.Fp8GemmLayer * 2)(l0, same_y), 2, None, None) == pg.ERR_INVALID_ARG
    into_w = pg.Fp8GemmLayer(aq1, sa1, wq, sw, wq + 4096, 600, 512, 512)   # output over the weights
    assert f((pg.Fp8GemmLayer * 2)(l0, into_w), 2, None, None) == pg.ERR_INVALID_ARG
    o = pg.LinearOpts(pg.PATH_TILED, 0, 0, 0)
    assert f((pg.Fp8GemmLayer * 2)(l0, l1), 2, ctypes.byref(o), None) == pg.ERR_UNSUPPORTED


def test_nested_group_checks_layers_aliasing_and_workspace_first():
    """pgf8_nestedfp_linear_group: the mode, every layer (FP8 mode: with its
    workspace), independence and the group workspace checked before anything
    is enqueued."""
    f = pg.lib.pgf8_nestedfp_linear_group
    ws_need = pg.lib.pgf8_fp8_linear_group_workspace_size(64)
    base = 1 << 33
    x0, x1, y0, y1, hi, lo, wsp0, wsp1, gws = (base + i * (1 << 27) for i in range(9))
    lw = pg.nestedfp_linear_workspace_size(64, 512, 512, pg.NESTED_FP8)
    l0 = pg.NestedLayer(x0, hi, lo, y0, wsp0, lw, 64, 512, 512)
    l1 = pg.NestedLayer(x1, hi, lo, y1, wsp1, lw, 8, 512, 512)     # layers may share weight planes
    ok2 = (pg.NestedLayer * 2)(l0, l1)
    for mode in (pg.NESTED_FP16, pg.NESTED_FP8):
        assert f(ok2, 2, 7, gws, ws_need, None, None) == pg.ERR_INVALID_ARG          # mode
        assert f(ok2, 2, mode, None, 0, None, None) == pg.ERR_INVALID_ARG           # group workspace missing
        assert f(ok2, 2, mode, gws, ws_need - 16, None, None) == pg.ERR_INVALID_ARG
        assert f(ok2, 2, mode, gws + 8, ws_need, None, None) == pg.ERR_ALIGNMENT
        dep = pg.NestedLayer(y0, hi, lo, y1, wsp1, lw, 8, 512, 512)                 # reads layer 0's output
        assert f((pg.NestedLayer * 2)(l0, dep), 2, mode, gws, ws_need, None, None) == pg.ERR_INVALID_ARG
        same_y = pg.NestedLayer(x1, hi, lo, y0, wsp1, lw, 8, 512, 512)
        assert f((pg.NestedLayer * 2)(l0, same_y), 2, mode, gws, ws_need, None, None) == pg.ERR_INVALID_ARG
        bad_k = pg.NestedLayer(x1, hi, lo, y1, wsp1, lw, 8, 520, 512)               # K % 16
        assert f((pg.NestedLayer * 2)(l0, bad_k), 2, mode, gws, ws_need, None, None) == pg.ERR_ALIGNMENT
        assert f(None, 2, mode, gws, ws_need, None, None) == pg.ERR_INVALID_ARG
        assert f(None, 0, mode, None, 0, None, None) == pg.OK
    # FP16 mode needs the lo plane; FP8 mode needs each layer's workspace
    no_lo = pg.NestedLayer(x1, hi, None, y1, None, 0, 8, 512, 512)
    assert f((pg.NestedLayer * 1)(no_lo), 1, pg.NESTED_FP16, gws, ws_need, None, None) == pg.ERR_INVALID_ARG
    small_ws = pg.NestedLayer(x1, hi, None, y1, wsp1, lw - 256, 64, 512, 512)
    assert f((pg.NestedLayer * 1)(small_ws), 1, pg.NESTED_FP8, gws, ws_need, None, None) == pg.ERR_INVALID_ARG
    shared_ws = pg.NestedLayer(x1, hi, None, y1, wsp0, lw, 8, 512, 512)
    assert f((pg.NestedLayer * 2)(l0, shared_ws), 2, pg.NESTED_FP8, gws, ws_need, None, None) == pg.ERR_INVALID_ARG


def test_tensor_parallel_blocks_argument_checks():
    lib = pg.lib
    assert lib.pgf8_fp8_row_amax(A16, pg.F32, 4, 512, 512, A16 + 2, None) == pg.ERR_ALIGNMENT
    assert lib.pgf8_fp8_row_amax(A16, pg.F32, 4, 520, 520, B16, None) == pg.ERR_ALIGNMENT     # cols % 16
    assert lib.pgf8_fp8_row_amax(A16, pg.F32, 4, 512, 256, B16, None) == pg.ERR_INVALID_ARG   # ldx < cols
    assert lib.pgf8_fp8_row_amax(A16, pg.F32, 0, 512, 512, None, None) == pg.OK
    assert lib.pgf8_fp8_quantize_rows_amax(A16, pg.F32, 4, 512, 512, B16 + 8, C16, None) == pg.ERR_ALIGNMENT
    assert lib.pgf8_fp8_quantize_rows_amax(None, pg.F32, 4, 512, 512, B16, C16, None) == pg.ERR_INVALID_ARG
    ws = lib.pgf8_fp8_linear_partial_workspace_size(8, 512, 512)
    assert ws == lib.pgf8_fp8_linear_group_workspace_size(8)
    assert lib.pgf8_fp8_linear_partial_workspace_size(300, 512, 512) > 16 << 20
    f = lib.pgf8_fp8_linear_partial
    assert f(A16, B16, 8, 512, C16, D16, 512, A16, B16, ws - 16, None) == pg.ERR_INVALID_ARG
    assert f(A16, B16, 8, 512, C16, D16, 512, A16, None, ws, None) == pg.ERR_INVALID_ARG
    assert f(A16, B16, 8, 512, C16, D16, 512, A16 + 4, B16, ws, None) == pg.ERR_ALIGNMENT
    assert f(A16, B16, 8, 520, C16, D16, 512, A16, B16, ws, None) == pg.ERR_ALIGNMENT
    assert lib.pgf8_round_bf16(A16, 12, B16, None) == pg.ERR_ALIGNMENT
    assert lib.pgf8_round_bf16(None, 16, B16, None) == pg.ERR_INVALID_ARG
    assert lib.pgf8_round_bf16(None, 0, None, None) == pg.OK


def test_selftest_row_division_argument_checks():
    f = pg.lib.pgf8_selftest_row_division
    buf = (ctypes.c_uint64 * 4)()
    assert f(None, 1, ctypes.addressof(buf), None) == pg.ERR_INVALID_ARG
    assert f(ctypes.addressof(buf), 0, ctypes.addressof(buf), None) == pg.ERR_INVALID_ARG
    assert f(ctypes.addressof(buf), 65, ctypes.addressof(buf), None) == pg.ERR_INVALID_ARG
    assert f(ctypes.addressof(buf), 1, None, None) == pg.ERR_INVALID_ARG
    assert f(ctypes.addressof(buf) + 1, 1, ctypes.addressof(buf), None) == pg.ERR_ALIGNMENT
    assert f(ctypes.addressof(buf), 1, ctypes.addressof(buf) + 4, None) == pg.ERR_ALIGNMENT


def test_dynamic_plan_is_host_only_and_follows_the_flag():
    # decode-sized M on the skinny path: split chosen, fused only when asked for
    fused, split = pg.fp8_linear_dynamic_plan(1, 4096, 4096, flags=pg.FLAG_FUSED_QUANT)
    assert fused and 1 <= split <= 8
    assert pg.fp8_linear_dynamic_plan(1, 4096, 4096) == (False, split)
    # a slice too long for the registers (f32: 4 x 16 per thread): two-kernel form
    assert pg.fp8_linear_dynamic_plan(8, 22016, 4096, flags=pg.FLAG_FUSED_QUANT)[0] is False
    # prefill-sized M: tiled kernels, no split reported
    assert pg.fp8_linear_dynamic_plan(2048, 4096, 4096, flags=pg.FLAG_FUSED_QUANT) == (False, 0)
    with pytest.raises(pg.Pgf8Error):
        pg.fp8_linear_dynamic_plan(1, 4096, 4000 + 8)   # K % 16 != 0


def test_per_tensor_scaling_argument_checks():
    buf = (ctypes.c_uint8 * 4096)()
    a = ctypes.addressof(buf)
    a16 = (a + 15) // 16 * 16
    amax = pg.lib.pgf8_fp8_amax_accumulate
    assert amax(a16, pg.F32, 0, 16, 16, a16, None) == pg.OK            # empty: nothing enqueued
    assert amax(a16, pg.F32, 2, 15, 16, a16, None) == pg.ERR_INVALID_ARG
    assert amax(a16, pg.F32, 2, 16, 16, None, None) == pg.ERR_INVALID_ARG
    assert amax(a16 + 4, pg.F32, 2, 16, 16, a16, None) == pg.ERR_ALIGNMENT
    assert amax(a16, pg.BF16, 2, 16, 16, a16, None) == pg.ERR_UNSUPPORTED
    qt = pg.lib.pgf8_fp8_quantize_tensor
    assert qt(a16, pg.F32, 2, 16, 16, a16, None, None, 0, None) == pg.ERR_INVALID_ARG      # no q
    assert qt(a16, pg.F32, 2, 16, 16, None, a16, None, 0, None) == pg.ERR_INVALID_ARG      # no amax
    assert qt(a16, pg.F32, 2, 16, 16, a16, a16 + 8, None, 0, None) == pg.ERR_ALIGNMENT
    init = pg.lib.pgf8_delayed_state_init
    assert init(a16, a16, 0, 1.0, None) == pg.ERR_INVALID_ARG
    assert init(a16, a16, 1024, 0.0, None) == pg.ERR_INVALID_ARG
    assert init(a16, a16, 1024, float("inf"), None) == pg.ERR_INVALID_ARG
    assert init(a16 + 4, a16, 1024, 1.0, None) == pg.ERR_ALIGNMENT
    qd = pg.lib.pgf8_fp8_quantize_delayed
    assert qd(a16, pg.F32, 2, 16, 16, a16, None, a16, 0, a16, 0, 0, None) == pg.ERR_INVALID_ARG
    assert qd(a16, pg.F32, 2, 16, 16, a16, None, a16, 1024, None, 0, 0, None) == pg.ERR_INVALID_ARG
    assert qd(a16, pg.F32, 2, 16, 16, a16, None, a16, 1024, a16 + 8, 0, 0, None) == pg.ERR_ALIGNMENT
    assert qd(a16, pg.F32, 0, 16, 16, a16, None, a16, 1024, a16, 0, 0, None) == pg.ERR_INVALID_ARG   # a step needs rows
    assert qd(a16, pg.F32, 2, 16, 16, a16, None, a16, 1024, a16, -1, 0, None) == pg.ERR_INVALID_ARG  # step < 0


def test_kv_write_paged_argument_checks():
    buf = (ctypes.c_uint8 * 8192)()
    a16 = (ctypes.addressof(buf) + 15) // 16 * 16
    f = pg.lib.pgf8_fp8_kv_write_paged
    # (kv, dt, tokens, heads, head_dim, ldkv, scales, first_pos, block_size, table, table_len, num_blocks, cache, bad, flags, stream)
    assert f(a16, pg.F32, 0, 2, 64, 128, a16, 0, 16, a16, 1, 1, a16, None, 0, None) == pg.OK           # nothing to write
    assert f(a16, pg.F32, 20, 2, 64, 128, a16, 0, 16, a16, 1, 2, a16, None, 0, None) == pg.ERR_INVALID_ARG  # table too short
    assert f(a16, pg.F32, 4, 2, 8, 16, a16, 0, 16, a16, 1, 1, a16, None, 0, None) == pg.ERR_INVALID_ARG    # head_dim < 16
    assert f(a16, pg.F32, 4, 2, 64, 100, a16, 0, 16, a16, 1, 1, a16, None, 0, None) == pg.ERR_INVALID_ARG  # ldkv < H*D
    assert f(a16, pg.F32, 4, 2, 40, 80, a16, 0, 16, a16, 1, 1, a16, None, 0, None) == pg.ERR_ALIGNMENT    # D % 16
    assert f(a16 + 4, pg.F32, 4, 2, 64, 128, a16, 0, 16, a16, 1, 1, a16, None, 0, None) == pg.ERR_ALIGNMENT
    assert f(a16, 7, 4, 2, 64, 128, a16, 0, 16, a16, 1, 1, a16, None, 0, None) == pg.ERR_UNSUPPORTED
    assert f(a16, pg.F32, 4, 2, 64, 128, None, 0, 16, a16, 1, 1, a16, None, 0, None) == pg.ERR_INVALID_ARG


def test_attention_decode_plan_covers_the_context():
    # automatic split: chunks of whole warp steps (64 positions), none empty
    for seqs, hq, hkv, ctx in [(8, 32, 32, 4096), (8, 64, 8, 4096), (1, 32, 32, 100000), (64, 64, 8, 1024),
                               (1, 8, 1, 17), (3, 12, 4, 333)]:
        ns, ch = pg.fp8_attention_decode_plan(seqs, hq, hkv, 128, ctx)
        assert ch % 64 == 0 and ns >= 1
        assert ns * ch >= ctx > (ns - 1) * ch
        if ns > 1:
            assert ch >= 256
        ws = pg.lib.pgf8_fp8_attention_decode_workspace_size(seqs, hq, hkv, 128, ctx, 0)
        assert ws == (seqs * hq * ns * 130 * 4 if ns > 1 else 0)
    # a small batch is split for the grid, a large one is not
    assert pg.fp8_attention_decode_plan(1, 32, 32, 128, 4096)[0] > 1
    assert pg.fp8_attention_decode_plan(256, 32, 32, 128, 4096)[0] == 1
    # forced: at most the requested chunks, multiples of 16 positions
    for ctx, splits in [(100, 3), (4096, 7), (40, 9), (16, 4), (0, 2)]:
        ns, ch = pg.fp8_attention_decode_plan(2, 8, 8, 64, ctx, splits)
        assert 1 <= ns <= splits and ch % 16 == 0
        assert ns * ch >= ctx and (ns == 1 or (ns - 1) * ch < ctx)
    assert pg.fp8_attention_decode_plan(2, 8, 8, 64, 100, 3) == (3, 48)
    with pytest.raises(pg.Pgf8Error):
        pg.fp8_attention_decode_plan(2, 12, 8, 128, 64)     # q_heads not a multiple of kv_heads
    with pytest.raises(pg.Pgf8Error):
        pg.fp8_attention_decode_plan(2, 8, 8, 96, 64)      # head_dim not 64 / 128 / 256


def test_attention_decode_argument_checks():
    buf = (ctypes.c_uint8 * 16384)()
    a16 = (ctypes.addressof(buf) + 15) // 16 * 16
    f = pg.lib.pgf8_fp8_attention_decode_paged

    def cache(**kw):
        c = dict(k_cache=a16, v_cache=a16, k_scales=a16, v_scales=a16, num_blocks=4, kv_heads=2, block_size=16,
                 head_dim=64)
        c.update(kw)
        return ctypes.byref(pg.PagedKVCache(**c))

    def call(c=None, seqs=2, hq=4, ldq=256, q=a16, qdt=pg.F32, table_stride=2, max_ctx=32, out=a16, odt=pg.F32,
             ldo=256, splits=1, ws=None, wsb=0, errors=None):
        # (q, q_dt, seqs, q_heads, ldq, cache, tables, table_stride, ctx_lens, max_context, out, out_dt, ldo,
        #  splits, workspace, workspace_bytes, errors, flags, stream)
        return f(q, qdt, seqs, hq, ldq, cache() if c is None else c, a16, table_stride, a16, max_ctx, out, odt, ldo,
                 splits, ws, wsb, errors, 0, None)

    assert call(seqs=0) == pg.OK                                      # nothing to do
    assert f(a16, pg.F32, 2, 4, 256, None, a16, 2, a16, 32, a16, pg.F32, 256, 1, None, 0, None, 0, None) \
        == pg.ERR_INVALID_ARG                                         # no cache
    assert call(c=cache(head_dim=96), ldq=384, ldo=384) == pg.ERR_INVALID_ARG
    assert call(c=cache(block_size=8)) == pg.ERR_INVALID_ARG          # block_size % 16
    assert call(c=cache(kv_heads=3)) == pg.ERR_INVALID_ARG            # q_heads % kv_heads
    assert call(c=cache(num_blocks=0)) == pg.ERR_INVALID_ARG
    assert call(max_ctx=33) == pg.ERR_INVALID_ARG                     # past the table (2 x 16)
    assert call(ldq=200) == pg.ERR_INVALID_ARG                        # ldq < q_heads * head_dim
    assert call(ldo=200) == pg.ERR_INVALID_ARG
    assert call(splits=-1) == pg.ERR_INVALID_ARG
    assert call(q=None) == pg.ERR_INVALID_ARG
    assert call(c=cache(v_scales=None)) == pg.ERR_INVALID_ARG
    assert call(qdt=5) == pg.ERR_UNSUPPORTED
    assert call(odt=5) == pg.ERR_UNSUPPORTED
    assert call(c=cache(k_cache=a16 + 8)) == pg.ERR_ALIGNMENT
    assert call(q=a16 + 2) == pg.ERR_ALIGNMENT                        # f32 query
    assert call(out=a16 + 1, odt=pg.BF16) == pg.ERR_ALIGNMENT
    assert call(errors=a16 + 2) == pg.ERR_ALIGNMENT
    # two chunks need the merge workspace
    need = pg.lib.pgf8_fp8_attention_decode_workspace_size(2, 4, 2, 64, 32, 2)
    assert need == 2 * 4 * 2 * 66 * 4
    assert call(splits=2) == pg.ERR_INVALID_ARG
    assert call(splits=2, ws=a16, wsb=need - 4) == pg.ERR_INVALID_ARG
    assert call(splits=2, ws=a16 + 2, wsb=need) == pg.ERR_ALIGNMENT


def test_attention_context_argument_checks():
    buf = (ctypes.c_uint8 * 16384)()
    a16 = (ctypes.addressof(buf) + 15) // 16 * 16
    f = pg.lib.pgf8_fp8_attention_context_paged

    def cache(**kw):
        c = dict(k_cache=a16, v_cache=a16, k_scales=a16, v_scales=a16, num_blocks=4, kv_heads=2, block_size=16,
                 head_dim=128)
        c.update(kw)
        return ctypes.byref(pg.PagedKVCache(**c))

    def call(c=None, qc=a16, seqs=2, total_q=40, max_q_len=20, hq=4, table_stride=2, max_ctx=32, out=a16,
             odt=pg.BF16, ldo=512, errors=None):
        # (q_codes, q_scales, q_start, seqs, total_q, max_q_len, q_heads, cache, tables, table_stride,
        #  ctx_lens, max_context, out, out_dt, ldo, errors, stream)
        return f(qc, a16, a16, seqs, total_q, max_q_len, hq, cache() if c is None else c, a16, table_stride, a16,
                 max_ctx, out, odt, ldo, errors, None)

    assert call(seqs=0) == pg.OK and call(total_q=0) == pg.OK and call(max_q_len=0) == pg.OK   # nothing to do
    assert f(a16, a16, a16, 2, 40, 20, 4, None, a16, 2, a16, 32, a16, pg.BF16, 512, None, None) == pg.ERR_INVALID_ARG
    assert call(c=cache(head_dim=64)) == pg.ERR_UNSUPPORTED           # head_dim 128 only
    assert call(c=cache(block_size=24)) == pg.ERR_INVALID_ARG         # block_size % 16
    assert call(c=cache(kv_heads=3)) == pg.ERR_INVALID_ARG            # q_heads % kv_heads
    assert call(max_ctx=33) == pg.ERR_INVALID_ARG                     # past the table (2 x 16)
    assert call(ldo=500) == pg.ERR_INVALID_ARG                        # ldo < q_heads * 128
    assert call(seqs=70000) == pg.ERR_INVALID_ARG
    assert call(c=cache(num_blocks=1 << 27)) == pg.ERR_INVALID_ARG    # cache rows past 2^31
    assert call(qc=None) == pg.ERR_INVALID_ARG
    assert call(c=cache(k_scales=None)) == pg.ERR_INVALID_ARG
    assert call(odt=9) == pg.ERR_UNSUPPORTED
    assert call(qc=a16 + 8) == pg.ERR_ALIGNMENT                       # TMA base
    assert call(c=cache(v_cache=a16 + 4)) == pg.ERR_ALIGNMENT
    assert call(out=a16 + 1) == pg.ERR_ALIGNMENT
    assert call(errors=a16 + 1) == pg.ERR_ALIGNMENT


def test_attention_bindings_check_shapes_before_any_pointer():
    """The attention bindings reject inconsistent tensors with their own
    messages before a pointer is taken (CPU tensors: nothing is launched)."""
    import torch
    u8 = lambda *s: torch.zeros(s, dtype=torch.uint8)       # noqa: E731
    i32 = lambda *s: torch.zeros(s, dtype=torch.int32)      # noqa: E731
    f32 = lambda *s: torch.zeros(s, dtype=torch.float32)    # noqa: E731
    q = f32(2, 4, 64)
    kc, vc = u8(4, 2, 16, 64), u8(4, 2, 16, 64)
    ok = dict(k_scales=f32(2), v_scales=f32(2), block_tables=i32(2, 2), context_lens=i32(2), max_context=32)

    def dec(**kw):
        a = dict(ok)
        a.update(kw)
        return pg.fp8_attention_decode_paged(q, kc, vc, **a)

    with pytest.raises(ValueError, match="caches must be"):
        pg.fp8_attention_decode_paged(q, kc, u8(4, 2, 16, 32), **ok)
    with pytest.raises(ValueError, match="one entry and block_tables one row"):
        dec(context_lens=i32(3))
    with pytest.raises(ValueError, match="one entry per KV head"):
        dec(v_scales=f32(1))
    with pytest.raises(ValueError, match="longer than the block tables"):
        dec(max_context=33)
    with pytest.raises(ValueError, match="int32"):
        dec(block_tables=torch.zeros((2, 2), dtype=torch.int64))
    with pytest.raises(ValueError, match="device tensors"):
        dec()                                                # consistent: only the device check remains

    qc, qs = u8(40, 4, 128), f32(160)
    kc2, vc2 = u8(4, 2, 16, 128), u8(4, 2, 16, 128)
    okc = dict(k_scales=f32(2), v_scales=f32(2), block_tables=i32(2, 2), max_context=32, max_q_len=20)

    def ctx(**kw):
        a = dict(okc)
        a.update(kw)
        qsc = a.pop("q_scales", qs)
        qst = a.pop("q_start", i32(3))
        lens = a.pop("context_lens", i32(2))
        return pg.fp8_attention_context_paged(qc, qsc, qst, lens, kc2, vc2, **a)

    with pytest.raises(ValueError, match="seqs \\+ 1 offsets"):
        ctx(q_start=i32(2))
    with pytest.raises(ValueError, match="one scale per"):
        ctx(q_scales=f32(100))
    with pytest.raises(ValueError, match="one row per sequence"):
        ctx(block_tables=i32(1, 2))
    with pytest.raises(ValueError, match="one entry per KV head"):
        ctx(k_scales=f32(1))
    with pytest.raises(ValueError, match="longer than the block tables"):
        ctx(max_context=40)
    with pytest.raises(ValueError, match="device tensors"):
        ctx()


def test_binding_constants_match_the_header():
    """Every enum value and flag the binding names equals the header's."""
    import re
    text = open(pg.HEADER_PATH).read()
    values = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(PGF8_[A-Z0-9_]+)\s*=\s*(\d+)", text)}
    values.update({m.group(1): int(m.group(2)) for m in re.finditer(r"#define\s+(PGF8_FLAG_\w+)\s+(\d+)", text)})
    names = ["OK", "ERR_INVALID_ARG", "ERR_ALIGNMENT", "ERR_UNSUPPORTED", "ERR_CUDA", "ERR_TIMEOUT", "ERR_TOO_LARGE",
             "F32", "F16", "BF16", "SCALE_DYNAMIC", "SCALE_STATIC", "NESTED_FP16", "NESTED_FP8", "PATH_AUTO",
             "PATH_SKINNY", "PATH_TILED", "PATH_STREAMK", "PATH_TILED_PAIR", "FLAG_OVERLAP_PREVIOUS",
             "FLAG_FUSED_QUANT", "FLAG_ATTN_MMA", "FLAG_STREAM_K_TAIL"]
    for n in names:
        assert getattr(pg, n) == values["PGF8_" + n], n
    flags = [values[k] for k in values if k.startswith("PGF8_FLAG_")]
    assert len(set(flags)) == len(flags) and all(f & (f - 1) == 0 for f in flags)   # distinct single bits


def test_layer_records_take_device_tensors_only():
    """The grouped bindings store device addresses the GPU reads later: host
    tensors are refused before any record is built."""
    import torch
    x = torch.zeros(4, 64)
    wq = torch.zeros(64, 64, dtype=torch.uint8)
    sw = torch.ones(64)
    y = torch.zeros(4, 64, dtype=torch.bfloat16)
    ws = torch.zeros(1 << 12, dtype=torch.uint8)
    with pytest.raises(ValueError):
        pg.LayerSequence([(x, wq, sw, y, ws)])
    with pytest.raises(ValueError):
        pg.NestedLayerGroup([(x.half(), wq, wq, y.half(), None)], group_workspace=ws)
    with pytest.raises(ValueError):
        pg.fp8_linear_group([(wq[:4], sw[:4], wq, sw, y)])
