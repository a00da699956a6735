"""The allocation-free dynamic FP8 linear entry point, called through the C ABI.

It serves callers that cannot hand the library a workspace (a host program
that links only the C library and has no device allocator, or a runtime that
plans all device memory before serving and forbids allocating on the request
path).  Its codes and scales live in the library's fixed device array, which
every call shares and which keeps the previous call's contents.  It runs the
same kernels as the workspace-taking entry point, so the test makes two calls
in a row with different inputs and different token counts (M = 8, then 64:
the scales move inside the shared array between the two), and checks each
output bit for bit against the workspace-taking entry point, whose codes and
scales it checks bit for bit against the oracle, and the output against the
oracle's binary64 layer within the stated bound.  The file sorts last so a
run that stops at the first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synthetic
from _parity import assert_within, fp8_row_max, linear_bound

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _call_noalloc(x, wq, sw, y):
    st = pg.lib.pgf8_fp8_linear_dynamic_noalloc(
        ctypes.c_void_p(x.data_ptr()), pg.F32 if x.dtype == torch.float32 else pg.F16, x.shape[0], x.shape[1],
        x.stride(0), ctypes.c_void_p(wq.data_ptr()), ctypes.c_void_p(sw.data_ptr()), wq.shape[0],
        ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def test_noalloc_matches_workspace_entry_point_twice():
    torch.cuda.set_device(0)
    g = np.random.default_rng(2024)
    K, N = 4096, 4096
    w = synthetic.weights_f16(N, K, 0.02, g)
    wq, sw = pg.fp8_quantize_rows(torch.from_numpy(w).to(DEV))
    wq0, sw0 = oracle.quantize_rows(w)
    for call, M in enumerate((8, 64)):          # two calls in a row share the fixed array
        x = synthetic.activations("normal_outl_0p5pct_x30", M, K, g)
        xt = torch.from_numpy(x).to(DEV)
        y_na = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _call_noalloc(xt, wq, sw, y_na) == pg.OK
        ws = torch.zeros(pg.fp8_linear_dynamic_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
        y_ws = pg.fp8_linear_dynamic(xt, wq, sw, workspace=ws)
        torch.cuda.synchronize()
        assert pg.device_status() == pg.OK
        assert torch.equal(y_na.view(torch.int16), y_ws.view(torch.int16)), f"call {call}: outputs differ"
        aq0, sa0 = oracle.quantize_rows(x)
        aq, sa = pg.dynamic_workspace_views(ws, M, K)
        assert np.array_equal(aq.cpu().numpy(), aq0), f"call {call}: codes differ from the oracle"
        assert np.array_equal(sa.cpu().numpy().view(np.uint32), sa0.view(np.uint32)), f"call {call}: scales"
        ref = oracle.fp8_linear(aq0, sa0, wq0, sw0)
        bound = linear_bound(ref, K, fp8_row_max(aq0, sa0), fp8_row_max(wq0, sw0))
        assert_within(y_na.float().cpu().numpy(), ref, bound, f"no-alloc call {call} (M={M})")


def test_noalloc_rejects_problems_beyond_the_array():
    M, K, N = 4096, 4096, 4096                 # 16 MiB of codes > the 8 MiB array
    assert pg.lib.pgf8_fp8_linear_dynamic_workspace_size(M, N, K) > pg.NOALLOC_SCRATCH_BYTES
    st = pg.lib.pgf8_fp8_linear_dynamic_noalloc(ctypes.c_void_p(0x10000), pg.F32, M, K, K,
                                                ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000), N,
                                                ctypes.c_void_p(0x40000), None)
    assert st == pg.ERR_TOO_LARGE
