"""B200 (sm_100a) FP8 E4M3 quantised linear layer and NestedFP dual-precision
linear layer.

This module is the Python binding of ``libpgf8.so`` (the C ABI declared in
``include/pgf8.h``).  It only marshals arguments: tensors are plain device
buffers (PyTorch is used for device memory and streams), every computation
runs in the library's CUDA kernels, and there is no other code path.  If the
library has not been built the import fails; build it with
``python precision_gemm_fp8_b200/build.py``.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpgf8.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "pgf8.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python precision_gemm_fp8_b200/build.py` "
                      "(the CUDA library is the only implementation)")

lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_ALIGNMENT, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_TOO_LARGE = range(7)
NOALLOC_SCRATCH_BYTES = 8 << 20
F32, F16, BF16 = 0, 1, 2
SCALE_DYNAMIC, SCALE_STATIC = 0, 1
NESTED_FP16, NESTED_FP8 = 0, 1
PATH_AUTO, PATH_SKINNY, PATH_TILED, PATH_STREAMK, PATH_TILED_PAIR = 0, 1, 2, 3, 4
FLAG_OVERLAP_PREVIOUS = 1
FLAG_FUSED_QUANT = 2
FLAG_ATTN_MMA = 4
FLAG_STREAM_K_TAIL = 8


class LinearOpts(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("split_k", ctypes.c_int32), ("tile_n", ctypes.c_int32),
                ("flags", ctypes.c_int32)]


class PagedKVCache(ctypes.Structure):
    _fields_ = [("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p), ("k_scales", ctypes.c_void_p),
                ("v_scales", ctypes.c_void_p), ("num_blocks", ctypes.c_int64), ("kv_heads", ctypes.c_int64),
                ("block_size", ctypes.c_int64), ("head_dim", ctypes.c_int64)]


class Fp8Layer(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("xdt", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("M", ctypes.c_int64), ("K", ctypes.c_int64), ("ldx", ctypes.c_int64), ("N", ctypes.c_int64),
                ("wq", ctypes.c_void_p), ("sw", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


class Fp8GemmLayer(ctypes.Structure):
    _fields_ = [("aq", ctypes.c_void_p), ("sa", ctypes.c_void_p), ("wq", ctypes.c_void_p), ("sw", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("M", ctypes.c_int64), ("K", ctypes.c_int64), ("N", ctypes.c_int64)]


class NestedLayer(ctypes.Structure):
    _fields_ = [("x_f16", ctypes.c_void_p), ("hi", ctypes.c_void_p), ("lo", ctypes.c_void_p),
                ("y_f16", ctypes.c_void_p), ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("M", ctypes.c_int64), ("K", ctypes.c_int64), ("N", ctypes.c_int64)]


_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t
_i32 = ctypes.c_int
_optp = ctypes.POINTER(LinearOpts)

_SIGS = {
    "pgf8_fp8_quantize_rows": ([_vp, _i32, _i64, _i64, _i64, _vp, _vp, _i32, _vp], _i32),
    "pgf8_fp8_amax_accumulate": ([_vp, _i32, _i64, _i64, _i64, _vp, _vp], _i32),
    "pgf8_fp8_kv_write_paged": ([_vp, _i32, _i64, _i64, _i64, _i64, _vp, _i64, _i64, _vp, _i64, _i64, _vp, _vp, _i32,
                                 _vp], _i32),
    "pgf8_fp8_attention_decode_plan": ([_i64, _i64, _i64, _i64, _i64, _i64, _vp, _vp], _i32),
    "pgf8_fp8_attention_decode_workspace_size": ([_i64, _i64, _i64, _i64, _i64, _i64], _sz),
    "pgf8_fp8_attention_decode_paged": ([_vp, _i32, _i64, _i64, _i64, ctypes.POINTER(PagedKVCache), _vp, _i64, _vp,
                                         _i64, _vp, _i32, _i64, _i64, _vp, _sz, _vp, _i32, _vp], _i32),
    "pgf8_fp8_attention_context_paged": ([_vp, _vp, _vp, _i64, _i64, _i64, _i64, ctypes.POINTER(PagedKVCache),
                                          _vp, _i64, _vp, _i64, _vp, _i32, _i64, _vp, _vp], _i32),
    "pgf8_fp8_norm_quantize": ([_vp, _i32, _i64, _i64, _i64, _vp, _vp, ctypes.c_float, _vp, _vp, _i32, _vp], _i32),
    "pgf8_fp8_silu_mul_quantize": ([_vp, _i32, _i64, _i64, _i64, _vp, _vp, _i32, _vp], _i32),
    "pgf8_fp8_quantize_tensor": ([_vp, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _i32, _vp], _i32),
    "pgf8_delayed_state_init": ([_vp, _vp, _i32, ctypes.c_float, _vp], _i32),
    "pgf8_fp8_quantize_delayed": ([_vp, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _i32, _vp, _i64, _i32, _vp], _i32),
    "pgf8_fp8_linear": ([_vp, _vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _sz, _vp], _i32),
    "pgf8_fp8_linear_ex": ([_vp, _vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _sz, _optp, _vp], _i32),
    "pgf8_fp8_linear_workspace_size": ([_i64, _i64, _i64], _sz),
    "pgf8_fp8_linear_dynamic": ([_vp, _i32, _i64, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _sz, _optp, _vp], _i32),
    "pgf8_fp8_linear_dynamic_workspace_size": ([_i64, _i64, _i64], _sz),
    "pgf8_fp8_linear_dynamic_codes_offset": ([_i64, _i64], _sz),
    "pgf8_fp8_linear_dynamic_many": ([ctypes.POINTER(Fp8Layer), _i64, _optp, _vp], _i32),
    "pgf8_fp8_linear_dynamic_scales_offset": ([_i64, _i64], _sz),
    "pgf8_fp8_linear_dynamic_group": ([ctypes.POINTER(Fp8Layer), _i64, _vp, _sz, _optp, _vp], _i32),
    "pgf8_fp8_linear_group_workspace_size": ([_i64], _sz),
    "pgf8_fp8_linear_group": ([ctypes.POINTER(Fp8GemmLayer), _i64, _optp, _vp], _i32),
    "pgf8_fp8_row_amax": ([_vp, _i32, _i64, _i64, _i64, _vp, _vp], _i32),
    "pgf8_fp8_quantize_rows_amax": ([_vp, _i32, _i64, _i64, _i64, _vp, _vp, _vp], _i32),
    "pgf8_fp8_linear_partial": ([_vp, _vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _sz, _vp], _i32),
    "pgf8_fp8_linear_partial_workspace_size": ([_i64, _i64, _i64], _sz),
    "pgf8_round_bf16": ([_vp, _i64, _vp, _vp], _i32),
    "pgf8_nestedfp_split": ([_vp, _i64, _i64, _vp, _vp, _vp], _i32),
    "pgf8_nestedfp_linear": ([_vp, _i64, _i64, _vp, _vp, _i64, _i32, _vp, _vp, _sz, _vp], _i32),
    "pgf8_nestedfp_linear_ex": ([_vp, _i64, _i64, _vp, _vp, _i64, _i32, _vp, _vp, _sz, _optp, _vp], _i32),
    "pgf8_nestedfp_linear_group": ([ctypes.POINTER(NestedLayer), _i64, _i32, _vp, _sz, _optp, _vp], _i32),
    "pgf8_nestedfp_linear_workspace_size": ([_i64, _i64, _i64, _i32], _sz),
    "pgf8_fp8_linear_dynamic_noalloc": ([_vp, _i32, _i64, _i64, _i64, _vp, _vp, _i64, _vp, _vp], _i32),
    "pgf8_last_cuda_error": ([ctypes.POINTER(ctypes.c_int)], _i32),
    "pgf8_device_status": ([_vp], _i32),
    "pgf8_selftest_bounded_wait": ([_i64, _vp], _i32),
    "pgf8_selftest_row_division": ([_vp, _i32, _vp, _vp], _i32),
    "pgf8_fp8_linear_dynamic_plan": ([_i64, _i64, _i64, _i32, _vp, _vp, _vp], _i32),
    "pgf8_status_str": ([_i32], ctypes.c_char_p),
    "pgf8_version": ([], _i32),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def header_symbols() -> list[str]:
    """Names of the functions declared in include/pgf8.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:pgf8_status|size_t|const char \*|int)\s*(pgf8_\w+)\s*\(", text, re.M)))


class Pgf8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.pgf8_status_str(status).decode()
        if status == ERR_CUDA:
            e = ctypes.c_int(0)
            lib.pgf8_last_cuda_error(ctypes.byref(e))
            msg += f" (cudaError {e.value})"
        super().__init__(f"{where}: {msg}")
        self.status = status


def _check(status: int, where: str):
    if status != OK:
        raise Pgf8Error(status, where)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("pgf8 takes device tensors")
    return ctypes.c_void_p(t.data_ptr())


def _dptr(t: torch.Tensor) -> int:
    """The device address of a tensor bound into a layer record (the
    library reads it on the GPU later): device tensors only."""
    if not t.is_cuda:
        raise ValueError("pgf8 takes device tensors")
    return t.data_ptr()


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _opts(path=PATH_AUTO, split_k=0, tile_n=0, flags=0):
    if path == PATH_AUTO and split_k == 0 and tile_n == 0 and flags == 0:
        return None
    return ctypes.byref(LinearOpts(path, split_k, tile_n, flags))


_ws_cache: dict = {}


def default_workspace(device, nbytes: int) -> torch.Tensor | None:
    """A zero-filled workspace of at least `nbytes`, cached per device and
    shared by every call that is not given its own.  The library leaves its
    synchronisation words zero after each completed call, so the buffer is
    reused as is; calls running concurrently on several streams must each be
    given their own (zero-filled) workspace instead."""
    if nbytes <= 0:
        return None
    dev = torch.device(device)
    t = _ws_cache.get(dev)
    if t is None or t.numel() < nbytes:
        t = torch.zeros(max(nbytes, 1 << 22), dtype=torch.uint8, device=dev)
        _ws_cache[dev] = t
    return t


def _lead(t: torch.Tensor) -> int:
    """Element stride between consecutive entries of the leading dimension.
    A size-1 leading dimension may carry any stride (torch keeps numpy's 0),
    so there the rows are taken as packed: the product of the other sizes."""
    if t.shape[0] > 1:
        return t.stride(0)
    n = 1
    for d in t.shape[1:]:
        n *= d
    return max(t.stride(0), n)


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.float16:
        return F16
    raise TypeError(f"unsupported activation dtype {t.dtype}")


# ----------------------------------------------------------------- entry points
def fp8_quantize_rows(x: torch.Tensor, q: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                      mode: int = SCALE_DYNAMIC, stream=None):
    """Per-row E4M3 quantisation of x [rows, cols] (f32 or f16, row stride
    x.stride(0)).  Returns (q uint8 [rows, cols], scales f32 [rows]).  In
    static mode ``scales`` holds the given scales."""
    rows, cols = x.shape
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        if mode == SCALE_STATIC:
            raise ValueError("static mode needs scales")
        scales = torch.empty(rows, dtype=torch.float32, device=x.device)
    _check(lib.pgf8_fp8_quantize_rows(_ptr(x), _dtype_code(x), rows, cols, _lead(x), _ptr(q), _ptr(scales),
                                      mode, _stream(stream)), "fp8_quantize_rows")
    return q, scales


def fp8_kv_write_paged(kv: torch.Tensor, scales: torch.Tensor, cache: torch.Tensor, block_table: torch.Tensor,
                       first_pos: int, bad_blocks: torch.Tensor | None = None, flags: int = 0, stream=None):
    """Quantise kv [tokens, heads, head_dim] (f32 / f16 / bf16; token rows may
    be strided) into the paged E4M3 cache [num_blocks, heads, block_size,
    head_dim] at positions first_pos.. through block_table (int32)."""
    tokens, heads, head_dim = kv.shape
    if kv.stride(2) != 1 or kv.stride(1) != head_dim:
        raise ValueError("kv heads must be contiguous within a token")
    code = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}.get(kv.dtype)
    if code is None:
        raise TypeError(f"unsupported kv dtype {kv.dtype}")
    num_blocks, ch, block_size, cd = cache.shape
    if (ch, cd) != (heads, head_dim) or cache.dtype != torch.uint8 or not cache.is_contiguous():
        raise ValueError("cache must be a contiguous uint8 [num_blocks, heads, block_size, head_dim] tensor")
    if block_table.dtype != torch.int32 or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous int32 tensor")
    _check(lib.pgf8_fp8_kv_write_paged(_ptr(kv), code, tokens, heads, head_dim, _lead(kv), _ptr(scales), first_pos,
                                       block_size, _ptr(block_table), block_table.numel(), num_blocks, _ptr(cache),
                                       None if bad_blocks is None else _ptr(bad_blocks), flags, _stream(stream)),
           "fp8_kv_write_paged")
    return cache


def fp8_attention_decode_plan(seqs: int, q_heads: int, kv_heads: int, head_dim: int, max_context: int,
                              splits: int = 0) -> tuple[int, int]:
    """(number of context chunks, positions per chunk) the decode attention
    uses for these sizes (host only)."""
    ns, ch = ctypes.c_int64(0), ctypes.c_int64(0)
    _check(lib.pgf8_fp8_attention_decode_plan(seqs, q_heads, kv_heads, head_dim, max_context, splits,
                                              ctypes.byref(ns), ctypes.byref(ch)), "fp8_attention_decode_plan")
    return ns.value, ch.value


def fp8_attention_decode_paged(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                               k_scales: torch.Tensor, v_scales: torch.Tensor, block_tables: torch.Tensor,
                               context_lens: torch.Tensor, max_context: int, out: torch.Tensor | None = None,
                               out_dtype: torch.dtype = torch.float32, splits: int = 0,
                               workspace: torch.Tensor | None = None, errors: torch.Tensor | None = None,
                               flags: int = 0, stream=None) -> torch.Tensor:
    """Decode attention of q [seqs, q_heads, head_dim] (one query per
    sequence, at its last position) over the paged E4M3 K / V caches
    [num_blocks, kv_heads, block_size, head_dim] with per-KV-head scales,
    block_tables int32 [seqs, table_stride], context_lens int32 [seqs].
    Returns out [seqs, q_heads, head_dim]."""
    seqs, q_heads, head_dim = q.shape
    if q.stride(2) != 1 or q.stride(1) != head_dim:
        raise ValueError("q heads must be contiguous within a sequence")
    num_blocks, kv_heads, block_size, cd = k_cache.shape
    for c in (k_cache, v_cache):
        if c.shape != k_cache.shape or c.dtype != torch.uint8 or not c.is_contiguous() or cd != head_dim:
            raise ValueError("caches must be contiguous uint8 [num_blocks, kv_heads, block_size, head_dim] tensors")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.stride(1) != 1:
        raise ValueError("block_tables must be an int32 [seqs, table_stride] tensor with contiguous rows")
    if context_lens.dtype != torch.int32 or not context_lens.is_contiguous():
        raise ValueError("context_lens must be a contiguous int32 tensor")
    if context_lens.numel() != seqs or block_tables.shape[0] < seqs:
        raise ValueError("context_lens needs one entry and block_tables one row per sequence")
    if k_scales.numel() < kv_heads or v_scales.numel() < kv_heads:
        raise ValueError("k_scales and v_scales need one entry per KV head")
    if max_context > block_tables.shape[1] * block_size:
        raise ValueError("max_context is longer than the block tables cover")
    if out is None:
        out = torch.empty((seqs, q_heads, head_dim), dtype=out_dtype, device=q.device)
    if out.stride(2) != 1 or out.stride(1) != head_dim:
        raise ValueError("out heads must be contiguous within a sequence")
    codes = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}
    if q.dtype not in codes or out.dtype not in codes:
        raise TypeError("q and out must be float32, float16 or bfloat16")
    need = lib.pgf8_fp8_attention_decode_workspace_size(seqs, q_heads, kv_heads, head_dim, max_context, splits)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    cache = PagedKVCache(_ptr(k_cache), _ptr(v_cache), _ptr(k_scales), _ptr(v_scales), num_blocks, kv_heads,
                         block_size, head_dim)
    _check(lib.pgf8_fp8_attention_decode_paged(
        _ptr(q), codes[q.dtype], seqs, q_heads, _lead(q), ctypes.byref(cache), _ptr(block_tables),
        _lead(block_tables), _ptr(context_lens), max_context, _ptr(out), codes[out.dtype], _lead(out), splits,
        _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
        None if errors is None else _ptr(errors), flags, _stream(stream)), "fp8_attention_decode_paged")
    return out


def fp8_attention_context_paged(q_codes: torch.Tensor, q_scales: torch.Tensor, q_start: torch.Tensor,
                                context_lens: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                k_scales: torch.Tensor, v_scales: torch.Tensor, block_tables: torch.Tensor,
                                max_context: int, max_q_len: int, out: torch.Tensor | None = None,
                                out_dtype: torch.dtype = torch.bfloat16, errors: torch.Tensor | None = None,
                                stream=None) -> torch.Tensor:
    """Causal context attention of the packed queries (E4M3 codes q_codes
    [total_q, q_heads, 128] with per-(token, head) scales q_scales
    [total_q * q_heads], as fp8_quantize_rows writes them) over the paged
    E4M3 K / V caches; sequence s owns query tokens q_start[s] ..
    q_start[s+1] - 1 (int32 [seqs + 1]), the last positions of its
    context_lens[s] cached ones.  Returns out [total_q, q_heads, 128]."""
    total_q, q_heads, head_dim = q_codes.shape
    if q_codes.dtype != torch.uint8 or not q_codes.is_contiguous():
        raise ValueError("q_codes must be a contiguous uint8 [total_q, q_heads, head_dim] tensor")
    num_blocks, kv_heads, block_size, cd = k_cache.shape
    for c in (k_cache, v_cache):
        if c.shape != k_cache.shape or c.dtype != torch.uint8 or not c.is_contiguous() or cd != head_dim:
            raise ValueError("caches must be contiguous uint8 [num_blocks, kv_heads, block_size, head_dim] tensors")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.stride(1) != 1:
        raise ValueError("block_tables must be an int32 [seqs, table_stride] tensor with contiguous rows")
    for t in (q_start, context_lens):
        if t.dtype != torch.int32 or not t.is_contiguous():
            raise ValueError("q_start and context_lens must be contiguous int32 tensors")
    seqs = context_lens.numel()
    if q_start.numel() != seqs + 1:
        raise ValueError("q_start must hold seqs + 1 offsets")
    if q_scales.numel() < total_q * q_heads:
        raise ValueError("q_scales needs one scale per (token, head) row")
    if block_tables.shape[0] < seqs:
        raise ValueError("block_tables needs one row per sequence")
    if k_scales.numel() < kv_heads or v_scales.numel() < kv_heads:
        raise ValueError("k_scales and v_scales need one entry per KV head")
    if max_context > block_tables.shape[1] * block_size:
        raise ValueError("max_context is longer than the block tables cover")
    if out is None:
        out = torch.empty((total_q, q_heads, head_dim), dtype=out_dtype, device=q_codes.device)
    codes = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}
    if out.dtype not in codes or out.stride(2) != 1 or out.stride(1) != head_dim:
        raise ValueError("out must be float32 / float16 / bfloat16 with heads contiguous within a token")
    cache = PagedKVCache(_ptr(k_cache), _ptr(v_cache), _ptr(k_scales), _ptr(v_scales), num_blocks, kv_heads,
                         block_size, head_dim)
    _check(lib.pgf8_fp8_attention_context_paged(
        _ptr(q_codes), _ptr(q_scales), _ptr(q_start), seqs, total_q, max_q_len, q_heads, ctypes.byref(cache),
        _ptr(block_tables), _lead(block_tables), _ptr(context_lens), max_context, _ptr(out), codes[out.dtype],
        _lead(out), None if errors is None else _ptr(errors), _stream(stream)), "fp8_attention_context_paged")
    return out


def fp8_norm_quantize(x: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor | None = None, eps: float = 1e-5,
                      q: torch.Tensor | None = None, scales: torch.Tensor | None = None, flags: int = 0, stream=None):
    """LayerNorm (beta given) or RMSNorm (beta None) of each row of x [rows,
    cols] (f32/f16), quantised per token to E4M3.  Returns (q uint8 [rows,
    cols], scales f32 [rows])."""
    rows, cols = x.shape
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(rows, dtype=torch.float32, device=x.device)
    _check(lib.pgf8_fp8_norm_quantize(_ptr(x), _dtype_code(x), rows, cols, _lead(x), _ptr(gamma),
                                      None if beta is None else _ptr(beta), float(eps), _ptr(q), _ptr(scales), flags,
                                      _stream(stream)), "fp8_norm_quantize")
    return q, scales


def fp8_silu_mul_quantize(gu: torch.Tensor, q: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                          flags: int = 0, stream=None):
    """silu(gate) * up of the gate+up output gu [rows, 2I] (bf16 or f32; gate
    = first I columns), quantised per token to E4M3.  Returns (q uint8
    [rows, I], scales f32 [rows])."""
    rows, two_i = gu.shape
    if gu.stride(1) != 1 or two_i % 2:
        raise ValueError("gu rows must be contiguous with an even width")
    inter = two_i // 2
    code = {torch.bfloat16: BF16, torch.float32: F32}.get(gu.dtype)
    if code is None:
        raise TypeError(f"unsupported gate/up dtype {gu.dtype}")
    if q is None:
        q = torch.empty((rows, inter), dtype=torch.uint8, device=gu.device)
    if scales is None:
        scales = torch.empty(rows, dtype=torch.float32, device=gu.device)
    _check(lib.pgf8_fp8_silu_mul_quantize(_ptr(gu), code, rows, inter, _lead(gu), _ptr(q), _ptr(scales), flags,
                                          _stream(stream)), "fp8_silu_mul_quantize")
    return q, scales


def fp8_amax_accumulate(x: torch.Tensor, amax: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """amax = max(amax, max |x|) as a device float32 [1] tensor (a new zero
    one when not given): the MINMAX calibration statistic, accumulated over
    calibration batches."""
    rows, cols = x.shape
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    if amax is None:
        amax = torch.zeros(1, dtype=torch.float32, device=x.device)
    _check(lib.pgf8_fp8_amax_accumulate(_ptr(x), _dtype_code(x), rows, cols, _lead(x), _ptr(amax),
                                        _stream(stream)), "fp8_amax_accumulate")
    return amax


def fp8_quantize_tensor(x: torch.Tensor, amax: torch.Tensor, q: torch.Tensor | None = None,
                        scales: torch.Tensor | None = None, flags: int = 0, stream=None):
    """Static per-tensor quantisation with the scale of a calibrated amax
    (device float32 [1]).  Returns (q uint8 [rows, cols], scales f32 [rows],
    every row holding the tensor's scale)."""
    rows, cols = x.shape
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(rows, dtype=torch.float32, device=x.device)
    _check(lib.pgf8_fp8_quantize_tensor(_ptr(x), _dtype_code(x), rows, cols, _lead(x), _ptr(amax), _ptr(q),
                                        _ptr(scales), flags, _stream(stream)), "fp8_quantize_tensor")
    return q, scales


class DelayedScaling:
    """Delayed per-tensor scaling of one activation tensor: a device amax
    history of ``history_len`` entries and the pending amax of the last
    step.  Each ``step(x)`` quantises x with the scale carried out of the
    previous step, RN(max of the last history_len amaxes / 448), and records
    amax(x) (one kernel)."""

    def __init__(self, history_len: int = 1024, initial_scale: float = 1.0, device="cuda", stream=None):
        self.history_len = int(history_len)
        self.history = torch.empty(self.history_len, dtype=torch.float32, device=device)
        self.state = torch.empty(4, dtype=torch.int32, device=device)   # pgf8_delayed_state, 16 bytes
        self.steps = 0
        self.initial_scale = float(initial_scale)
        _check(lib.pgf8_delayed_state_init(_ptr(self.state), _ptr(self.history), self.history_len,
                                           self.initial_scale, _stream(stream)), "delayed_state_init")

    def step(self, x: torch.Tensor, q: torch.Tensor | None = None, scales: torch.Tensor | None = None, flags: int = 0,
             stream=None):
        """Returns (q uint8 [rows, cols], scales f32 [rows]: the step's scale)."""
        rows, cols = x.shape
        if x.stride(1) != 1:
            raise ValueError("x rows must be contiguous")
        if q is None:
            q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
        if scales is None:
            scales = torch.empty(rows, dtype=torch.float32, device=x.device)
        _check(lib.pgf8_fp8_quantize_delayed(_ptr(x), _dtype_code(x), rows, cols, _lead(x), _ptr(q),
                                             _ptr(scales), _ptr(self.history), self.history_len, _ptr(self.state),
                                             self.steps, flags, _stream(stream)), "fp8_quantize_delayed")
        self.steps += 1
        return q, scales

    def window(self):
        """The last history_len amaxes as the ring holds them after the steps
        so far (the newest, still pending on the device, filed in its slot);
        read back (synchronises)."""
        import numpy as _np
        h = self.history.cpu().numpy().copy()
        if self.steps:
            t = self.steps - 1
            pend = self.state.cpu().numpy().view(_np.uint32)[1 + t % 3]
            h[t % self.history_len] = _np.array([pend], dtype=_np.uint32).view(_np.float32)[0]
        return h


def fp8_linear(aq, sa, wq, sw, y=None, workspace=None, path=PATH_AUTO, split_k=0, tile_n=0, flags=0,
               stream=None):
    """y [M,N] bf16 = (E4M3 aq [M,K] x E4M3 wq [N,K]^T) * sa[m] * sw[n].
    workspace: zero-filled device buffer (default: the per-device shared one)."""
    M, K = aq.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=aq.device)
    if workspace is None:
        workspace = default_workspace(aq.device, int(lib.pgf8_fp8_linear_workspace_size(M, N, K)))
    _check(lib.pgf8_fp8_linear_ex(_ptr(aq), _ptr(sa), M, K, _ptr(wq), _ptr(sw), N, _ptr(y), _ptr(workspace),
                                  _nbytes(workspace), _opts(path, split_k, tile_n, flags), _stream(stream)),
           "fp8_linear")
    return y


def fp8_row_amax(x: torch.Tensor, amax: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """amax [rows] f32 = max_c |x[r, c]| of x [rows, cols] (f32 or f16)."""
    rows, cols = x.shape
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    if amax is None:
        amax = torch.empty(rows, dtype=torch.float32, device=x.device)
    _check(lib.pgf8_fp8_row_amax(_ptr(x), _dtype_code(x), rows, cols, _lead(x), _ptr(amax), _stream(stream)),
           "fp8_row_amax")
    return amax


def fp8_quantize_rows_amax(x: torch.Tensor, amax: torch.Tensor, q: torch.Tensor | None = None, stream=None):
    """Codes and scales of x [rows, cols] from the given per-row amax (taken
    over the whole rows, of which x may hold a slice).  `amax` is replaced
    by the scales in place.  Returns (q uint8 [rows, cols], scales = amax)."""
    rows, cols = x.shape
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    if amax.dtype != torch.float32 or amax.numel() != rows or not amax.is_contiguous():
        raise ValueError("amax must be a contiguous float32 tensor with one entry per row")
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    _check(lib.pgf8_fp8_quantize_rows_amax(_ptr(x), _dtype_code(x), rows, cols, _lead(x), _ptr(q), _ptr(amax),
                                           _stream(stream)), "fp8_quantize_rows_amax")
    return q, amax


def fp8_linear_partial(aq, sa, wq, sw, y=None, workspace=None, stream=None):
    """y [M,N] f32 = (E4M3 aq [M,K] x E4M3 wq [N,K]^T) * sa[m] * sw[n], summed
    in f32 and not rounded: one rank's share of a layer split along K."""
    M, K = aq.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=aq.device)
    need = int(lib.pgf8_fp8_linear_partial_workspace_size(M, N, K))
    if workspace is None:
        workspace = default_workspace(aq.device, need)
    _check(lib.pgf8_fp8_linear_partial(_ptr(aq), _ptr(sa), M, K, _ptr(wq), _ptr(sw), N, _ptr(y), _ptr(workspace),
                                       _nbytes(workspace), _stream(stream)), "fp8_linear_partial")
    return y


def round_bf16(x: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = bf16_RN(x) for a contiguous f32 tensor (numel % 8 == 0)."""
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 tensor")
    if y is None:
        y = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    _check(lib.pgf8_round_bf16(_ptr(x), x.numel(), _ptr(y), _stream(stream)), "round_bf16")
    return y


def fp8_linear_dynamic_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib.pgf8_fp8_linear_dynamic_workspace_size(M, N, K))


def fp8_linear_dynamic(x, wq, sw, y=None, workspace=None, path=PATH_AUTO, split_k=0, tile_n=0, flags=0,
                       stream=None):
    """Per-token dynamic quantisation of x [M,K] (f32/f16) followed by the FP8
    linear with weights wq [N,K] / sw [N].  Returns y [M,N] bf16.  A given
    workspace must be zero-filled before its first use."""
    M, K = x.shape
    N = wq.shape[0]
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    need = fp8_linear_dynamic_workspace_size(M, N, K)
    if workspace is None:
        workspace = default_workspace(x.device, need)
    _check(lib.pgf8_fp8_linear_dynamic(_ptr(x), _dtype_code(x), M, K, _lead(x), _ptr(wq), _ptr(sw), N, _ptr(y),
                                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _opts(path, split_k, tile_n, flags), _stream(stream)), "fp8_linear_dynamic")
    return y


def fp8_linear_dynamic_plan(M: int, N: int, K: int, x_dtype=torch.float32, path=PATH_AUTO, split_k=0, tile_n=0,
                            flags=0):
    """(fused, split_k) the dynamic FP8 linear would use for these arguments:
    fused True when the GEMM quantises the activations itself; split_k the
    skinny GEMM's K-split (0 for a tiled kernel)."""
    code = {torch.float32: F32, torch.float16: F16}.get(x_dtype)
    if code is None:
        raise TypeError(f"unsupported activation dtype {x_dtype}")
    fused, split = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib.pgf8_fp8_linear_dynamic_plan(M, N, K, code, _opts(path, split_k, tile_n, flags),
                                            ctypes.addressof(fused), ctypes.addressof(split)),
           "fp8_linear_dynamic_plan")
    return bool(fused.value), int(split.value)


def fp8_linear_dynamic_noalloc(x, wq, sw, y=None, stream=None):
    """fp8_linear_dynamic without a workspace, for callers that cannot allocate
    one: the codes and scales live in the library's fixed 8 MiB device array
    (shared by all calls on a device; keep such calls on one stream).  Raises
    Pgf8Error(ERR_TOO_LARGE) when the problem does not fit.  (Allocating y
    here is this wrapper's convenience; pass y to allocate nothing.)"""
    M, K = x.shape
    N = wq.shape[0]
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(lib.pgf8_fp8_linear_dynamic_noalloc(_ptr(x), _dtype_code(x), M, K, _lead(x), _ptr(wq), _ptr(sw), N,
                                               _ptr(y), _stream(stream)), "fp8_linear_dynamic_noalloc")
    return y


class LayerSequence:
    """A fixed sequence of dynamic FP8 layers (device tensors bound once), run
    by one call of pgf8_fp8_linear_dynamic_many.  Each entry is a tuple
    (x, wq, sw, y, workspace); workspaces must be zero-filled before first use."""

    def __init__(self, layers):
        self._keep = list(layers)
        arr = (Fp8Layer * len(self._keep))()
        for i, (x, wq, sw, y, ws) in enumerate(self._keep):
            if x.stride(1) != 1:
                raise ValueError("x rows must be contiguous")
            arr[i] = Fp8Layer(_dptr(x), _dtype_code(x), 0, x.shape[0], x.shape[1], _lead(x), wq.shape[0],
                              _dptr(wq), _dptr(sw), _dptr(y), _dptr(ws), _nbytes(ws))
        self._arr = arr
        self.count = len(self._keep)

    def run(self, flags=0, stream=None):
        _check(lib.pgf8_fp8_linear_dynamic_many(self._arr, self.count, _opts(flags=flags), _stream(stream)),
               "fp8_linear_dynamic_many")


class LayerGroup(LayerSequence):
    """A fixed group of INDEPENDENT dynamic FP8 layers (no layer reads another
    layer's output), run by one call of pgf8_fp8_linear_dynamic_group: the
    layers with M <= 256 stream their weights through the grouped kernel.
    Entries as LayerSequence; the group workspace is allocated (zero-filled)
    here unless given."""

    def __init__(self, layers, group_workspace=None):
        super().__init__(layers)
        max_m = max((x.shape[0] for (x, _, _, _, _) in self._keep), default=0)
        need = group_workspace_size(max_m)
        if group_workspace is None:
            dev = self._keep[0][0].device if self._keep else "cuda"
            group_workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
        elif _nbytes(group_workspace) < need:
            raise ValueError(f"group workspace needs {need} bytes")
        self.group_workspace = group_workspace

    def run(self, flags=0, stream=None):
        _check(lib.pgf8_fp8_linear_dynamic_group(self._arr, self.count, _ptr(self.group_workspace),
                                                 _nbytes(self.group_workspace), _opts(flags=flags), _stream(stream)),
               "fp8_linear_dynamic_group")


def fp8_linear_group(layers, flags=0, stream=None):
    """pgf8_fp8_linear_group: independent pre-quantised FP8 GEMMs in one
    launch on SM pairs.  Each entry (aq [M,K] uint8, sa [M] f32, wq [N,K]
    uint8, sw [N] f32, y [M,N] bf16 or None); returns the outputs."""
    arr = (Fp8GemmLayer * len(layers))()
    outs = []
    for i, (aq, sa, wq, sw, y) in enumerate(layers):
        if not (aq.is_contiguous() and wq.is_contiguous() and sa.is_contiguous() and sw.is_contiguous()):
            raise ValueError("operands must be contiguous")
        M, K = aq.shape
        N = wq.shape[0]
        if y is None:
            y = torch.empty((M, N), dtype=torch.bfloat16, device=aq.device)
        outs.append(y)
        arr[i] = Fp8GemmLayer(_dptr(aq), _dptr(sa), _dptr(wq), _dptr(sw), _dptr(y), M, K, N)
    _check(lib.pgf8_fp8_linear_group(arr, len(layers), _opts(flags=flags), _stream(stream)), "fp8_linear_group")
    return outs


def group_workspace_size(max_m: int) -> int:
    return int(lib.pgf8_fp8_linear_group_workspace_size(max_m))


def dynamic_workspace_views(workspace: torch.Tensor, M: int, K: int):
    """(aq [M,K] uint8, sa [M] f32) views of a dynamic-linear workspace."""
    c0 = int(lib.pgf8_fp8_linear_dynamic_codes_offset(M, K))
    off = int(lib.pgf8_fp8_linear_dynamic_scales_offset(M, K))
    aq = workspace[c0:c0 + M * K].view(M, K)
    sa = workspace[off:off + 4 * M].view(torch.float32)
    return aq, sa


def nestedfp_split(w: torch.Tensor, hi=None, lo=None, stream=None):
    """hi/lo byte planes [N,K] of an FP16 weight [N,K]."""
    if w.dtype != torch.float16 or not w.is_contiguous():
        raise ValueError("w must be a contiguous float16 tensor")
    N, K = w.shape
    if hi is None:
        hi = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    if lo is None:
        lo = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    _check(lib.pgf8_nestedfp_split(_ptr(w), N, K, _ptr(hi), _ptr(lo), _stream(stream)), "nestedfp_split")
    return hi, lo


def nestedfp_linear_workspace_size(M: int, N: int, K: int, mode: int) -> int:
    return int(lib.pgf8_nestedfp_linear_workspace_size(M, N, K, mode))


def nestedfp_linear(x, hi, lo, mode=NESTED_FP16, y=None, workspace=None, path=PATH_AUTO, split_k=0, tile_n=0,
                    flags=0, stream=None):
    """NestedFP linear: x [M,K] f16, hi/lo [N,K] uint8 planes -> y [M,N] f16.
    FP16 mode rebuilds (hi << 8) | lo; FP8 mode uses hi as E5M2 and
    quantises x per token to E4M3 (lo unused)."""
    if x.dtype != torch.float16 or not x.is_contiguous():
        raise ValueError("x must be a contiguous float16 tensor")
    M, K = x.shape
    N = hi.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    need = nestedfp_linear_workspace_size(M, N, K, mode)
    if workspace is None:
        workspace = default_workspace(x.device, need)
    wbytes = _nbytes(workspace)
    _check(lib.pgf8_nestedfp_linear_ex(_ptr(x), M, K, _ptr(hi), _ptr(lo) if lo is not None else None, N, mode,
                                       _ptr(y), _ptr(workspace), wbytes, _opts(path, split_k, tile_n, flags),
                                       _stream(stream)), "nestedfp_linear")
    return y


class NestedLayerGroup:
    """A fixed group of INDEPENDENT NestedFP layers in one mode, run by one
    call of pgf8_nestedfp_linear_group: the layers with M <= 256 stream their
    weight planes through the grouped kernel.  Entries are tuples
    (x [M,K] f16, hi [N,K], lo [N,K] or None, y [M,N] f16, workspace or None);
    FP8 mode needs each layer's workspace (nestedfp_linear_workspace_size
    bytes), FP16 mode none.  The group workspace is allocated (zero-filled)
    here unless given."""

    def __init__(self, layers, mode=NESTED_FP16, group_workspace=None):
        self._keep = list(layers)
        self.mode = mode
        arr = (NestedLayer * len(self._keep))()
        for i, (x, hi, lo, y, ws) in enumerate(self._keep):
            if x.dtype != torch.float16 or not x.is_contiguous():
                raise ValueError("x must be a contiguous float16 tensor")
            arr[i] = NestedLayer(_dptr(x), _dptr(hi), _dptr(lo) if lo is not None else None,
                                 _dptr(y), _dptr(ws) if ws is not None else None, _nbytes(ws),
                                 x.shape[0], x.shape[1], hi.shape[0])
        self._arr = arr
        self.count = len(self._keep)
        max_m = max((x.shape[0] for (x, *_rest) in self._keep if x.shape[0] <= 256), default=0)
        need = group_workspace_size(max_m) if max_m else 0
        if group_workspace is None:
            dev = self._keep[0][0].device if self._keep else "cuda"
            group_workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=dev)
        elif _nbytes(group_workspace) < need:
            raise ValueError(f"group workspace needs {need} bytes")
        self.group_workspace = group_workspace

    def run(self, flags=0, stream=None):
        _check(lib.pgf8_nestedfp_linear_group(self._arr, self.count, self.mode, _ptr(self.group_workspace),
                                              _nbytes(self.group_workspace), _opts(flags=flags), _stream(stream)),
               "nestedfp_linear_group")


def selftest_row_division(divisors: torch.Tensor, stream=None):
    """[count, 2] int64 mismatch counts of the quantisation's division against
    the device's IEEE division over every binary32 x with |x| <= 512 s:
    column 0 quotients (where |x| >= 2^-11 s), column 1 E4M3 codes (see
    pgf8_selftest_row_division)."""
    if divisors.dtype != torch.float32 or not divisors.is_contiguous():
        raise ValueError("divisors must be a contiguous float32 tensor")
    counts = torch.zeros((divisors.numel(), 2), dtype=torch.int64, device=divisors.device)
    _check(lib.pgf8_selftest_row_division(_ptr(divisors), divisors.numel(), _ptr(counts), _stream(stream)),
           "selftest_row_division")
    return counts


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return int(lib.pgf8_device_status(_stream(stream)))


def version() -> int:
    return int(lib.pgf8_version())
