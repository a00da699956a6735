"""CPU oracle for the FP8 linear layer and NestedFP — TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  The product (``precision_gemm_fp8_b200``) never imports
it, and this package never imports the product: the two share no code.

The arithmetic lives in ``pgf8_oracle.c`` (plain scalar C, binary64 wherever
the method does not fix a precision).  This module compiles it with gcc on
first use and wraps each function with numpy marshalling only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pgf8_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

MODE_DYNAMIC = 0
MODE_STATIC = 1


def build(force: bool = False) -> str:
    """Compile pgf8_oracle.c into liboracle.so (plain gcc, no fast-math, no
    contraction, so every operation is the IEEE one written in the source)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-frounding-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i64 = ctypes.c_int64
        lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_decode.restype = ctypes.c_double
        lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        lib.orc_e5m2_decode.argtypes = [ctypes.c_uint8]
        lib.orc_e5m2_decode.restype = ctypes.c_double
        lib.orc_e5m2_encode.argtypes = [ctypes.c_float]
        lib.orc_e5m2_encode.restype = ctypes.c_uint8
        lib.orc_fp16_decode.argtypes = [ctypes.c_uint16]
        lib.orc_fp16_decode.restype = ctypes.c_double
        lib.orc_quantize_rows_f32.argtypes = [f32p, i64, i64, i64, u8p, f32p, ctypes.c_int]
        lib.orc_quantize_rows_f32.restype = ctypes.c_int
        lib.orc_quantize_rows_f16.argtypes = [u16p, i64, i64, i64, u8p, f32p, ctypes.c_int, f32p]
        lib.orc_quantize_rows_f16.restype = ctypes.c_int
        lib.orc_fp8_linear.argtypes = [u8p, f32p, i64, i64, u8p, f32p, i64, f64p]
        lib.orc_fp8_linear.restype = None
        lib.orc_nestedfp_split.argtypes = [u16p, i64, u8p, u8p]
        lib.orc_nestedfp_split.restype = None
        lib.orc_nestedfp_rebuild.argtypes = [ctypes.c_uint8, ctypes.c_uint8]
        lib.orc_nestedfp_rebuild.restype = ctypes.c_uint16
        lib.orc_nestedfp_linear_fp16.argtypes = [u16p, i64, i64, u8p, u8p, i64, f64p]
        lib.orc_nestedfp_linear_fp16.restype = None
        lib.orc_nestedfp_linear_fp8.argtypes = [u16p, i64, i64, u8p, i64, f64p, u8p, f32p, f32p]
        lib.orc_amax_accumulate_f32.argtypes = [f32p, i64, i64, i64, f32p]
        lib.orc_amax_accumulate_f32.restype = ctypes.c_int
        lib.orc_quantize_tensor_f32.argtypes = [f32p, i64, i64, i64, ctypes.c_float, u8p, f32p]
        lib.orc_quantize_tensor_f32.restype = ctypes.c_int
        lib.orc_delayed_step_f32.argtypes = [f32p, i64, i64, i64, u8p, f32p, ctypes.c_int32,
                                             ctypes.POINTER(ctypes.c_int32), f32p, f32p]
        lib.orc_delayed_step_f32.restype = ctypes.c_int
        lib.orc_norm_rows.argtypes = [f32p, i64, i64, i64, f32p, f32p, ctypes.c_double, f64p]
        lib.orc_norm_rows.restype = ctypes.c_int
        lib.orc_silu_mul.argtypes = [f64p, f64p, i64, f64p]
        lib.orc_silu_mul.restype = None
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.orc_kv_calibrate_scales.argtypes = [f32p, i64, i64, i64, f32p]
        lib.orc_kv_calibrate_scales.restype = ctypes.c_int
        lib.orc_kv_write_paged.argtypes = [f32p, i64, i64, i64, i64, f32p, i64, i32p, i64, u8p]
        lib.orc_kv_write_paged.restype = ctypes.c_int
        lib.orc_attention_paged.argtypes = [f64p, i64, i64, i64, u8p, u8p, f32p, f32p, i64, i64, i32p, i64, i64,
                                            f64p, f64p]
        lib.orc_attention_paged.restype = ctypes.c_int
        lib.orc_nestedfp_linear_fp8.restype = ctypes.c_int
        _lib = lib
        return lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ctype))


class OracleError(RuntimeError):
    pass


_ERRS = {1: "non-finite input", 2: "scale not positive and finite", 3: "bad argument"}


def _check(st: int):
    if st != 0:
        raise OracleError(_ERRS.get(st, f"oracle status {st}"))


# ---------------------------------------------------------------- scalar codecs
def e4m3_decode(code: int) -> float:
    return _load().orc_e4m3_decode(int(code) & 0xFF)


def e4m3_encode(v: float) -> int:
    return int(_load().orc_e4m3_encode(float(v)))


def e5m2_decode(code: int) -> float:
    return _load().orc_e5m2_decode(int(code) & 0xFF)


def e5m2_encode(v: float) -> int:
    return int(_load().orc_e5m2_encode(float(v)))


def fp16_decode(bits: int) -> float:
    return _load().orc_fp16_decode(int(bits) & 0xFFFF)


def e4m3_table() -> np.ndarray:
    """The 256 E4M3 code values (binary64), NaN at 0x7F / 0xFF."""
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e5m2_table() -> np.ndarray:
    return np.array([e5m2_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.ascontiguousarray(v, dtype=np.float32).ravel()
    return np.fromiter((lib.orc_e4m3_encode(float(x)) for x in flat), dtype=np.uint8,
                       count=flat.size).reshape(np.shape(v))


def e5m2_encode_array(v: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.ascontiguousarray(v, dtype=np.float32).ravel()
    return np.fromiter((lib.orc_e5m2_encode(float(x)) for x in flat), dtype=np.uint8,
                       count=flat.size).reshape(np.shape(v))


# ---------------------------------------------------------------- row quantisation
def quantize_rows(x: np.ndarray, scales: np.ndarray | None = None):
    """Per-row E4M3 quantisation of a 2-D float32 or float16 array.

    Dynamic mode (``scales is None``): returns (codes uint8 [R,C], scales f32 [R]).
    Static mode: uses the given scales and returns (codes, scales)."""
    lib = _load()
    x = np.ascontiguousarray(x)
    if x.ndim != 2:
        raise ValueError("x must be 2-D")
    R, C = x.shape
    q = np.empty((R, C), dtype=np.uint8)
    mode = MODE_DYNAMIC if scales is None else MODE_STATIC
    s = np.zeros(R, dtype=np.float32) if scales is None else np.array(scales, dtype=np.float32)
    if x.dtype == np.float32:
        st = lib.orc_quantize_rows_f32(_ptr(x, ctypes.c_float), R, C, C,
                                       _ptr(q, ctypes.c_uint8), _ptr(s, ctypes.c_float), mode)
    elif x.dtype == np.float16:
        bits = x.view(np.uint16)
        tmp = np.empty(max(C, 1), dtype=np.float32)
        st = lib.orc_quantize_rows_f16(_ptr(bits, ctypes.c_uint16), R, C, C,
                                       _ptr(q, ctypes.c_uint8), _ptr(s, ctypes.c_float), mode,
                                       _ptr(tmp, ctypes.c_float))
    else:
        raise TypeError("x must be float32 or float16")
    _check(st)
    return q, s


# ---------------------------------------------------------------- FP8 linear
def fp8_linear(aq: np.ndarray, sa: np.ndarray, wq: np.ndarray, sw: np.ndarray) -> np.ndarray:
    """ref[m,n] = (sum_k dec(aq[m,k]) dec(wq[n,k])) * sa[m] * sw[n] in binary64."""
    lib = _load()
    aq = np.ascontiguousarray(aq, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = aq.shape
    N, K2 = wq.shape
    if K != K2 or sa.shape != (M,) or sw.shape != (N,):
        raise ValueError("shape mismatch")
    ref = np.empty((M, N), dtype=np.float64)
    lib.orc_fp8_linear(_ptr(aq, ctypes.c_uint8), _ptr(sa, ctypes.c_float), M, K,
                       _ptr(wq, ctypes.c_uint8), _ptr(sw, ctypes.c_float), N,
                       _ptr(ref, ctypes.c_double))
    return ref


# ---------------------------------------------------------------- NestedFP
def nestedfp_split(w: np.ndarray):
    """hi = bits >> 8, lo = bits & 0xFF of a float16 (or uint16 bit) array."""
    lib = _load()
    bits = np.ascontiguousarray(w).view(np.uint16)
    hi = np.empty(bits.shape, dtype=np.uint8)
    lo = np.empty(bits.shape, dtype=np.uint8)
    lib.orc_nestedfp_split(_ptr(bits, ctypes.c_uint16), bits.size,
                           _ptr(hi, ctypes.c_uint8), _ptr(lo, ctypes.c_uint8))
    return hi, lo


def nestedfp_rebuild(hi: int, lo: int) -> int:
    return int(_load().orc_nestedfp_rebuild(int(hi) & 0xFF, int(lo) & 0xFF))


def nestedfp_linear_fp16(x16: np.ndarray, hi: np.ndarray, lo: np.ndarray) -> np.ndarray:
    lib = _load()
    xb = np.ascontiguousarray(x16).view(np.uint16)
    hi = np.ascontiguousarray(hi, dtype=np.uint8)
    lo = np.ascontiguousarray(lo, dtype=np.uint8)
    M, K = xb.shape
    N = hi.shape[0]
    if hi.shape != (N, K) or lo.shape != (N, K):
        raise ValueError("shape mismatch")
    ref = np.empty((M, N), dtype=np.float64)
    lib.orc_nestedfp_linear_fp16(_ptr(xb, ctypes.c_uint16), M, K, _ptr(hi, ctypes.c_uint8),
                                 _ptr(lo, ctypes.c_uint8), N, _ptr(ref, ctypes.c_double))
    return ref


def nestedfp_linear_fp8(x16: np.ndarray, hi: np.ndarray):
    """Returns (ref [M,N] binary64, aq [M,K] codes, sa [M])."""
    lib = _load()
    xb = np.ascontiguousarray(x16).view(np.uint16)
    hi = np.ascontiguousarray(hi, dtype=np.uint8)
    M, K = xb.shape
    N = hi.shape[0]
    if hi.shape != (N, K):
        raise ValueError("shape mismatch")
    ref = np.empty((M, N), dtype=np.float64)
    aq = np.empty((M, K), dtype=np.uint8)
    sa = np.empty(M, dtype=np.float32)
    tmp = np.empty(max(K, 1), dtype=np.float32)
    st = lib.orc_nestedfp_linear_fp8(_ptr(xb, ctypes.c_uint16), M, K, _ptr(hi, ctypes.c_uint8), N,
                                     _ptr(ref, ctypes.c_double), _ptr(aq, ctypes.c_uint8),
                                     _ptr(sa, ctypes.c_float), _ptr(tmp, ctypes.c_float))
    _check(st)
    return ref, aq, sa


# ---------------------------------------------------------------- per-tensor scaling
def _as_f32_2d(x: np.ndarray) -> np.ndarray:
    """float32 copy of a 2-D float32 / float16 array (float16 widens exactly)."""
    x = np.asarray(x)
    if x.ndim != 2 or x.dtype not in (np.float32, np.float16):
        raise ValueError("x must be a 2-D float32 or float16 array")
    return np.ascontiguousarray(x, dtype=np.float32)


def amax_accumulate(x: np.ndarray, amax: float = 0.0) -> float:
    """max(amax, max |x|) — the MINMAX calibration statistic of a tensor."""
    lib = _load()
    x = _as_f32_2d(x)
    a = np.array([amax], dtype=np.float32)
    _check(lib.orc_amax_accumulate_f32(_ptr(x, ctypes.c_float), x.shape[0], x.shape[1], x.shape[1],
                                       _ptr(a, ctypes.c_float)))
    return float(a[0])


def quantize_tensor(x: np.ndarray, amax: float):
    """Static per-tensor quantisation with the scale of a calibrated amax.
    Returns (codes uint8 [R,C], scale f32)."""
    lib = _load()
    x = _as_f32_2d(x)
    q = np.empty(x.shape, dtype=np.uint8)
    s = np.zeros(1, dtype=np.float32)
    _check(lib.orc_quantize_tensor_f32(_ptr(x, ctypes.c_float), x.shape[0], x.shape[1], x.shape[1],
                                       np.float32(amax), _ptr(q, ctypes.c_uint8), _ptr(s, ctypes.c_float)))
    return q, np.float32(s[0])


class DelayedScaling:
    """Delayed per-tensor scaling over an amax history of length H: each
    step quantises with the scale carried from the previous step, then
    records its amax and carries max(history) / 448."""

    def __init__(self, history_len: int, initial_scale: float = 1.0):
        if history_len < 1:
            raise ValueError("history_len must be >= 1")
        self.history = np.zeros(history_len, dtype=np.float32)
        self.pos = 0
        self.scale = np.float32(initial_scale)

    def step(self, x: np.ndarray):
        """Returns (codes uint8 [R,C], the scale they were made with)."""
        lib = _load()
        x = _as_f32_2d(x)
        q = np.empty(x.shape, dtype=np.uint8)
        pos = ctypes.c_int32(self.pos)
        sc = np.array([self.scale], dtype=np.float32)
        used = np.zeros(1, dtype=np.float32)
        _check(lib.orc_delayed_step_f32(_ptr(x, ctypes.c_float), x.shape[0], x.shape[1], x.shape[1],
                                        _ptr(q, ctypes.c_uint8), _ptr(self.history, ctypes.c_float),
                                        len(self.history), ctypes.byref(pos), _ptr(sc, ctypes.c_float),
                                        _ptr(used, ctypes.c_float)))
        self.pos = pos.value
        self.scale = np.float32(sc[0])
        return q, np.float32(used[0])


# ---------------------------------------------------------------- normalisation / gated activation
def norm_rows(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray | None = None, eps: float = 1e-5) -> np.ndarray:
    """LayerNorm (beta given) or RMSNorm (beta None) of each row, binary64."""
    lib = _load()
    x = _as_f32_2d(x)
    R, C = x.shape
    gamma = np.ascontiguousarray(gamma, dtype=np.float32)
    y = np.empty((R, C), dtype=np.float64)
    bp = None if beta is None else _ptr(np.ascontiguousarray(beta, dtype=np.float32), ctypes.c_float)
    _check(lib.orc_norm_rows(_ptr(x, ctypes.c_float), R, C, C, _ptr(gamma, ctypes.c_float), bp, float(eps),
                             _ptr(y, ctypes.c_double)))
    return y


def silu_mul(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """g / (1 + exp(-g)) * u elementwise, binary64 (inputs widened exactly)."""
    lib = _load()
    g = np.ascontiguousarray(g, dtype=np.float64)
    u = np.ascontiguousarray(u, dtype=np.float64)
    if g.shape != u.shape:
        raise ValueError("g and u must have the same shape")
    h = np.empty(g.shape, dtype=np.float64)
    lib.orc_silu_mul(_ptr(g, ctypes.c_double), _ptr(u, ctypes.c_double), g.size, _ptr(h, ctypes.c_double))
    return h


# ---------------------------------------------------------------- FP8 KV cache
def kv_calibrate_scales(kv: np.ndarray) -> np.ndarray:
    """Per-KV-head MINMAX scales of kv [T, H, D]: fl32(max |kv[:, h, :]| / 448), 1 when 0."""
    lib = _load()
    kv = np.ascontiguousarray(kv, dtype=np.float32)
    T, H, D = kv.shape
    s = np.empty(H, dtype=np.float32)
    _check(lib.orc_kv_calibrate_scales(_ptr(kv, ctypes.c_float), T, H, D, _ptr(s, ctypes.c_float)))
    return s


class PagedKV:
    """An FP8 (E4M3) paged cache [num_blocks, H, B, D] with per-head scales
    and a block table (logical block -> physical block)."""

    def __init__(self, num_blocks: int, heads: int, head_dim: int, block_size: int, scales: np.ndarray,
                 block_table: np.ndarray):
        self.cache = np.zeros((num_blocks, heads, block_size, head_dim), dtype=np.uint8)
        self.scales = np.ascontiguousarray(scales, dtype=np.float32)
        self.block_table = np.ascontiguousarray(block_table, dtype=np.int32)
        self.B, self.H, self.D = block_size, heads, head_dim

    def write(self, kv: np.ndarray, t0: int):
        """Quantise kv [T, H, D] into positions t0 .. t0 + T - 1."""
        lib = _load()
        kv = np.ascontiguousarray(kv, dtype=np.float32)
        T = kv.shape[0]
        if (t0 + T + self.B - 1) // self.B > len(self.block_table):
            raise ValueError("block table too short")
        _check(lib.orc_kv_write_paged(_ptr(kv, ctypes.c_float), t0, T, self.H, self.D, _ptr(self.scales, ctypes.c_float),
                                      self.B, self.block_table.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                      self.cache.shape[0], _ptr(self.cache, ctypes.c_uint8)))

    def gather(self, ctx: int) -> np.ndarray:
        """Codes of positions 0 .. ctx - 1 as [ctx, H, D] (logical order)."""
        idx = np.arange(ctx)
        return self.cache[self.block_table[idx // self.B], :, idx % self.B, :]


def attention_paged(q: np.ndarray, k: PagedKV, v: PagedKV, ctx: int) -> np.ndarray:
    """Causal attention of q [Tq, Hq, D] at positions ctx - Tq .. ctx - 1
    over the dequantised paged K / V caches (binary64)."""
    lib = _load()
    q = np.ascontiguousarray(q, dtype=np.float64)
    Tq, Hq, D = q.shape
    if not (np.array_equal(k.block_table, v.block_table) and k.B == v.B and k.H == v.H and k.D == D == v.D):
        raise ValueError("K and V caches must share block size, table and shape")
    out = np.empty((Tq, Hq, D), dtype=np.float64)
    scratch = np.empty(max(ctx, 1), dtype=np.float64)
    bt = k.block_table.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    _check(lib.orc_attention_paged(_ptr(q, ctypes.c_double), Tq, Hq, D, _ptr(k.cache, ctypes.c_uint8),
                                   _ptr(v.cache, ctypes.c_uint8), _ptr(k.scales, ctypes.c_float),
                                   _ptr(v.scales, ctypes.c_float), k.H, k.B, bt, k.cache.shape[0], ctx,
                                   _ptr(out, ctypes.c_double), _ptr(scratch, ctypes.c_double)))
    return out
