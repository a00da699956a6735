"""GPU parity of the FP8 paged decode attention against the oracle ("7B on
an RTX 4060 with FP8": K/V held in FP8; "C++ and FP8" §3.2 paged cache of
16-token blocks, §3.3 attention in the FP8 dataflow).

The CUDA-core kernel works in binary32 on the dequantised cache; the oracle
in binary64 on the same codes and the same (binary32) queries.  Bound per
output element d of a (sequence, head), from the binary32 steps:
  logit error (base 2)  D_t <= (D + 4) 2^-24 sum_d |q_d k_td| s_k log2(e)/sqrt(D)
  weight error          |dp_t / p_t| <= 2 ln2 max_t D_t + 2^-21 (two exp2f)
  sums over T positions (T + 16) 2^-24 (sequential accumulation per warp)
  |out - ref| <= (2 (2 ln2 D + 2^-21) + (T + 16) 2^-24) max_t |v_td s_v|
                 + rounding of the output (2^-24, 2^-11 or 2^-8 of |ref|),
taken twice for margin.  The tensor-core kernel (PGF8_FLAG_ATTN_MMA) also
rounds q and the probabilities to binary16 (2^-11 relative, 2^-25 absolute
below the normal range) and accumulates on the tensor cores: its logit term
gains 2^-11 sum_d |q_d k_td| (and 2^-22 per addition), its weights 2^-11 plus
2^-25 T absolute."""
import math

import numpy as np
import pytest
import torch

import oracle

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"
E4 = oracle.e4m3_table()
OUT_ULP = {torch.float32: 2.0 ** -24, torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


def _to(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _tolerance(q, K, V, ctx, out_dtype, mma=False):
    """Per-element bound [Hq, D] for one sequence (see the module docstring)."""
    Hq, D = q.shape
    Hkv = K.H
    G = Hq // Hkv
    kd = E4[K.gather(ctx)]                       # [T, Hkv, D] codes' values
    vd = E4[V.gather(ctx)] * V.scales.astype(np.float64)[None, :, None]
    tol = np.empty((Hq, D))
    for h in range(Hq):
        hk = h // G
        rel = (2.0 ** -11 + (D + 4) * 2.0 ** -22) if mma else (D + 4) * 2.0 ** -24
        dl = rel * np.abs(kd[:, hk, :] * q[h][None, :]).sum(axis=1).max() * \
            K.scales[hk] * math.log2(math.e) / math.sqrt(D)
        eps = 2 * (2 * math.log(2) * dl + 2.0 ** -21) + (ctx + 16) * 2.0 ** -24
        if mma:
            eps += 2.0 ** -11 + 2.0 ** -25 * ctx + (ctx + 16) * 2.0 ** -22
        tol[h] = 2 * eps * np.abs(vd[:, hk, :]).max(axis=0)
    return tol, OUT_ULP[out_dtype]


def _build(seqs, Hkv, D, B, ctxs, seed, kv_scale=1.0):
    g = np.random.default_rng(seed)
    max_ctx = max(ctxs)
    tstride = max(1, -(-max_ctx // B)) + 1
    nb = seqs * tstride + 2
    tables = g.permutation(nb)[:seqs * tstride].astype(np.int32).reshape(seqs, tstride)
    kk = [(g.standard_normal((c, Hkv, D)) * kv_scale).astype(np.float32) for c in ctxs]
    vv = [g.standard_normal((c, Hkv, D)).astype(np.float32) for c in ctxs]
    allk = np.concatenate(kk) if sum(ctxs) else np.ones((1, Hkv, D), np.float32)
    allv = np.concatenate(vv) if sum(ctxs) else np.ones((1, Hkv, D), np.float32)
    sk, sv = oracle.kv_calibrate_scales(allk), oracle.kv_calibrate_scales(allv)
    kc = np.full((nb, Hkv, B, D), 0x7F, np.uint8)   # NaN codes in every unwritten slot: never read
    vc = np.full((nb, Hkv, B, D), 0x7F, np.uint8)
    refs = []
    for s in range(seqs):
        K = oracle.PagedKV(nb, Hkv, D, B, sk, tables[s])
        V = oracle.PagedKV(nb, Hkv, D, B, sv, tables[s])
        K.cache, V.cache = kc, vc
        if ctxs[s]:
            K.write(kk[s], 0)
            V.write(vv[s], 0)
        refs.append((K, V))
    return dict(kc=kc, vc=vc, sk=sk, sv=sv, tables=tables, refs=refs, max_ctx=max_ctx)


def _run(c, q_dev, ctxs, out_dtype=torch.float32, splits=0, max_ctx=None, errors=None, mma=False):
    return pg.fp8_attention_decode_paged(q_dev, _to(c["kc"]), _to(c["vc"]), _to(c["sk"]), _to(c["sv"]),
                                         _to(c["tables"]), _to(np.array(ctxs, np.int32)),
                                         c["max_ctx"] if max_ctx is None else max_ctx, out_dtype=out_dtype,
                                         splits=splits, errors=errors, flags=pg.FLAG_ATTN_MMA if mma else 0)


def _check(c, q, out, ctxs, out_dtype, mma=False):
    got = out.to(torch.float32).cpu().numpy().astype(np.float64)
    for s, ctx in enumerate(ctxs):
        if ctx == 0:
            assert not got[s].any()
            continue
        K, V = c["refs"][s]
        ref = oracle.attention_paged(q[s:s + 1].astype(np.float64), K, V, ctx)[0]
        tol, ulp = _tolerance(q[s], K, V, ctx, out_dtype, mma)
        err = np.abs(got[s] - ref)
        bad = err > tol + ulp * np.abs(ref)
        assert not bad.any(), (s, ctx, float(err.max()), float(tol.max()))


@pytest.mark.parametrize("mma", [False, True])
@pytest.mark.parametrize("seqs,Hq,Hkv,D,B,ctxs,splits", [
    (3, 8, 8, 128, 16, [1, 77, 300], 0),          # MHA, ragged
    (3, 8, 8, 128, 16, [1, 77, 300], 1),          # one chunk: no merge kernel
    (2, 16, 2, 128, 16, [513, 1000], 5),          # grouped heads (8 per KV head)
    (2, 12, 2, 64, 32, [16, 129], 3),             # 6 per KV head: 3 CTAs of 2
    (2, 8, 2, 256, 16, [250, 31], 0),             # head_dim 256, 4 per KV head
    (4, 4, 4, 64, 16, [0, 15, 16, 17], 2),        # empty and block-edge contexts
])
def test_decode_attention_matches_the_oracle(seqs, Hq, Hkv, D, B, ctxs, splits, mma):
    c = _build(seqs, Hkv, D, B, ctxs, seed=seqs * 100 + Hq + D)
    q = np.random.default_rng(D).standard_normal((seqs, Hq, D)).astype(np.float32)
    out = _run(c, _to(q), ctxs, splits=splits, mma=mma)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    _check(c, q, out, ctxs, torch.float32, mma)


@pytest.mark.parametrize("G", [1, 3, 8, 16])
def test_tensor_core_path_across_group_sizes(G):
    """Padding heads (G not a multiple of 8) and several CTAs per KV head (G = 16)."""
    seqs, Hkv, D = 2, 2, 128
    ctxs = [333, 64]
    c = _build(seqs, Hkv, D, 16, ctxs, seed=50 + G)
    q = np.random.default_rng(G).standard_normal((seqs, Hkv * G, D)).astype(np.float32)
    out = _run(c, _to(q), ctxs, mma=True)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    _check(c, q, out, ctxs, torch.float32, mma=True)


@pytest.mark.parametrize("qdt,odt", [(torch.float16, torch.bfloat16), (torch.bfloat16, torch.float16),
                                     (torch.float32, torch.bfloat16)])
def test_query_and_output_types_and_strided_query(qdt, odt):
    seqs, Hq, Hkv, D = 3, 8, 2, 128
    ctxs = [200, 64, 1]
    c = _build(seqs, Hkv, D, 16, ctxs, seed=11)
    g = np.random.default_rng(12)
    q = torch.from_numpy(g.standard_normal((seqs, Hq, D)).astype(np.float32)).to(qdt)
    # the query is a slice of a QKV-projection-like row: [q | k | v]
    wide = torch.zeros((seqs, (Hq + 2 * Hkv) * D), dtype=qdt)
    wide[:, :Hq * D] = q.reshape(seqs, Hq * D)
    q_dev = wide.to(DEV)[:, :Hq * D].view(seqs, Hq, D)
    assert q_dev.stride(0) == (Hq + 2 * Hkv) * D
    out = _run(c, q_dev, ctxs, out_dtype=odt)
    torch.cuda.synchronize()
    assert out.dtype == odt
    _check(c, q.to(torch.float32).numpy(), out, ctxs, odt)


def test_split_count_changes_only_rounding():
    seqs, Hq, Hkv, D = 2, 8, 8, 128
    ctxs = [4000, 1234]
    c = _build(seqs, Hkv, D, 16, ctxs, seed=21)
    q = _to(np.random.default_rng(22).standard_normal((seqs, Hq, D)).astype(np.float32))
    outs = [_run(c, q, ctxs, splits=sp).cpu() for sp in (1, 2, 7, 0)]
    for o in outs[1:]:
        torch.testing.assert_close(o, outs[0], rtol=1e-5, atol=1e-6)
    # same split: identical bits on a second run (no scheduling dependence)
    assert torch.equal(_run(c, q, ctxs, splits=7).cpu(), outs[2])


def test_written_by_the_cache_writer():
    """The cache as pgf8_fp8_kv_write_paged leaves it, attended in place."""
    Hq, Hkv, D, B, T = 16, 4, 128, 16, 157
    g = np.random.default_rng(31)
    k = g.standard_normal((T, Hkv, D)).astype(np.float32)
    v = g.standard_normal((T, Hkv, D)).astype(np.float32)
    sk, sv = oracle.kv_calibrate_scales(k), oracle.kv_calibrate_scales(v)
    nb = 16
    table = g.permutation(nb)[:10].astype(np.int32)
    kc = torch.zeros((nb, Hkv, B, D), dtype=torch.uint8, device=DEV)
    vc = torch.zeros_like(kc)
    pg.fp8_kv_write_paged(_to(k), _to(sk), kc, _to(table), 0)
    pg.fp8_kv_write_paged(_to(v), _to(sv), vc, _to(table), 0)
    q = g.standard_normal((1, Hq, D)).astype(np.float32)
    out = pg.fp8_attention_decode_paged(_to(q), kc, vc, _to(sk), _to(sv), _to(table[None, :]),
                                        _to(np.array([T], np.int32)), T)
    torch.cuda.synchronize()
    K = oracle.PagedKV(nb, Hkv, D, B, sk, table)
    V = oracle.PagedKV(nb, Hkv, D, B, sv, table)
    K.write(k, 0)
    V.write(v, 0)
    np.testing.assert_array_equal(kc.cpu().numpy(), K.cache)
    ref = oracle.attention_paged(q.astype(np.float64), K, V, T)[0]
    tol, ulp = _tolerance(q[0], K, V, T, torch.float32)
    assert (np.abs(out.cpu().numpy()[0] - ref) <= tol + ulp * np.abs(ref)).all()


def test_bad_table_entries_and_long_contexts_are_counted():
    seqs, Hq, Hkv, D, B = 2, 4, 2, 64, 16
    ctxs = [40, 40]
    c = _build(seqs, Hkv, D, B, ctxs, seed=41)
    c["tables"] = c["tables"].copy()
    c["tables"][0, 1] = 10 ** 6                   # positions 16..31 of sequence 0: out of range
    q = np.random.default_rng(42).standard_normal((seqs, Hq, D)).astype(np.float32)
    errors = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = _run(c, _to(q), ctxs, splits=1, errors=errors)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    assert errors.item() == 1                     # one 16-position step
    assert torch.isfinite(out).all()
    # sequence 1 is untouched by sequence 0's bad entry
    K, V = c["refs"][1]
    ref = oracle.attention_paged(q[1:2].astype(np.float64), K, V, 40)[0]
    tol, ulp = _tolerance(q[1], K, V, 40, torch.float32)
    assert (np.abs(out[1].cpu().numpy() - ref) <= tol + ulp * np.abs(ref)).all()
    # a context longer than max_context is clamped to it and counted
    errors.zero_()
    out2 = _run(c, _to(q), [40, 40], max_ctx=32, splits=1, errors=errors)
    torch.cuda.synchronize()
    assert errors.item() >= 2
    K, V = c["refs"][1]
    ref32 = oracle.attention_paged(q[1:2].astype(np.float64), K, V, 32)[0]
    tol, ulp = _tolerance(q[1], K, V, 32, torch.float32)
    assert (np.abs(out2[1].cpu().numpy() - ref32) <= tol + ulp * np.abs(ref32)).all()


@pytest.mark.parametrize("qdt", [torch.float32, torch.bfloat16])
def test_tensor_core_path_queries_beyond_binary16_range(qdt):
    """Queries of magnitude up to 2^20 (beyond binary16's 65504): the
    tensor-core path scales each head's query by a power of two into binary16
    range and its scores back, so it stays finite and within the bound like
    the CUDA-core path."""
    seqs, Hq, Hkv, D, B, ctxs = 2, 8, 2, 128, 16, [200, 77]
    c = _build(seqs, Hkv, D, B, ctxs, seed=91)
    g = np.random.default_rng(92)
    q = g.standard_normal((seqs, Hq, D)).astype(np.float32)
    q[:, ::2] *= 2.0 ** 20                          # every other head far beyond 65504
    q[0, 1] *= 2.0 ** 13                            # and one just below
    qt = _to(q).to(qdt)
    qref = qt.float().cpu().numpy()
    for mma in (False, True):
        out = _run(c, qt, ctxs, mma=mma)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all(), f"mma={mma}: non-finite outputs"
        _check(c, qref, out, ctxs, torch.float32, mma=mma)
