"""CPU models of the attention kernels (tests/kernel_models.py) against the
oracle: the kernels' index arithmetic, masks, chunking and merges checked
before they run on a GPU.  The chunk plans come from the library's own host
planner.  Unwritten cache slots hold NaN codes, so a model that read one
would fail; every address the models form is asserted inside the cache."""
import math

import numpy as np
import pytest

import oracle
import precision_gemm_fp8_b200 as pg
import kernel_models as km

E4 = oracle.e4m3_table()


def _cache(seqs, Hkv, D, B, ctxs, seed, exact=False):
    g = np.random.default_rng(seed)
    max_ctx = max(ctxs)
    tstride = max(1, -(-max_ctx // B)) + 1
    nb = seqs * tstride + 2
    tables = g.permutation(nb)[:seqs * tstride].astype(np.int32).reshape(seqs, tstride)
    kc = np.full((nb, Hkv, B, D), 0x7F, np.uint8)
    vc = np.full((nb, Hkv, B, D), 0x7F, np.uint8)
    vv = [g.standard_normal((c, Hkv, D)).astype(np.float32) for c in ctxs]
    if exact:
        kk = [(-g.integers(0, 17, (c, Hkv, D)) / 16.0).astype(np.float32) for c in ctxs]
        sk = np.full(Hkv, 1.0 / 16, np.float32)
    else:
        kk = [g.standard_normal((c, Hkv, D)).astype(np.float32) for c in ctxs]
        sk = oracle.kv_calibrate_scales(np.concatenate(kk))
    sv = oracle.kv_calibrate_scales(np.concatenate(vv))
    refs = []
    for s in range(seqs):
        K, V = oracle.PagedKV(nb, Hkv, D, B, sk, tables[s]), oracle.PagedKV(nb, Hkv, D, B, sv, tables[s])
        K.cache, V.cache = kc, vc
        if ctxs[s]:
            K.write(kk[s], 0)
            V.write(vv[s], 0)
        refs.append((K, V))
    vfin = E4[vc][np.isfinite(E4[vc])]
    return dict(kc=kc, vc=vc, sk=sk, sv=sv, tables=tables, refs=refs, max_ctx=max_ctx,
                vmax=float(np.abs(vfin).max() * sv.max()))


@pytest.mark.parametrize("seqs,Hq,Hkv,D,B,ctxs,splits", [
    (2, 4, 2, 64, 16, [37, 70], 0),
    (2, 4, 2, 64, 16, [37, 70], 3),
    (3, 8, 1, 64, 32, [1, 16, 65], 2),
    (2, 3, 3, 64, 16, [0, 50], 4),
    (1, 6, 2, 128, 16, [300], 0),
])
def test_decode_cuda_core_model(seqs, Hq, Hkv, D, B, ctxs, splits):
    c = _cache(seqs, Hkv, D, B, ctxs, seed=seqs * 10 + Hq + D)
    q = np.random.default_rng(D + Hq).standard_normal((seqs, Hq, D)).astype(np.float32)
    nsplit, chunk = pg.fp8_attention_decode_plan(seqs, Hq, Hkv, D, c["max_ctx"], splits)
    out, errors = km.decode_cuda_core(q, c["kc"], c["vc"], c["sk"], c["sv"], c["tables"], ctxs, c["max_ctx"],
                                      nsplit, chunk)
    assert errors == 0
    for s, ctx in enumerate(ctxs):
        if ctx == 0:
            assert not out[s].any()
            continue
        ref = oracle.attention_paged(q[s:s + 1].astype(np.float64), *c["refs"][s], ctx)[0]
        assert np.abs(out[s] - ref).max() <= 1e-5 * c["vmax"]


def test_decode_cuda_core_model_counts_bad_entries():
    c = _cache(2, 2, 64, 16, [40, 40], seed=3)
    c["tables"][0, 1] = 10 ** 6
    q = np.random.default_rng(4).standard_normal((2, 4, 64)).astype(np.float32)
    out, errors = km.decode_cuda_core(q, c["kc"], c["vc"], c["sk"], c["sv"], c["tables"], [40, 41], 40, 1, 48)
    assert errors == 2                                  # one 16-position step, one clamped context
    assert np.isfinite(out).all()


@pytest.mark.parametrize("seqs,Hq,Hkv,D,B,ctxs,splits", [
    (1, 8, 1, 64, 16, [37], 1),
    (2, 16, 2, 128, 16, [70, 129], 2),
    (1, 6, 2, 64, 32, [50], 1),
    (1, 2, 2, 256, 16, [20], 1),
])
def test_decode_tensor_core_model(seqs, Hq, Hkv, D, B, ctxs, splits):
    c = _cache(seqs, Hkv, D, B, ctxs, seed=seqs * 20 + Hq + D)
    q = np.random.default_rng(D).standard_normal((seqs, Hq, D)).astype(np.float32)
    nsplit, chunk = pg.fp8_attention_decode_plan(seqs, Hq, Hkv, D, c["max_ctx"], splits)
    out = km.decode_tensor_core(q, c["kc"], c["vc"], c["sk"], c["sv"], c["tables"], ctxs, c["max_ctx"], nsplit,
                                chunk)
    for s, ctx in enumerate(ctxs):
        ref = oracle.attention_paged(q[s:s + 1].astype(np.float64), *c["refs"][s], ctx)[0]
        # binary16 query and probabilities: a few 2^-11 of the largest value
        assert np.abs(out[s] - ref).max() <= 8 * 2.0 ** -11 * c["vmax"]


def _context_case(seqs, Hq, Hkv, B, q_lens, ctxs, seed, exact):
    c = _cache(seqs, Hkv, 128, B, ctxs, seed, exact)
    q_start = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    total_q = int(q_start[-1])
    g = np.random.default_rng(seed + 1)
    if exact:                                           # power-of-two probabilities (temperature ln 2)
        q = np.zeros((total_q, Hq, 128), np.float32)
        for t in range(total_q):
            for h in range(Hq):
                q[t, h, (t * 7 + h * 3) % 128] = 16 * math.sqrt(128) * math.log(2)
    else:
        q = (g.standard_normal((total_q, Hq, 128)) * 2).astype(np.float32)
    qc, qs = oracle.quantize_rows(q.reshape(total_q * Hq, 128))
    qc = qc.reshape(total_q, Hq, 128)
    out = km.context(qc, qs, q_start, ctxs, c["kc"], c["vc"], c["sk"], c["sv"], c["tables"], c["max_ctx"],
                     max(q_lens))
    qdeq = E4[qc] * qs.reshape(total_q, Hq)[:, :, None].astype(np.float64)
    ref = np.zeros_like(qdeq)
    for s, ctx in enumerate(ctxs):
        a, b = q_start[s], q_start[s + 1]
        ref[a:b] = oracle.attention_paged(qdeq[a:b], *c["refs"][s], ctx)
    return out, ref, c


@pytest.mark.parametrize("seqs,Hq,Hkv,B,q_lens,ctxs", [
    (2, 2, 1, 16, [130, 40], [130, 300]),
    (1, 2, 2, 32, [200], [333]),
    (1, 1, 1, 16, [1], [17]),
])
def test_context_model_exact_probabilities(seqs, Hq, Hkv, B, q_lens, ctxs):
    out, ref, c = _context_case(seqs, Hq, Hkv, B, q_lens, ctxs, seed=seqs + Hq + B, exact=True)
    assert np.abs(out - ref).max() <= 2.0 ** -14 * c["vmax"]


def test_context_model_random_within_the_fp8_bound():
    out, ref, c = _context_case(2, 4, 2, 16, [77, 129], [77, 129], seed=3, exact=False)
    T = 129
    assert np.abs(out - ref).max() <= (2.0 ** -4 + 2.0 ** -18 * (T + 1) + 2.0 ** -16) * c["vmax"]
