"""Pins of the oracle's FP8 paged KV cache and attention over it ("7B on an
RTX 4060 with FP8": FP8 K/V storage; "C++ and FP8" §3.2 paged cache in
blocks of 16 tokens, §3.3 FP8 context attention).  Readings: per-KV-head
MINMAX scales, saturating E4M3 codes in [block][kv head][slot][d] through a
block table, attention softmax(q.k/sqrt(D)) v in binary64 over the
dequantised cache, grouped query heads, causal for context queries."""
import numpy as np
import pytest

import oracle

E4 = oracle.e4m3_table()
B = 16


def _caches(kv_k, kv_v, table, num_blocks):
    T, H, D = kv_k.shape
    sk, sv = oracle.kv_calibrate_scales(kv_k), oracle.kv_calibrate_scales(kv_v)
    K = oracle.PagedKV(num_blocks, H, D, B, sk, table)
    V = oracle.PagedKV(num_blocks, H, D, B, sv, table)
    K.write(kv_k, 0)
    V.write(kv_v, 0)
    return K, V


def _deq(cache: oracle.PagedKV, ctx):
    return E4[cache.gather(ctx)] * cache.scales.astype(np.float64)[None, :, None]


def test_scales_and_codes_reduce_to_the_row_quantiser():
    g = np.random.default_rng(1)
    kv = (g.standard_normal((37, 3, 64)) * np.array([0.5, 4.0, 30.0])[None, :, None]).astype(np.float32)
    s = oracle.kv_calibrate_scales(kv)
    for h in range(3):
        assert s[h] == oracle.quantize_tensor(kv[:, h, :], oracle.amax_accumulate(kv[:, h, :]))[1]
    table = np.array([5, 1, 3], np.int32)
    K = oracle.PagedKV(6, 3, 64, B, s, table)
    K.write(kv[:20], 0)
    K.write(kv[20:], 20)                                     # written in two pieces
    codes = K.gather(37)
    for h in range(3):
        ref, _ = oracle.quantize_rows(kv[:, h, :], np.full(37, s[h], np.float32))
        np.testing.assert_array_equal(codes[:, h, :], ref)
        i = np.unravel_index(np.argmax(np.abs(kv[:, h, :])), (37, 64))
        assert codes[i[0], h, i[1]] in (0x7E, 0xFE)          # the amax element lands on 448
    # physical placement: token t at [table[t // B], h, t % B]
    assert np.array_equal(K.cache[3, 2, 4], codes[36, 2])
    assert not K.cache[0].any() and not K.cache[2].any()     # untouched blocks


def test_attention_closed_forms():
    g = np.random.default_rng(2)
    D = 32
    kv_v = g.standard_normal((24, 1, D)).astype(np.float32)
    # identical keys: uniform weights, output = mean of the dequantised values
    kv_k = np.tile(g.standard_normal((1, 1, D)).astype(np.float32), (24, 1, 1))
    K, V = _caches(kv_k, kv_v, np.array([1, 0], np.int32), 2)
    q = g.standard_normal((1, 1, D))
    out = oracle.attention_paged(q, K, V, 24)
    np.testing.assert_allclose(out[0, 0], _deq(V, 24)[:, 0].mean(axis=0), rtol=1e-13, atol=1e-15)
    # one key: the output is its value
    out1 = oracle.attention_paged(q, K, V, 1)
    np.testing.assert_allclose(out1[0, 0], _deq(V, 1)[0, 0], rtol=0, atol=1e-15)
    # a dominant key (q along it, large): the output is that key's value
    kv_k2 = g.standard_normal((24, 1, D)).astype(np.float32)
    K2, V2 = _caches(kv_k2, kv_v, np.array([1, 0], np.int32), 2)
    kd = _deq(K2, 24)[:, 0]
    j = 17
    q2 = (kd[j] / np.linalg.norm(kd[j]) * 400.0)[None, None, :]
    assert np.argmax(kd @ q2[0, 0]) == j
    np.testing.assert_allclose(oracle.attention_paged(q2, K2, V2, 24)[0, 0], _deq(V2, 24)[j, 0], atol=1e-6)
    # causal context queries: query 0 of a full-length prompt sees key 0 only
    qc = g.standard_normal((24, 1, D))
    outc = oracle.attention_paged(qc, K2, V2, 24)
    np.testing.assert_allclose(outc[0, 0], _deq(V2, 24)[0, 0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(outc[23, 0], oracle.attention_paged(qc[23:], K2, V2, 24)[0, 0], rtol=0, atol=0)


def test_attention_invariants_gqa_block_table_and_value_scale():
    g = np.random.default_rng(3)
    T, Hkv, D, G = 40, 2, 16, 3
    kk = g.standard_normal((T, Hkv, D)).astype(np.float32)
    vv = g.standard_normal((T, Hkv, D)).astype(np.float32)
    q = g.standard_normal((2, Hkv * G, D))
    K, V = _caches(kk, vv, np.array([2, 0, 1], np.int32), 3)
    out = oracle.attention_paged(q, K, V, T)
    # another physical placement of the same logical cache: identical results
    Kp, Vp = _caches(kk, vv, np.array([0, 2, 1], np.int32), 3)
    np.testing.assert_array_equal(oracle.attention_paged(q, Kp, Vp, T), out)
    # grouped heads = multi-head attention over KV heads repeated G times
    rep = lambda a: np.repeat(a, G, axis=1)
    Km, Vm = _caches(rep(kk), rep(vv), np.array([2, 0, 1], np.int32), 3)
    np.testing.assert_allclose(oracle.attention_paged(q, Km, Vm, T), out, rtol=1e-13, atol=1e-14)
    # the value scale multiplies the output
    V.scales = V.scales * np.float32(2.0)
    np.testing.assert_allclose(oracle.attention_paged(q, K, V, T), 2.0 * out, rtol=1e-14, atol=1e-15)


def test_argument_errors():
    kv = np.ones((4, 2, 8), np.float32)
    s = oracle.kv_calibrate_scales(kv)
    K = oracle.PagedKV(1, 2, 8, B, s, np.array([0], np.int32))
    with pytest.raises(ValueError):
        K.write(np.ones((20, 2, 8), np.float32), 0)          # past the block table
    bad = oracle.PagedKV(1, 2, 8, B, s, np.array([5], np.int32))
    with pytest.raises(oracle.OracleError):
        bad.write(kv, 0)                                      # physical block out of range
    K.write(kv, 0)
    with pytest.raises(oracle.OracleError):
        oracle.attention_paged(np.ones((1, 3, 8)), K, K, 4)  # 3 query heads over 2 KV heads


def test_attention_equals_the_library_routine():
    """torch's scaled_dot_product_attention (binary64, default scale 1/sqrt(D))
    on the dequantised cache: pins the temperature, the key scale, the
    softmax and the causal alignment (a full prompt: query i sees 0..i)."""
    import torch
    import torch.nn.functional as F
    g = np.random.default_rng(4)
    T, Hkv, D, G = 45, 2, 32, 2
    kk = (g.standard_normal((T, Hkv, D)) * 3).astype(np.float32)
    vv = g.standard_normal((T, Hkv, D)).astype(np.float32)
    K, V = _caches(kk, vv, np.array([2, 0, 1], np.int32), 3)
    kd = torch.from_numpy(np.repeat(_deq(K, T), G, axis=1)).permute(1, 0, 2)   # [Hq, T, D]
    vd = torch.from_numpy(np.repeat(_deq(V, T), G, axis=1)).permute(1, 0, 2)
    # decode: one query at the last position sees every key
    q1 = g.standard_normal((1, Hkv * G, D))
    ref1 = F.scaled_dot_product_attention(torch.from_numpy(q1).permute(1, 0, 2), kd, vd)
    np.testing.assert_allclose(oracle.attention_paged(q1, K, V, T), ref1.permute(1, 0, 2).numpy(),
                               rtol=1e-12, atol=1e-13)
    # context: T queries over T keys, causal
    qc = g.standard_normal((T, Hkv * G, D))
    refc = F.scaled_dot_product_attention(torch.from_numpy(qc).permute(1, 0, 2), kd, vd, is_causal=True)
    np.testing.assert_allclose(oracle.attention_paged(qc, K, V, T), refc.permute(1, 0, 2).numpy(),
                               rtol=1e-12, atol=1e-13)
    # the last Tq queries of a longer context (bottom-right causal alignment): explicit mask
    Tq = 5
    qt = qc[-Tq:]
    mask = torch.from_numpy(np.arange(T)[None, :] <= (T - Tq + np.arange(Tq))[:, None])
    reft = F.scaled_dot_product_attention(torch.from_numpy(qt).permute(1, 0, 2), kd, vd, attn_mask=mask)
    np.testing.assert_allclose(oracle.attention_paged(qt, K, V, T), reft.permute(1, 0, 2).numpy(),
                               rtol=1e-12, atol=1e-13)
