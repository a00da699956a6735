"""GPU parity of the FP8 context attention over the paged cache ("C++ and
FP8" §3.2-3.3) against the oracle.

The query is quantised by the row quantiser (bit-exact with the oracle's);
the oracle then attends with the dequantised query in binary64.  The kernel
rounds the probabilities to E4M3 (x 2^8): at most 2^-4 relative above 2^-14,
2^-18 absolute below, with l summing the unrounded values and the largest
probability exactly 1, so
  |out - ref| <= (2^-4 + 2^-18 (T + 1)) max_t |v_t s_v|   (plus binary32 terms).
Cases built so that every probability is a power of two (one-hot queries,
integer keys, softmax temperature ln 2 per unit) make that rounding exact:
there the kernel must agree within 2^-14 max |v s_v|."""
import math

import numpy as np
import pytest
import torch

import oracle

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"
E4 = oracle.e4m3_table()


def _to(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _case(seqs, Hq, Hkv, B, q_lens, ctxs, seed, exact):
    g = np.random.default_rng(seed)
    D = 128
    max_ctx = max(ctxs)
    tstride = -(-max_ctx // B) + 1
    nb = seqs * tstride + 3
    tables = g.permutation(nb)[:seqs * tstride].astype(np.int32).reshape(seqs, tstride)
    kc = np.full((nb, Hkv, B, D), 0x7F, np.uint8)           # NaN codes in every unwritten slot
    vc = np.full((nb, Hkv, B, D), 0x7F, np.uint8)
    vv = [g.standard_normal((c, Hkv, D)).astype(np.float32) for c in ctxs]
    sv = oracle.kv_calibrate_scales(np.concatenate(vv))
    if exact:
        sk = np.full(Hkv, 1.0 / 16, np.float32)
        kk = [(-g.integers(0, 17, (c, Hkv, D)) / 16.0).astype(np.float32) for c in ctxs]
    else:
        kk = [g.standard_normal((c, Hkv, D)).astype(np.float32) for c in ctxs]
        sk = oracle.kv_calibrate_scales(np.concatenate(kk))
    refs = []
    for s in range(seqs):
        K = oracle.PagedKV(nb, Hkv, D, B, sk, tables[s])
        V = oracle.PagedKV(nb, Hkv, D, B, sv, tables[s])
        K.cache, V.cache = kc, vc
        K.write(kk[s], 0)
        V.write(vv[s], 0)
        refs.append((K, V))
    q_start = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    total_q = int(q_start[-1])
    if exact:
        q = np.zeros((total_q, Hq, D), np.float32)
        for t in range(total_q):
            for h in range(Hq):
                q[t, h, (t * 7 + h * 3) % D] = 16 * math.sqrt(128) * math.log(2)
    else:
        q = (g.standard_normal((total_q, Hq, D)) * 2).astype(np.float32)
    return dict(q=q, q_start=q_start, ctxs=ctxs, kc=kc, vc=vc, sk=sk, sv=sv, tables=tables, refs=refs,
                max_ctx=max_ctx, max_q_len=max(q_lens))


def _reference(c, qc, qs):
    total_q, Hq, D = qc.shape
    qdeq = E4[qc] * qs.reshape(total_q, Hq)[:, :, None].astype(np.float64)
    out = np.zeros((total_q, Hq, D))
    for s, ctx in enumerate(c["ctxs"]):
        a, b = c["q_start"][s], c["q_start"][s + 1]
        if b > a:
            out[a:b] = oracle.attention_paged(qdeq[a:b], c["refs"][s][0], c["refs"][s][1], ctx)
    return out


def _run(c, errors=None, out_dtype=torch.float32, max_q_len=None):
    total_q, Hq, D = c["q"].shape
    qc_dev, qs_dev = pg.fp8_quantize_rows(_to(c["q"]).view(total_q * Hq, D))
    out = pg.fp8_attention_context_paged(qc_dev.view(total_q, Hq, D), qs_dev, _to(c["q_start"]),
                                         _to(np.array(c["ctxs"], np.int32)), _to(c["kc"]), _to(c["vc"]),
                                         _to(c["sk"]), _to(c["sv"]), _to(c["tables"]), c["max_ctx"],
                                         c["max_q_len"] if max_q_len is None else max_q_len, out_dtype=out_dtype,
                                         errors=errors)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    return out, qc_dev.view(total_q, Hq, D).cpu().numpy(), qs_dev.cpu().numpy()


def _vmax(c):
    v = E4[c["vc"]]
    return np.abs(v[np.isfinite(v)]).max() * float(c["sv"].max())


@pytest.mark.parametrize("seqs,Hq,Hkv,B,q_lens,ctxs", [
    (1, 1, 1, 16, [1], [17]),                      # one query, ragged block
    (2, 2, 1, 16, [130, 40], [130, 300]),          # a prompt; a continuation after a cached prefix
    (1, 2, 2, 32, [200], [333]),                   # block size 32
    (2, 8, 2, 16, [256, 100], [256, 612]),         # grouped heads, several key tiles, exact tile edges
])
def test_exact_probabilities_match_the_oracle(seqs, Hq, Hkv, B, q_lens, ctxs):
    c = _case(seqs, Hq, Hkv, B, q_lens, ctxs, seed=seqs + Hq + B, exact=True)
    out, qc, qs = _run(c)
    ref_codes, ref_scales = oracle.quantize_rows(c["q"].reshape(-1, 128))
    np.testing.assert_array_equal(qc.reshape(-1, 128), ref_codes)
    np.testing.assert_array_equal(qs, ref_scales)
    ref = _reference(c, qc, qs)
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref)
    assert err.max() <= 2.0 ** -14 * _vmax(c), err.max()


@pytest.mark.parametrize("odt", [torch.float32, torch.bfloat16])
def test_random_within_the_fp8_probability_bound(odt):
    c = _case(2, 4, 2, 16, [77, 129], [77, 400], seed=5, exact=False)
    out, qc, qs = _run(c, out_dtype=odt)
    ref = _reference(c, qc, qs)
    T = max(c["ctxs"])
    bound = (2.0 ** -4 + 2.0 ** -18 * (T + 1) + 2.0 ** -16) * _vmax(c)
    ulp = 2.0 ** -8 if odt == torch.bfloat16 else 2.0 ** -24
    err = np.abs(out.to(torch.float32).cpu().numpy().astype(np.float64) - ref)
    assert (err <= bound + ulp * np.abs(ref)).all(), err.max()
    assert torch.isfinite(out).all()


def test_bad_entries_and_lengths_are_counted():
    c = _case(2, 2, 2, 16, [40, 40], [40, 60], seed=7, exact=True)
    c["tables"] = c["tables"].copy()
    c["tables"][1, 2] = 10 ** 6                    # positions 32..47 of sequence 1: out of range
    errors = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, qc, qs = _run(c, errors=errors)
    assert errors.item() == 1                      # the one bad entry, counted once
    assert torch.isfinite(out[:40]).all()          # sequence 0 is unaffected
    ref = _reference(c, qc, qs)
    assert np.abs(out[:40].cpu().numpy() - ref[:40]).max() <= 2.0 ** -14 * _vmax(c)
    # q_len beyond max_q_len: counted, the covered rows still right
    errors.zero_()
    c2 = _case(1, 1, 1, 16, [200], [200], seed=8, exact=True)
    o2, qc2, qs2 = _run(c2, errors=errors, max_q_len=128)
    assert errors.item() == 1
    ref2 = _reference(c2, qc2, qs2)
    assert np.abs(o2[:128].cpu().numpy() - ref2[:128]).max() <= 2.0 ** -14 * _vmax(c2)


def test_one_hot_values_expose_each_key_probability():
    """V row t = e_(t mod 128) (code 0x38 = 1.0): output column d is the
    probability mass of the keys t = d (mod 128).  With exact power-of-two
    probabilities this checks the P layout (swizzle) and the MN-major V
    operand column by column; a wrong layout shows up as a permutation."""
    seqs, Hq, Hkv, B, D = 1, 1, 1, 16, 128
    q_len, ctx = 1, 256                            # one query at the last position sees all 256 keys
    c = _case(seqs, Hq, Hkv, B, [q_len], [ctx], seed=9, exact=True)
    vc = c["vc"]
    vc[:] = 0
    for t in range(ctx):
        blk = c["tables"][0, t // B]
        vc[blk, 0, t % B, t % 128] = 0x38
    c["sv"] = np.ones(1, np.float32)
    for K, V in c["refs"]:
        V.scales = c["sv"]
    out, qc, qs = _run(c)
    ref = _reference(c, qc, qs)
    got = out.cpu().numpy()[0, 0].astype(np.float64)
    np.testing.assert_allclose(got, ref[0, 0], rtol=0, atol=2.0 ** -14)
    assert abs(got.sum() - 1.0) < 1e-5            # the probabilities of all keys add up to 1


def test_strided_output_rows():
    """Output rows with a padded token stride: 16-byte-aligned strides take the
    packed stores, others the element stores; both land in place."""
    c = _case(1, 2, 1, 16, [140], [140], seed=11, exact=True)
    total_q, Hq, D = c["q"].shape
    qc_dev, qs_dev = pg.fp8_quantize_rows(_to(c["q"]).view(total_q * Hq, D))
    ref = _reference(c, qc_dev.view(total_q, Hq, D).cpu().numpy(), qs_dev.cpu().numpy())
    for pad, dt in ((8, torch.bfloat16), (2, torch.bfloat16), (1, torch.float32)):
        wide = torch.full((total_q, Hq * D + pad), float("nan"), dtype=dt, device=DEV)
        out = torch.as_strided(wide, (total_q, Hq, D), (Hq * D + pad, D, 1))
        pg.fp8_attention_context_paged(qc_dev.view(total_q, Hq, D), qs_dev, _to(c["q_start"]),
                                       _to(np.array(c["ctxs"], np.int32)), _to(c["kc"]), _to(c["vc"]),
                                       _to(c["sk"]), _to(c["sv"]), _to(c["tables"]), c["max_ctx"], c["max_q_len"],
                                       out=out)
        torch.cuda.synchronize()
        assert pg.device_status() == pg.OK
        ulp = 2.0 ** -8 if dt == torch.bfloat16 else 2.0 ** -24
        got = out.to(torch.float32).cpu().numpy()
        assert (np.abs(got - ref) <= 2.0 ** -14 * _vmax(c) + ulp * np.abs(ref)).all()
        assert torch.isnan(wide[:, Hq * D:].to(torch.float32)).all()     # the padding is untouched
