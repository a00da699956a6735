"""CPU models of the attention kernels' index arithmetic and arithmetic order.

Test infrastructure only: no entry point of the library uses them.  Each
model follows its kernel step by step (grid, chunks, 16-position warp
steps, the lanes' row pieces, masks, the online softmax, merges) and
asserts that every cache address it forms lies inside the cache, so that a
CPU run checks the kernels' design against the oracle before a GPU does.

- decode_cuda_core: attn_decode_paged_kernel + attn_decode_combine_kernel.
- decode_tensor_core: attn_decode_mma_kernel, lane by lane: every register
  is built as the kernel builds it, and mma.sync m16n8k16 follows the PTX
  fragment layouts (A: rows g / g+8, cols 2q+e / 2q+8+e; B: rows 2q+e /
  2q+8+e, col g; C: rows g / g+8, cols 2q+e; g = lane / 4, q = lane % 4).
- context: attn_context_kernel (128-query tiles, 16-row pieces, E4M3
  probabilities x 2^8 with the scale folded into the exponent, two softmax
  threads per row each summing its half of l, V rows past the context
  cleared, PV one tile late).

E4M3 values come from torch's float8_e4m3fn; binary16 rounding from numpy.
"""
import math

import numpy as np
import torch

f32 = np.float32
E4 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)
LOG2E = 1.4426950408889634


def _h(x):
    return float(np.float16(x))


def _e4m3_round(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).to(
        torch.float32).numpy()


# ---------------------------------------------------------------- decode, CUDA cores
def decode_cuda_core(q, kc, vc, sk, sv, tables, lens, max_ctx, nsplit, chunk):
    """Returns (out [seqs, Hq, D], error count)."""
    seqs, Hq, D = q.shape
    nb, Hkv, B, _ = kc.shape
    G = Hq // Hkv
    GT = next(g for g in (8, 4, 2, 1) if G % g == 0)
    groups = G // GT
    qscale = f32(LOG2E / math.sqrt(D))
    kflat, vflat = kc.reshape(-1), vc.reshape(-1)
    DPL = D // 32
    out = np.zeros((seqs, Hq, D), np.float32)
    part = np.full((seqs, Hq, nsplit, D + 2), np.nan, np.float32)
    errors = 0
    for s in range(seqs):
        for y in range(Hkv * groups):
            hk, gi = y // groups, y % groups
            h0 = hk * G + gi * GT
            for sp in range(nsplit):
                qs = (q[s, h0:h0 + GT].astype(np.float32) * f32(sk[hk] * qscale)).astype(np.float32)
                ctx = int(lens[s])
                if ctx < 0 or ctx > max_ctx:
                    if sp == 0 and y == 0:
                        errors += 1
                    ctx = 0 if ctx < 0 else max_ctx
                tb, te = sp * chunk, min(sp * chunk + chunk, ctx)
                red = []
                for w in range(4):
                    m = np.full(GT, -np.inf, np.float32)
                    l = np.zeros(GT, np.float32)
                    o = np.zeros((GT, D), np.float32)
                    base = tb + 16 * w
                    while base < te:
                        nvalid = min(16, te - base)
                        assert base // B < tables.shape[1]
                        blk = int(tables[s, base // B])
                        if blk < 0 or blk >= nb:
                            if y == 0:
                                errors += 1
                            base += 64
                            continue
                        row0 = (blk * Hkv + hk) * B + base % B
                        assert base % B + 15 < B
                        dots = np.zeros((16, GT), np.float32)
                        for tq in range(nvalid):
                            for hf in range(2):            # lanes 2t, 2t+1: interleaved 16-byte pieces
                                for i in range(D // 32):
                                    off = (row0 + tq) * D + 16 * (2 * i + hf)
                                    assert 0 <= off and off + 16 <= kflat.size
                                    kf = E4[kflat[off:off + 16]].astype(np.float32)
                                    d0 = 16 * (2 * i + hf)
                                    dots[tq] += (qs[:, d0:d0 + 16] * kf[None, :]).sum(axis=1, dtype=np.float32)
                        valid = np.arange(16) < nvalid
                        for g in range(GT):
                            sc = np.where(valid, dots[:, g], -np.inf).astype(np.float32)
                            mn = max(m[g], sc.max())
                            alpha = f32(0) if m[g] == -np.inf else f32(np.exp2(f32(m[g] - mn)))
                            p = np.where(valid, np.exp2(np.where(valid, sc - mn, 0)), 0).astype(np.float32)
                            l[g] = f32(l[g] * alpha + p.sum(dtype=np.float32))
                            m[g] = mn
                            o[g] *= alpha
                            for t in range(nvalid):
                                for lane in range(32):         # lane owns dims lane*DPL .. +DPL-1
                                    off = (row0 + t) * D + lane * DPL
                                    assert off + DPL <= vflat.size
                                    o[g, lane * DPL:(lane + 1) * DPL] += p[t] * E4[vflat[off:off + DPL]]
                        base += 64
                    red.append((m, l, o))
                for g in range(GT):
                    M = max(r[0][g] for r in red)
                    L, O = f32(0), np.zeros(D, np.float32)
                    for r in red:
                        if r[0][g] != -np.inf:
                            fct = f32(np.exp2(f32(r[0][g] - M)))
                            L = f32(L + r[1][g] * fct)
                            O = (O + r[2][g] * fct).astype(np.float32)
                    if nsplit == 1:
                        out[s, h0 + g] = (O / L * sv[hk]) if L > 0 else 0
                    else:
                        part[s, h0 + g, sp, :D], part[s, h0 + g, sp, D], part[s, h0 + g, sp, D + 1] = O, M, L
    if nsplit > 1:
        assert not np.isnan(part).any()                # every chunk state written
        for s in range(seqs):
            for h in range(Hq):
                pp = part[s, h]
                M = pp[:, D].max()
                L, O = f32(0), np.zeros(D, np.float32)
                for i in range(nsplit):                # chunk order
                    if pp[i, D] != -np.inf:
                        fct = f32(np.exp2(f32(pp[i, D] - M)))
                        L = f32(L + pp[i, D + 1] * fct)
                        O = (O + pp[i, :D] * fct).astype(np.float32)
                out[s, h] = (O / L * sv[h // G]) if L > 0 else 0
    return out, errors


# ---------------------------------------------------------------- decode, tensor cores
def _dec2(word):
    return (E4[word & 0xFF], E4[(word >> 8) & 0xFF])


def _byte_perm(x, y, sel):
    src = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(src[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))


def _mma_16816(c, a, b):
    """c[lane][4] += A.B from the lanes' fragments (PTX m16n8k16 layouts)."""
    A, Bm = np.zeros((16, 16)), np.zeros((16, 8))
    for lane in range(32):
        g, q = lane >> 2, lane & 3
        for e in range(2):
            A[g][2 * q + e], A[g + 8][2 * q + e] = a[lane][0][e], a[lane][1][e]
            A[g][2 * q + 8 + e], A[g + 8][2 * q + 8 + e] = a[lane][2][e], a[lane][3][e]
            Bm[2 * q + e][g], Bm[2 * q + 8 + e][g] = b[lane][0][e], b[lane][1][e]
    Dm = A @ Bm
    for lane in range(32):
        g, q = lane >> 2, lane & 3
        for e in range(2):
            c[lane][e] = f32(c[lane][e] + Dm[g][2 * q + e])
            c[lane][2 + e] = f32(c[lane][2 + e] + Dm[g + 8][2 * q + e])


def _words(buf):
    return [int.from_bytes(bytes(buf[4 * i:4 * i + 4]), "little") for i in range(len(buf) // 4)]


def decode_tensor_core(q, kc, vc, sk, sv, tables, lens, max_ctx, nsplit, chunk):
    """Returns out [seqs, Hq, D] (block tables must be in range)."""
    seqs, Hq, D = q.shape
    nb, Hkv, B, _ = kc.shape
    G = Hq // Hkv
    groups = -(-G // 8)
    KSTEPS, KSEG, VSEG, DB = D // 16, D // 4, D // 8, D // 16
    qscale = f32(LOG2E / math.sqrt(D))
    kflat, vflat = kc.reshape(-1), vc.reshape(-1)
    states = {}

    def piece(flat, row, off, n, ok):
        if not ok:
            return [0] * (n // 4)
        st = row * D + off
        assert 0 <= st and st + n <= flat.size and st % min(n, 16) == 0
        return _words(flat[st:st + n])

    for s in range(seqs):
        for y in range(Hkv * groups):
            hk, gi = y // groups, y % groups
            nh, h0 = min(8, G - gi * 8), hk * G + gi * 8
            qb = [[[(_h(q[s, h0 + (ln >> 2), KSEG * (ln & 3) + 4 * j + 2 * e]) if (ln >> 2) < nh else 0.0,
                     _h(q[s, h0 + (ln >> 2), KSEG * (ln & 3) + 4 * j + 2 * e + 1]) if (ln >> 2) < nh else 0.0)
                    for e in range(2)] for j in range(KSTEPS)] for ln in range(32)]
            ctx = max(0, min(int(lens[s]), max_ctx))
            scale = f32(sk[hk] * qscale)
            for sp in range(nsplit):
                tb, te = sp * chunk, min(sp * chunk + chunk, ctx)
                red = []
                for w in range(4):
                    m = [[-np.inf, -np.inf] for _ in range(32)]
                    l = [[0.0, 0.0] for _ in range(32)]
                    o = [[[0.0] * 4 for _ in range(DB)] for _ in range(32)]
                    for base in range(tb + 16 * w, te, 64):
                        nvalid = min(16, te - base)
                        blk = int(tables[s, base // B])
                        assert 0 <= blk < nb
                        row0 = (blk * Hkv + hk) * B + base % B
                        k0 = [piece(kflat, row0 + (ln >> 2), KSEG * (ln & 3), KSEG, (ln >> 2) < nvalid)
                              for ln in range(32)]
                        k1 = [piece(kflat, row0 + (ln >> 2) + 8, KSEG * (ln & 3), KSEG, (ln >> 2) + 8 < nvalid)
                              for ln in range(32)]
                        vw = [[piece(vflat, row0 + 4 * (ln & 3) + r, VSEG * (ln >> 2), VSEG, 4 * (ln & 3) + r < nvalid)
                               for r in range(4)] for ln in range(32)]
                        c = [[0.0] * 4 for _ in range(32)]
                        for j in range(KSTEPS):
                            _mma_16816(c, [[_dec2(k0[ln][j]), _dec2(k1[ln][j]), _dec2(k0[ln][j] >> 16),
                                            _dec2(k1[ln][j] >> 16)] for ln in range(32)],
                                       [qb[ln][j] for ln in range(32)])
                        pr = [[0.0] * 4 for _ in range(32)]
                        alpha = [[0.0, 0.0] for _ in range(32)]
                        for hh in range(2):
                            sc = [(f32(c[ln][hh] * scale) if (ln >> 2) < nvalid else -np.inf,
                                   f32(c[ln][2 + hh] * scale) if (ln >> 2) + 8 < nvalid else -np.inf)
                                  for ln in range(32)]
                            for q4 in range(4):
                                lanes = [4 * g + q4 for g in range(8)]
                                mx = max(max(sc[ln]) for ln in lanes)
                                psum = 0.0
                                for ln in lanes:
                                    mn = max(m[ln][hh], mx)
                                    alpha[ln][hh] = 0.0 if m[ln][hh] == -np.inf else f32(np.exp2(f32(m[ln][hh] - mn)))
                                    pr[ln][hh] = f32(np.exp2(f32(sc[ln][0] - mn))) if (ln >> 2) < nvalid else 0.0
                                    pr[ln][2 + hh] = f32(np.exp2(f32(sc[ln][1] - mn))) if (ln >> 2) + 8 < nvalid else 0.0
                                    psum += pr[ln][hh] + pr[ln][2 + hh]
                                for ln in lanes:
                                    l[ln][hh] = f32(l[ln][hh] * alpha[ln][hh] + psum)
                                    m[ln][hh] = max(m[ln][hh], mx)
                        for ln in range(32):
                            for bb in range(DB):
                                for i, hh in enumerate((0, 1, 0, 1)):
                                    o[ln][bb][i] *= alpha[ln][hh]
                        ps = np.zeros((8, 16))                 # [head][position] in binary16
                        for ln in range(32):
                            g, t4 = ln >> 2, ln & 3
                            ps[2 * t4][g], ps[2 * t4 + 1][g] = _h(pr[ln][0]), _h(pr[ln][1])
                            ps[2 * t4][g + 8], ps[2 * t4 + 1][g + 8] = _h(pr[ln][2]), _h(pr[ln][3])
                        pb = [((ps[ln >> 2][4 * (ln & 3)], ps[ln >> 2][4 * (ln & 3) + 1]),
                               (ps[ln >> 2][4 * (ln & 3) + 2], ps[ln >> 2][4 * (ln & 3) + 3])) for ln in range(32)]
                        for bb in range(DB):
                            wi, sh = bb >> 1, 2 * (bb & 1)
                            sel = sh | ((4 + sh) << 4) | ((sh + 1) << 8) | ((5 + sh) << 12)
                            a = []
                            for ln in range(32):
                                x01 = _byte_perm(vw[ln][0][wi], vw[ln][1][wi], sel)
                                x23 = _byte_perm(vw[ln][2][wi], vw[ln][3][wi], sel)
                                a.append([_dec2(x01), _dec2(x01 >> 16), _dec2(x23), _dec2(x23 >> 16)])
                            cc = [o[ln][bb] for ln in range(32)]
                            _mma_16816(cc, a, pb)
                    rm, rl, ro = np.full(8, -np.inf), np.zeros(8), np.zeros((8, D))
                    for ln in range(32):
                        g, t4 = ln >> 2, ln & 3
                        if g == 0:
                            rm[2 * t4], rm[2 * t4 + 1] = m[ln]
                            rl[2 * t4], rl[2 * t4 + 1] = l[ln]
                        for bb in range(DB):
                            d = VSEG * g + 2 * bb
                            ro[2 * t4][d], ro[2 * t4 + 1][d] = o[ln][bb][0], o[ln][bb][1]
                            ro[2 * t4][d + 1], ro[2 * t4 + 1][d + 1] = o[ln][bb][2], o[ln][bb][3]
                    red.append((rm, rl, ro))
                for hh in range(nh):
                    M = max(r[0][hh] for r in red)
                    L, O = 0.0, np.zeros(D)
                    for r in red:
                        if r[0][hh] != -np.inf:
                            L += r[1][hh] * np.exp2(r[0][hh] - M)
                            O += r[2][hh] * np.exp2(r[0][hh] - M)
                    states[(s, h0 + hh, sp)] = (M, L, O)
    out = np.zeros((seqs, Hq, D), np.float32)
    for s in range(seqs):
        for h in range(Hq):
            ps_ = [states[(s, h, sp)] for sp in range(nsplit)]
            M = max(p[0] for p in ps_)
            L, O = 0.0, np.zeros(D)
            for p in ps_:
                if p[0] != -np.inf:
                    L += p[1] * np.exp2(p[0] - M)
                    O += p[2] * np.exp2(p[0] - M)
            out[s, h] = O / L * sv[h // G] if L > 0 else 0
    return out


# ---------------------------------------------------------------- context, tcgen05
def context(qc, qs, q_start, lens, kc, vc, sk, sv, tables, max_ctx, max_q_len):
    """Returns out [total_q, Hq, 128] (NaN where the kernel writes nothing)."""
    total_q, Hq, D = qc.shape
    nb, Hkv, B, _ = kc.shape
    assert D == 128
    cache_rows = nb * Hkv * B
    kflat, vflat = kc.reshape(cache_rows, D), vc.reshape(cache_rows, D)
    out = np.full((total_q, Hq, D), np.nan, np.float32)
    nqt = -(-max_q_len // 128)
    for s in range(len(lens)):
        q0, q_len, ctx = int(q_start[s]), int(q_start[s + 1] - q_start[s]), int(lens[s])
        if q_len < 0 or q0 < 0 or q0 + q_len > total_q or ctx < q_len or ctx > max_ctx:
            continue
        for x in range(nqt * Hq):                     # heaviest tiles of every head first
            h, qt = x % Hq, nqt - 1 - x // Hq
            if q_len <= qt * 128:
                continue
            hk = h // (Hq // Hkv)
            nrows = min(128, q_len - qt * 128)
            pos0 = ctx - q_len + qt * 128
            nkt = (pos0 + nrows - 1) // 128 + 1
            Qt = np.zeros((128, D))
            for r in range(128):
                if q0 + qt * 128 + r < total_q:
                    Qt[r] = E4[qc[q0 + qt * 128 + r, h]]
            rows = np.arange(128)
            row_ok, pos = rows < nrows, pos0 + rows
            sq = np.array([qs[(q0 + qt * 128 + r) * Hq + h] if r < nrows else 0 for r in range(128)], np.float32)
            scale = (sq * f32(sk[hk]) * (f32(LOG2E) * f32(0.08838834764831845))).astype(np.float32)
            m, l = np.full(128, -np.inf, np.float32), np.zeros((2, 128), np.float32)
            o = np.zeros((128, D), np.float32)
            pending = alpha_prev = None
            for j in range(nkt):
                Kt, Vt = np.zeros((128, D)), np.zeros((128, D))
                piece_ok = 0
                for i in range(8):
                    key = j * 128 + i * 16
                    row = cache_rows
                    if key < ctx:
                        blk = tables[s, key // B]
                        if 0 <= blk < nb:
                            row = (blk * Hkv + hk) * B + key % B
                            piece_ok |= 1 << i
                    assert 0 <= row <= cache_rows
                    if row < cache_rows:
                        assert row + 16 <= cache_rows and row % B + 16 <= B
                        Kt[16 * i:16 * i + 16], Vt[16 * i:16 * i + 16] = E4[kflat[row:row + 16]], E4[vflat[row:row + 16]]
                S = (Qt @ Kt.T).astype(np.float32)
                keys = j * 128 + np.arange(128)
                pok = np.array([(piece_ok >> (c // 16)) & 1 for c in range(128)], bool)
                valid = pok[None, :] & row_ok[:, None] & (keys[None, :] <= pos[:, None])
                sc = (S * scale[:, None]).astype(np.float32)
                mn = np.maximum(m, np.where(valid, sc, -np.inf).max(axis=1)).astype(np.float32)
                safe = np.where(m == -np.inf, 0, m - np.where(m == -np.inf, 0, mn))
                alpha = np.where(m == -np.inf, 0, np.exp2(safe)).astype(np.float32)
                # probabilities times 2^8 (the code scale folded into the exponent:
                # exp2(fma(S, scale, 8 - m))), l in the same units
                nm8 = (f32(8) - mn).astype(np.float32)
                arg = np.where(valid, S.astype(np.float64) * scale[:, None] + nm8[:, None], 0).astype(np.float32)
                pr = np.where(valid, np.exp2(arg), 0).astype(np.float32)
                P = _e4m3_round(pr)
                cut = ctx - j * 128
                if 0 < cut < 128 and cut % 16 and (piece_ok >> (cut // 16)) & 1:
                    Vt[cut:(cut // 16 + 1) * 16] = 0
                PV = (P.astype(np.float64) @ Vt).astype(np.float32)
                # each of the two softmax threads of a row keeps its half's share
                rs = np.stack([pr[:, :64].sum(axis=1, dtype=np.float32), pr[:, 64:].sum(axis=1, dtype=np.float32)])
                m, l = mn, (l * alpha[None, :] + rs).astype(np.float32)
                if pending is not None:
                    o = (o * alpha_prev[:, None] + pending).astype(np.float32)
                pending, alpha_prev = PV, alpha
            o = (o * alpha_prev[:, None] + pending).astype(np.float32)
            lsum = (l[0] + l[1]).astype(np.float32)
            f = np.where(lsum > 0, sv[hk] / np.where(lsum > 0, lsum, 1), 0).astype(np.float32)
            out[q0 + qt * 128:q0 + qt * 128 + nrows, h] = o[:nrows] * f[:nrows, None]
    return out
