"""CPU models of the work split of the two stream-K kernels (the grouped
weight-streaming kernel and the stream-K region of the pair kernel),
restating their index arithmetic: every (tile, k-block) unit is computed by
exactly one CTA (pair); a CTA publishes at most one partial tile, and only
as its first stream-K segment; a tile shared by several CTAs is finished by
the one holding its first k-block, as its last segment, with the partials
of exactly the following CTAs that hold the rest of the tile; every
published partial is consumed exactly once.  Those properties make the
fix-up free of deadlock (a finishing CTA never waits on a CTA that waits)
and every output written once."""
import random

import pytest


def unit_begin(c, units, G):
    return (c * units) // G


def owner(u, units, G):
    c = (u * G) // units
    while c + 1 < G and unit_begin(c + 1, units, G) <= u:
        c += 1
    while c > 0 and unit_begin(c, units, G) > u:
        c -= 1
    return c


def group_segments(layers, c, G, units):
    """gemm_group_kernel: the segments (layer, tile, kb0, kb1) of CTA c."""
    u0, u1 = unit_begin(c, units, G), unit_begin(c + 1, units, G)
    u, lh, segs = u0, 0, []
    while u < u1:
        l = lh
        while l + 1 < len(layers) and layers[l + 1]["unit0"] <= u:
            l += 1
        lh = l
        g = layers[l]
        local = u - g["unit0"]
        t, kb0 = local // g["kb"], local % g["kb"]
        tile_end = g["unit0"] + (t + 1) * g["kb"]
        kb1 = min(u1, tile_end) - g["unit0"] - t * g["kb"]
        segs.append((l, t, kb0, kb1))
        u = g["unit0"] + t * g["kb"] + kb1
    return segs


def check_group(shapes, sms):
    layers, units = [], 0
    for (M, K, N) in shapes:
        kb, tiles = (K + 127) // 128, (N + 127) // 128
        layers.append({"unit0": units, "kb": kb})
        units += tiles * kb
    G = min(sms, units, 256)
    cover, publish, fin = {}, [0] * G, {}
    for c in range(G):
        segs = group_segments(layers, c, G, units)
        for i, (l, t, kb0, kb1) in enumerate(segs):
            for k in range(kb0, kb1):
                assert (l, t, k) not in cover
                cover[(l, t, k)] = c
            if kb0 > 0:
                assert i == 0
                publish[c] += 1
            elif kb1 < layers[l]["kb"]:
                assert i == len(segs) - 1
                fin[(l, t)] = c
    assert len(cover) == units
    consumed = [0] * G
    for (l, t), c in fin.items():
        last = layers[l]["unit0"] + (t + 1) * layers[l]["kb"] - 1
        cl = owner(last, units, G)
        assert sorted({cover[(l, t, k)] for k in range(layers[l]["kb"])}) == list(range(c, cl + 1))
        for cc in range(c + 1, cl + 1):
            consumed[cc] += 1
    assert consumed == publish


def pair_plan(tiles, kb, pairs_fit, max_ctas=160):
    """Host side of the pair kernel's stream-K region (launch_pair)."""
    sk_pairs = min(pairs_fit, max_ctas // 2)
    pairs, t0, units = min(tiles, pairs_fit), tiles, 0
    if tiles % sk_pairs != 0:
        rounds = tiles // sk_pairs
        t0 = (rounds - 1 if rounds > 1 else 0) * sk_pairs
        units = (tiles - t0) * kb
        pairs = min(sk_pairs, units)
    return pairs, t0, units


def pair_walk(p, npairs, t0, units, tiles, kb):
    """PairWalk: whole tiles round-robin below t0, then the pair's k-block range."""
    T0 = t0 if units > 0 else tiles
    t = p
    while t < T0:
        yield (t, 0, kb)
        t += npairs
    if units:
        u, u1 = p * units // npairs, (p + 1) * units // npairs
        while u < u1:
            lt, k0 = u // kb, u % kb
            se = min(u1, (lt + 1) * kb)
            yield (T0 + lt, k0, se - lt * kb)
            u = se


def check_pair(tiles, kb, pairs_fit):
    npairs, t0, units = pair_plan(tiles, kb, pairs_fit)
    assert 2 * npairs <= 160
    cover, publish, fin = {}, {}, {}
    for p in range(npairs):
        segs = list(pair_walk(p, npairs, t0, units, tiles, kb))
        n_rr = sum(1 for s in segs if s[0] < t0) if units else len(segs)
        for i, (t, k0, k1) in enumerate(segs):
            for k in range(k0, k1):
                assert (t, k) not in cover
                cover[(t, k)] = p
            if k0 == 0 and k1 < kb:
                assert i == len(segs) - 1
                fin[t] = p
            elif k0 > 0:
                assert i == n_rr
                publish[p] = publish.get(p, 0) + 1
    assert len(cover) == tiles * kb
    ways = 1
    for t, p in fin.items():
        pl = owner((t - t0 + 1) * kb - 1, units, npairs)
        holders = sorted({cover[(t, k)] for k in range(kb)})
        assert holders == list(range(p, pl + 1))
        ways = max(ways, len(holders))
    assert all(v == 1 for v in publish.values())
    return ways


@pytest.mark.parametrize("sms", [148, 147, 7, 1])
def test_group_kernel_split(sms):
    rnd = random.Random(sms)
    cases = [[(m, k, n) for m in (1, 4, 8) for (k, n) in ((4096, 12288), (4096, 4096), (4096, 22016), (11008, 4096))],
             [(m, k, n) for m in (1, 2, 4, 8, 16, 32, 64, 128)
              for (k, n) in ((8192, 10240), (8192, 8192), (8192, 57344), (28672, 8192))],
             [(8, 4096, 512)], [(1, 16, 16), (2, 32, 16)], [(8, 11008, 256), (3, 128, 2048)]]
    cases += [[(rnd.randint(1, 128), 16 * rnd.randint(1, 700), 16 * rnd.randint(1, 700))
               for _ in range(rnd.randint(1, 32))] for _ in range(60)]
    for shapes in cases:
        check_group(shapes, sms)


def test_pair_kernel_stream_k_region():
    worst = 1
    for tiles in list(range(1, 300)) + [3584, 1792, 896, 768, 448, 320, 160, 80]:
        for kb in (1, 2, 4, 16, 64, 224):
            for pf in (74, 73, 1):
                w = check_pair(tiles, kb, pf)
                if tiles >= pf:
                    worst = max(worst, w)
    assert worst <= 2      # with at least one round of tiles, a tile spans two pairs at most
