"""CPU model of the tiled launches of a grouped call's M > 128 layers
(tiled_group_launch and gemm_pair_group_kernel), restating their host
partition and the kernel's walk: the layers with at most 296 tiles of
256 x 256 share one launch, in order of K (stable); every larger layer runs
its own launch; in the shared launch every tile of every layer is visited
exactly once, by one pair, and each role's forward-moving layer hint finds
the layer the tile belongs to; the tile's token and weight rows stay inside
the layer (rows past M or N read as zeros and are not stored)."""
import random

import pytest

MAX_TILES = 296          # kPairGroupMaxTiles
MAX_LAYERS = 32          # kPairGroupMaxLayers


def tiles(M, N):
    return ((M + 255) // 256) * ((N + 255) // 256)


def partition(layers):
    """(shared list in launch order, layers run alone) as tiled_group_launch
    builds them; layers = [(M, K, N)]."""
    order = sorted(range(len(layers)), key=lambda i: layers[i][1])   # stable
    shared, tile0 = [], 0
    for i in order:
        M, K, N = layers[i]
        if tiles(M, N) > MAX_TILES:
            continue
        shared.append({"layer": i, "M": M, "N": N, "K": K, "m_tiles": (M + 255) // 256, "tile0": tile0})
        tile0 += tiles(M, N)
    alone = [i for i in range(len(layers)) if tiles(layers[i][0], layers[i][2]) > MAX_TILES]
    return shared, tile0, alone


def walk(shared, total, pair, npairs):
    """One role's visits (layer, m-tile, n-tile) in the pair's order, with the
    kernel's forward-moving hint."""
    out, l = [], 0
    for t in range(pair, total, npairs):
        while l + 1 < len(shared) and shared[l + 1]["tile0"] <= t:
            l += 1
        g = shared[l]
        lt = t - g["tile0"]
        assert 0 <= lt < tiles(g["M"], g["N"]), (t, l)
        out.append((g["layer"], lt % g["m_tiles"], lt // g["m_tiles"]))
    return out


def llama70b_large():
    shapes = [(8192, 10240), (8192, 8192), (8192, 57344), (28672, 8192)]
    return [(M, K, N) for M in (256, 512, 1024, 2048, 4096) for (K, N) in shapes]


@pytest.mark.parametrize("npairs", [74, 73, 1, 5])
def test_llama70b_partition_and_walk(npairs):
    layers = llama70b_large()
    shared, total, alone = partition(layers)
    assert len(shared) + len(alone) == len(layers) == 20
    assert len(alone) == 8 and len(shared) == 12
    ks = [g["K"] for g in shared]
    assert ks == sorted(ks)
    seen = {}
    for p in range(npairs):
        for v in walk(shared, total, p, npairs):
            assert v not in seen, v
            seen[v] = p
    want = {(g["layer"], m, n) for g in shared for m in range(g["m_tiles"]) for n in range((g["N"] + 255) // 256)}
    assert set(seen) == want


def test_random_groups_cover_every_tile_once():
    rng = random.Random(7)
    for _ in range(200):
        n = rng.randint(1, MAX_LAYERS)
        layers = [(rng.randint(129, 5000), 16 * rng.randint(1, 2000), 16 * rng.randint(1, 1200)) for _ in range(n)]
        shared, total, alone = partition(layers)
        npairs = rng.randint(1, 80)
        seen = set()
        for p in range(npairs):
            for v in walk(shared, total, p, npairs):
                assert v not in seen
                seen.add(v)
                g = next(x for x in shared if x["layer"] == v[0])
                assert v[1] * 256 < g["M"] and v[2] * 256 < g["N"]   # the tile starts inside the layer
        assert len(seen) == total
        assert all(tiles(layers[i][0], layers[i][2]) > MAX_TILES for i in alone)
        # the stable order: equal K keeps the call order
        for a, b in zip(shared, shared[1:]):
            assert a["K"] < b["K"] or (a["K"] == b["K"] and a["layer"] < b["layer"])
