"""GPU parity of the FP8 paged KV-cache writer against the oracle ("7B on an
RTX 4060 with FP8": K/V stored in FP8; "C++ and FP8" §3.2: a paged cache of
token blocks): codes bit-exact in their physical blocks, strided input,
pieces written at different positions, and out-of-range block-table
entries skipped and counted without writing outside the cache."""
import numpy as np
import pytest
import torch

import oracle

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _to(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


@pytest.mark.parametrize("T,H,D,B,dtype,pad", [(37, 4, 128, 16, torch.float32, 0), (50, 8, 64, 16, torch.float16, 64),
                                               (33, 2, 128, 8, torch.bfloat16, 32), (1, 1, 16, 16, torch.float32, 0)])
def test_kv_write_matches_the_oracle(T, H, D, B, dtype, pad):
    g = np.random.default_rng(T * 10 + H)
    kv_host = (torch.from_numpy(g.standard_normal((T, H, D)).astype(np.float32)) *
               torch.from_numpy(np.exp(g.uniform(-2, 2, (1, H, 1))).astype(np.float32))).to(dtype)
    kv64 = kv_host.to(torch.float32).numpy()
    scales = oracle.kv_calibrate_scales(kv64)
    nlog = (T + B - 1) // B
    num_blocks = nlog + 3
    table = np.random.default_rng(5).permutation(num_blocks)[:nlog].astype(np.int32)
    ref = oracle.PagedKV(num_blocks, H, D, B, scales, table)
    split = T // 2
    ref.write(kv64[:split], 0)
    ref.write(kv64[split:], split)
    # strided token rows: kv is a slice of a wider buffer
    wide = torch.zeros((T, H * D + pad), dtype=dtype)
    wide[:, :H * D] = kv_host.reshape(T, H * D)
    kv_dev = wide.to(DEV)[:, :H * D].view(T, H, D) if pad == 0 else \
        torch.as_strided(wide.to(DEV), (T, H, D), (H * D + pad, D, 1))
    cache = torch.zeros((num_blocks, H, B, D), dtype=torch.uint8, device=DEV)
    sc, tb = _to(scales), _to(table)
    pg.fp8_kv_write_paged(kv_dev[:split], sc, cache, tb, 0)
    pg.fp8_kv_write_paged(kv_dev[split:], sc, cache, tb, split, flags=pg.FLAG_OVERLAP_PREVIOUS)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    np.testing.assert_array_equal(cache.cpu().numpy(), ref.cache)


def test_out_of_range_blocks_are_skipped_and_counted():
    T, H, D, B = 40, 2, 32, 16
    g = np.random.default_rng(8)
    kv = g.standard_normal((T, H, D)).astype(np.float32)
    scales = oracle.kv_calibrate_scales(kv)
    table = np.array([1, 7, 0], np.int32)            # logical block 1 -> physical 7: out of range (2 blocks)
    guard = torch.full((4, H, B, D), 0xAA, dtype=torch.uint8, device=DEV)
    cache = guard[:2]                                 # the writer sees 2 blocks; blocks 2-3 are a guard zone
    bad = torch.zeros(1, dtype=torch.int32, device=DEV)
    pg.fp8_kv_write_paged(_to(kv), _to(scales), cache, _to(table), 0, bad_blocks=bad)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    assert bad.item() == 16                           # the 16 tokens of logical block 1
    assert (guard[2:] == 0xAA).all()                  # nothing written past the cache
    ref = oracle.PagedKV(2, H, D, B, scales, np.array([1, 0, 0], np.int32))
    ref.write(kv[:16], 0)                             # logical block 0 -> physical 1
    ref.write(kv[32:], 32)                            # logical block 2 -> physical 0
    got = cache.cpu().numpy()
    np.testing.assert_array_equal(got[1], ref.cache[1])
    np.testing.assert_array_equal(got[0, :, :8], ref.cache[0, :, :8])
    assert (got[0, :, 8:] == 0xAA).all()              # slots 8.. of block 0 were never written
