"""The quantisation's per-row division (one correctly rounded reciprocal per
row, two FMA remainder corrections per element) against the device's IEEE
division x / s, exhaustively over every binary32 x with |x| <= 512 s — the
domain the quantisation uses, since |x| <= amax and s = RN(amax / 448)
("7B on an RTX 4060 with FP8" §2.2 and §6.1: the code is E4M3(RN(x / s))):
bit-identical quotients wherever |x / s| >= 2^-11, identical E4M3 codes
everywhere (below 2^-11 every quotient encodes to a zero code)."""
import numpy as np
import pytest
import torch

pg = pytest.importorskip("precision_gemm_fp8_b200")
pytestmark = pytest.mark.gpu


def _f32(bits):
    return float(np.array([bits], dtype=np.uint32).view(np.float32)[0])


DIVISORS = [
    1.0,
    float(np.float32(1.0) / np.float32(448.0)),
    2.0 ** -60, 2.0 ** 96,                     # ends of the FMA path's range
    2.0 ** -61, 2.0 ** 97, 1e-40, 3e38,        # outside it: the IEEE division itself
    _f32(0x3F800001), _f32(0x3FFFFFFF),        # 1 + ulp, 2 - ulp
    _f32(0x3F7FFFFF), _f32(0x00800000),        # 1 - ulp/2, smallest normal (outside the range)
    0.0223, 3.3e-5, 7.5e3, 0.6696428571428571,
]


def test_row_division_exhaustive():
    rng = np.random.default_rng(2024)
    rand = (2.0 ** rng.uniform(-50, 60, 8)).astype(np.float32).tolist()
    d = torch.tensor(DIVISORS + rand, dtype=torch.float32, device="cuda:0")
    counts = pg.selftest_row_division(d)
    torch.cuda.synchronize()
    assert pg.device_status() == pg.OK
    c = counts.cpu().numpy()
    bad = {float(v): (int(q), int(k)) for v, (q, k) in zip(d.cpu().numpy(), c) if q or k}
    assert not bad, f"(quotient, code) mismatches against IEEE division: {bad}"
