"""Tensor-parallel FP8 linear on two gloo ranks (CPU): the sharding and
collective logic of precision_gemm_fp8_b200.tensor_parallel, with the
oracle's arithmetic standing in for the kernels (test infrastructure: the
product binds the CUDA library).

Row-parallel (K split): the all-reduce MAX of the slices' amax must give
every rank the codes and scales of the unsplit rows, bit for bit against
the oracle's per-token quantisation of the whole rows; the all-reduce SUM of
the f32 partial products, rounded once to bf16, must lie within the layer's
bound |y - ref| <= 2^-8 |ref| + 1e-4 sqrt(K) A_m W_n of the oracle's binary64
layer.  Column-parallel (N split): every rank's channel block and the
all-gathered output within the same bound."""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The oracle's arithmetic behind the Fp8Ops interface (CPU tensors)."""

    def __init__(self):
        import oracle
        self.o = oracle

    def row_amax(self, x):
        return torch.from_numpy(np.abs(x.numpy()).max(axis=1).astype(np.float32))

    def quantize_rows_amax(self, x, amax):
        # s = fl32(amax / 448) (IEEE binary32 division), 1 for a zero row;
        # codes from the oracle's static-scale quantisation with that s
        a = amax.numpy().astype(np.float32)
        s = (a / np.float32(448.0)).astype(np.float32)
        s[s == 0] = np.float32(1.0)
        q, s2 = self.o.quantize_rows(x.numpy(), scales=s)
        amax.copy_(torch.from_numpy(s2))
        return torch.from_numpy(q), amax

    def linear_partial(self, aq, sa, wq, sw):
        y = self.o.fp8_linear(aq.numpy(), sa.numpy(), wq.numpy(), sw.numpy())
        return torch.from_numpy(y.astype(np.float32))

    def round_bf16(self, y):
        return y.to(torch.bfloat16)

    def linear_dynamic(self, x, wq, sw):
        aq, sa = self.o.quantize_rows(x.numpy())
        y = self.o.fp8_linear(aq, sa, wq.numpy(), sw.numpy())
        return torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16)


def _case(M, K, N, seed):
    sys.path.insert(0, ROOT)
    import oracle
    import synthetic
    g = np.random.default_rng(seed)
    x = synthetic.activations("student_t3", M, K, g)
    # one row of the first slice all zero: its slice amax is 0 on rank 0 only
    x[1, : K // 2] = 0.0
    w = synthetic.weights_f16(N, K, 0.01, g)
    wq, sw = oracle.quantize_rows(w)
    return x, wq, sw


def _worker(rank, world, port, q, M, K, N, seed):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from precision_gemm_fp8_b200.tensor_parallel import (ColumnParallelFP8Linear, RowParallelFP8Linear,
                                                         TPGroup)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, wq, sw = _case(M, K, N, seed)
        tp = TPGroup.current()
        ops = OracleOps()
        row = RowParallelFP8Linear(torch.from_numpy(wq), torch.from_numpy(sw), tp, ops)
        x_r = row.slice_input(torch.from_numpy(x))
        aq_r, sa = row.quantize(x_r.clone())
        y_row = row.forward(x_r)
        col = ColumnParallelFP8Linear(torch.from_numpy(wq), torch.from_numpy(sw), tp, ops)
        y_blk = col.forward(torch.from_numpy(x))
        y_all = col.forward(torch.from_numpy(x), gather=True)
        q.put((rank, row.k0, row.k1, aq_r.numpy(), sa.numpy(), y_row.float().numpy(), col.n0, col.n1,
               y_blk.float().numpy(), y_all.float().numpy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_row_and_column_parallel_against_the_oracle():
    sys.path.insert(0, ROOT)
    import oracle
    from _parity import assert_within, fp8_row_max, linear_bound

    M, K, N, seed = 12, 1024, 96, 77
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, M, K, N, seed)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in procs], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    x, wq, sw = _case(M, K, N, seed)
    aq0, sa0 = oracle.quantize_rows(x)
    ref = oracle.fp8_linear(aq0, sa0, wq, sw)
    bound = linear_bound(ref, K, fp8_row_max(aq0, sa0), fp8_row_max(wq, sw))
    codes = np.zeros_like(aq0)
    for rank, k0, k1, aq_r, sa, y_row, n0, n1, y_blk, y_all in res:
        # the scales of the whole rows on every rank, the codes of this slice
        assert np.array_equal(sa.view(np.uint32), sa0.view(np.uint32)), f"rank {rank}: scales"
        codes[:, k0:k1] = aq_r
        assert_within(y_row, ref, bound, f"row-parallel rank {rank}")
        assert_within(y_blk, ref[:, n0:n1], bound[:, n0:n1], f"column block rank {rank}")
        assert_within(y_all, ref, bound, f"column-parallel gathered, rank {rank}")
    assert np.array_equal(codes, aq0), "row-parallel codes differ from the unsplit rows' codes"
    assert sorted((r[1], r[2]) for r in res) == [(0, K // 2), (K // 2, K)]
    assert sorted((r[6], r[7]) for r in res) == [(0, N // 2), (N // 2, N)]


def test_split_range_rejects_unaligned_blocks():
    sys.path.insert(0, ROOT)
    import pytest
    from precision_gemm_fp8_b200.tensor_parallel import split_range
    assert split_range(4096, 4, 3) == (3072, 4096)
    with pytest.raises(ValueError):
        split_range(4096 + 16, 2, 0)
