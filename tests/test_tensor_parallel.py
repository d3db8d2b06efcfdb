"""Tensor-parallel sharding on CPU: gloo ranks run ColumnParallelLinear / RowParallelLinear with
every per-rank step computed by the CPU oracle, and the gathered / all-reduced result must equal
the oracle's unsharded forward exactly (the fp64 y the oracle computes from acc, s_x and s_w:
equal acc and s_x give equal y). This checks the partition logic — the rank ranges, the weight
and scale slices, the amax all-reduce (max), the int32 partial-sum all-reduce and the gather —
independently of the GPU kernels, which the GPU tests check step by step.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleOps:
    """The per-rank steps on CPU tensors, each computed by the oracle. The quantiser with a
    supplied amax runs as the oracle's own per-token quantiser on the slice with one extra
    column holding amax (a bf16 value no smaller than any |x| of the slice), whose amax is then
    exactly the supplied one; the extra column is dropped."""

    def __init__(self, oracle):
        self.o = oracle

    @staticmethod
    def _bits(x):
        return x.contiguous().view(torch.int16).numpy().view(np.uint16)

    def linear(self, x, packed, s_w, per_row, out_dtype):
        K = packed.shape[1] * 4
        y = self.o.bitlinear(self._bits(x), packed.numpy(), s_w.numpy(), per_row, K)["y"]
        return torch.from_numpy(y)

    def act_amax(self, x):
        v = self._bits(x).astype(np.uint32) & 0x7FFF
        return torch.from_numpy((v.max(axis=1) << 16).astype(np.uint32).view(np.float32).copy())

    def quant_act_amax(self, x, amax):
        bits = self._bits(x)
        col = (amax.numpy().view(np.uint32) >> 16).astype(np.uint16)[:, None]
        q, s_x = self.o.quant_act(np.concatenate([bits, col], axis=1))
        return torch.from_numpy(np.ascontiguousarray(q[:, :-1])), torch.from_numpy(s_x)

    def linear_i32(self, q, packed):
        K = packed.shape[1] * 4
        return torch.from_numpy(self.o.ternary_matmul(q.numpy(), self.o.unpack(packed.numpy(), K)))

    def dequant(self, acc, s_x, s_w, per_row, out_dtype):
        return torch.from_numpy(self.o.dequant(acc.numpy(), s_x.numpy(), s_w.numpy(), per_row))


def _case(M, N, K, per_row, seed):
    import synth
    g = synth.rng(seed, 90, M, N + K, synth.KIND_T)
    x = synth.normal_x(M, K, g)
    x[0, 5] = synth.to_bf16_bits(np.array([40.0], dtype=np.float32))[0]  # one outlier channel
    if M > 2:
        x[1] = 0  # an all-zero token
    t = synth.ternary(N, K, g, 0.4)
    s_w = synth.uniform_scale(N if per_row else 1, g)
    return x, t, s_w


def _worker(rank, world, port, cases, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    from ternary_w2a8_linear_token_b200.tensor_parallel import (ColumnParallelLinear,
                                                                RowParallelLinear)
    ops = OracleOps(oracle)
    res = []
    for (M, N, K, per_row, seed) in cases:
        x, t, s_w = _case(M, N, K, per_row, seed)
        packed = torch.from_numpy(oracle.pack(t))
        sw = torch.from_numpy(s_w)
        xt = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16)
        ref = oracle.bitlinear(x, oracle.pack(t), s_w, per_row, K)["y"]
        col = ColumnParallelLinear(packed, sw, per_row, ops=ops).forward(xt)
        row_l = RowParallelLinear(packed, sw, per_row, ops=ops)
        row = row_l.forward(row_l.slice_input(xt))
        res.append((bool(np.array_equal(col.numpy(), ref)), bool(np.array_equal(row.numpy(), ref)),
                    (row_l.k0, row_l.k1)))
    out[rank] = res
    dist.barrier()
    dist.destroy_process_group()


CASES = [  # (M, N, K, per_row, seed): ragged N, K of odd 64-units, both scale modes
    (3, 37, 192, False, 1),
    (5, 64, 640, True, 2),
    (1, 130, 1024, True, 3),
]


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_forward_equals_unsharded(world):
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, CASES, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for ci, (M, N, K, per_row, seed) in enumerate(CASES):
        ranges = []
        for r in range(world):
            col_ok, row_ok, kr = out[r][ci]
            assert col_ok, f"column split, case {ci}, rank {r}"
            assert row_ok, f"row split, case {ci}, rank {r}"
            ranges.append(kr)
        # the K slices tile [0, K) in rank order, in multiples of 64
        assert ranges[0][0] == 0 and ranges[-1][1] == K
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
        assert all((b - a) % 64 == 0 and b > a for a, b in ranges)


def test_split_range():
    from ternary_w2a8_linear_token_b200.tensor_parallel import split_range
    for n, world, align in [(10, 3, 1), (640, 3, 64), (2560, 8, 64), (7, 7, 1), (128, 2, 64)]:
        rs = [split_range(n, world, r, align) for r in range(world)]
        assert rs[0][0] == 0 and rs[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
        sizes = [b - a for a, b in rs]
        assert max(sizes) - min(sizes) <= align and all(s % align == 0 for s in sizes)
    with pytest.raises(ValueError):
        split_range(100, 2, 0, 64)
