"""Host logic of the token-split layer on CPU: two gloo ranks each hold a
contiguous slice of one block's rows and exchange the block-wide scalars
through the library's collective helpers (``sharded.allreduce_sum_`` for
Gamma's two sums, ``sharded.allreduce_max_`` for the tensor amax).  The
per-rank arithmetic here is the oracle's; what is under test is the split
and the exchange: the combined Gamma, the amax and every rank's NVFP4 codes
must be those of the unsplit block."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch.multiprocessing as mp

M, K = 301, 384      # ragged: rank 0 takes 151 rows, rank 1 150


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _block():
    from bit_quantized_linear_block_b200 import synthetic as S
    x = S.activations_fixed_outliers(M, K, 8, 50.0, 5, 1)
    y = S.to_bf16(x.float().numpy() + S.normal((M, K), 0.2, 5, 2))
    return S.bf16_bits(x), S.bf16_bits(y)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from bit_quantized_linear_block_b200 import sharded as SH
        from oracle import qlinear_oracle as O
        xb, yb = _block()
        lo, hi = SH.shard_rows(M, world, rank)
        xs, ys = O.bf16_bits_to_f32(xb[lo:hi]), O.bf16_bits_to_f32(yb[lo:hi])
        d = (ys - xs).astype(np.float32)
        sums = torch.tensor([np.abs(d).astype(np.float64).sum(), np.abs(xs).astype(np.float64).sum()],
                            dtype=torch.float64)
        SH.allreduce_sum_(sums)
        h = O.block_hadamard(xs)
        amax = torch.tensor([np.abs(h).max()], dtype=torch.float32)
        SH.allreduce_max_(amax)
        g = O.nvfp4_tensor_scale(amax.numpy().reshape(1, 1))
        packed, sb, _ = O.nvfp4_quantize(h, g)
        q.put((rank, lo, hi, sums.tolist(), float(amax.item()), packed, sb))
    finally:
        dist.destroy_process_group()


def test_shard_rows_partitions_every_row_once():
    from bit_quantized_linear_block_b200.sharded import shard_rows
    for m in (0, 1, 7, 301, 17776):
        for world in (1, 2, 3, 8):
            parts = [shard_rows(m, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == m
            assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


def test_collectives_are_no_ops_without_a_process_group():
    import torch
    from bit_quantized_linear_block_b200 import sharded as SH
    t = torch.tensor([1.0, 2.0])
    assert SH.world_size() == 1
    assert SH.allreduce_sum_(t).tolist() == [1.0, 2.0]
    assert SH.allreduce_max_(t).tolist() == [1.0, 2.0]


def test_two_gloo_ranks_reproduce_the_unsplit_block():
    from oracle import qlinear_oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(2)), key=lambda r: r[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert [(r[1], r[2]) for r in res] == [(0, 151), (151, 301)]
    # every rank holds the same exchanged scalars
    assert res[0][3] == res[1][3] and res[0][4] == res[1][4]
    xb, yb = _block()
    s1, s0 = res[0][3]
    assert s1 / s0 == pytest.approx(O.dmpq_gamma(xb, yb), rel=1e-12)
    h = O.block_hadamard(O.bf16_bits_to_f32(xb))
    assert res[0][4] == float(np.abs(h).max())
    packed, sb, _ = O.nvfp4_quantize(h)
    assert np.array_equal(np.concatenate([res[0][5], res[1][5]]), packed)
    assert np.array_equal(np.concatenate([res[0][6], res[1][6]]), sb)


def test_activation_format_follows_the_forward():
    """Which activation format the token-split forward quantizes to, whether
    it rotates, and whether it needs the block-wide amax: the choices
    qlinear_forward makes for each weight format and route."""
    import torch
    from bit_quantized_linear_block_b200 import qlinear as Q, sharded as SH

    def packed(fmt, hadamard):
        return Q.PackedWeights(Q.Weights(fmt=fmt, N=64, K=128, hadamard=hadamard), torch.zeros(1), 64, 128, fmt)

    nv, qa, de = packed(Q.QL_W_NVFP4, 1), packed(Q.QL_W_QARVD_INT4, 0), packed(Q.QL_W_NVFP4_DECOMP, 1)
    assert SH.activation_format(nv, Q.QL_ROUTE_NVFP4) == (Q.QL_ROUTE_NVFP4, True, True)
    for route in (Q.QL_ACT_INT8_F16, Q.QL_ACT_INT6_F16, Q.QL_ROUTE_BF16):
        assert SH.activation_format(nv, route) == (route, True, False)      # per token or unquantized
    # the per-token integer routes quantize to f16-coded integers, as qlinear_forward does
    assert SH.activation_format(nv, Q.QL_ROUTE_INT8) == (Q.QL_ACT_INT8_F16, True, False)
    assert SH.activation_format(nv, Q.QL_ROUTE_INT6) == (Q.QL_ACT_INT6_F16, True, False)
    assert SH.activation_format(qa, Q.QL_ACT_INT8_TENSOR) == (Q.QL_ACT_INT8_TENSOR, False, True)
    assert SH.activation_format(qa, Q.QL_ROUTE_INT6) == (Q.QL_ACT_INT6_TENSOR, False, True)
    assert SH.activation_format(qa, Q.QL_ACT_INT6_TENSOR) == (Q.QL_ACT_INT6_TENSOR, False, True)
    assert SH.activation_format(de, Q.QL_ROUTE_NVFP4) == (Q.QL_ACT_NVFP4_DECOMP, True, True)
    with pytest.raises(ValueError):
        SH.activation_format(de, Q.QL_ROUTE_INT8)
