"""Token-split (sequence-parallel) form of the quantized linear layer.

A block's M tokens are split into contiguous row slices, one per rank, and
every rank holds the same packed weights.  Each output row depends only on
its own input row, except for two block-wide statistics, each of which
takes one scalar exchange:

  * the tensor amax behind the NVFP4 tensor scale g = amax / (6 * 448)
    (6Bit-Diffusion, Methodology B.1, with the NVFP4 two-level recipe) and
    behind Q-ARVD's per-tensor INT8 / INT6 scale (Q-ARVD, Technical
    details).  One all-reduce(max) of an fp32.  A max does not depend on
    the order of its operands, so every rank's codes, scales and output
    rows are those of the unsplit block;
  * the DMPQ statistic Gamma = sum|out - in| / sum|in| (6Bit-Diffusion,
    Methodology A.1 / B.1).  One all-reduce(sum) of two fp64.  Only the
    order of the fp64 additions differs from the unsplit reduction.

The per-token integer routes and the BF16 route need no exchange.  Every
step on the data runs in the library's kernels; torch.distributed carries
the scalars (NCCL over NVLink between GPUs).  With no process group, or a
group of one rank, no collective is made.
"""
from __future__ import annotations

from contextlib import nullcontext

import torch
import torch.distributed as dist

from . import qlinear as Q


def world_size(group=None) -> int:
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group)
    return 1


def shard_rows(M: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of rank's contiguous row slice; the first M % world
    ranks take one row more."""
    if world <= 0 or not 0 <= rank < world or M < 0:
        raise ValueError(f"bad split: M={M}, world={world}, rank={rank}")
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def _on(stream):
    return torch.cuda.stream(stream) if stream is not None else nullcontext()


def allreduce_max_(t: torch.Tensor, group=None, stream=None) -> torch.Tensor:
    """In place: every rank ends with the elementwise max over ranks."""
    if world_size(group) > 1:
        with _on(stream):
            dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t


def allreduce_sum_(t: torch.Tensor, group=None, stream=None) -> torch.Tensor:
    """In place: every rank ends with the elementwise sum over ranks."""
    if world_size(group) > 1:
        with _on(stream):
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


def token_split_route(inp_local: torch.Tensor, out_local: torch.Tensor, threshold: float = 0.05, group=None,
                      stream=None):
    """DMPQ route of a block whose rows are split across ranks: this rank's
    two sums, their sum over ranks, then the decision.  Returns device
    tensors (gamma float64 [1], route int32 [1]), equal on every rank."""
    sums = Q.qlinear_gamma_sums(inp_local, out_local, stream=stream)
    allreduce_sum_(sums, group, stream)
    return Q.qlinear_route_from_sums(sums, threshold, stream=stream)


def token_split_amax(x_local: torch.Tensor, hadamard: bool, group=None, stream=None) -> torch.Tensor:
    """Device fp32 [1]: max |H x| (|x| without the rotation) over the rows of
    every rank."""
    amax = Q.qlinear_tensor_amax(x_local, hadamard, stream=stream)
    return allreduce_max_(amax, group, stream)


def activation_format(w: Q.PackedWeights, route: int) -> tuple[int, bool, bool]:
    """(activation format, Hadamard, needs the block-wide amax) of the
    forward of weights `w` on `route`, as qlinear_forward chooses them."""
    if w.fmt == Q.QL_W_QARVD_INT4:   # per-tensor codes; 6-bit when the route asks for W4A6
        six = route in (Q.QL_ROUTE_INT6, Q.QL_ACT_INT6_TENSOR)
        return (Q.QL_ACT_INT6_TENSOR if six else Q.QL_ACT_INT8_TENSOR), False, True
    if w.fmt == Q.QL_W_NVFP4_DECOMP:
        if route != Q.QL_ROUTE_NVFP4:
            raise ValueError("decomposed weights run on the NVFP4 route only")
        return Q.QL_ACT_NVFP4_DECOMP, bool(w.desc.hadamard), True
    if route == Q.QL_ROUTE_NVFP4:
        return Q.QL_ROUTE_NVFP4, bool(w.desc.hadamard), True
    # per-token integer codes are kept as f16 values, the f16 MMA's operand type
    per_token_f16 = {Q.QL_ROUTE_INT8: Q.QL_ACT_INT8_F16, Q.QL_ROUTE_INT6: Q.QL_ACT_INT6_F16}
    return per_token_f16.get(route, route), bool(w.desc.hadamard), False


def forward_with_amax(x_local: torch.Tensor, w: Q.PackedWeights, route: int, amax: torch.Tensor,
                      Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """This rank's rows of the layer with a given block-wide amax (device
    fp32 [1]): quantize with it, then the GEMM."""
    act, hadamard, _ = activation_format(w, route)
    q = Q.qlinear_quantize_act(x_local, act, hadamard, w=w if w.fmt == Q.QL_W_QARVD_INT4 else None,
                               rowmajor_scales=False, amax_in=amax, stream=stream)
    return Q.qlinear_gemm(act, q, x_local.shape[0], w, Y=Y, stream=stream)


def token_split_forward(x_local: torch.Tensor, w: Q.PackedWeights, route: int = Q.QL_ROUTE_NVFP4, group=None,
                        Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """This rank's output rows of the layer whose input rows are split
    across ranks; the same rows as qlinear_forward on the whole block."""
    _, hadamard, needs_amax = activation_format(w, route)
    if not needs_amax:   # per-token scales or no quantization: rows are independent
        return Q.qlinear_forward(x_local, w, route, Y=Y, stream=stream)
    amax = token_split_amax(x_local, hadamard, group, stream)
    return forward_with_amax(x_local, w, route, amax, Y=Y, stream=stream)
