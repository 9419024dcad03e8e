"""Tensor-parallel BitLinear across GPUs (one process per GPU, torch.distributed).

BitNet b1.58's 70B model was served on two GPUs (dmarx anthology record LIT-380, Key
takeaways bullet 5); the pages do not say how the layers were split. Both classic splits
of a linear layer are provided, each exact: the result on G GPUs is bit for bit the
single-GPU forward.

Column-parallel (N split): GPU r holds the weight rows [n0, n1) (`dist.row_shard`), every
GPU the whole batch. Each GPU computes its own output columns; no collective is needed
unless the caller wants y gathered.

Row-parallel (K split): GPU r holds the weight columns [k0, k1) (`col_shard`, multiples
of 64) and the same columns of the batch. The per-token absmax is a MAX all-reduce of
the shards' maxima, each GPU quantizes its columns with it and forms its exact int32
partial product, the partial products are SUM all-reduced (integers: exact, any order)
and every GPU rescales.

Both splits need gamma = mean |W| over the WHOLE matrix: each GPU forms the exact sum of
|w| over its shard (integer words), the words are SUM all-reduced, and each GPU finishes
gamma and codes its own shard.

Every arithmetic step runs in the library's kernels (the `bitlinear` binding); this
module only orders the calls and the collectives. `ops` and `comm` are parameters so
that the same orchestration can be driven by other implementations of those calls.
"""

from __future__ import annotations

import torch

from . import bitlinear as _bitlinear
from .dist import row_shard  # noqa: F401  (the N split)


def col_shard(K: int, world: int, rank: int, align: int = 64) -> tuple[int, int]:
    """Contiguous columns [k0, k1) of a K-wide matrix owned by `rank`: whole blocks of
    `align` columns (K % align == 0), block counts differing by at most one."""
    if K % align:
        raise ValueError(f"K = {K} is not a multiple of {align}")
    b0, b1 = row_shard(K // align, world, rank)
    return b0 * align, b1 * align


class TorchDistComm:
    """The collectives this module needs, on a torch.distributed process group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group

    @property
    def rank(self) -> int:
        return self.dist.get_rank(self.group)

    @property
    def world(self) -> int:
        return self.dist.get_world_size(self.group)

    def all_reduce(self, t: torch.Tensor, op: str) -> None:
        ops = {"sum": self.dist.ReduceOp.SUM, "max": self.dist.ReduceOp.MAX}
        self.dist.all_reduce(t, op=ops[op], group=self.group)

    def all_gather(self, t: torch.Tensor) -> list[torch.Tensor]:
        out = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(out, t, group=self.group)
        return out


def quantize_weights_sharded(W_shard: torch.Tensor, n_total: int, eps: float = 1e-5,
                             comm=None, ops=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Absmean ternary quantization of this GPU's shard of a matrix of n_total weights:
    (packed codes of the shard, gamma of the whole matrix)."""
    ops = ops or _bitlinear
    comm = comm or TorchDistComm()
    sums = ops.weight_abssum(W_shard)
    comm.all_reduce(sums, "sum")  # exact: integer words
    return ops.quantize_weights_from_abssum(W_shard, n_total, sums, eps)


def forward_column_parallel(x: torch.Tensor, packed_shard: torch.Tensor, gamma: torch.Tensor,
                            out_dtype: torch.dtype = torch.bfloat16, gather: bool = False,
                            comm=None, ops=None) -> torch.Tensor:
    """y[:, n0:n1] of the whole batch x for this GPU's weight rows; with gather=True the
    whole y [M][N] on every GPU (shards all-gathered, padded to the largest)."""
    ops = ops or _bitlinear
    y = ops.forward(x, packed_shard, gamma, out_dtype=out_dtype)
    if not gather:
        return y
    comm = comm or TorchDistComm()
    rows = torch.tensor([y.shape[1]], dtype=torch.int64, device=y.device)
    widths = [int(w.item()) for w in comm.all_gather(rows)]
    pad = max(widths)
    yp = y if y.shape[1] == pad else torch.nn.functional.pad(y, (0, pad - y.shape[1]))
    parts = comm.all_gather(yp.contiguous())
    return torch.cat([p[:, :w] for p, w in zip(parts, widths)], dim=1)


def forward_row_parallel(x_shard: torch.Tensor, packed_shard: torch.Tensor,
                         gamma: torch.Tensor, out_dtype: torch.dtype = torch.bfloat16,
                         comm=None, ops=None) -> torch.Tensor:
    """The whole y [M][N] from this GPU's columns x[:, k0:k1] and W[:, k0:k1] (packed),
    identical on every GPU."""
    ops = ops or _bitlinear
    comm = comm or TorchDistComm()
    amax = ops.act_absmax(x_shard)
    comm.all_reduce(amax, "max")  # the absmax of the whole token rows
    xq, scale = ops.quantize_acts_absmax(x_shard, amax)
    acc = ops.contract_i32(xq, packed_shard)
    comm.all_reduce(acc, "sum")  # exact int32 sum of the partial products
    return ops.rescale(acc, scale, gamma, out_dtype=out_dtype)
