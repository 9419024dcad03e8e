"""Tensor-parallel BitLinear (ternary_weight_linear_03_b200/tp.py).

CPU: world-size-2 gloo process groups run the module's orchestration (collectives and
call order) with the oracle's steps standing in for the library's kernels, and the
results must equal the single-device oracle bit for bit: gamma of the whole matrix from
the shards' exact sums, the shards' packed codes, the column-parallel output (gathered)
and the row-parallel output (absmax MAX all-reduce, int32 SUM all-reduce).

GPU: the same orchestration with the library's kernels, two ranks emulated by two host
threads on one GPU whose collectives are host-side (no kernel waits on another rank).
"""

import datetime
import os
import socket
import threading

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import oracle as orc
from ternary_weight_linear_03_b200 import synthetic as syn
from ternary_weight_linear_03_b200 import tp
from ternary_weight_linear_03_b200.dist import row_shard

M, N, K, EPS = 6, 200, 384, 1e-5


class OracleOps:
    """The calls tp.py makes, answered by the oracle on CPU tensors (test stand-in for the
    library's kernels)."""

    @staticmethod
    def _bits(t):
        return syn.bf16_bits(t) if t.dtype == torch.bfloat16 else t.numpy()

    def weight_abssum(self, W):
        return torch.from_numpy(orc.abs_buckets(self._bits(W)).view(np.int64).copy())

    def quantize_weights_from_abssum(self, W, n_total, sums, eps):
        g = orc.absmean_from_buckets(sums.numpy().view(np.uint64), n_total)
        packed = orc.pack(orc.ternarize(self._bits(W), g, eps))
        return torch.from_numpy(packed), torch.tensor([g], dtype=torch.float32)

    def act_absmax(self, x):
        return torch.from_numpy(orc.act_absmax(self._bits(x)))

    def quantize_acts_absmax(self, x, amax):
        q, s = orc.quantize_acts_absmax(self._bits(x), amax.numpy())
        return torch.from_numpy(q), torch.from_numpy(s)

    def contract_i32(self, xq, packed):
        codes = orc.unpack(packed.numpy(), xq.shape[1])
        return torch.from_numpy(orc.contract_i32(xq.numpy(), codes))

    def rescale(self, acc, scale, gamma, out_dtype):
        y = orc.rescale(acc.numpy(), scale.numpy(), float(gamma.item()))
        return _to_torch(y, out_dtype)

    def forward(self, x, packed, gamma, out_dtype):
        y = orc.forward(self._bits(x), packed.numpy(), float(gamma.item()))
        return _to_torch(y, out_dtype)


def _to_torch(y, out_dtype):
    if out_dtype == torch.float32:
        return torch.from_numpy(y)
    return torch.from_numpy(orc.to_bf16(y).view(np.int16)).view(torch.bfloat16)


def _inputs():
    W = syn.weights(N, K, 0.02, seed=41)
    W[: N // 2] *= 3.0  # the shards' sums differ
    x = syn.activations(M, K, seed=42, dtype=torch.bfloat16, outlier_frac=0.01)
    x[2, K - 5] = 60.0  # a token's maximum in the last K shard
    return W, x


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ops, comm = OracleOps(), tp.TorchDistComm()
        W, x = _inputs()
        # column-parallel: weight rows
        n0, n1 = row_shard(N, world, rank)
        pc, gc = tp.quantize_weights_sharded(W[n0:n1].contiguous(), N * K, EPS, comm, ops)
        yc = tp.forward_column_parallel(x, pc, gc, torch.float32, gather=True, comm=comm, ops=ops)
        # row-parallel: weight and activation columns
        k0, k1 = tp.col_shard(K, world, rank)
        pr, gr = tp.quantize_weights_sharded(W[:, k0:k1].contiguous(), N * K, EPS, comm, ops)
        yr = tp.forward_row_parallel(x[:, k0:k1].contiguous(), pr, gr, torch.bfloat16, comm, ops)
        results[rank] = (pc.numpy(), float(gc.item()), yc.numpy(), pr.numpy(), float(gr.item()),
                         yr.view(torch.int16).numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_tensor_parallel_matches_single_device():
    world = 2
    results = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), results), nprocs=world, join=True)
    W, x = _inputs()
    ref_packed, ref_gamma = orc.quantize_weights(W.numpy(), EPS)
    xb = syn.bf16_bits(x)
    ref_y = orc.forward(xb, ref_packed, ref_gamma)
    ref_y16 = orc.to_bf16(ref_y).view(np.int16)
    for rank in range(world):
        pc, gc, yc, pr, gr, yr = results[rank]
        n0, n1 = row_shard(N, world, rank)
        k0, k1 = tp.col_shard(K, world, rank)
        assert gc == float(ref_gamma) and gr == float(ref_gamma)
        np.testing.assert_array_equal(pc, ref_packed[n0:n1])
        np.testing.assert_array_equal(pr, ref_packed[:, k0 // 4:k1 // 4])
        np.testing.assert_array_equal(yc, ref_y)
        np.testing.assert_array_equal(yr, ref_y16)


@pytest.mark.parametrize("K_,world", [(384, 2), (8192, 8), (64, 1), (640, 3)])
def test_col_shards_tile_k_in_blocks_of_64(K_, world):
    shards = [tp.col_shard(K_, world, r) for r in range(world)]
    assert shards[0][0] == 0 and shards[-1][1] == K_
    for (a0, a1), (b0, b1) in zip(shards, shards[1:]):
        assert a1 == b0
    assert all(a % 64 == 0 and b % 64 == 0 for a, b in shards)
    with pytest.raises(ValueError):
        tp.col_shard(100, 2, 0)


# ----------------------------------------------------------------------------- GPU


class ThreadComm:
    """Collectives between host threads of one process (one thread per emulated rank):
    each deposits its tensor, the reduction is formed on the device, every thread copies
    the result. Host-side only: no kernel waits on another rank."""

    def __init__(self, world):
        self.world = world
        self._bar = threading.Barrier(world)
        self._slots = [None] * world
        self._local = threading.local()

    def bind(self, rank):
        self._local.rank = rank
        return self

    @property
    def rank(self):
        return self._local.rank

    def all_reduce(self, t, op):
        torch.cuda.synchronize()
        self._slots[self.rank] = t
        self._bar.wait()
        stack = torch.stack([s for s in self._slots])
        red = stack.sum(0, dtype=t.dtype) if op == "sum" else stack.max(0).values
        self._bar.wait()
        t.copy_(red)
        torch.cuda.synchronize()
        self._bar.wait()

    def all_gather(self, t):
        torch.cuda.synchronize()
        self._slots[self.rank] = t
        self._bar.wait()
        out = [s.clone() for s in self._slots]
        self._bar.wait()
        return out


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(16, 8640, 3200), (3, 1000, 1536), (300, 520, 1536)])
def test_tensor_parallel_kernels_two_emulated_ranks(shape):
    """Both splits through the library's kernels, two ranks as two host threads on one GPU,
    against the single-device oracle (gamma, packed shards and outputs bit for bit)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import ternary_weight_linear_03_b200 as bl
    Mg, Ng, Kg = shape
    W = syn.weights(Ng, Kg, 0.02, seed=Ng)
    W[: Ng // 3] *= 2.0
    x = syn.activations(Mg, Kg, seed=Mg, dtype=torch.bfloat16, outlier_frac=0.01)
    ref_packed, ref_gamma = orc.quantize_weights(W.numpy(), EPS)
    ref_y = orc.forward(syn.bf16_bits(x), ref_packed, ref_gamma, out="bf16").view(np.int16)
    world, comm = 2, ThreadComm(2)
    out, errors = {}, []

    def rank_main(rank):
        try:
            torch.cuda.set_device(0)
            c = comm.bind(rank)
            Wd, xd = W.cuda(), x.cuda()
            n0, n1 = row_shard(Ng, world, rank)
            pc, gc = tp.quantize_weights_sharded(Wd[n0:n1].contiguous(), Ng * Kg, EPS, c)
            yc = tp.forward_column_parallel(xd, pc, gc, torch.bfloat16, gather=True, comm=c)
            k0, k1 = tp.col_shard(Kg, world, rank)
            pr, gr = tp.quantize_weights_sharded(Wd[:, k0:k1].contiguous(), Ng * Kg, EPS, c)
            yr = tp.forward_row_parallel(xd[:, k0:k1].contiguous(), pr, gr, torch.bfloat16, c)
            torch.cuda.synchronize()
            out[rank] = (pc.cpu().numpy(), gc.item(), yc.cpu().view(torch.int16).numpy(),
                         pr.cpu().numpy(), gr.item(), yr.cpu().view(torch.int16).numpy())
        except Exception as e:  # noqa: BLE001
            errors.append(e)
            comm._bar.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    assert bl.get_device_status() == 0
    for rank in range(world):
        pc, gc, yc, pr, gr, yr = out[rank]
        n0, n1 = row_shard(Ng, world, rank)
        k0, k1 = tp.col_shard(Kg, world, rank)
        assert gc == float(ref_gamma) and gr == float(ref_gamma)
        np.testing.assert_array_equal(pc, ref_packed[n0:n1])
        np.testing.assert_array_equal(pr, ref_packed[:, k0 // 4:k1 // 4])
        np.testing.assert_array_equal(yc, ref_y)
        np.testing.assert_array_equal(yr, ref_y)
