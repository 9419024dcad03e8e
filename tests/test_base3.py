"""Base-3 weight format (5 trits per byte) through the C ABI: the 2-bit -> base-3 repack
and the decode GEMV on base-3 weights, against the oracle's pack_base3 and forward
(bit for bit). CPU: the row size and the host-side argument checks."""

import numpy as np
import pytest
import torch

import ternary_weight_linear_03_b200 as bl
from oracle import oracle as orc
from ternary_weight_linear_03_b200 import synthetic as syn

FAKE = 0x10000


@pytest.mark.parametrize("K", [64, 128, 1536, 3200, 8192, 8640, 28672])
def test_row_bytes_agree_with_the_oracle(K):
    assert bl.base3_row_bytes(K) == orc.base3_row_bytes(K)


def test_base3_argument_checks():
    lib = bl.load_library()
    assert lib.bitlinear_base3_row_bytes(100) == 0
    assert lib.bitlinear_pack_base3(None, 16, 64, FAKE, None) == 1
    assert lib.bitlinear_pack_base3(FAKE, 16, 96, FAKE, None) == 2
    assert lib.bitlinear_pack_base3(FAKE, 16, 64, FAKE + 4, None) == 3
    f = lib.bitlinear_forward_base3
    assert f(FAKE, 1, FAKE, FAKE, FAKE, 1, 5, 16, 64, None) == 2        # M > 4
    assert f(FAKE, 1, FAKE, FAKE, FAKE, 1, 4, 16, 28672 * 2, None) == 2  # 4 rows too long
    assert f(FAKE, 2, FAKE, FAKE, FAKE, 1, 1, 16, 64, None) == 1
    assert f(FAKE, 1, FAKE + 8, FAKE, FAKE, 1, 1, 16, 64, None) == 3


def _np_in(t):
    return syn.bf16_bits(t) if t.dtype == torch.bfloat16 else t.numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,x_dtype,out", [
    (1, 4096, 1536, torch.bfloat16, "bf16"), (4, 4096, 1536, torch.bfloat16, "f32"),
    (1, 8640, 3200, torch.float32, "f32"), (2, 3200, 8640, torch.bfloat16, "bf16"),
    (3, 1001, 8192, torch.bfloat16, "bf16"), (1, 300, 28672, torch.bfloat16, "bf16"),
    (1, 7, 64, torch.float32, "f32"),
])
def test_base3_repack_and_forward_match_oracle(M, N, K, x_dtype, out):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    W = syn.weights(N, K, 0.02, seed=N + K)
    x = syn.activations(M, K, seed=M + K, dtype=x_dtype, outlier_frac=0.01)
    packed, gamma = bl.quantize_weights(W.cuda())
    packed3 = bl.pack_base3(packed)
    codes = orc.unpack(packed.cpu().numpy(), K)
    np.testing.assert_array_equal(packed3.cpu().numpy(), orc.pack_base3(codes))
    od = torch.float32 if out == "f32" else torch.bfloat16
    y3 = bl.forward_base3(x.cuda(), packed3, gamma, out_dtype=od)
    y2 = bl.forward(x.cuda(), packed, gamma, out_dtype=od)
    torch.cuda.synchronize()
    assert bl.get_device_status() == 0
    ref = orc.forward(_np_in(x), packed.cpu().numpy(), gamma.item(), out=out)
    got = y3.cpu()
    got = got.numpy() if out == "f32" else got.view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, ref)
    assert torch.equal(y3, y2)


@pytest.mark.gpu
def test_base3_full_size_70b_down_decode():
    """The 70B down projection (K = 28672, 358.4 chunks per row: a ragged last chunk) at
    M = 1: every packed byte and output against the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    name = "70b_down_28672x8192"
    wl = syn.WORKLOADS[name]
    N, K = wl["N"], wl["K"]
    W = syn.weights(N, K, wl["sigma"], seed=syn.w_seed(name))
    x = syn.activations(1, K, seed=syn.x_seed(name, 1))
    packed, gamma = bl.quantize_weights(W.cuda())
    packed3 = bl.pack_base3(packed)
    np.testing.assert_array_equal(packed3.cpu().numpy(),
                                  orc.pack_base3(orc.unpack(packed.cpu().numpy(), K)))
    y = bl.forward_base3(x.cuda(), packed3, gamma)
    ref = orc.forward(syn.bf16_bits(x), packed.cpu().numpy(), gamma.item(), out="bf16")
    np.testing.assert_array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), ref)
