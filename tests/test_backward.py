"""Straight-through BitLinear backward (bitlinear_backward, bitlinear_pack_transpose).

The transposed 2-bit weights are compared byte for byte with the oracle's packing of the
transposed codes. The gradients are compared with the oracle's float64 sums, within the
bound the fp32 accumulation allows: every product G c and G X~ is exact in fp32 (bf16 x
bf16, or bf16 x +-1), so the only error is the rounding of the additions. A sum of n
terms accumulated in fp32 in any order is off by at most (n - 1) u sum|terms| with
u = 2^-24 per correctly rounded addition; the bar allows 4 u per addition (2^-22) for the
tensor core's accumulation, plus one rounding (2^-23 relative) for the scaling by gamma:
    |got - ref| <= n 2^-22 sum|terms| + 2^-23 |ref|."""

import numpy as np
import pytest
import torch

import ternary_weight_linear_03_b200 as bl
from oracle import oracle as orc
from ternary_weight_linear_03_b200 import synthetic as syn

FAKE = 0x10000


def test_backward_argument_checks():
    lib = bl.load_library()
    assert lib.bitlinear_backward_workspace_size(16, 100, 64) == 0     # N % 64
    assert lib.bitlinear_backward_workspace_size(16, 128, 64) > 0
    assert lib.bitlinear_pack_transpose(FAKE, 100, 64, FAKE, None) == 2
    f = lib.bitlinear_backward
    assert f(FAKE, 1, FAKE, FAKE, FAKE, None, None, 4, 128, 64, FAKE, 1 << 20, None) == 1
    assert f(FAKE, 1, FAKE, None, FAKE, FAKE, None, 4, 128, 64, FAKE, 1 << 20, None) == 1
    assert f(FAKE, 1, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 100, 64, FAKE, 1 << 20, None) == 2
    assert f(FAKE, 1, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 128, 64, FAKE, 16, None) == 7
    assert f(FAKE, 1, FAKE + 2, FAKE, FAKE, FAKE, None, 4, 128, 64, FAKE, 1 << 20, None) == 3


def _within_bound(got, ref, abs_terms, n):
    bound = n * 2.0 ** -22 * abs_terms + 2.0 ** -23 * np.abs(ref)
    err = np.abs(got.astype(np.float64) - ref)
    assert np.all(err <= bound), float(np.max(err / np.maximum(bound, 1e-300)))


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,x_dtype", [
    (8, 256, 256, torch.float32), (300, 640, 1536, torch.bfloat16),
    (130, 4096, 1536, torch.bfloat16), (64, 3200, 8640, torch.bfloat16),
    (520, 1024, 1536, torch.bfloat16), (5, 128, 64, torch.float32),
])
def test_backward_matches_oracle(M, N, K, x_dtype):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    W = syn.weights(N, K, 0.02, seed=N + 3 * K)
    x = syn.activations(M, K, seed=M + K, dtype=x_dtype, outlier_frac=0.01)
    G = (torch.randn((M, N), generator=syn.gen(M * N)) * 0.01).bfloat16()
    packed, gamma = bl.quantize_weights(W.cuda())
    packedT = bl.pack_transpose(packed)
    codes = orc.unpack(packed.cpu().numpy(), K)
    np.testing.assert_array_equal(packedT.cpu().numpy(), orc.pack(np.ascontiguousarray(codes.T)))
    gx, gw = bl.backward(x.cuda(), G.cuda(), packedT, gamma)
    torch.cuda.synchronize()
    assert bl.get_device_status() == 0
    Gb = G.view(torch.int16).numpy().view(np.uint16)
    Gf = G.float().numpy().astype(np.float64)
    g = float(gamma.item())
    ref_x = orc.ste_grad_x(Gb, codes, g)
    _within_bound(gx.cpu().numpy(), ref_x, abs(g) * (np.abs(Gf) @ np.abs(codes).astype(np.float64)), N)
    xin = syn.bf16_bits(x) if x_dtype == torch.bfloat16 else x.numpy()
    q, s = orc.quantize_acts(xin)
    xt = orc.dequant_acts_bf16(q, s)
    ref_w = orc.ste_grad_w(Gb, xt)
    xtf = (xt.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    _within_bound(gw.cpu().numpy(), ref_w, np.abs(Gf).T @ np.abs(xtf), M)


@pytest.mark.gpu
def test_backward_single_gradients_and_exact_cases():
    """grad_x alone and grad_w alone; with G holding one non-zero entry per row every sum
    has one term, so both gradients are exact (bit for bit the oracle's)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    M, N, K = 128, 512, 1024
    W = syn.weights(N, K, 0.02, seed=3)
    x = syn.activations(M, K, seed=4)
    packed, gamma = bl.quantize_weights(W.cuda())
    packedT = bl.pack_transpose(packed)
    G = torch.zeros((M, N))
    G[torch.arange(M), (torch.arange(M) * 37) % N] = 0.5 + torch.arange(M) / 256.0
    G = G.bfloat16()
    gx, none_w = bl.backward(x.cuda(), G.cuda(), packedT, gamma, need_w=False)
    none_x, gw = bl.backward(x.cuda(), G.cuda(), packedT, gamma, need_x=False)
    assert none_w is None and none_x is None
    codes = orc.unpack(packed.cpu().numpy(), K)
    Gb = G.view(torch.int16).numpy().view(np.uint16)
    ref_x = orc.ste_grad_x(Gb, codes, float(gamma.item()))
    np.testing.assert_array_equal(gx.cpu().numpy(), ref_x.astype(np.float32))
    q, s = orc.quantize_acts(syn.bf16_bits(x))
    ref_w = orc.ste_grad_w(Gb, orc.dequant_acts_bf16(q, s))
    # token t's one entry is at n = 37 t mod 512, distinct for the 128 tokens (37 is odd),
    # so every grad_w entry has at most one term
    assert np.bincount((np.arange(M) * 37) % N, minlength=N).max() == 1
    np.testing.assert_array_equal(gw.cpu().numpy(), ref_w.astype(np.float32))
