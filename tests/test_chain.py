"""Layer chains (bitlinear_chain_forward): several BitLinear layers over one batch, each
reading the chain input or an earlier layer's bf16 output, with the next layer's absmax
formed in the producing kernel's epilogue and every launch chained by programmatic
dependent launch.

CPU: the host-side plan (workspace size, argument checks). GPU: every output of the
chain against the oracle applied layer by layer (bf16 intermediates), bit for bit, on the
three kernel paths and the feed-forward pattern (gate and up read the same input)."""

import ctypes

import numpy as np
import pytest
import torch

import ternary_weight_linear_03_b200 as bl
from ternary_weight_linear_03_b200 import synthetic as syn

FAKE = 0x10000  # 16-byte aligned, never dereferenced by the host-only size query


def _fake_layers(specs):
    arr = (bl.Layer * len(specs))()
    for i, (N, K, src) in enumerate(specs):
        arr[i] = bl.Layer(FAKE, FAKE, N, K, src, None)
    return arr


def test_chain_workspace_size_checks_the_chain():
    lib = bl.load_library()
    ok = _fake_layers([(1536, 512, -1), (1536, 512, -1), (512, 1536, 1)])
    assert lib.bitlinear_chain_workspace_size(16, ok, 3) > 0
    assert lib.bitlinear_chain_workspace_size(16, ok, 0) == 0               # no layers
    assert lib.bitlinear_chain_workspace_size(0, ok, 3) == 0                # M = 0
    bad_src = _fake_layers([(1536, 512, -1), (512, 1536, 1)])               # reads itself
    assert lib.bitlinear_chain_workspace_size(16, bad_src, 2) == 0
    bad_k = _fake_layers([(1536, 512, -1), (512, 1024, 0)])                 # K != N of src
    assert lib.bitlinear_chain_workspace_size(16, bad_k, 2) == 0
    two_x = _fake_layers([(1536, 512, -1), (512, 640, -1)])                 # x with two K
    assert lib.bitlinear_chain_workspace_size(16, two_x, 2) == 0
    # bigger batches need more room (activation buffers and staged codes scale with M)
    assert (lib.bitlinear_chain_workspace_size(300, ok, 3)
            > lib.bitlinear_chain_workspace_size(16, ok, 3))


def test_chain_forward_rejects_bad_arguments():
    lib = bl.load_library()
    ok = _fake_layers([(1536, 512, -1), (512, 1536, 0)])
    f = lib.bitlinear_chain_forward
    assert f(None, 1, 4, ok, 2, FAKE, 1, FAKE, 1 << 30, None) == 1
    assert f(FAKE, 2, 4, ok, 2, FAKE, 1, FAKE, 1 << 30, None) == 1   # int32 x
    assert f(FAKE, 1, 4, ok, 2, FAKE + 8, 1, FAKE, 1 << 30, None) == 3
    assert f(FAKE, 1, 4, ok, 2, FAKE, 1, FAKE, 16, None) == 7        # workspace too small
    bad = _fake_layers([(1536, 512, -1), (512, 1000, 0)])
    assert f(FAKE, 1, 4, bad, 2, FAKE, 1, FAKE, 1 << 30, None) == 2


# ----------------------------------------------------------------------------- GPU


def _ffn_chain(blocks, d, h, sigma, device, gate_out):
    """Layers of `blocks` feed-forward blocks: gate (d -> h, output kept), up (d -> h,
    same input), down (h -> d, reads up); the next block reads down."""
    layers, fp32 = [], []
    src = -1
    for b in range(blocks):
        for i, (N, K) in enumerate([(h, d), (h, d), (d, h)]):
            W = syn.weights(N, K, sigma, seed=7000 + 3 * b + i)
            fp32.append(W)
            packed, gamma = bl.quantize_weights(W.to(device))
            if i == 0:
                layers.append((packed, gamma, src, gate_out[b]))
            elif i == 1:
                layers.append((packed, gamma, src))
            else:
                layers.append((packed, gamma, len(layers) - 1))
        src = len(layers) - 1
    return layers


def _oracle_chain(x_in, layers, out):
    from oracle import oracle as orc
    bufs = [x_in]
    for i, ly in enumerate(layers):
        last = i == len(layers) - 1
        y = orc.forward(bufs[ly[2] + 1], ly[0].cpu().numpy(), ly[1].item(),
                        out=out if last else "bf16")
        bufs.append(y)
    return bufs


@pytest.mark.gpu
@pytest.mark.parametrize("M,x_dtype,out", [(1, torch.bfloat16, "bf16"), (2, torch.float32, "f32"),
                                           (16, torch.bfloat16, "bf16"), (64, torch.bfloat16, "f32"),
                                           (300, torch.bfloat16, "bf16")])
def test_ffn_chain_matches_oracle_layer_by_layer(M, x_dtype, out):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    d, h, blocks = 1024, 3200, 2
    gate_out = [torch.full((M, h), float("nan"), dtype=torch.bfloat16, device="cuda")
                for _ in range(blocks)]
    layers = _ffn_chain(blocks, d, h, 0.02, "cuda", gate_out)
    x = syn.activations(M, d, seed=31 + M, dtype=x_dtype, outlier_frac=0.01)
    y = bl.chain_forward(x.cuda(), layers,
                         out_dtype=torch.float32 if out == "f32" else torch.bfloat16)
    torch.cuda.synchronize()
    assert bl.get_device_status() == 0
    x_in = syn.bf16_bits(x) if x_dtype == torch.bfloat16 else x.numpy()
    bufs = _oracle_chain(x_in, layers, out)
    got = y.cpu()
    got = got.numpy() if out == "f32" else got.view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, bufs[-1])
    for b in range(blocks):  # the gate outputs the chain handed back
        g = gate_out[b].cpu().view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(g, bufs[3 * b + 1])


@pytest.mark.gpu
@pytest.mark.parametrize("M", [16, 64])
def test_chain_equals_separate_forwards_and_repeats(M):
    """The chain gives the bits of separate bitlinear_forward calls; a second call on the
    same workspace (whose absmax and split-K sums start from what the first left) agrees.
    At 64 tokens the chain splits K where a single forward does not."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    d, h = 3200, 8640  # the 3B feed-forward shapes
    gate_out = [torch.empty((M, h), dtype=torch.bfloat16, device="cuda")]
    layers = _ffn_chain(1, d, h, 0.02, "cuda", gate_out)
    x = syn.activations(M, d, seed=5).cuda()
    ws = bl.chain_workspace(M, layers)
    y1 = bl.chain_forward(x, layers, ws=ws).clone()
    y2 = bl.chain_forward(x, layers, ws=ws)
    g = bl.forward(x, layers[0][0], layers[0][1])
    u = bl.forward(x, layers[1][0], layers[1][1])
    yd = bl.forward(u, layers[2][0], layers[2][1])
    torch.cuda.synchronize()
    assert torch.equal(y1, yd) and torch.equal(y2, yd)
    assert torch.equal(gate_out[0], g)
