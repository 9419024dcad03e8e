"""The library's shard-level entry points against the oracle (gpu marker): the exact |w|
sums of weight shards and gamma from their total, the activation absmax and quantization
with a given absmax, and the stand-alone rescale. Integer results bit for bit; fp32 and
bf16 outputs identical (same operation order on both sides)."""

import numpy as np
import pytest
import torch

import ternary_weight_linear_03_b200 as bl
from oracle import oracle as orc
from ternary_weight_linear_03_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bl.load_library()
    assert bl.get_device_status() == 0
    yield
    assert bl.get_device_status() == 0


def _np_in(t):
    return syn.bf16_bits(t) if t.dtype == torch.bfloat16 else t.numpy()


@pytest.mark.parametrize("N,K,dtype,parts", [
    (512, 1536, torch.float32, 2), (4096, 8192, torch.float32, 2),   # second: streamed pass B
    (300, 8640, torch.bfloat16, 3), (64, 64, torch.float32, 1),
])
def test_gamma_from_shard_sums_equals_whole(N, K, dtype, parts):
    """Row shards: words added on the device, then each shard coded against the total;
    gamma and the concatenated codes equal bitlinear_quantize_weights on the whole matrix
    and the oracle."""
    W = syn.weights(N, K, 0.02, seed=N + K, dtype=dtype)
    W[: N // 2] *= 7.0
    Wd = W.cuda()
    edges = np.linspace(0, N, parts + 1).astype(int)
    shards = [Wd[a:b].contiguous() for a, b in zip(edges[:-1], edges[1:])]
    total = sum(bl.weight_abssum(s) for s in shards)
    got = [bl.quantize_weights_from_abssum(s, N * K, total, 1e-5) for s in shards]
    packed_whole, gamma_whole = bl.quantize_weights(Wd)
    ref_packed, ref_gamma = orc.quantize_weights(_np_in(W), 1e-5)
    for _, g in got:
        assert g.item() == float(ref_gamma) == gamma_whole.item()
    cat = torch.cat([p for p, _ in got]).cpu().numpy()
    np.testing.assert_array_equal(cat, ref_packed)
    np.testing.assert_array_equal(packed_whole.cpu().numpy(), ref_packed)


def test_abssum_words_of_one_matrix_give_its_gamma():
    W = syn.weights(256, 640, 0.02, seed=3)
    s = bl.weight_abssum(W.cuda())
    p, g = bl.quantize_weights_from_abssum(W.cuda(), W.numel(), s, 0.0)
    rp, rg = orc.quantize_weights(W.numpy(), 0.0)
    assert g.item() == float(rg)
    np.testing.assert_array_equal(p.cpu().numpy(), rp)


@pytest.mark.parametrize("M,K,dtype", [(5, 1536, torch.bfloat16), (64, 8640, torch.float32)])
def test_act_absmax_and_quantize_with_given_absmax(M, K, dtype):
    x = syn.activations(M, K, seed=M * 3, dtype=dtype, outlier_frac=0.01)
    x[0].zero_()
    xd = x.cuda()
    a = bl.act_absmax(xd)
    np.testing.assert_array_equal(a.cpu().numpy(), orc.act_absmax(_np_in(x)))
    # K-shards quantized with the whole rows' absmax reproduce the whole-row codes
    q, s = orc.quantize_acts(_np_in(x))
    half = (K // 2) // 64 * 64
    for k0, k1 in [(0, half), (half, K)]:
        xq, sc = bl.quantize_acts_absmax(xd[:, k0:k1].contiguous(), a)
        np.testing.assert_array_equal(xq.cpu().numpy(), q[:, k0:k1])
        np.testing.assert_array_equal(sc.cpu().numpy(), s)


@pytest.mark.parametrize("M,N,out", [(7, 1000, "f32"), (64, 8192, "bf16"), (3, 999, "bf16")])
def test_rescale_matches_oracle(M, N, out):
    rng = np.random.default_rng(M + N)
    acc = rng.integers(-127 * 8192, 127 * 8192, size=(M, N)).astype(np.int32)
    scale = (rng.random(M) * 0.3).astype(np.float32)
    scale[0] = 0.0
    gamma = np.float32(0.0137)
    y = bl.rescale(torch.from_numpy(acc).cuda(), torch.from_numpy(scale).cuda(),
                   torch.tensor([gamma]).cuda(),
                   out_dtype=torch.float32 if out == "f32" else torch.bfloat16)
    ref = orc.rescale(acc, scale, float(gamma))
    if out == "f32":
        np.testing.assert_array_equal(y.cpu().numpy(), ref)
    else:
        np.testing.assert_array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16),
                                      orc.to_bf16(ref))
