"""CUDA path vs the oracle, element by element, through the C ABI (gpu marker).

Bars: ternary codes, packed bytes, int8 codes, scales and int32 accumulators are compared
bit-exactly; fp32 outputs within 1e-6 relative error and bf16 outputs within 1 ulp (in
practice both are bit-identical, because both sides fix the same fp32 operation order).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import ternary_weight_linear_03_b200 as bl
from oracle import oracle as orc
from ternary_weight_linear_03_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

FP32_RTOL = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bl.load_library()
    assert bl.get_device_status() == 0
    yield
    assert bl.get_device_status() == 0


def _np_in(t: torch.Tensor):
    return syn.bf16_bits(t) if t.dtype == torch.bfloat16 else t.numpy()


def _bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def assert_f32_close(got: np.ndarray, ref: np.ndarray):
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    assert np.all(err <= FP32_RTOL * np.abs(ref.astype(np.float64))), float(err.max())


def assert_bf16_within_1ulp(got_bits: np.ndarray, ref_bits: np.ndarray):
    g = got_bits.astype(np.int32)
    r = ref_bits.astype(np.int32)
    # same sign and adjacent bit patterns (bf16 ordering is monotone within a sign)
    same_sign = (g >> 15) == (r >> 15)
    close = np.abs(g - r) <= 1
    zeros = ((g & 0x7FFF) == 0) & ((r & 0x7FFF) == 0)
    assert np.all((same_sign & close) | zeros)


# ----------------------------------------------------------------------------- weights


@pytest.mark.parametrize("N,K,dtype", [
    (256, 256, torch.float32), (293, 192, torch.float32), (4096, 1536, torch.float32),
    (300, 8640, torch.bfloat16), (8, 64, torch.bfloat16), (1, 64, torch.float32),
    # more than 64 KB of W per block (the ring of four 16 KB stages): the second pass
    # streams the block's range again instead of reading it from shared memory
    (1024, 8192, torch.float32), (2048, 8192, torch.bfloat16), (1111, 8256, torch.float32),
])
def test_quantize_weights_bit_exact(N, K, dtype):
    W = syn.weights(N, K, 0.02, seed=N * 7 + K, dtype=dtype)
    packed, gamma = bl.quantize_weights(W.cuda(), eps=1e-5)
    ref_packed, ref_gamma = orc.quantize_weights(_np_in(W), 1e-5)
    assert gamma.item() == float(ref_gamma)
    np.testing.assert_array_equal(packed.cpu().numpy(), ref_packed)


@pytest.mark.parametrize("kind", ["wide", "subnormal", "zeros", "constant", "sparse"])
def test_quantize_weights_exact_sum_edge_cases(kind):
    rng = np.random.default_rng(17)
    N, K = 96, 640
    if kind == "wide":
        w = rng.choice([-1, 1], N * K) * 10.0 ** rng.uniform(-30, 30, N * K)
    elif kind == "subnormal":
        w = rng.standard_normal(N * K) * 1e-40
        w[::5] = rng.standard_normal(len(w[::5])) * 0.02
    elif kind == "zeros":
        w = np.zeros(N * K)
    elif kind == "constant":
        w = np.full(N * K, -0.013)
    else:
        w = rng.standard_normal(N * K) * 0.02
        w[rng.random(N * K) < 0.9] = 0.0
    W = np.ascontiguousarray(w.astype(np.float32).reshape(N, K))
    for eps in (1e-5, 0.0):
        packed, gamma = bl.quantize_weights(torch.from_numpy(W).cuda(), eps=eps)
        ref_packed, ref_gamma = orc.quantize_weights(W, eps)
        assert gamma.item() == float(ref_gamma), (kind, eps)
        np.testing.assert_array_equal(packed.cpu().numpy(), ref_packed)


def test_quantize_weights_rows_of_very_different_scale():
    """Row blocks whose scale differs 100x, so the blocks' own shares of the sum of |w|
    differ by as much: gamma still comes out exact and every code with it."""
    N, K = 2048, 1536
    W = syn.weights(N, K, 1.0, seed=77)
    scale = torch.where((torch.arange(N) // 64) % 2 == 0, 0.001, 0.1)
    W = (W * scale[:, None]).contiguous()
    packed, gamma = bl.quantize_weights(W.cuda())
    ref_packed, ref_gamma = orc.quantize_weights(W.numpy(), 1e-5)
    assert gamma.item() == float(ref_gamma)
    np.testing.assert_array_equal(packed.cpu().numpy(), ref_packed)


@pytest.mark.parametrize("ws_kind", ["full", "tiny"])
def test_quantize_weights_many_ambiguous(ws_kind):
    """Half of the weights sit within 1% of (gamma + eps)/2, right at the threshold between
    0 and +-1, so a threshold off by one float would flip codes; also with the smallest
    workspace the call accepts."""
    rng = np.random.default_rng(5)
    N, K = 512, 2048
    mag = np.where(rng.random(N * K) < 0.5, 0.5 * (1 + 0.01 * rng.uniform(-1, 1, N * K)), 1.5)
    W = (mag * rng.choice([-1.0, 1.0], N * K) * 0.02).astype(np.float32).reshape(N, K)
    Wd = torch.from_numpy(W).cuda()
    lib = bl.load_library()
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    gamma = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = bl.workspace(1, N, K) if ws_kind == "full" else torch.empty(4096, dtype=torch.uint8, device="cuda")
    rc = lib.bitlinear_quantize_weights(Wd.data_ptr(), 0, N, K, 1e-5, packed.data_ptr(),
                                        gamma.data_ptr(), ws.data_ptr(), ws.numel(),
                                        torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    ref_packed, ref_gamma = orc.quantize_weights(W, 1e-5)
    assert gamma.item() == float(ref_gamma)
    np.testing.assert_array_equal(packed.cpu().numpy(), ref_packed)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_weights_single_read_band_overflow(dtype):
    """A matrix large enough for the single-read mode (each block's range exceeds its
    ring) whose weights crowd the threshold: half of them within 0.1% of (gamma + eps)/2,
    far more than a block's band list holds, so every block falls back to reading its
    range again. Codes stay exact, as they do on Gaussian matrices (patched lists)."""
    rng = np.random.default_rng(8)
    N, K = 2048, 8192
    mag = np.where(rng.random(N * K) < 0.5, 0.5 * (1 + 0.001 * rng.uniform(-1, 1, N * K)), 1.5)
    W = (mag * rng.choice([-1.0, 1.0], N * K) * 0.02).astype(np.float32).reshape(N, K)
    Wt = torch.from_numpy(W).to(dtype)
    packed, gamma = bl.quantize_weights(Wt.cuda())
    ref_packed, ref_gamma = orc.quantize_weights(_np_in(Wt), 1e-5)
    assert gamma.item() == float(ref_gamma)
    np.testing.assert_array_equal(packed.cpu().numpy(), ref_packed)


def test_ternarize_ties_on_device():
    """Weights exactly at 0.5 (gamma + eps) and one ulp either side."""
    d = np.float32(0.71875)
    half = np.float32(0.5) * d  # exact
    up = np.nextafter(half, np.float32(1))
    dn = np.nextafter(half, np.float32(0))
    row = [half, -half, up, -up, dn, -dn, np.float32(1.5) * d, -np.float32(1.5) * d]
    W = np.array(row * 8, np.float32)  # 64 values
    # pad a second row so that mean|W| is exactly d: need sum|W| = 128 d
    s = float(np.abs(W).astype(np.float64).sum())
    rest = np.full(64, np.float32((128 * float(d) - s) / 64), np.float32)
    W = np.stack([W, rest])
    ref_gamma = orc.absmean(W)
    packed, gamma = bl.quantize_weights(torch.from_numpy(W).cuda(), eps=0.0)
    assert gamma.item() == float(ref_gamma)
    ref_packed, _ = orc.quantize_weights(W, 0.0)
    np.testing.assert_array_equal(packed.cpu().numpy(), ref_packed)
    if ref_gamma == d:
        codes = orc.unpack(ref_packed, 64)[0, :8]
        np.testing.assert_array_equal(codes, [0, 0, 1, -1, 0, 0, 1, -1])


# ----------------------------------------------------------------------------- activations


@pytest.mark.parametrize("M,K,dtype,outliers", [
    (8, 256, torch.float32, 0.0), (16, 1536, torch.bfloat16, 0.01),
    (5, 8640, torch.bfloat16, 0.0), (64, 3200, torch.float32, 0.01),
])
def test_quantize_acts_bit_exact(M, K, dtype, outliers):
    x = syn.activations(M, K, seed=M + K, dtype=dtype, outlier_frac=outliers)
    x[0].zero_()                       # all-zero row
    if M > 2:
        x[1].zero_()
        x[1, 7] = -3.25                # one-hot row
    xq, scale = bl.quantize_acts(x.cuda())
    ref_q, ref_s = orc.quantize_acts(_np_in(x))
    np.testing.assert_array_equal(xq.cpu().numpy(), ref_q)
    np.testing.assert_array_equal(scale.cpu().numpy(), ref_s)


# ----------------------------------------------------------------------------- contraction


CONTRACT_SHAPES = [
    (1, 256, 256), (2, 293, 192), (3, 1000, 1536), (4, 777, 64),       # CUDA-core path
    (1, 4099, 8192), (1, 3001, 2048),            # one token, activations in registers
    (1, 5000, 28672), (2, 4800, 2048), (4, 4737, 4096),  # large K: two rows per warp
    (1, 3001, 16384), (1, 600, 57344), (1, 200, 131072),  # one token, long rows
    (5, 300, 640), (16, 4096, 1536), (130, 293, 8640), (300, 520, 1536),  # tensor-core path
    (129, 257, 128), (64, 64, 64), (256, 1000, 3200), (257, 300, 640), (17, 8640, 3200),
    (48, 129, 8640), (176, 520, 8192),
]


@pytest.mark.parametrize("M,N,K", CONTRACT_SHAPES)
def test_contract_i32_bit_exact(M, N, K):
    rng = np.random.default_rng(M * 1000 + N + K)
    q = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    q[0, :] = 127  # extreme row
    codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    codes[0, :] = 1
    packed = orc.pack(codes)
    acc = bl.contract_i32(torch.from_numpy(q).cuda(), torch.from_numpy(packed).cuda())
    np.testing.assert_array_equal(acc.cpu().numpy(), orc.contract_i32(q, codes))


# ----------------------------------------------------------------------------- forward


@pytest.mark.parametrize("M,N,K,x_dtype", [
    (8, 256, 256, torch.float32),          # tiny config
    (1, 4096, 1536, torch.bfloat16), (4, 4096, 1536, torch.bfloat16),
    (16, 4096, 1536, torch.bfloat16),
    (3, 1000, 3200, torch.float32), (200, 600, 8640, torch.bfloat16),
])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_forward_matches_oracle(M, N, K, x_dtype, out):
    W = syn.weights(N, K, 0.02, seed=1000 + N)
    x = syn.activations(M, K, seed=2000 + M, dtype=x_dtype, outlier_frac=0.01)
    packed, gamma = bl.quantize_weights(W.cuda())
    y = bl.forward(x.cuda(), packed, gamma,
                   out_dtype=torch.float32 if out == "f32" else torch.bfloat16)
    ref = orc.forward(_np_in(x), packed.cpu().numpy(), gamma.item(), out=out)
    if out == "f32":
        assert_f32_close(y.cpu().numpy(), ref)
        np.testing.assert_array_equal(y.cpu().numpy(), ref)  # same op order: identical
    else:
        got = y.cpu().view(torch.int16).numpy().view(np.uint16)
        assert_bf16_within_1ulp(got, ref)
        np.testing.assert_array_equal(got, ref)


def _edge_row(kind: str, K: int, seed: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    v = torch.randn(K, generator=g)
    if kind == "tiny":          # absmax ~4e-38: 127 / absmax overflows fp32 to +inf
        v = v * 1e-38
    elif kind == "zeros":
        v = torch.zeros(K)
    elif kind == "onehot":
        v = torch.zeros(K)
        v[K // 3] = -2.75
    elif kind == "subnormal_mix":  # bf16 subnormals next to a few ordinary values
        v = v * 1e-39
        v[::997] = torch.randn(len(v[::997]), generator=g)
    return v.bfloat16()


@pytest.mark.parametrize("K", [1536, 8192, 28672])
@pytest.mark.parametrize("kinds", [("normal",), ("tiny",), ("zeros",), ("onehot",),
                                   ("subnormal_mix",), ("tiny", "normal"), ("zeros", "onehot")])
def test_gemv_prologue_edge_rows(K, kinds):
    """bf16 tokens through the CUDA-core path (one or two tokens, activations in registers
    or in shared memory): ordinary rows, rows whose 127 / absmax overflows (every nonzero
    value quantizes to +-127), all-zero, one-hot and subnormal rows, bit for bit."""
    N = {1536: 4096, 8192: 2048, 28672: 4800}[K]  # registers, registers, two rows per warp
    W = syn.weights(N, K, 0.02, seed=K + 5)
    x = torch.stack([_edge_row(k, K, 31 * i + K) for i, k in enumerate(kinds)]).contiguous()
    packed, gamma = bl.quantize_weights(W.cuda())
    path, _ = bl.debug_plan(x.shape[0], N, K)
    assert path == "gemv"
    for out in ("f32", "bf16"):
        y = bl.forward(x.cuda(), packed, gamma,
                       out_dtype=torch.float32 if out == "f32" else torch.bfloat16)
        ref = orc.forward(_np_in(x), packed.cpu().numpy(), gamma.item(), out=out)
        got = y.cpu().numpy() if out == "f32" else y.cpu().view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(got, ref)
    assert bl.get_device_status() == 0


def test_forward_tiny_config_end_to_end():
    """Tiny config: W 256x256 ~N(0,0.02), x 8x256 ~N(0,1) fp32, seed 0, fp32 out."""
    W = syn.weights(256, 256, 0.02, seed=0)
    x = syn.activations(8, 256, seed=0, dtype=torch.float32)
    packed, gamma = bl.quantize_weights(W.cuda())
    y = bl.forward(x.cuda(), packed, gamma, out_dtype=torch.float32)
    ref_packed, ref_gamma = orc.quantize_weights(W.numpy(), 1e-5)
    ref = orc.forward(x.numpy(), ref_packed, ref_gamma)
    np.testing.assert_array_equal(y.cpu().numpy(), ref)


@pytest.mark.parametrize("m_small,m_big,N,K", [(4, 5, 1000, 1536), (2, 3, 4800, 2048),
                                               (256, 257, 1000, 1536)])
def test_forward_paths_agree_at_the_switch(m_small, m_big, N, K):
    """CUDA-core GEMV -> skinny tensor-core kernel at M = 4 | 5 for small packed weights and
    at M = 2 | 3 for larger ones; skinny -> prefill GEMM at M = 256 | 257. Rows present in
    both calls must agree bit for bit (the per-token quantization does not depend on the
    other tokens)."""
    W = syn.weights(N, K, 0.02, seed=5)
    x = syn.activations(m_big, K, seed=6)
    packed, gamma = bl.quantize_weights(W.cuda())
    yb = bl.forward(x.cuda(), packed, gamma, out_dtype=torch.float32)
    ys = bl.forward(x[:m_small].contiguous().cuda(), packed, gamma, out_dtype=torch.float32)
    torch.testing.assert_close(yb[:m_small], ys, rtol=0, atol=0)


# ----------------------------------------------------------------------------- full sizes


def oracle_forward_parallel(x_in, packed: np.ndarray, gamma: float, out: str):
    """The oracle's forward over every weight row, the rows cut into contiguous ranges run
    on one host thread each (the oracle itself stays single-threaded; ctypes releases the
    interpreter lock). Returns [M][N] and the thread count."""
    from concurrent.futures import ThreadPoolExecutor
    threads = max(1, min(os.cpu_count() or 1, 32))
    edges = np.linspace(0, packed.shape[0], threads + 1).astype(int)
    ranges = [(a, b) for a, b in zip(edges[:-1], edges[1:]) if b > a]
    with ThreadPoolExecutor(len(ranges)) as ex:
        parts = list(ex.map(
            lambda r: orc.forward(x_in, np.ascontiguousarray(packed[r[0]:r[1]]), gamma, out=out),
            ranges))
    return np.concatenate(parts, axis=1), len(ranges)


FULL = [
    ("700m_up_1536x4096", 16), ("3b_gate_up_3200x8640", 64), ("3b_down_8640x3200", 1),
    ("70b_up_8192x28672", 176), ("70b_down_28672x8192", 16),
]


@pytest.mark.parametrize("name,M", FULL)
def test_full_size_every_packed_byte(name, M):
    """Full-size matrices: gamma and every packed byte against the oracle (the 3B and 70B
    ones take the second pass's streaming branch), then the forward on sampled rows."""
    wl = syn.WORKLOADS[name]
    N, K = wl["N"], wl["K"]
    W = syn.weights(N, K, wl["sigma"], seed=syn.w_seed(name))
    x = syn.activations(M, K, seed=syn.x_seed(name, M), dtype=wl["x_dtype"],
                        outlier_frac=wl["outlier_frac"])
    packed, gamma = bl.quantize_weights(W.cuda())
    ref_gamma = orc.absmean(W.numpy())
    assert gamma.item() == float(ref_gamma)
    ref_packed = orc.pack(orc.ternarize(W.numpy(), ref_gamma, 1e-5))
    got_packed = packed.cpu().numpy()
    np.testing.assert_array_equal(got_packed, ref_packed)
    rows = np.sort(np.random.default_rng(0).choice(N, size=min(N, 96), replace=False))
    y = bl.forward(x.cuda(), packed, gamma, out_dtype=torch.bfloat16)
    ref = orc.forward(_np_in(x), np.ascontiguousarray(ref_packed[rows]), ref_gamma, out="bf16")
    got = y.cpu().view(torch.int16).numpy().view(np.uint16)[:, rows]
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("N,K", [(8192, 8192), (1024, 8192)])
def test_70b_layer_shapes_every_packed_byte(N, K):
    """The other 70B-shaped layer matrices the weight quantization serves (attention
    projections): gamma and every packed byte."""
    W = syn.weights(N, K, 0.015, seed=5000 + N)
    packed, gamma = bl.quantize_weights(W.cuda())
    ref_packed, ref_gamma = orc.quantize_weights(W.numpy(), 1e-5)
    assert gamma.item() == float(ref_gamma)
    np.testing.assert_array_equal(packed.cpu().numpy(), ref_packed)


@pytest.mark.parametrize("name,M", [("70b_up_8192x28672", 16), ("70b_down_28672x8192", 16)])
def test_70b_decode_forward_every_output(name, M):
    """One 70B decode forward (M = 16, the skinny tensor-core kernel), every one of its
    M x N bf16 outputs against the oracle, the oracle run over disjoint row ranges on the
    host's cores."""
    wl = syn.WORKLOADS[name]
    N, K = wl["N"], wl["K"]
    W = syn.weights(N, K, wl["sigma"], seed=syn.w_seed(name))
    x = syn.activations(M, K, seed=syn.x_seed(name, M), dtype=wl["x_dtype"])
    packed, gamma = bl.quantize_weights(W.cuda())
    y = bl.forward(x.cuda(), packed, gamma, out_dtype=torch.bfloat16)
    ref, threads = oracle_forward_parallel(_np_in(x), packed.cpu().numpy(), gamma.item(), "bf16")
    got = y.cpu().view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, ref)
    assert threads >= 1


@pytest.mark.parametrize("fixture", ["hand_worked_2x16.json", "hand_worked_eps_scale_2x16.json"])
def test_hand_worked_examples_on_device(fixture):
    """The hand-worked examples (tests/golden/) through the library: gamma, packed bytes
    and the fp32 outputs, bit for bit."""
    with open(os.path.join(os.path.dirname(__file__), "golden", fixture)) as f:
        d = json.load(f)
    W = torch.tensor(d["W"], dtype=torch.float32)
    # The library needs K % 64 == 0: the 16 columns are padded to 64 with weights equal to
    # gamma (so the mean of |W| over all 128 entries is still exactly gamma, the codes of
    # the real weights unchanged) facing zero activations (absmax and acc unchanged).
    K0 = W.shape[1]
    Wp = torch.full((W.shape[0], 64), d["gamma"], dtype=torch.float32)
    Wp[:, :K0] = W
    x = torch.zeros((1, 64))
    x[:, :K0] = torch.tensor(d["x"], dtype=torch.float32)
    packed, gamma = bl.quantize_weights(Wp.cuda(), eps=d["eps"])
    assert gamma.item() == d["gamma"]
    np.testing.assert_array_equal(packed.cpu().numpy()[:, :K0 // 4], np.array(d["packed"], np.uint8))
    y = bl.forward(x.cuda(), packed, gamma, out_dtype=torch.float32)
    np.testing.assert_array_equal(y.cpu().numpy(), np.array(d["y"], np.float32))


def test_prefill_shape_sampled_rows():
    """M = 4096, K = 8192, N = 28672 through the tensor-core path, sampled outputs."""
    name = "70b_prefill_4096x8192x28672"
    wl = syn.WORKLOADS[name]
    N, K, M = wl["N"], wl["K"], 4096
    W = syn.weights(N, K, wl["sigma"], seed=syn.w_seed(name))
    x = syn.activations(M, K, seed=syn.x_seed(name, M), dtype=torch.bfloat16)
    packed, gamma = bl.quantize_weights(W.cuda())
    y = bl.forward(x.cuda(), packed, gamma, out_dtype=torch.bfloat16)
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(N, 64, replace=False))
    toks = np.sort(rng.choice(M, 48, replace=False))
    codes = orc.ternarize(np.ascontiguousarray(W.numpy()[rows]), gamma.item(), 1e-5)
    xs = x[torch.from_numpy(toks)].contiguous()
    ref = orc.forward(syn.bf16_bits(xs), orc.pack(codes), gamma.item(), out="bf16")
    got = y.cpu()[torch.from_numpy(toks)][:, torch.from_numpy(rows)]
    np.testing.assert_array_equal(got.contiguous().view(torch.int16).numpy().view(np.uint16), ref)


# ----------------------------------------------------------------------------- status word


def test_nonfinite_inputs_set_status():
    W = torch.randn(64, 64, device="cuda")
    W[3, 5] = float("nan")
    bl.quantize_weights(W)
    assert bl.get_device_status() == 6
    x = torch.randn(2, 64, device="cuda")
    x[1, 1] = float("inf")
    bl.quantize_acts(x)
    assert bl.get_device_status() == 6
    assert bl.get_device_status() == 0  # read clears


def test_timeout_probe_reports_and_context_survives():
    bl.debug_timeout_probe(2_000_000)  # 2 ms wait on a barrier nobody arrives on
    assert bl.get_device_status() == 5
    W = syn.weights(256, 256, 0.02, seed=0)
    packed, gamma = bl.quantize_weights(W.cuda())
    assert gamma.item() == float(orc.absmean(W.numpy()))
    assert bl.get_device_status() == 0


def test_repeatable():
    W = syn.weights(2048, 1536, 0.02, seed=3).cuda()
    x = syn.activations(64, 1536, seed=4).cuda()
    p1, g1 = bl.quantize_weights(W)
    p2, g2 = bl.quantize_weights(W)
    assert torch.equal(p1, p2) and torch.equal(g1, g2)
    assert torch.equal(bl.forward(x, p1, g1), bl.forward(x, p2, g2))
