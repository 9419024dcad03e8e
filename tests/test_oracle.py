"""Pins for the oracle: each test ties one oracle function to something other than itself
(a hand-worked example, a correctly rounded library sum, closed forms, brute force, a
library routine, or an invariant the method fixes). CPU only."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fsum_gamma(w: np.ndarray) -> np.float32:
    """Correctly rounded double of the exact sum (math.fsum), / n in double, -> fp32."""
    a = np.abs(w.astype(np.float64)).ravel()
    return np.float32(math.fsum(a.tolist()) / a.size)


# ----------------------------------------------------------------------------- golden


@pytest.mark.parametrize("fixture", ["hand_worked_2x16.json", "hand_worked_eps_scale_2x16.json"])
def test_hand_worked_example(fixture):
    """Every stage of a hand-worked 2x16 example (tests/golden/): the first with eps = 0
    and unit scale, the second with eps > 0 and a scale that is not a power of two, where
    the rescale's operation order and its use of gamma (not gamma + eps) show in the bits."""
    with open(os.path.join(GOLDEN, fixture)) as f:
        d = json.load(f)
    W = np.array(d["W"], np.float32)
    x = np.array(d["x"], np.float32)
    gamma = orc.absmean(W)
    assert gamma == np.float32(d["gamma"])
    codes = orc.ternarize(W, gamma, d["eps"])
    np.testing.assert_array_equal(codes, np.array(d["codes"], np.int8))
    packed = orc.pack(codes)
    np.testing.assert_array_equal(packed, np.array(d["packed"], np.uint8))
    q, s = orc.quantize_acts(x)
    np.testing.assert_array_equal(q, np.array(d["q"], np.int8))
    np.testing.assert_array_equal(s, np.array(d["scale"], np.float32))
    acc = orc.contract_i32(q, codes)
    np.testing.assert_array_equal(acc, np.array(d["acc"], np.int32))
    y = orc.forward(x, packed, gamma)
    np.testing.assert_array_equal(y, np.array(d["y"], np.float32))
    for wrong in ("y_wrong_order", "y_rescaled_by_gamma_plus_eps"):
        if wrong in d:  # the fixture's alternatives really differ from the answer
            assert np.all(np.array(d[wrong], np.float32) != y), wrong


# ----------------------------------------------------------------------------- absmean


@pytest.mark.parametrize("kind", ["gauss", "wide", "subnormal", "huge", "bf16"])
def test_absmean_equals_correctly_rounded_sum(kind):
    rng = np.random.default_rng(7)
    n = 50_000
    if kind == "gauss":
        w = (rng.standard_normal(n) * 0.02).astype(np.float32)
    elif kind == "wide":  # exponents over most of the fp32 range, both signs
        w = (rng.choice([-1, 1], n) * 10.0 ** rng.uniform(-37, 37, n)).astype(np.float32)
    elif kind == "subnormal":
        w = (rng.standard_normal(n) * 1e-40).astype(np.float32)
        w[::7] = rng.standard_normal(len(w[::7])).astype(np.float32)
    elif kind == "huge":
        w = (rng.uniform(-1, 1, n) * 3.0e38).astype(np.float32)
    else:
        t = torch.from_numpy((rng.standard_normal(n) * 0.02).astype(np.float32)).bfloat16()
        bits = t.view(torch.int16).numpy().view(np.uint16)
        g = orc.absmean(bits)
        assert g == _fsum_gamma(t.float().numpy())
        return
    g = orc.absmean(w)
    assert g == _fsum_gamma(w), (g, _fsum_gamma(w))
    ref = np.mean(np.abs(w.astype(np.float64)))
    assert abs(float(g) - ref) <= 1e-7 * ref


def test_absmean_special_cases():
    a = np.float32(0.0123)
    assert orc.absmean(np.full(4096, a, np.float32)) == a
    assert orc.absmean(np.full(1000, -a, np.float32)) == a
    assert orc.absmean(np.zeros(64, np.float32)) == 0.0
    # many equal terms whose fp32 running sum would drift: exact sum still gives a
    assert orc.absmean(np.full(3_000_000, np.float32(0.1), np.float32)) == np.float32(0.1)
    with pytest.raises(ValueError):
        orc.absmean(np.array([1.0, np.inf], np.float32))
    with pytest.raises(ValueError):
        orc.absmean(np.array([np.nan, 1.0], np.float32))


# ----------------------------------------------------------------------------- ternarize


def test_ternarize_ties_and_saturation():
    # gamma = 1, eps = 0 -> d = 1, so w / d = w exactly
    w = np.array([0.5, np.nextafter(np.float32(0.5), np.float32(1)), 1.5, 2.5, -0.5,
                  np.nextafter(np.float32(-0.5), np.float32(0)), -1.5, 0.0, 1e-30, 1e30,
                  -1e30, 0.49999997], np.float32)
    expect = [0, 1, 1, 1, 0, 0, -1, 0, 0, 1, -1, 0]
    np.testing.assert_array_equal(orc.ternarize(w, 1.0, 0.0), np.array(expect, np.int8))
    # d = gamma + eps rounds in fp32: gamma = 2, eps = 2 -> d = 4; 2.0 / 4 = 0.5 tie -> 0
    np.testing.assert_array_equal(orc.ternarize(np.array([2.0, 2.5, -6.0], np.float32), 2.0, 2.0),
                                  np.array([0, 1, -1], np.int8))
    # gamma = eps = 0: every code is 0
    np.testing.assert_array_equal(orc.ternarize(np.array([1.0, -3.0, 0.0], np.float32), 0.0, 0.0),
                                  np.zeros(3, np.int8))


def test_ternarize_constant_matrix():
    W = np.full((8, 64), np.float32(0.37), np.float32)
    packed, gamma = orc.quantize_weights(W, 1e-5)
    assert gamma == np.float32(0.37)
    np.testing.assert_array_equal(orc.unpack(packed, 64), np.ones((8, 64), np.int8))


def test_ternarize_gaussian_closed_form():
    """W ~ N(0, sigma): E|W| = sigma*sqrt(2/pi), P(code 0) = erf(0.5 d / (sigma sqrt 2))."""
    sigma, eps, n = 0.02, 1e-5, 2_000_000
    w = (np.random.default_rng(3).standard_normal(n) * sigma).astype(np.float32)
    gamma = orc.absmean(w)
    assert abs(float(gamma) - sigma * math.sqrt(2 / math.pi)) < 5 * sigma / math.sqrt(n)
    codes = orc.ternarize(w, gamma, eps)
    assert set(np.unique(codes).tolist()) <= {-1, 0, 1}
    d = float(gamma) + eps
    p0 = math.erf(0.5 * d / (sigma * math.sqrt(2)))
    assert abs(0.310 - p0) < 0.002
    tol = 5 * math.sqrt(p0 * (1 - p0) / n)
    assert abs(np.mean(codes == 0) - p0) < tol
    pplus = (1 - p0) / 2
    assert abs(np.mean(codes == 1) - pplus) < 5 * math.sqrt(pplus * (1 - pplus) / n)


# ----------------------------------------------------------------------------- pack


def _codes_by(fn, N=3, K=64):
    return np.array([[fn(k) for k in range(K)] for _ in range(N)], np.int8)


def test_pack_closed_form_bytes():
    assert np.all(orc.pack(_codes_by(lambda k: 1)) == 0xAA)
    assert np.all(orc.pack(_codes_by(lambda k: 0)) == 0x55)
    assert np.all(orc.pack(_codes_by(lambda k: -1)) == 0x00)
    # depends only on i = k % 4: (+1, 0, -1, 0) -> bytes AA 55 00 55 repeating
    p = orc.pack(_codes_by(lambda k: [1, 0, -1, 0][k % 4]))
    np.testing.assert_array_equal(p[0, :8], [0xAA, 0x55, 0x00, 0x55] * 2)
    # depends only on j = (k % 16) // 4: (+1, 0, -1, 0) -> every byte 2 | 1<<2 | 0<<4 | 1<<6
    p = orc.pack(_codes_by(lambda k: [1, 0, -1, 0][(k % 16) // 4]))
    assert np.all(p == 0x46)
    # a single +1 at k = 21 (g = 1, j = 1, i = 1) among -1: row byte 4*1+1 = 5 holds 2 << 2
    c = _codes_by(lambda k: 1 if k == 21 else -1, N=1, K=32)
    expect = np.zeros(8, np.uint8)
    expect[5] = 0x08
    np.testing.assert_array_equal(orc.pack(c)[0], expect)


def test_pack_roundtrip_and_bad_code():
    rng = np.random.default_rng(11)
    codes = rng.integers(-1, 2, size=(37, 160)).astype(np.int8)
    np.testing.assert_array_equal(orc.unpack(orc.pack(codes), 160), codes)
    bad = orc.pack(codes)
    bad[3, 7] |= 0x3 << 4
    with pytest.raises(ValueError):
        orc.unpack(bad, 160)


# ----------------------------------------------------------------------------- activations


def test_quantize_acts_rounding_and_ties():
    # absmax 127 -> r = 1 exactly, s = 1: q = rne(x)
    x = np.array([[127.0, 2.5, 3.5, -2.5, 0.5, 1.5, 126.5, -0.5, -126.5, 0.0]], np.float32)
    q, s = orc.quantize_acts(x)
    np.testing.assert_array_equal(q[0], [127, 2, 4, -2, 0, 2, 126, 0, -126, 0])
    assert s[0] == 1.0


def test_quantize_acts_invariants():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 1536)).astype(np.float32)
    x[:, rng.choice(1536, 16, replace=False)] *= 20
    q, s = orc.quantize_acts(x)
    assert np.all(np.abs(q.astype(int)).max(axis=1) == 127)  # per-row max |q| = 127
    assert q.min() >= -127
    a = np.abs(x).max(axis=1)
    np.testing.assert_array_equal(s, (a / np.float32(127)).astype(np.float32))
    err = np.abs(x - q.astype(np.float32) * s[:, None])
    assert np.all(err <= s[:, None] * (0.5 + 1e-5))  # half a step, up to fp32 rounding
    assert np.all(np.sign(q) == np.sign(np.where(np.abs(x) < s[:, None] / 2, 0, x)))
    # monotone within a row
    o = np.argsort(x[0], kind="stable")
    assert np.all(np.diff(q[0][o].astype(int)) >= 0)


def test_quantize_acts_special_rows():
    x = np.zeros((4, 32), np.float32)
    x[1, 5] = 3.0
    x[2, 7] = -0.001
    x[3, :] = np.float32(1e-45)  # subnormal absmax: 127 / a overflows to inf
    x[3, 3] = 0.0
    x[3, 4] = np.float32(-1e-45)
    q, s = orc.quantize_acts(x)
    assert np.all(q[0] == 0) and s[0] == 0.0
    assert q[1, 5] == 127 and np.count_nonzero(q[1]) == 1
    assert q[2, 7] == -127 and np.count_nonzero(q[2]) == 1
    assert np.isclose(s[1], 3.0 / 127, rtol=1e-7)
    assert q[3, 0] == 127 and q[3, 3] == 0 and q[3, 4] == -127
    with pytest.raises(ValueError):
        orc.quantize_acts(np.array([[1.0, np.nan]], np.float32))


def test_quantize_acts_bf16_matches_widened_fp32():
    t = torch.randn(8, 256, generator=torch.Generator().manual_seed(1)).bfloat16()
    bits = t.view(torch.int16).numpy().view(np.uint16)
    q1, s1 = orc.quantize_acts(bits)
    q2, s2 = orc.quantize_acts(t.float().numpy())
    np.testing.assert_array_equal(q1, q2)
    np.testing.assert_array_equal(s1, s2)


# ----------------------------------------------------------------------------- contraction


def test_contract_brute_force_all_code_vectors():
    """Every one of the 3^5 code rows against numpy's int64 matmul."""
    K = 5
    grids = np.array(np.meshgrid(*[[-1, 0, 1]] * K, indexing="ij")).reshape(K, -1).T
    codes = np.ascontiguousarray(grids.astype(np.int8))  # [243][5]
    rng = np.random.default_rng(2)
    q = rng.integers(-127, 128, size=(6, K)).astype(np.int8)
    q[0] = 127
    q[1] = -127
    acc = orc.contract_i32(q, codes)
    np.testing.assert_array_equal(acc, q.astype(np.int64) @ codes.astype(np.int64).T)


def test_contract_matches_library_matmul_and_extremes():
    rng = np.random.default_rng(9)
    q = rng.integers(-127, 128, size=(8, 1024)).astype(np.int8)
    codes = rng.integers(-1, 2, size=(40, 1024)).astype(np.int8)
    np.testing.assert_array_equal(orc.contract_i32(q, codes),
                                  q.astype(np.int64) @ codes.astype(np.int64).T)
    # extremes: |acc| = 127 * K
    K = 8192
    q = np.full((2, K), 127, np.int8)
    q[1] = -127
    codes = np.ones((2, K), np.int8)
    codes[1] = -1
    acc = orc.contract_i32(q, codes)
    np.testing.assert_array_equal(acc, [[127 * K, -127 * K], [-127 * K, 127 * K]])
    # zero codes contribute nothing ("feature filtering")
    codes = rng.integers(-1, 2, size=(4, 64)).astype(np.int8)
    q = rng.integers(-127, 128, size=(3, 64)).astype(np.int8)
    q2 = q.copy()
    q2[:, codes[0] == 0] = rng.integers(-127, 128, size=(3, int((codes[0] == 0).sum())))
    np.testing.assert_array_equal(orc.contract_i32(q, codes[:1]), orc.contract_i32(q2, codes[:1]))


# ----------------------------------------------------------------------------- rescale


def test_rescale_exact_powers_of_two():
    acc = np.array([[3, -5, 0], [1 << 20, -(1 << 20), 7]], np.int32)
    y = orc.rescale(acc, np.array([0.5, 0.25], np.float32), 0.25)
    np.testing.assert_array_equal(y, [[0.375, -0.625, 0.0], [65536.0, -65536.0, 0.4375]])


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(4)
    y = rng.standard_normal(10_000).astype(np.float32) * 100
    # exact ties: low half 0x8000 with even and odd upper halves
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x47000000 | 0x8000], np.uint32)
    y = np.concatenate([y, ties.view(np.float32)])
    ref = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(orc.to_bf16(y), ref)


def test_forward_quantization_error_bound():
    """y approximates x @ (gamma*c)^T within the activation quantization error."""
    rng = np.random.default_rng(12)
    M, N, K = 4, 32, 256
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    packed, gamma = orc.quantize_weights(W, 1e-5)
    codes = orc.unpack(packed, K)
    y = orc.forward(x, packed, gamma).astype(np.float64)
    exact = x.astype(np.float64) @ (float(gamma) * codes.astype(np.float64)).T
    s = np.abs(x).max(axis=1) / 127.0
    bound = float(gamma) * (s[:, None] / 2) * np.abs(codes).sum(axis=1)[None, :] * (1 + 1e-5)
    assert np.all(np.abs(y - exact) <= bound + 1e-5 * np.abs(exact))


# ----------------------------------------------------------------------------- shards


@pytest.mark.parametrize("split", ["rows", "cols"])
def test_abs_buckets_of_shards_add_to_the_whole(split):
    """The two halves of absmean: the bucket arrays of the parts of a matrix add up to the
    whole's, and gamma formed from the added buckets is the correctly rounded mean of the
    whole (math.fsum), also when the parts differ in scale by 10^6."""
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((64, 320)) * 0.02).astype(np.float32)
    W[:32] *= 1e-6 if split == "rows" else 1.0
    W[:, :128] *= 1e3 if split == "cols" else 1.0
    parts = [W[:32], W[32:]] if split == "rows" else [W[:, :128], W[:, 128:]]
    b = sum(orc.abs_buckets(np.ascontiguousarray(p)) for p in parts)
    np.testing.assert_array_equal(b, orc.abs_buckets(W))
    assert orc.absmean_from_buckets(b, W.size) == _fsum_gamma(W)
    assert orc.absmean_from_buckets(b, W.size) == orc.absmean(W)


def test_act_absmax_is_numpy_max():
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((7, 192)) * 3).astype(np.float32)
    x[2] = 0.0
    np.testing.assert_array_equal(orc.act_absmax(x), np.max(np.abs(x), axis=1))


def test_quantize_acts_absmax_on_k_shards_matches_whole_rows():
    """A row held in K-shards: each shard quantized with the absmax of the whole row gives
    exactly the whole row's codes and scale."""
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((5, 512)) * 2).astype(np.float32)
    x[1, 300] = 40.0  # the row's maximum lies in the second shard
    q, s = orc.quantize_acts(x)
    a = np.max(np.abs(x), axis=1)
    for k0, k1 in [(0, 192), (192, 512)]:
        qs, ss = orc.quantize_acts_absmax(np.ascontiguousarray(x[:, k0:k1]), a)
        np.testing.assert_array_equal(qs, q[:, k0:k1])
        np.testing.assert_array_equal(ss, s)


def test_quantize_acts_absmax_closed_form():
    """With a_t = 2 * 127 / 127 = 2 and x = 1 the code is rne(1 * fl(127/2)) = rne(63.5) =
    64 (ties to even); x = a_t gives 127; x above a_t clips to 127."""
    x = np.array([[1.0, 2.0, 3.0, -5.0, 0.0, 0.5, -1.0, 1.5]], np.float32)
    x = np.tile(x, (1, 8))
    q, s = orc.quantize_acts_absmax(x, np.array([2.0], np.float32))
    np.testing.assert_array_equal(q[0, :8], [64, 127, 127, -127, 0, 32, -64, 95])
    assert s[0] == np.float32(2.0) / np.float32(127.0)


# ----------------------------------------------------------------------------- base 3


def test_base3_every_trit_group_encodes_to_its_fixed_point_byte():
    """All 3^5 groups of five trits: the byte is ceil(256 v / 243) of the group's base-3
    value v (u_0 leading, u = c + 1), computed here with Python integers; the 243 bytes
    are distinct and rise with v (so the encoding is injective), and unpacking restores
    every group."""
    import itertools
    groups = list(itertools.product((-1, 0, 1), repeat=5))
    codes = np.zeros((len(groups), 80), np.int8)
    for r, g in enumerate(groups):
        for p, c in enumerate(g):
            codes[r, 16 * p] = c  # byte 0 of the chunk holds trits 0, 16, 32, 48, 64
    packed = orc.pack_base3(codes)
    assert packed.shape == (243, 16)
    vs = [sum((c + 1) * 3 ** (4 - p) for p, c in enumerate(g)) for g in groups]
    want = [-(-256 * v // 243) for v in vs]
    np.testing.assert_array_equal(packed[:, 0], want)
    order = np.argsort(vs)
    assert np.all(np.diff(packed[order, 0].astype(int)) > 0)
    np.testing.assert_array_equal(orc.unpack_base3(packed, 80), codes)


def test_base3_closed_form_bytes_and_positions():
    """All +1 -> 255, all 0 -> 128, all -1 -> 0 (v = 242, 121, 0); one +1 among zeros at
    digit p gives v = 121 + 3^(4-p) = 202, 148, 130, 124, 122: bytes ceil(256 v / 243) =
    213, 156, 137, 131, 129 for p = 0..4 (e.g. 256 * 148 / 243 = 155.9), in byte
    i of chunk j for trit k = 80 j + 16 p + i."""
    K = 160
    for c, b in ((1, 255), (0, 128), (-1, 0)):
        np.testing.assert_array_equal(orc.pack_base3(np.full((1, K), c, np.int8)), b)
    for p, b in enumerate((213, 156, 137, 131, 129)):
        for j, i in ((0, 0), (1, 7), (1, 15)):
            codes = np.zeros((1, K), np.int8)
            codes[0, 80 * j + 16 * p + i] = 1
            packed = orc.pack_base3(codes)
            expect = np.full(32, 128, np.uint8)
            expect[16 * j + i] = b
            np.testing.assert_array_equal(packed[0], expect)


def test_base3_ragged_rows_pad_with_zero_trits():
    """K not a multiple of 80: the last chunk's missing trits are zeros (u = 1), the row
    size is ceil(K / 80) * 16 bytes (1648 for K = 8192, 0.805 of the 2-bit 2048), and
    non-zero padding is rejected on unpacking."""
    assert orc.base3_row_bytes(8192) == 1648 and orc.base3_row_bytes(80) == 16
    assert orc.base3_row_bytes(64) == 16 and orc.base3_row_bytes(28672) == 5744
    rng = np.random.default_rng(21)
    codes = rng.integers(-1, 2, size=(9, 192)).astype(np.int8)
    packed = orc.pack_base3(codes)
    np.testing.assert_array_equal(orc.unpack_base3(packed, 192), codes)
    bad = packed.copy()
    bad[0, 16 * 2 + 0] = 255  # chunk 2 byte 0 holds trits 160, 176 (real) and 192.. (padding)
    with pytest.raises(ValueError):
        orc.unpack_base3(bad, 192)


# ----------------------------------------------------------------------------- backward


def _bilinear_loss(G, Xt, Wt):
    """L = sum_{t,n} G[t,n] (Xt Wt^T)[t,n] by explicit loops in float64 (tiny sizes)."""
    M, K = Xt.shape
    N = Wt.shape[0]
    total = 0.0
    for t in range(M):
        for n in range(N):
            total += float(G[t, n]) * sum(float(Xt[t, k]) * float(Wt[n, k]) for k in range(K))
    return total


def _bf16_bits_to_f64(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_ste_gradients_are_the_bilinear_derivatives():
    """The straight-through gradients are the partial derivatives of the bilinear
    surrogate L = sum G * (X~ W~^T) in X~ and W~: unit perturbations of single entries, by
    brute force, change L by exactly grad_x[t,k] (as X~ moves) and grad_w[n,k] (as W~
    moves); the loss is linear in each, so the difference quotient is exact."""
    rng = np.random.default_rng(31)
    M, N, K = 3, 4, 16
    G = (rng.standard_normal((M, N))).astype(np.float32)
    codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    gamma = np.float32(0.0625)
    q = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    s = np.float32([0.5, 0.25, 0.125])  # q * s exact in bf16? (|q| <= 127: 7 bits) yes
    xt_bits = orc.dequant_acts_bf16(q, s)
    Xt = _bf16_bits_to_f64(xt_bits)
    Wt = codes.astype(np.float64) * float(gamma)
    gx = orc.ste_grad_x(G, codes, gamma)
    gw = orc.ste_grad_w(G, xt_bits)
    base = _bilinear_loss(G, Xt, Wt)
    for (t, k) in [(0, 0), (2, 15), (1, 7)]:
        X2 = Xt.copy()
        X2[t, k] += 1.0
        assert _bilinear_loss(G, X2, Wt) - base == pytest.approx(gx[t, k], rel=1e-12, abs=1e-12)
    for (n, k) in [(0, 0), (3, 15), (2, 9)]:
        W2 = Wt.copy()
        W2[n, k] += 1.0
        assert _bilinear_loss(G, Xt, W2) - base == pytest.approx(gw[n, k], rel=1e-12, abs=1e-12)


def test_ste_gradients_special_cases_and_adjoint_identity():
    """One-hot G picks a weight row (grad_x = gamma c[n0]) and an activation row (grad_w
    row n0 = X~[t0]); and both gradients pair with the forward: sum grad_x * X~ =
    sum G * y = sum grad_w * W~ (y = X~ W~^T in float64)."""
    rng = np.random.default_rng(32)
    M, N, K = 5, 7, 64
    codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    gamma = np.float32(0.013)
    x = rng.standard_normal((M, K)).astype(np.float32)
    q, s = orc.quantize_acts(x)
    xt_bits = orc.dequant_acts_bf16(q, s)
    Xt = _bf16_bits_to_f64(xt_bits)
    G = np.zeros((M, N), np.float32)
    G[2, 5] = 1.0
    np.testing.assert_array_equal(orc.ste_grad_x(G, codes, gamma)[2],
                                  float(gamma) * codes[5].astype(np.float64))
    np.testing.assert_array_equal(orc.ste_grad_w(G, xt_bits)[5], Xt[2])
    G = rng.standard_normal((M, N)).astype(np.float32)
    gx = orc.ste_grad_x(G, codes, gamma)
    gw = orc.ste_grad_w(G, xt_bits)
    Wt = codes.astype(np.float64) * float(gamma)
    y = Xt @ Wt.T
    a = float(np.sum(gx * Xt))
    b = float(np.sum(G.astype(np.float64) * y))
    c = float(np.sum(gw * Wt))
    assert a == pytest.approx(b, rel=1e-12) and c == pytest.approx(b, rel=1e-12)
    # bf16 G is read as its exact value
    Gb = torch.from_numpy(G).bfloat16()
    gb = orc.ste_grad_x(Gb.view(torch.int16).numpy().view(np.uint16), codes, gamma)
    np.testing.assert_allclose(gb, orc.ste_grad_x(Gb.float().numpy(), codes, gamma), rtol=0, atol=0)


def test_dequant_acts_bf16_rounds_half_to_even():
    """X~ = bf16(fl32(q * s)) equals torch's own fp32 -> bf16 conversion (a library
    routine, round half to even) for every q and three scales, the first with low bits
    (2^-8 + 2^-9) that the 8-bit bf16 significand must round away."""
    q = np.arange(-127, 128, dtype=np.int8).reshape(1, -1)[:, :240]
    for s in (np.float32(1.0 + 2**-8 + 2**-9), np.float32(0.0123), np.float32(3.0)):
        got = orc.dequant_acts_bf16(q, np.array([s], np.float32))
        want = torch.from_numpy(q.astype(np.float32) * s).bfloat16()
        np.testing.assert_array_equal(got, want.view(torch.int16).numpy().view(np.uint16))
