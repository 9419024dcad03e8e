"""Host-side kernel choice of bitlinear_forward (pure host code, runs without a GPU).

Pins the measured rules: the CUDA-core GEMV for one or two tokens, or up to four when the
packed weights are at most 2 MB; the skinny tensor-core kernel up to 256 tokens, splitting K
into as many parts as the CTA slots (two per SM for up to 64 tokens, one above) hold in one
wave, while each split keeps at least 8 K blocks and the int32 sums the splits exchange stay
within a quarter of the packed weight bytes; the prefill GEMM above 256 tokens."""
import ctypes

import pytest

import ternary_weight_linear_03_b200 as bl

PLANS = [
    # (M, N, K) -> (path, K splits) on a 148-SM B200
    ((1, 28672, 8192), ("gemv", 1)),
    ((2, 5000, 28672), ("gemv", 1)),          # two tokens: always the GEMV
    ((3, 28672, 8192), ("skinny", 1)),        # three tokens, 58.7 MB of packed weights
    ((4, 4096, 1536), ("gemv", 1)),           # four tokens, 1.57 MB of packed weights
    ((4, 28672, 8192), ("skinny", 1)),
    ((16, 4096, 1536), ("skinny", 1)),        # 12 K blocks: too few to split
    ((16, 8640, 3200), ("skinny", 3)),
    ((64, 8640, 3200), ("skinny", 1)),        # the sums of a split would outweigh W / 4
    ((16, 3200, 8640), ("skinny", 6)),
    ((16, 8192, 28672), ("skinny", 4)),       # 64 tiles x 4 splits = 256 CTAs <= 296 slots
    ((176, 8192, 28672), ("skinny", 2)),      # one CTA per SM above 64 tokens: 128 CTAs
    ((16, 28672, 8192), ("skinny", 1)),       # 224 weight tiles already fill the GPU
    ((256, 1000, 3200), ("skinny", 1)),
    ((257, 1000, 3200), ("prefill", 1)),
    ((4096, 28672, 8192), ("prefill", 1)),
]


@pytest.mark.parametrize("shape,plan", PLANS)
def test_forward_kernel_choice(shape, plan):
    assert bl.debug_plan(*shape, sms=148) == plan


def test_split_rule_invariants():
    for M in (5, 8, 16, 32, 64, 128, 176, 256):
        for N in (300, 1024, 3200, 4096, 8192, 8640, 28672):
            for K in (640, 1536, 3200, 8192, 8640, 28672):
                path, splits = bl.debug_plan(M, N, K, sms=148)
                if path != "skinny":
                    continue
                kb = (K + 127) // 128
                if splits > 1:
                    assert kb // splits >= 4  # whole 4-block super-tiles, no empty split
                    assert splits <= kb // 8
                    assert M * N * 4 * splits * 4 <= N * K // 4 + M * N * 4 * 4
                    slots = (2 if (M + 15) // 16 * 16 <= 64 else 1) * 148
                    assert (N + 127) // 128 * splits <= slots  # one wave of CTAs


def test_argument_errors():
    lib = bl.load_library()
    p, s = ctypes.c_int(), ctypes.c_int()
    assert lib.bitlinear_debug_plan(16, 4096, 1536, 148, None, ctypes.byref(s)) == 1
    assert lib.bitlinear_debug_plan(16, 4096, 1536, 0, ctypes.byref(p), ctypes.byref(s)) == 1
    assert lib.bitlinear_debug_plan(16, 4096, 100, 148, ctypes.byref(p), ctypes.byref(s)) == 2
