"""bitlinear_forward_noalloc: the forward for callers that cannot allocate device memory
(for instance code running under another runtime's memory planner, or latency-critical
paths that avoid cudaMalloc because it can synchronize the device). Its scratch is a fixed
16 MiB array inside the library instead of a caller workspace.

Checked through the C ABI against bitlinear_forward on two calls in a row, with the
same bar as the other parity tests (identical bits; fp32 within 1e-6 relative). This
file is collected last on purpose."""

import ctypes

import numpy as np
import pytest
import torch

import ternary_weight_linear_03_b200 as bl
from ternary_weight_linear_03_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bl.load_library()


def _call_noalloc(lib, x, packed, gamma, y, M, N, K):
    return lib.bitlinear_forward_noalloc(
        x.data_ptr(), bl.BL_BF16 if x.dtype == torch.bfloat16 else bl.BL_F32, packed.data_ptr(),
        gamma.data_ptr(), y.data_ptr(), bl.BL_F32 if y.dtype == torch.float32 else bl.BL_BF16,
        M, N, K, torch.cuda.current_stream().cuda_stream)


def _call_forward(lib, x, packed, gamma, y, ws, M, N, K):
    return lib.bitlinear_forward(
        x.data_ptr(), bl.BL_BF16 if x.dtype == torch.bfloat16 else bl.BL_F32, packed.data_ptr(),
        gamma.data_ptr(), y.data_ptr(), bl.BL_F32 if y.dtype == torch.float32 else bl.BL_BF16,
        M, N, K, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    lib = bl.load_library()
    cases = [(200, 1000, 1536, torch.bfloat16, torch.float32),   # skinny tensor-core kernel
             (64, 4096, 3200, torch.float32, torch.bfloat16),    # second call, other shape
             (16, 8640, 3200, torch.bfloat16, torch.bfloat16),   # bitlinear_forward splits K
             (300, 520, 1536, torch.bfloat16, torch.float32)]    # prefill GEMM
    for i, (M, N, K, xdt, ydt) in enumerate(cases):
        W = syn.weights(N, K, 0.02, seed=300 + i).cuda()
        x = syn.activations(M, K, seed=400 + i, dtype=xdt, outlier_frac=0.01).cuda()
        packed, gamma = bl.quantize_weights(W)
        ws = bl.workspace(M, N, K)
        y_ref = torch.empty((M, N), dtype=ydt, device="cuda")
        y_new = torch.full((M, N), float("nan"), dtype=ydt, device="cuda")
        assert _call_forward(lib, x, packed, gamma, y_ref, ws, M, N, K) == 0
        assert _call_noalloc(lib, x, packed, gamma, y_new, M, N, K) == 0
        torch.cuda.synchronize()
        assert bl.get_device_status() == 0
        a = y_new.float().cpu().numpy().astype(np.float64)
        b = y_ref.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(a - b) <= 1e-6 * np.abs(b))
        assert torch.equal(y_new, y_ref)


def test_noalloc_small_m_and_capacity_limit():
    lib = bl.load_library()
    M, N, K = 3, 512, 1536  # CUDA-core path: needs no scratch at all
    W = syn.weights(N, K, 0.02, seed=9).cuda()
    x = syn.activations(M, K, seed=10).cuda()
    packed, gamma = bl.quantize_weights(W)
    y = bl.forward_noalloc(x, packed, gamma, out_dtype=torch.float32)
    assert torch.equal(y, bl.forward(x, packed, gamma, out_dtype=torch.float32))
    # beyond the 16 MiB scratch: rejected before anything is queued
    big_m, big_k = 4096, 8192
    rc = lib.bitlinear_forward_noalloc(ctypes.c_void_p(0x10000), 1, ctypes.c_void_p(0x10000),
                                       ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), 1,
                                       big_m, 256, big_k, None)
    assert rc == 7  # BL_ERR_WORKSPACE
