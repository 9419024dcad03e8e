"""ctypes front end of the BitLinear oracle (``bitlinear_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this module; the library never does.

Each function mirrors one step of the BitLinear forward of BitNet b1.58 ("The Era of
1-bit LLMs", dmarx anthology record LIT-380, Key takeaways bullets 1 and 4): absmean
ternary weights, per-token absmax int8 activations, the integer contraction and the
rescale. Inputs are numpy arrays (fp32, or bf16 carried as uint16 bit patterns); the
work happens in the single-threaded C++ code.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitlinear_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

F32 = 0
BF16 = 1

GXX_FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (plain g++, no GPU)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["g++", *GXX_FLAGS, _SRC, "-o", _LIB])
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        p, i64, f32, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int
        _lib.oracle_absmean.argtypes = [p, i32, i64, p]
        _lib.oracle_absmean.restype = i32
        _lib.oracle_ternarize.argtypes = [p, i32, i64, f32, f32, p]
        _lib.oracle_ternarize.restype = i32
        _lib.oracle_pack.argtypes = [p, i64, i64, p]
        _lib.oracle_pack.restype = None
        _lib.oracle_unpack.argtypes = [p, i64, i64, p]
        _lib.oracle_unpack.restype = i32
        _lib.oracle_quantize_acts.argtypes = [p, i32, i64, i64, p, p]
        _lib.oracle_quantize_acts.restype = i32
        _lib.oracle_base3_row_bytes.argtypes = [i64]
        _lib.oracle_base3_row_bytes.restype = i64
        _lib.oracle_pack_base3.argtypes = [p, i64, i64, p]
        _lib.oracle_pack_base3.restype = None
        _lib.oracle_unpack_base3.argtypes = [p, i64, i64, p]
        _lib.oracle_unpack_base3.restype = i32
        _lib.oracle_dequant_acts_bf16.argtypes = [p, p, i64, i64, p]
        _lib.oracle_dequant_acts_bf16.restype = None
        _lib.oracle_ste_grad_x.argtypes = [p, i32, p, f32, i64, i64, i64, p]
        _lib.oracle_ste_grad_x.restype = None
        _lib.oracle_ste_grad_w.argtypes = [p, i32, p, i64, i64, i64, p]
        _lib.oracle_ste_grad_w.restype = None
        _lib.oracle_abs_buckets.argtypes = [p, i32, i64, p]
        _lib.oracle_abs_buckets.restype = i32
        _lib.oracle_absmean_from_buckets.argtypes = [p, i64, p]
        _lib.oracle_absmean_from_buckets.restype = None
        _lib.oracle_act_absmax.argtypes = [p, i32, i64, i64, p]
        _lib.oracle_act_absmax.restype = i32
        _lib.oracle_quantize_acts_absmax.argtypes = [p, i32, i64, i64, p, p, p]
        _lib.oracle_quantize_acts_absmax.restype = i32
        _lib.oracle_contract_i32.argtypes = [p, p, i64, i64, i64, p]
        _lib.oracle_contract_i32.restype = None
        _lib.oracle_rescale.argtypes = [p, p, f32, i64, i64, p]
        _lib.oracle_rescale.restype = None
        _lib.oracle_to_bf16.argtypes = [p, i64, p]
        _lib.oracle_to_bf16.restype = None
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _as_input(a: np.ndarray) -> tuple[np.ndarray, int]:
    """fp32 arrays pass as fp32; uint16 arrays are bf16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"oracle inputs are float32 or bf16-as-uint16, got {a.dtype}")


def absmean(W: np.ndarray) -> np.float32:
    """gamma = mean|W|: exact sum of |w|, rounded once to double, / n, rounded to fp32."""
    W, dt = _as_input(W)
    out = np.zeros(1, np.float32)
    rc = lib().oracle_absmean(_ptr(W), dt, W.size, _ptr(out))
    if rc != 0:
        raise ValueError("non-finite weight")
    return out[0]


def base3_row_bytes(K: int) -> int:
    """Bytes per row of the base-3 (5 trits per byte) format: ceil(K / 80) * 16."""
    return int(lib().oracle_base3_row_bytes(int(K)))


def pack_base3(codes: np.ndarray) -> np.ndarray:
    """int8 codes [N][K] -> base-3 bytes [N][ceil(K/80)*16] (5 trits per byte)."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    N, K = codes.shape
    out = np.zeros((N, base3_row_bytes(K)), np.uint8)
    lib().oracle_pack_base3(_ptr(codes), N, K, _ptr(out))
    return out


def unpack_base3(packed3: np.ndarray, K: int) -> np.ndarray:
    packed3 = np.ascontiguousarray(packed3, dtype=np.uint8)
    N = packed3.shape[0]
    assert packed3.shape[1] == base3_row_bytes(K)
    codes = np.zeros((N, K), np.int8)
    if lib().oracle_unpack_base3(_ptr(packed3), N, K, codes.ctypes.data) != 0:
        raise ValueError("bytes that no trit group encodes")
    return codes


def dequant_acts_bf16(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """X~ = bf16(fl32(q * s_t)) as bf16 bit patterns (uint16 [M][K])."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    M, K = q.shape
    out = np.zeros((M, K), np.uint16)
    lib().oracle_dequant_acts_bf16(_ptr(q), _ptr(scale), M, K, _ptr(out))
    return out


def ste_grad_x(G: np.ndarray, codes: np.ndarray, gamma: float) -> np.ndarray:
    """Straight-through dL/dx = gamma * G C, float64 [M][K] (G fp32 or bf16 bits)."""
    G, dt = _as_input(G)
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    M, N = G.shape
    K = codes.shape[1]
    assert codes.shape[0] == N
    out = np.zeros((M, K), np.float64)
    lib().oracle_ste_grad_x(_ptr(G), dt, _ptr(codes), float(gamma), M, N, K, _ptr(out))
    return out


def ste_grad_w(G: np.ndarray, xt_bf16: np.ndarray) -> np.ndarray:
    """Straight-through dL/dW = G^T X~, float64 [N][K] (X~ as bf16 bits [M][K])."""
    G, dt = _as_input(G)
    xt = np.ascontiguousarray(xt_bf16, dtype=np.uint16)
    M, N = G.shape
    K = xt.shape[1]
    assert xt.shape[0] == M
    out = np.zeros((N, K), np.float64)
    lib().oracle_ste_grad_w(_ptr(G), dt, _ptr(xt), M, N, K, _ptr(out))
    return out


def abs_buckets(W: np.ndarray) -> np.ndarray:
    """The 256 exponent buckets (uint64) of the exact sum of |W|; the buckets of the parts
    of a matrix add up (as integers) to those of the whole."""
    W, dt = _as_input(W)
    out = np.zeros(256, np.uint64)
    if lib().oracle_abs_buckets(_ptr(W), dt, W.size, _ptr(out)) != 0:
        raise ValueError("non-finite weight")
    return out


def absmean_from_buckets(buckets: np.ndarray, n: int) -> np.float32:
    """gamma from the buckets of n values in all (the second half of absmean)."""
    b = np.ascontiguousarray(buckets, dtype=np.uint64)
    assert b.shape == (256,)
    out = np.zeros(1, np.float32)
    lib().oracle_absmean_from_buckets(_ptr(b), int(n), _ptr(out))
    return out[0]


def act_absmax(x: np.ndarray) -> np.ndarray:
    """a_t = max_k |x[t,k]| (fp32 [M])."""
    x, dt = _as_input(x)
    M, K = x.shape
    a = np.zeros(M, np.float32)
    if lib().oracle_act_absmax(_ptr(x), dt, M, K, _ptr(a)) != 0:
        raise ValueError("non-finite activation")
    return a


def quantize_acts_absmax(x: np.ndarray, amax: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Per-token int8 quantization with a_t given (the absmax of the whole rows when x is a
    K-shard of them)."""
    x, dt = _as_input(x)
    M, K = x.shape
    a = np.ascontiguousarray(amax, dtype=np.float32)
    q = np.zeros((M, K), np.int8)
    s = np.zeros(M, np.float32)
    if lib().oracle_quantize_acts_absmax(_ptr(x), dt, M, K, _ptr(a), _ptr(q), _ptr(s)) != 0:
        raise RuntimeError("FPU rounding mode is not round-to-nearest")
    return q, s


def ternarize(W: np.ndarray, gamma: float, eps: float) -> np.ndarray:
    """c = RoundClip(w / (gamma + eps), -1, 1), fp32 quotient, ties to even."""
    W, dt = _as_input(W)
    codes = np.zeros(W.shape, np.int8)
    rc = lib().oracle_ternarize(_ptr(W), dt, W.size, float(gamma), float(eps), _ptr(codes))
    if rc != 0:
        raise RuntimeError("FPU rounding mode is not round-to-nearest")
    return codes


def pack(codes: np.ndarray) -> np.ndarray:
    """2-bit packing of an int8 [N][K] code array (K % 16 == 0) -> uint8 [N][K/4]."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    N, K = codes.shape
    assert K % 16 == 0
    out = np.zeros((N, K // 4), np.uint8)
    lib().oracle_pack(_ptr(codes), N, K, _ptr(out))
    return out


def unpack(packed: np.ndarray, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    assert packed.shape[1] * 4 == K
    codes = np.zeros((N, K), np.int8)
    if lib().oracle_unpack(_ptr(packed), N, K, _ptr(codes)) != 0:
        raise ValueError("packed buffer holds the unused 2-bit code 3")
    return codes


def quantize_weights(W: np.ndarray, eps: float = 1e-5) -> tuple[np.ndarray, np.float32]:
    """absmean -> ternarize -> pack. Returns (packed uint8 [N][K/4], gamma)."""
    gamma = absmean(W)
    return pack(ternarize(W, gamma, eps)), gamma


def quantize_acts(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Per-token absmax int8: returns (q int8 [M][K], scale fp32 [M] = absmax/127)."""
    x, dt = _as_input(x)
    M, K = x.shape
    q = np.zeros((M, K), np.int8)
    s = np.zeros(M, np.float32)
    rc = lib().oracle_quantize_acts(_ptr(x), dt, M, K, _ptr(q), _ptr(s))
    if rc == 1:
        raise ValueError("non-finite activation")
    if rc != 0:
        raise RuntimeError("FPU rounding mode is not round-to-nearest")
    return q, s


def contract_i32(q: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """acc[t,n] = sum_{c=+1} q[t,k] - sum_{c=-1} q[t,k] (int32)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    M, K = q.shape
    N = codes.shape[0]
    assert codes.shape[1] == K
    acc = np.zeros((M, N), np.int32)
    lib().oracle_contract_i32(_ptr(q), _ptr(codes), M, N, K, _ptr(acc))
    return acc


def rescale(acc: np.ndarray, scale: np.ndarray, gamma: float) -> np.ndarray:
    """y = float(acc) * (scale_t * gamma), fp32."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    M, N = acc.shape
    y = np.zeros((M, N), np.float32)
    lib().oracle_rescale(_ptr(acc), _ptr(scale), float(gamma), M, N, _ptr(y))
    return y


def to_bf16(y: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round half to even."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    out = np.zeros(y.shape, np.uint16)
    lib().oracle_to_bf16(_ptr(y), y.size, _ptr(out))
    return out


def forward(x: np.ndarray, packed: np.ndarray, gamma: float, out: str = "f32") -> np.ndarray:
    """Whole BitLinear forward from packed weights: y [M][N] fp32 (or bf16 bits)."""
    K = x.shape[1]
    q, s = quantize_acts(x)
    acc = contract_i32(q, unpack(packed, K))
    y = rescale(acc, s, gamma)
    return to_bf16(y) if out == "bf16" else y
