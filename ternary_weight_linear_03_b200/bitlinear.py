"""Thin Python binding of libbitlinear.so (C ABI in include/bitlinear.h).

Argument marshalling only: every step of the BitLinear forward runs in the library's
sm_100a kernels. PyTorch supplies device memory and the current stream. There is no
fallback: if the shared library is missing or no CUDA device is present, the calls raise.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbitlinear.so")

BL_F32, BL_BF16, BL_I32 = 0, 1, 2
STATUS = {
    0: "BL_OK", 1: "BL_ERR_INVALID_ARG", 2: "BL_ERR_UNSUPPORTED_SHAPE", 3: "BL_ERR_MISALIGNED",
    4: "BL_ERR_CUDA", 5: "BL_ERR_TIMEOUT", 6: "BL_ERR_NONFINITE", 7: "BL_ERR_WORKSPACE",
}

# Every symbol declared in include/bitlinear.h.
EXPORTS = (
    "bitlinear_workspace_size", "bitlinear_quantize_weights", "bitlinear_quantize_acts",
    "bitlinear_weight_abssum", "bitlinear_quantize_weights_from_abssum", "bitlinear_act_absmax",
    "bitlinear_quantize_acts_absmax", "bitlinear_rescale", "bitlinear_chain_workspace_size",
    "bitlinear_chain_forward", "bitlinear_base3_row_bytes", "bitlinear_pack_base3",
    "bitlinear_forward_base3", "bitlinear_pack_transpose", "bitlinear_backward_workspace_size",
    "bitlinear_backward",
    "bitlinear_forward", "bitlinear_forward_noalloc", "bitlinear_contract_i32",
    "bitlinear_get_device_status",
    "bitlinear_debug_timeout_probe", "bitlinear_debug_plan", "bitlinear_status_string",
)


class Layer(ctypes.Structure):
    """bl_layer of include/bitlinear.h: one layer of a chain."""
    _fields_ = [("packed", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("N", ctypes.c_int),
                ("K", ctypes.c_int), ("src", ctypes.c_int), ("out", ctypes.c_void_p)]


class BitLinearError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def load_library() -> ctypes.CDLL:
    """Loads the in-tree libbitlinear.so (built by ternary_weight_linear_03_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m ternary_weight_linear_03_b200.build`"
            " (or __graft_entry__.build()); there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    p, i, f, sz, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64
    lib.bitlinear_workspace_size.argtypes = [i, i, i]
    lib.bitlinear_workspace_size.restype = sz
    lib.bitlinear_quantize_weights.argtypes = [p, i, i, i, f, p, p, p, sz, p]
    lib.bitlinear_quantize_weights.restype = i
    lib.bitlinear_quantize_acts.argtypes = [p, i, i, i, p, p, p]
    lib.bitlinear_quantize_acts.restype = i
    i64 = ctypes.c_longlong
    lib.bitlinear_weight_abssum.argtypes = [p, i, i, i, p, p, sz, p]
    lib.bitlinear_weight_abssum.restype = i
    lib.bitlinear_quantize_weights_from_abssum.argtypes = [p, i, i, i, i64, p, f, p, p, p]
    lib.bitlinear_quantize_weights_from_abssum.restype = i
    lib.bitlinear_act_absmax.argtypes = [p, i, i, i, p, p]
    lib.bitlinear_act_absmax.restype = i
    lib.bitlinear_quantize_acts_absmax.argtypes = [p, i, i, i, p, p, p, p]
    lib.bitlinear_quantize_acts_absmax.restype = i
    lib.bitlinear_rescale.argtypes = [p, p, p, p, i, i, i, p]
    lib.bitlinear_rescale.restype = i
    lib.bitlinear_chain_workspace_size.argtypes = [i, ctypes.POINTER(Layer), i]
    lib.bitlinear_chain_workspace_size.restype = sz
    lib.bitlinear_chain_forward.argtypes = [p, i, i, ctypes.POINTER(Layer), i, p, i, p, sz, p]
    lib.bitlinear_chain_forward.restype = i
    lib.bitlinear_base3_row_bytes.argtypes = [i]
    lib.bitlinear_base3_row_bytes.restype = sz
    lib.bitlinear_pack_base3.argtypes = [p, i, i, p, p]
    lib.bitlinear_pack_base3.restype = i
    lib.bitlinear_forward_base3.argtypes = [p, i, p, p, p, i, i, i, i, p]
    lib.bitlinear_forward_base3.restype = i
    lib.bitlinear_pack_transpose.argtypes = [p, i, i, p, p]
    lib.bitlinear_pack_transpose.restype = i
    lib.bitlinear_backward_workspace_size.argtypes = [i, i, i]
    lib.bitlinear_backward_workspace_size.restype = sz
    lib.bitlinear_backward.argtypes = [p, i, p, p, p, p, p, i, i, i, p, sz, p]
    lib.bitlinear_backward.restype = i
    lib.bitlinear_forward.argtypes = [p, i, p, p, p, i, i, i, i, p, sz, p]
    lib.bitlinear_forward.restype = i
    lib.bitlinear_forward_noalloc.argtypes = [p, i, p, p, p, i, i, i, i, p]
    lib.bitlinear_forward_noalloc.restype = i
    lib.bitlinear_contract_i32.argtypes = [p, p, p, i, i, i, p, sz, p]
    lib.bitlinear_contract_i32.restype = i
    lib.bitlinear_get_device_status.argtypes = [p]
    lib.bitlinear_get_device_status.restype = i
    lib.bitlinear_debug_timeout_probe.argtypes = [u64, p]
    lib.bitlinear_debug_timeout_probe.restype = i
    lib.bitlinear_debug_plan.argtypes = [i, i, i, i, p, p]
    lib.bitlinear_debug_plan.restype = i
    lib.bitlinear_status_string.argtypes = [i]
    lib.bitlinear_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(status: int, what: str) -> None:
    if status != 0:
        raise BitLinearError(status, what)


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return BL_F32
    if t.dtype == torch.bfloat16:
        return BL_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (fp32 or bf16)")


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def workspace_size(M: int, N: int, K: int) -> int:
    return int(load_library().bitlinear_workspace_size(M, N, K))


def workspace(M: int, N: int, K: int, device="cuda") -> torch.Tensor:
    """A caller-owned device workspace large enough for (M, N, K)."""
    n = workspace_size(M, N, K)
    if n == 0:
        raise BitLinearError(2, "workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def quantize_weights(W: torch.Tensor, eps: float = 1e-5, packed: torch.Tensor | None = None,
                     gamma: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                     stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Absmean ternary quantization of W [N][K] -> (packed uint8 [N][K/4], gamma fp32 [1])."""
    lib = load_library()
    N, K = W.shape
    if packed is None:
        packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    if ws is None:
        ws = workspace(1, N, K, W.device)
    _check(lib.bitlinear_quantize_weights(
        _dev(W, "W"), _dtype_code(W), N, K, float(eps), _dev(packed, "packed"),
        _dev(gamma, "gamma"), _dev(ws, "ws"), ws.numel(), _stream(stream)),
        "bitlinear_quantize_weights")
    return packed, gamma


def quantize_acts(x: torch.Tensor, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Per-token absmax int8: x [M][K] -> (xq int8 [M][K], scale fp32 [M])."""
    lib = load_library()
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    scale = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib.bitlinear_quantize_acts(_dev(x, "x"), _dtype_code(x), M, K, _dev(xq, "xq"),
                                       _dev(scale, "scale"), _stream(stream)),
           "bitlinear_quantize_acts")
    return xq, scale


ABSSUM_WORDS = 14


def weight_abssum(W: torch.Tensor, sums: torch.Tensor | None = None,
                  ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Exact sum of |w| over W (a shard of a matrix) as ABSSUM_WORDS int64 words (uint64
    bit patterns): the words of several shards add up exactly to those of their union."""
    lib = load_library()
    N, K = W.shape
    if sums is None:
        sums = torch.empty(ABSSUM_WORDS, dtype=torch.int64, device=W.device)
    if ws is None:
        ws = workspace(1, N, K, W.device)
    _check(lib.bitlinear_weight_abssum(_dev(W, "W"), _dtype_code(W), N, K, _dev(sums, "sums"),
                                       _dev(ws, "ws"), ws.numel(), _stream(stream)),
           "bitlinear_weight_abssum")
    return sums


def quantize_weights_from_abssum(W: torch.Tensor, n_total: int, sums: torch.Tensor,
                                 eps: float = 1e-5, packed: torch.Tensor | None = None,
                                 gamma: torch.Tensor | None = None,
                                 stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """gamma from the added words of every shard (over n_total weights), then this shard's
    packed codes."""
    lib = load_library()
    N, K = W.shape
    if packed is None:
        packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    _check(lib.bitlinear_quantize_weights_from_abssum(
        _dev(W, "W"), _dtype_code(W), N, K, int(n_total), _dev(sums, "sums"), float(eps),
        _dev(packed, "packed"), _dev(gamma, "gamma"), _stream(stream)),
        "bitlinear_quantize_weights_from_abssum")
    return packed, gamma


def act_absmax(x: torch.Tensor, amax: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Per-token max |x| (fp32 [M])."""
    lib = load_library()
    M, K = x.shape
    if amax is None:
        amax = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib.bitlinear_act_absmax(_dev(x, "x"), _dtype_code(x), M, K, _dev(amax, "amax"),
                                    _stream(stream)), "bitlinear_act_absmax")
    return amax


def quantize_acts_absmax(x: torch.Tensor, amax: torch.Tensor,
                         stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Per-token int8 quantization with the absmax given (of the whole rows)."""
    lib = load_library()
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    scale = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib.bitlinear_quantize_acts_absmax(_dev(x, "x"), _dtype_code(x), M, K,
                                              _dev(amax, "amax"), _dev(xq, "xq"),
                                              _dev(scale, "scale"), _stream(stream)),
           "bitlinear_quantize_acts_absmax")
    return xq, scale


def rescale(acc: torch.Tensor, scale: torch.Tensor, gamma: torch.Tensor,
            out_dtype: torch.dtype = torch.bfloat16, y: torch.Tensor | None = None,
            stream=None) -> torch.Tensor:
    """y = float(acc) * (scale_t * gamma) for an int32 product [M][N]."""
    lib = load_library()
    M, N = acc.shape
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=acc.device)
    _check(lib.bitlinear_rescale(_dev(acc, "acc"), _dev(scale, "scale"), _dev(gamma, "gamma"),
                                 _dev(y, "y"), _dtype_code(y), M, N, _stream(stream)),
           "bitlinear_rescale")
    return y


def chain_layers(layers) -> ctypes.Array:
    """ctypes array of bl_layer from (packed, gamma, src[, out]) tuples (device tensors;
    out a bf16 [M][N] tensor or None)."""
    arr = (Layer * len(layers))()
    for i, ly in enumerate(layers):
        packed, gamma, src = ly[0], ly[1], ly[2]
        out = ly[3] if len(ly) > 3 else None
        arr[i] = Layer(_dev(packed, "packed"), _dev(gamma, "gamma"), packed.shape[0],
                       packed.shape[1] * 4, int(src), _dev(out, "out") if out is not None else None)
    return arr


def chain_workspace(M: int, layers, device="cuda") -> torch.Tensor:
    arr = chain_layers(layers)
    n = int(load_library().bitlinear_chain_workspace_size(M, arr, len(layers)))
    if n == 0:
        raise BitLinearError(1, "bitlinear_chain_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def chain_forward(x: torch.Tensor, layers, out_dtype: torch.dtype = torch.bfloat16,
                  y: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    """A chain of BitLinear layers (bitlinear_chain_forward): layers are (packed, gamma,
    src[, out]) with src = -1 for x or the index of the layer whose output is the input."""
    lib = load_library()
    M = x.shape[0]
    arr = chain_layers(layers)
    if y is None:
        y = torch.empty((M, layers[-1][0].shape[0]), dtype=out_dtype, device=x.device)
    if ws is None:
        ws = chain_workspace(M, layers, x.device)
    _check(lib.bitlinear_chain_forward(_dev(x, "x"), _dtype_code(x), M, arr, len(layers),
                                       _dev(y, "y"), _dtype_code(y), _dev(ws, "ws"), ws.numel(),
                                       _stream(stream)), "bitlinear_chain_forward")
    return y


def base3_row_bytes(K: int) -> int:
    return int(load_library().bitlinear_base3_row_bytes(K))


def pack_base3(packed: torch.Tensor, stream=None) -> torch.Tensor:
    """2-bit packed weights [N][K/4] -> base-3 [N][ceil(K/80)*16] (same codes)."""
    lib = load_library()
    N, K = packed.shape[0], packed.shape[1] * 4
    out = torch.empty((N, base3_row_bytes(K)), dtype=torch.uint8, device=packed.device)
    _check(lib.bitlinear_pack_base3(_dev(packed, "packed"), N, K, _dev(out, "packed3"),
                                    _stream(stream)), "bitlinear_pack_base3")
    return out


def forward_base3(x: torch.Tensor, packed3: torch.Tensor, gamma: torch.Tensor,
                  out_dtype: torch.dtype = torch.bfloat16, y: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    """BitLinear forward on base-3 weights (M <= 4 tokens)."""
    lib = load_library()
    M, K = x.shape
    N = packed3.shape[0]
    if packed3.shape[1] != base3_row_bytes(K):
        raise ValueError("packed3 must be [N][ceil(K/80)*16]")
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check(lib.bitlinear_forward_base3(
        _dev(x, "x"), _dtype_code(x), _dev(packed3, "packed3"), _dev(gamma, "gamma"),
        _dev(y, "y"), _dtype_code(y), M, N, K, _stream(stream)), "bitlinear_forward_base3")
    return y


def pack_transpose(packed: torch.Tensor, stream=None) -> torch.Tensor:
    """2-bit weights [N][K/4] -> the transposed 2-bit weights [K][N/4] (N % 64 == 0)."""
    lib = load_library()
    N, K = packed.shape[0], packed.shape[1] * 4
    out = torch.empty((K, N // 4), dtype=torch.uint8, device=packed.device)
    _check(lib.bitlinear_pack_transpose(_dev(packed, "packed"), N, K, _dev(out, "packedT"),
                                        _stream(stream)), "bitlinear_pack_transpose")
    return out


def backward(x: torch.Tensor, grad_y: torch.Tensor, packedT: torch.Tensor, gamma: torch.Tensor,
             need_x: bool = True, need_w: bool = True, ws: torch.Tensor | None = None,
             stream=None):
    """Straight-through BitLinear backward: (grad_x fp32 [M][K] or None, grad_w fp32 [N][K]
    or None) from the forward input x, grad_y bf16 [M][N] and the transposed weights."""
    lib = load_library()
    M, K = x.shape
    N = grad_y.shape[1]
    if grad_y.dtype != torch.bfloat16:
        raise TypeError("grad_y must be bf16")
    gx = torch.empty((M, K), dtype=torch.float32, device=x.device) if need_x else None
    gw = torch.empty((N, K), dtype=torch.float32, device=x.device) if need_w else None
    if ws is None and need_w:
        n = int(lib.bitlinear_backward_workspace_size(M, N, K))
        if n == 0:
            raise BitLinearError(2, "bitlinear_backward_workspace_size")
        ws = torch.empty(n, dtype=torch.uint8, device=x.device)
    _check(lib.bitlinear_backward(
        _dev(x, "x"), _dtype_code(x), _dev(grad_y, "grad_y"), _dev(packedT, "packedT"),
        _dev(gamma, "gamma"), _dev(gx, "grad_x") if gx is not None else None,
        _dev(gw, "grad_w") if gw is not None else None, M, N, K,
        _dev(ws, "ws") if ws is not None else None, ws.numel() if ws is not None else 0,
        _stream(stream)), "bitlinear_backward")
    return gx, gw


def forward(x: torch.Tensor, packed: torch.Tensor, gamma: torch.Tensor,
            out_dtype: torch.dtype = torch.bfloat16, y: torch.Tensor | None = None,
            ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """BitLinear forward: y [M][N] = rescale(int32 contraction of quantized x with W)."""
    lib = load_library()
    M, K = x.shape
    N = packed.shape[0]
    if packed.shape[1] * 4 != K:
        raise ValueError("packed must be [N][K/4]")
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    if ws is None:
        ws = workspace(M, N, K, x.device)
    _check(lib.bitlinear_forward(
        _dev(x, "x"), _dtype_code(x), _dev(packed, "packed"), _dev(gamma, "gamma"), _dev(y, "y"),
        _dtype_code(y), M, N, K, _dev(ws, "ws"), ws.numel(), _stream(stream)),
        "bitlinear_forward")
    return y


def forward_noalloc(x: torch.Tensor, packed: torch.Tensor, gamma: torch.Tensor,
                    out_dtype: torch.dtype = torch.bfloat16, y: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """bitlinear_forward without a workspace: the library's built-in 16 MiB device scratch
    serves the tensor-core path (for callers that cannot allocate; calls must not overlap
    on the GPU)."""
    lib = load_library()
    M, K = x.shape
    N = packed.shape[0]
    if packed.shape[1] * 4 != K:
        raise ValueError("packed must be [N][K/4]")
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check(lib.bitlinear_forward_noalloc(
        _dev(x, "x"), _dtype_code(x), _dev(packed, "packed"), _dev(gamma, "gamma"), _dev(y, "y"),
        _dtype_code(y), M, N, K, _stream(stream)), "bitlinear_forward_noalloc")
    return y


def contract_i32(xq: torch.Tensor, packed: torch.Tensor, acc: torch.Tensor | None = None,
                 ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Integer stage only: acc [M][N] int32 = sum_k c[n,k] * xq[t,k]."""
    lib = load_library()
    M, K = xq.shape
    N = packed.shape[0]
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=xq.device)
    if ws is None:
        ws = workspace(M, N, K, xq.device)
    _check(lib.bitlinear_contract_i32(_dev(xq, "xq"), _dev(packed, "packed"), _dev(acc, "acc"),
                                      M, N, K, _dev(ws, "ws"), ws.numel(), _stream(stream)),
           "bitlinear_contract_i32")
    return acc


def get_device_status(stream=None) -> int:
    """Synchronizes the stream, returns and clears the device status word (0 = BL_OK)."""
    return int(load_library().bitlinear_get_device_status(_stream(stream)))


def debug_timeout_probe(timeout_ns: int, stream=None) -> None:
    _check(load_library().bitlinear_debug_timeout_probe(int(timeout_ns), _stream(stream)),
           "bitlinear_debug_timeout_probe")


PATHS = ("gemv", "skinny", "prefill")


def debug_plan(M: int, N: int, K: int, sms: int = 148) -> tuple[str, int]:
    """The kernel a forward of this shape runs and its K splits (host only, no device)."""
    path, splits = ctypes.c_int(-1), ctypes.c_int(0)
    _check(load_library().bitlinear_debug_plan(M, N, K, sms, ctypes.byref(path),
                                               ctypes.byref(splits)), "bitlinear_debug_plan")
    return PATHS[path.value], splits.value


def status_string(status: int) -> str:
    return load_library().bitlinear_status_string(status).decode()
