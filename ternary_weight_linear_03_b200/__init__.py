"""B200 (sm_100a) BitLinear forward of BitNet b1.58: absmean ternary weights, per-token
int8 activations, exact int32 contraction and rescale, as a C-ABI library
(libbitlinear.so, include/bitlinear.h) with a thin Python binding."""

from .bitlinear import (  # noqa: F401
    BL_BF16, BL_F32, BL_I32, EXPORTS, BitLinearError, contract_i32, debug_plan,
    debug_timeout_probe,
    forward, forward_noalloc, get_device_status, load_library, quantize_acts, quantize_weights, status_string,
    workspace, workspace_size,
)
