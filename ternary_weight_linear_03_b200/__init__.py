"""B200 (sm_100a) BitLinear forward of BitNet b1.58: absmean ternary weights, per-token
int8 activations, exact int32 contraction and rescale, as a C-ABI library
(libbitlinear.so, include/bitlinear.h) with a thin Python binding."""

from .bitlinear import (  # noqa: F401
    ABSSUM_WORDS, BL_BF16, BL_F32, BL_I32, EXPORTS, BitLinearError, Layer, act_absmax,
    backward, base3_row_bytes, chain_forward, chain_layers, chain_workspace, contract_i32, forward_base3,
    pack_base3, pack_transpose,
    debug_plan, debug_timeout_probe, forward, forward_noalloc, get_device_status, load_library,
    quantize_acts, quantize_acts_absmax, quantize_weights, quantize_weights_from_abssum,
    rescale, status_string, weight_abssum, workspace, workspace_size,
)
