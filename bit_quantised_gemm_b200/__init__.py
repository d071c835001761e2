"""B200-native BitNet a4.8 BitLinear forward (ternary 2-bit weights x
per-token INT4 / FP4 / top-k INT8 activations), as hand-written sm_100a CUDA
kernels behind a C ABI (include/bitlinear.h). This package is the thin
Python binding; see `_lib` for the calls."""
from ._lib import (  # noqa: F401
    MODE_FP4, MODE_INT4, MODE_INT8, BitlinearError, check_status, debug_wait_timeout,
    gemm_w2a4, gemm_w2a8, gemm_w2a8_acc, gemm_w2fp4, gemm_w2fp4_acc, gemv_w2, gemv_w2_quant,
    header_functions,
    kv_attention_3bit, kv_keep4_positions, kv_quant_3bit, kv_quant_3bit_kv, lib, quant_act, set_launch_overlap, set_wait_timeout_ns, status_buffer, ternarize_pack,
    tensor_peak, topk_sparsify_i8, version,
)
