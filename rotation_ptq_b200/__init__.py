"""B200 (sm_100a) SpinQuant W4A4 inference hot path: thin Python binding.

The compute lives in the C-ABI library ``libsq.so`` (CUDA kernels for
sm_100a); this module only marshals arguments.  Tensors are torch CUDA
tensors; every call enqueues on torch's current CUDA stream of the tensor's
device.  There is no CPU fallback: if the library is missing, importing this
package raises.

Entry points (same names as the C ABI without the ``sq_`` prefix):
  rotate_quant, rotate_quant8, swiglu_rotate_quant, w4a4_linear, w4a8_linear,
  w4a4_workspace_bytes, kv_rotate_quant,
  kv_dequant, kv4_decode_attention, kv4_decode_workspace_bytes, rope_tables,
  kv_rotate_quant8, kv8_dequant, kv8_decode_attention,
  R2Problem (sq_r2_prepare / sq_r2_loss_grad / sq_r2_cayley_learn), cayley_update,
  r2_random_hadamard, orth_error,
  device_status, debug_set_spin_limit.
"""
from __future__ import annotations

from .binding import (  # noqa: F401
    R2Problem,
    cayley_update,
    orth_error,
    r2_random_hadamard,
    SQ_IN_BF16,
    SQ_IN_F32,
    SQ_OUT_BF16,
    SQ_OUT_I32,
    SqError,
    debug_set_gemm_path,
    debug_set_spin_limit,
    SPIN_FAIL_AT_ONCE,
    device_status,
    kv4_decode_attention,
    kv4_decode_workspace_bytes,
    kv8_decode_attention,
    kv8_dequant,
    kv_dequant,
    kv_rotate_quant,
    kv_rotate_quant8,
    lib,
    library_path,
    quantize_weights,
    rope_tables,
    rotate_quant,
    rotate_quant8,
    swiglu_rotate_quant,
    version,
    w4a4_linear,
    w4a4_tail_workspace_bytes,
    w4a4_workspace_bytes,
    w4a8_linear,
)
from .hadamard import paley_h12  # noqa: F401
