"""ctypes marshalling for ``libsq.so``: torch CUDA tensors in, C-ABI calls out.

Nothing here computes: shapes are read off the tensors, outputs are allocated
with torch (device memory is the one service torch provides), and each call
goes straight to the matching ``sq_*`` entry point on torch's current stream.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(HERE, "libsq.so")

if not os.path.exists(library_path):
    raise ImportError(
        "rotation_ptq_b200: CUDA library %s is missing; build it with "
        "`python rotation_ptq_b200/build.py` (there is no CPU fallback)" % library_path)

lib = ctypes.CDLL(library_path)

SQ_IN_F32, SQ_IN_BF16 = 0, 1
SQ_OUT_BF16, SQ_OUT_I32 = 0, 1

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_f32 = ctypes.c_float

lib.sq_status_string.restype = ctypes.c_char_p
lib.sq_status_string.argtypes = [_i32]
lib.sq_last_error.restype = ctypes.c_char_p
lib.sq_last_error.argtypes = []
lib.sq_version.restype = _i32
lib.sq_rotate_quant.restype = _i32
lib.sq_rotate_quant.argtypes = [_vp, _i32, _i64, _i64, _i64, _vp, _i32, _i32, _f32, _vp, _vp, _vp]
lib.sq_w4a8_linear.restype = _i32
lib.sq_w4a8_linear.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i32, _vp,
                               ctypes.c_size_t, _vp]
lib.sq_rotate_quant8.restype = _i32
lib.sq_rotate_quant8.argtypes = [_vp, _i32, _i64, _i64, _i64, _vp, _i32, _i32, _f32, _vp, _vp, _vp]
lib.sq_swiglu_rotate_quant.restype = _i32
lib.sq_swiglu_rotate_quant.argtypes = [_vp, _i64, _i64, _i64, _vp, _i32, _i32, _f32, _vp, _vp, _vp]
lib.sq_w4a4_linear.restype = _i32
lib.sq_w4a4_linear.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i32, _vp,
                               ctypes.c_size_t, _vp]
lib.sq_kv4_decode_workspace_bytes.restype = ctypes.c_size_t
lib.sq_kv4_decode_workspace_bytes.argtypes = [_i64, _i64, _i32, _i32]
for _f in (lib.sq_kv4_decode_attention, lib.sq_kv8_decode_attention):
    _f.restype = _i32
    _f.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i32, _i32, _i32, _vp, _vp,
                   ctypes.c_size_t, _vp]
lib.sq_w4a4_workspace_bytes.restype = ctypes.c_size_t
lib.sq_w4a4_workspace_bytes.argtypes = [_i64, _i64, _i64]
lib.sq_w4a4_tail_workspace_bytes.restype = ctypes.c_size_t
lib.sq_w4a4_tail_workspace_bytes.argtypes = [_i64, _i64, _i64]
for _f in (lib.sq_kv_rotate_quant, lib.sq_kv_rotate_quant8):
    _f.restype = _i32
    _f.argtypes = [_vp, _vp, _vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp,
                   _vp, _vp, _vp, _vp]
for _f in (lib.sq_kv_dequant, lib.sq_kv8_dequant):
    _f.restype = _i32
    _f.argtypes = [_vp, _vp, _vp, _i64, _i32, _i32, _vp, _vp]
lib.sq_r2_workspace_bytes.restype = ctypes.c_size_t
lib.sq_r2_workspace_bytes.argtypes = [_i64, _i32, _i32, _i64]
lib.sq_r2_prepare.restype = _i32
lib.sq_r2_prepare.argtypes = [_vp, _vp, _i64, _i32, _i32, _i64, _vp, ctypes.c_size_t, _vp]
lib.sq_r2_loss_grad.restype = _i32
lib.sq_r2_loss_grad.argtypes = [_vp, _vp, _vp, _i64, _i32, _i32, _i64, _vp, _vp, _vp,
                                ctypes.c_size_t, _vp]
lib.sq_r2_cayley_learn.restype = _i32
lib.sq_r2_cayley_learn.argtypes = [_vp, _vp, _vp, _i64, _i32, _i32, _i64, ctypes.c_double, _i32,
                                   _vp, _vp, _vp, ctypes.c_size_t, _vp]
lib.sq_cayley_workspace_bytes.restype = ctypes.c_size_t
lib.sq_cayley_workspace_bytes.argtypes = [_i32, _i32]
lib.sq_cayley_update.restype = _i32
lib.sq_cayley_update.argtypes = [_vp, _vp, ctypes.c_double, _i32, _i32, _vp, _vp, _vp,
                                 ctypes.c_size_t, _vp]
lib.sq_r2_random_hadamard.restype = _i32
lib.sq_r2_random_hadamard.argtypes = [_vp, _i32, _i32, _vp, _vp]
lib.sq_orth_error.restype = _i32
lib.sq_orth_error.argtypes = [_vp, _i32, _i32, _vp, _vp]
lib.sq_rope_tables.restype = _i32
lib.sq_rope_tables.argtypes = [ctypes.c_double, _i32, _i32, _vp, _vp, _vp]
lib.sq_device_status.restype = _i32
lib.sq_device_status.argtypes = [_vp]
lib.sq_debug_set_spin_limit.restype = None
lib.sq_debug_set_spin_limit.argtypes = [ctypes.c_uint32]
lib.sq_debug_set_gemm_path.restype = None
lib.sq_debug_set_gemm_path.argtypes = [ctypes.c_int]


class SqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = lib.sq_status_string(status).decode()
        detail = lib.sq_last_error().decode()
        super().__init__("%s: %s (%s)" % (where, name, detail))


def _check(status: int, where: str) -> None:
    if status != 0:
        raise SqError(status, where)


def version() -> int:
    return lib.sq_version()


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("rotation_ptq_b200 takes CUDA tensors (no CPU path)")


SQ_ERR_TIMEOUT = 5


def _expect(t, name, dtype, shape):
    """Reject a tensor whose dtype, shape or layout the C entry point would
    misread (a short or mistyped buffer would be read or written past its end
    on the device)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _same_device(*ts):
    devs = {t.device for t in ts if t is not None}
    if len(devs) > 1:
        raise ValueError("all tensors must be on one device, got %s" % sorted(map(str, devs)))


def _expect_workspace(ws):
    if ws is None:
        return
    if not isinstance(ws, torch.Tensor) or ws.dtype != torch.uint8 or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 tensor")


def rotate_quant(x: torch.Tensor, had_small=None, n_pow2: int = 1, clip: float = 1.0,
                 a_q: torch.Tensor = None, a_scale: torch.Tensor = None):
    """Online rotation + per-token INT4 (``sq_rotate_quant``).

    x: CUDA [M, K] bf16 or float32 (unit stride along K).  had_small: None or a
    host +-1 int8 matrix [n, n].  Returns (a_q uint8 [M, K/2], a_scale f32 [M]).
    """
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit stride along K")
    if x.dtype == torch.bfloat16:
        dt = SQ_IN_BF16
    elif x.dtype == torch.float32:
        dt = SQ_IN_F32
    else:
        raise ValueError("x must be bf16 or float32")
    M, K = x.shape
    if had_small is None:
        hs, n_small, hs_ptr = None, 1, None
    else:
        hs = np.ascontiguousarray(np.asarray(had_small, dtype=np.int8))
        n_small = hs.shape[0]
        if hs.shape != (n_small, n_small):
            raise ValueError("had_small must be square")
        hs_ptr = hs.ctypes.data
    if K % 2:
        raise ValueError("K must be even")
    if a_q is not None:
        _expect(a_q, "a_q", torch.uint8, (M, K // 2))
    if a_scale is not None:
        _expect(a_scale, "a_scale", torch.float32, (M,))
    _same_device(x, a_q, a_scale)
    if a_q is None:
        a_q = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    if a_scale is None:
        a_scale = torch.empty((M,), dtype=torch.float32, device=x.device)
    _need_cuda(x, a_q, a_scale)
    st = lib.sq_rotate_quant(x.data_ptr(), dt, M, K, x.stride(0), hs_ptr, n_small, n_pow2,
                             float(clip), a_q.data_ptr(), a_scale.data_ptr(), _stream(x))
    _check(st, "sq_rotate_quant")
    return a_q, a_scale


def _small_hadamard(had_small):
    if had_small is None:
        return None, 1, None
    hs = np.ascontiguousarray(np.asarray(had_small, dtype=np.int8))
    n_small = hs.shape[0]
    if hs.shape != (n_small, n_small):
        raise ValueError("had_small must be square")
    return hs, n_small, hs.ctypes.data


def rotate_quant8(x: torch.Tensor, had_small=None, n_pow2: int = 1, clip: float = 1.0,
                  a_q: torch.Tensor = None, a_scale: torch.Tensor = None):
    """Online rotation + per-token INT8 (``sq_rotate_quant8``, the A side of W4A8).

    x: CUDA [M, K] bf16 or float32.  Returns (a_q int8 [M, K], a_scale f32 [M]).
    """
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit stride along K")
    if x.dtype == torch.bfloat16:
        dt = SQ_IN_BF16
    elif x.dtype == torch.float32:
        dt = SQ_IN_F32
    else:
        raise ValueError("x must be bf16 or float32")
    M, K = x.shape
    hs, n_small, hs_ptr = _small_hadamard(had_small)
    if a_q is not None:
        _expect(a_q, "a_q", torch.int8, (M, K))
    if a_scale is not None:
        _expect(a_scale, "a_scale", torch.float32, (M,))
    _same_device(x, a_q, a_scale)
    _need_cuda(x, a_q, a_scale)
    if a_q is None:
        a_q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if a_scale is None:
        a_scale = torch.empty((M,), dtype=torch.float32, device=x.device)
    st = lib.sq_rotate_quant8(x.data_ptr(), dt, M, K, x.stride(0), hs_ptr, n_small, n_pow2,
                              float(clip), a_q.data_ptr(), a_scale.data_ptr(), _stream(x))
    _check(st, "sq_rotate_quant8")
    return a_q, a_scale


def swiglu_rotate_quant(gate_up: torch.Tensor, had_small=None, n_pow2: int = 1,
                        clip: float = 1.0, a_q: torch.Tensor = None,
                        a_scale: torch.Tensor = None):
    """SwiGLU of [gate | up] + online rotation + per-token INT4 (``sq_swiglu_rotate_quant``).

    gate_up: CUDA bf16 [M, >= 2K] with unit stride along the columns; K is
    half its width (gate = columns [0, K), up = [K, 2K)).  Returns
    (a_q uint8 [M, K/2], a_scale f32 [M]).
    """
    if gate_up.dim() != 2 or gate_up.stride(1) != 1 or gate_up.dtype != torch.bfloat16:
        raise ValueError("gate_up must be a 2-D bf16 tensor with unit stride along columns")
    M, W2 = gate_up.shape
    if W2 % 4:
        raise ValueError("gate_up width must be 2K with K even ([gate | up])")
    K = W2 // 2
    hs, n_small, hs_ptr = _small_hadamard(had_small)
    if a_q is not None:
        _expect(a_q, "a_q", torch.uint8, (M, K // 2))
    if a_scale is not None:
        _expect(a_scale, "a_scale", torch.float32, (M,))
    _same_device(gate_up, a_q, a_scale)
    _need_cuda(gate_up, a_q, a_scale)
    if a_q is None:
        a_q = torch.empty((M, K // 2), dtype=torch.uint8, device=gate_up.device)
    if a_scale is None:
        a_scale = torch.empty((M,), dtype=torch.float32, device=gate_up.device)
    st = lib.sq_swiglu_rotate_quant(gate_up.data_ptr(), M, K, gate_up.stride(0), hs_ptr,
                                    n_small, n_pow2, float(clip), a_q.data_ptr(),
                                    a_scale.data_ptr(), _stream(gate_up))
    _check(st, "sq_swiglu_rotate_quant")
    return a_q, a_scale


def quantize_weights(w: torch.Tensor, had_small=None, n_pow2: int = 1):
    """Offline: fold the rotation into W [N, K] (float32) and RTN-quantize per channel.

    The same kernel as ``rotate_quant`` (clip 1.0), applied to weight rows:
    codes of W H / sqrt(g).  Returns (w_q uint8 [N, K/2], w_scale f32 [N]).
    """
    return rotate_quant(w.float().contiguous(), had_small, n_pow2, 1.0)


_ws_lock = threading.Lock()
_ws_cache = {}


def _reset_workspaces(device_index: int) -> None:
    """Zero every cached workspace of a device.  The library leaves a
    workspace zero after each call that completes; a call whose device waits
    ran out (SQ_ERR_TIMEOUT) can leave partial sums and arrival counters in
    it, which the next call would otherwise add to."""
    with _ws_lock:
        bufs = [b for (d, _), b in _ws_cache.items() if d == device_index]
    if bufs:
        torch.cuda.synchronize(device_index)
        for b in bufs:
            b.zero_()
        torch.cuda.synchronize(device_index)


def _workspace(device: torch.device, stream: int, nbytes: int) -> torch.Tensor:
    key = (device.index, stream)
    with _ws_lock:
        buf = _ws_cache.get(key)
        if buf is None or buf.numel() < nbytes:
            # zero-filled once; the library hands it back zero-filled after every call
            buf = torch.zeros((max(nbytes, 256),), dtype=torch.uint8, device=device)
            _ws_cache[key] = buf
        return buf


def w4a4_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib.sq_w4a4_workspace_bytes(M, N, K))


def w4a4_tail_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib.sq_w4a4_tail_workspace_bytes(M, N, K))


def w4a4_linear(a_q: torch.Tensor, a_scale: torch.Tensor, w_q: torch.Tensor,
                w_scale: torch.Tensor, out_int32: bool = False, out: torch.Tensor = None,
                workspace: torch.Tensor = None, use_workspace: bool = True):
    """W4A4 GEMM with fused dequant (``sq_w4a4_linear``).

    a_q [M, K/2], a_scale [M], w_q [N, K/2], w_scale [N] on one CUDA device.
    Returns bf16 [M, N] (or int32 accumulators with out_int32=True).
    """
    if a_q.dim() != 2 or w_q.dim() != 2:
        raise ValueError("a_q must be [M, K/2] and w_q [N, K/2]")
    M, Kh = a_q.shape
    N = w_q.shape[0]
    K = 2 * Kh
    _expect(a_q, "a_q", torch.uint8, (M, Kh))
    _expect(a_scale, "a_scale", torch.float32, (M,))
    _expect(w_q, "w_q", torch.uint8, (N, Kh))
    _expect(w_scale, "w_scale", torch.float32, (N,))
    if out is not None:
        _expect(out, "out", torch.int32 if out_int32 else torch.bfloat16, (M, N))
    _expect_workspace(workspace)
    _same_device(a_q, a_scale, w_q, w_scale, out, workspace)
    _need_cuda(a_q, a_scale, w_q, w_scale, out, workspace)
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32 if out_int32 else torch.bfloat16,
                          device=a_q.device)
    stream = _stream(a_q)
    ws_ptr, ws_bytes = None, 0
    if use_workspace:
        need = max(w4a4_workspace_bytes(M, N, K), w4a4_tail_workspace_bytes(M, N, K))
        if workspace is not None:
            ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
        elif need > 0:
            ws = _workspace(a_q.device, stream, need)
            ws_ptr, ws_bytes = ws.data_ptr(), ws.numel()
    st = lib.sq_w4a4_linear(a_q.data_ptr(), a_scale.data_ptr(), w_q.data_ptr(),
                            w_scale.data_ptr(), M, N, K, out.data_ptr(),
                            SQ_OUT_I32 if out_int32 else SQ_OUT_BF16, ws_ptr, ws_bytes, stream)
    _check(st, "sq_w4a4_linear")
    return out


def kv4_decode_workspace_bytes(B: int, S_max: int, hq: int, hkv: int) -> int:
    """Scratch bytes that let sq_kv4_decode_attention split sequences across CTAs."""
    return int(lib.sq_kv4_decode_workspace_bytes(B, S_max, hq, hkv))


def kv4_decode_attention(q: torch.Tensor, k_cache: torch.Tensor, k_scale: torch.Tensor,
                         k_zero: torch.Tensor, v_cache: torch.Tensor, v_scale: torch.Tensor,
                         v_zero: torch.Tensor, lengths: torch.Tensor, S_max: int,
                         out: torch.Tensor = None, workspace: torch.Tensor = None):
    """One decode step of attention over the 4-bit caches (``sq_kv4_decode_attention``).

    q: bf16 [B, hq, 128]; caches uint8 [B * S_max, hkv, 64]; scales f32 and
    zeros uint8 [B * S_max, hkv]; lengths int32 [B].  Returns bf16 [B, hq, 128].
    Without ``workspace`` a cached zero-filled buffer of the stream is used.
    """
    return _kv_decode(lib.sq_kv4_decode_attention, "sq_kv4_decode_attention", q, k_cache,
                      k_scale, k_zero, v_cache, v_scale, v_zero, lengths, S_max, out, workspace)


def kv8_decode_attention(q: torch.Tensor, k_cache: torch.Tensor, k_scale: torch.Tensor,
                         k_zero: torch.Tensor, v_cache: torch.Tensor, v_scale: torch.Tensor,
                         v_zero: torch.Tensor, lengths: torch.Tensor, S_max: int,
                         out: torch.Tensor = None, workspace: torch.Tensor = None):
    """kv4_decode_attention over 8-bit caches uint8 [B * S_max, hkv, 128]
    (``sq_kv8_decode_attention``)."""
    return _kv_decode(lib.sq_kv8_decode_attention, "sq_kv8_decode_attention", q, k_cache,
                      k_scale, k_zero, v_cache, v_scale, v_zero, lengths, S_max, out, workspace)


def _kv_decode(fn, name, q, k_cache, k_scale, k_zero, v_cache, v_scale, v_zero, lengths, S_max,
               out, workspace):
    if q.dim() != 3 or k_scale.dim() != 2:
        raise ValueError("q must be [B, hq, d] and the scales [B * S_max, hkv]")
    B, hq, d = q.shape
    hkv = k_scale.shape[1]
    rows = B * S_max
    row_bytes = k_cache.shape[-1] if k_cache.dim() == 3 else -1
    _expect(q, "q", torch.bfloat16, (B, hq, d))
    for nm, c, sc, z in (("k", k_cache, k_scale, k_zero), ("v", v_cache, v_scale, v_zero)):
        _expect(c, nm + "_cache", torch.uint8, (rows, hkv, row_bytes))
        _expect(sc, nm + "_scale", torch.float32, (rows, hkv))
        _expect(z, nm + "_zero", torch.uint8, (rows, hkv))
    if row_bytes != (d // 2 if fn is lib.sq_kv4_decode_attention else d):
        raise ValueError("cache rows must hold %s bytes per head vector"
                         % ("d/2" if fn is lib.sq_kv4_decode_attention else "d"))
    _expect(lengths, "lengths", torch.int32, (B,))
    if out is not None:
        _expect(out, "out", torch.bfloat16, (B, hq, d))
    _expect_workspace(workspace)
    _same_device(q, k_cache, k_scale, k_zero, v_cache, v_scale, v_zero, lengths, out, workspace)
    _need_cuda(q, k_cache, k_scale, k_zero, v_cache, v_scale, v_zero, lengths, out, workspace)
    if out is None:
        out = torch.empty((B, hq, d), dtype=torch.bfloat16, device=q.device)
    stream = _stream(q)
    need = kv4_decode_workspace_bytes(B, S_max, hq, hkv)
    if workspace is None and need > 0:
        workspace = _workspace(q.device, stream, need)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = fn(q.data_ptr(), k_cache.data_ptr(), k_scale.data_ptr(), k_zero.data_ptr(),
            v_cache.data_ptr(), v_scale.data_ptr(), v_zero.data_ptr(), lengths.data_ptr(), B, S_max,
            hq, hkv, d, out.data_ptr(), ws_ptr, ws_bytes, stream)
    _check(st, name)
    return out


def w4a8_linear(a_q: torch.Tensor, a_scale: torch.Tensor, w_q: torch.Tensor,
                w_scale: torch.Tensor, out: torch.Tensor = None, out_i32: bool = False,
                workspace: torch.Tensor = None):
    """INT8 activations x packed INT4 weights (``sq_w4a8_linear``).

    a_q: int8 [M, K] (from rotate_quant8); w_q: uint8 [N, K/2].  Returns bf16
    (or, with out_i32, the exact int32 sums) [M, N].
    """
    if a_q.dim() != 2 or w_q.dim() != 2:
        raise ValueError("a_q must be int8 [M, K] and w_q uint8 [N, K/2]")
    M, K = a_q.shape
    N = w_q.shape[0]
    if K % 2:
        raise ValueError("K must be even")
    _expect(a_q, "a_q", torch.int8, (M, K))
    _expect(a_scale, "a_scale", torch.float32, (M,))
    _expect(w_q, "w_q", torch.uint8, (N, K // 2))
    _expect(w_scale, "w_scale", torch.float32, (N,))
    if out is not None:
        _expect(out, "out", torch.int32 if out_i32 else torch.bfloat16, (M, N))
    _expect_workspace(workspace)
    _same_device(a_q, a_scale, w_q, w_scale, out, workspace)
    _need_cuda(a_q, a_scale, w_q, w_scale, out, workspace)
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32 if out_i32 else torch.bfloat16,
                          device=a_q.device)
    stream = _stream(a_q)
    if workspace is None:
        need = w4a4_tail_workspace_bytes(M, N, K)
        workspace = _workspace(a_q.device, stream, need) if need > 0 else None
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.sq_w4a8_linear(a_q.data_ptr(), a_scale.data_ptr(), w_q.data_ptr(),
                            w_scale.data_ptr(), M, N, K, out.data_ptr(),
                            SQ_OUT_I32 if out_i32 else SQ_OUT_BF16, ws_ptr, ws_bytes, stream)
    _check(st, "sq_w4a8_linear")
    return out


def rope_tables(theta: float, max_pos: int, d: int = 128, device=None):
    """cos/sin tables [max_pos, d/2] float32 computed on the device (``sq_rope_tables``)."""
    device = torch.device("cuda") if device is None else torch.device(device)
    cos = torch.empty((max_pos, d // 2), dtype=torch.float32, device=device)
    sin = torch.empty_like(cos)
    st = lib.sq_rope_tables(float(theta), max_pos, d, cos.data_ptr(), sin.data_ptr(),
                            _stream(cos))
    _check(st, "sq_rope_tables")
    return cos, sin


def kv_rotate_quant(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor,
                    cos: torch.Tensor = None, sin: torch.Tensor = None, out=None):
    """RoPE + head-wise H128 on Q/K, asymmetric 4-bit K/V caches (``sq_kv_rotate_quant``).

    q [T, hq, 128], k/v [T, hkv, 128] bf16; pos [T] int32.  Returns a dict with
    q_out, k_cache, k_scale, k_zero, v_cache, v_scale, v_zero.
    """
    return _kv_rotate_quant(lib.sq_kv_rotate_quant, "sq_kv_rotate_quant", 2, q, k, v, pos, cos,
                            sin, out)


def kv_rotate_quant8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor,
                     cos: torch.Tensor = None, sin: torch.Tensor = None, out=None):
    """kv_rotate_quant with 8-bit caches [T, hkv, 128] (``sq_kv_rotate_quant8``)."""
    return _kv_rotate_quant(lib.sq_kv_rotate_quant8, "sq_kv_rotate_quant8", 1, q, k, v, pos, cos,
                            sin, out)


def _kv_rotate_quant(fn, name, per_byte, q, k, v, pos, cos, sin, out):
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("q must be [T, hq, d] and k, v [T, hkv, d]")
    T, hq, d = q.shape
    hkv = k.shape[1]
    _expect(q, "q", torch.bfloat16, (T, hq, d))
    _expect(k, "k", torch.bfloat16, (T, hkv, d))
    _expect(v, "v", torch.bfloat16, (T, hkv, d))
    _expect(pos, "pos", torch.int32, (T,))
    if (cos is None) != (sin is None):
        raise ValueError("cos and sin must both be given or both be None")
    if cos is not None:
        if cos.dim() != 2:
            raise ValueError("cos must be [max_pos, d/2]")
        _expect(cos, "cos", torch.float32, (cos.shape[0], d // 2))
        _expect(sin, "sin", torch.float32, tuple(cos.shape))
    dev = q.device
    if out is not None:
        shapes = dict(q_out=((T, hq, d), torch.bfloat16),
                      k_cache=((T, hkv, d // per_byte), torch.uint8),
                      k_scale=((T, hkv), torch.float32), k_zero=((T, hkv), torch.uint8),
                      v_cache=((T, hkv, d // per_byte), torch.uint8),
                      v_scale=((T, hkv), torch.float32), v_zero=((T, hkv), torch.uint8))
        for key, (shp, dt) in shapes.items():
            if key not in out:
                raise ValueError("out is missing %s" % key)
            _expect(out[key], "out[%s]" % key, dt, shp)
    _same_device(q, k, v, pos, cos, sin, *(out.values() if out is not None else ()))
    _need_cuda(q, k, v, pos, cos, sin, *(out.values() if out is not None else ()))
    if out is None:
        out = dict(
            q_out=torch.empty_like(q),
            k_cache=torch.empty((T, hkv, d // per_byte), dtype=torch.uint8, device=dev),
            k_scale=torch.empty((T, hkv), dtype=torch.float32, device=dev),
            k_zero=torch.empty((T, hkv), dtype=torch.uint8, device=dev),
            v_cache=torch.empty((T, hkv, d // per_byte), dtype=torch.uint8, device=dev),
            v_scale=torch.empty((T, hkv), dtype=torch.float32, device=dev),
            v_zero=torch.empty((T, hkv), dtype=torch.uint8, device=dev))
    max_pos = cos.shape[0] if cos is not None else 0
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), T, hq, hkv, d, pos.data_ptr(), _ptr(cos),
            _ptr(sin), max_pos, out["q_out"].data_ptr(), out["k_cache"].data_ptr(),
            out["k_scale"].data_ptr(), out["k_zero"].data_ptr(), out["v_cache"].data_ptr(),
            out["v_scale"].data_ptr(), out["v_zero"].data_ptr(), _stream(q))
    _check(st, name)
    return out


def kv_dequant(cache: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor, out=None):
    """Packed asymmetric cache [T, h, 64] -> bf16 [T, h, 128] (``sq_kv_dequant``)."""
    if cache.dim() != 3:
        raise ValueError("cache must be [T, h, 64]")
    T, h, dh = cache.shape
    _expect(cache, "cache", torch.uint8, (T, h, dh))
    _expect(scale, "scale", torch.float32, (T, h))
    _expect(zero, "zero", torch.uint8, (T, h))
    if out is not None:
        _expect(out, "out", torch.bfloat16, (T, h, 2 * dh))
    _same_device(cache, scale, zero, out)
    _need_cuda(cache, scale, zero, out)
    if out is None:
        out = torch.empty((T, h, 2 * dh), dtype=torch.bfloat16, device=cache.device)
    st = lib.sq_kv_dequant(cache.data_ptr(), scale.data_ptr(), zero.data_ptr(), T, h, 2 * dh,
                           out.data_ptr(), _stream(cache))
    _check(st, "sq_kv_dequant")
    return out


def kv8_dequant(cache: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor, out=None):
    """8-bit asymmetric cache [T, h, 128] -> bf16 [T, h, 128] (``sq_kv8_dequant``)."""
    if cache.dim() != 3:
        raise ValueError("cache must be [T, h, 128]")
    T, h, d = cache.shape
    _expect(cache, "cache", torch.uint8, (T, h, d))
    _expect(scale, "scale", torch.float32, (T, h))
    _expect(zero, "zero", torch.uint8, (T, h))
    if out is not None:
        _expect(out, "out", torch.bfloat16, (T, h, d))
    _same_device(cache, scale, zero, out)
    _need_cuda(cache, scale, zero, out)
    if out is None:
        out = torch.empty((T, h, d), dtype=torch.bfloat16, device=cache.device)
    st = lib.sq_kv8_dequant(cache.data_ptr(), scale.data_ptr(), zero.data_ptr(), T, h, d,
                            out.data_ptr(), _stream(cache))
    _check(st, "sq_kv8_dequant")
    return out


class R2Problem:
    """One o_proj layer for the Cayley R2 learner: x float32 [T, H*d], w
    float32 [N, H*d] on the GPU, and the prepared workspace
    (``sq_r2_prepare``)."""

    def __init__(self, x: torch.Tensor, w: torch.Tensor, H: int, d: int = 128):
        _need_cuda(x, w)
        if x.dtype != torch.float32 or w.dtype != torch.float32:
            raise ValueError("x and w must be float32")
        self.x, self.w = x.contiguous(), w.contiguous()
        self.T, self.N, self.H, self.d = x.shape[0], w.shape[0], H, d
        need = int(lib.sq_r2_workspace_bytes(self.T, H, d, self.N))
        if need == 0:
            raise ValueError("unsupported R2 problem shape T=%d H=%d d=%d N=%d"
                             % (self.T, H, d, self.N))
        self.ws = torch.empty((need,), dtype=torch.uint8, device=x.device)
        st = lib.sq_r2_prepare(self.x.data_ptr(), self.w.data_ptr(), self.T, H, d, self.N,
                               self.ws.data_ptr(), need, _stream(x))
        _check(st, "sq_r2_prepare")

    def loss_grad(self, R: torch.Tensor, grad: bool = True):
        """Loss (device float64 [1]) and, with grad, G (device float64 [d, d]) at R
        (float32 [d, d]) (``sq_r2_loss_grad``)."""
        _need_cuda(R)
        R = R.to(torch.float32).contiguous()
        loss = torch.empty((1,), dtype=torch.float64, device=R.device)
        G = torch.empty((self.d, self.d), dtype=torch.float64, device=R.device) if grad else None
        st = lib.sq_r2_loss_grad(self.x.data_ptr(), self.w.data_ptr(), R.data_ptr(), self.T,
                                 self.H, self.d, self.N, loss.data_ptr(), _ptr(G),
                                 self.ws.data_ptr(), self.ws.numel(), _stream(R))
        _check(st, "sq_r2_loss_grad")
        return loss, G

    def learn(self, R0: torch.Tensor, alpha: float, iters: int):
        """iters Cayley SGD steps from R0 (float64 [d, d]) (``sq_r2_cayley_learn``).
        Returns (R float64 [d, d], losses float64 [iters + 1]) on the device."""
        _need_cuda(R0)
        R0 = R0.to(torch.float64).contiguous()
        R = torch.empty_like(R0)
        losses = torch.empty((iters + 1,), dtype=torch.float64, device=R0.device)
        st = lib.sq_r2_cayley_learn(self.x.data_ptr(), self.w.data_ptr(), R0.data_ptr(), self.T,
                                    self.H, self.d, self.N, float(alpha), int(iters),
                                    R.data_ptr(), losses.data_ptr(), self.ws.data_ptr(),
                                    self.ws.numel(), _stream(R0))
        _check(st, "sq_r2_cayley_learn")
        return R, losses


def cayley_update(R: torch.Tensor, G: torch.Tensor, alpha: float, out: torch.Tensor = None,
                  out_f32: torch.Tensor = None):
    """(I - alpha/2 Y)^-1 (I + alpha/2 Y) R with Y = R G^T - G R^T, float64, for
    R, G [n, n] or [batch, n, n] (``sq_cayley_update``)."""
    _need_cuda(R, G)
    if R.dtype != torch.float64 or G.dtype != torch.float64 or R.shape != G.shape:
        raise ValueError("R and G must be float64 of the same shape")
    R, G = R.contiguous(), G.contiguous()
    n = R.shape[-1]
    batch = R.numel() // (n * n)
    if out is None:
        out = torch.empty_like(R)
    need = int(lib.sq_cayley_workspace_bytes(n, max(batch, 1)))
    ws = torch.empty((max(need, 16),), dtype=torch.uint8, device=R.device)
    st = lib.sq_cayley_update(R.data_ptr(), G.data_ptr(), float(alpha), n, batch, out.data_ptr(),
                              _ptr(out_f32), ws.data_ptr(), ws.numel(), _stream(R))
    _check(st, "sq_cayley_update")
    return out


def r2_random_hadamard(signs: torch.Tensor) -> torch.Tensor:
    """diag(s) H_d / sqrt(d) (float64) for signs int8 [d] or [batch, d]
    (``sq_r2_random_hadamard``)."""
    _need_cuda(signs)
    if signs.dtype != torch.int8:
        raise ValueError("signs must be int8")
    signs = signs.contiguous()
    d = signs.shape[-1]
    batch = signs.numel() // d
    R = torch.empty(tuple(signs.shape[:-1]) + (d, d), dtype=torch.float64, device=signs.device)
    st = lib.sq_r2_random_hadamard(signs.data_ptr(), d, batch, R.data_ptr(), _stream(signs))
    _check(st, "sq_r2_random_hadamard")
    return R


def orth_error(R: torch.Tensor) -> torch.Tensor:
    """||R^T R - I||_F per matrix of R [n, n] or [batch, n, n] (float64)
    (``sq_orth_error``)."""
    _need_cuda(R)
    if R.dtype != torch.float64:
        raise ValueError("R must be float64")
    R = R.contiguous()
    n = R.shape[-1]
    batch = R.numel() // (n * n)
    out = torch.empty((batch,), dtype=torch.float64, device=R.device)
    st = lib.sq_orth_error(R.data_ptr(), n, batch, out.data_ptr(), _stream(R))
    _check(st, "sq_orth_error")
    return out


def device_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device status word.

    After SQ_ERR_TIMEOUT every cached workspace of the device is zeroed again
    (a kernel that gave up may have left partial sums in it)."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    st = int(lib.sq_device_status(torch.cuda.current_stream(dev).cuda_stream))
    if st == SQ_ERR_TIMEOUT:
        idx = dev.index if dev.index is not None else torch.cuda.current_device()
        _reset_workspaces(idx)
    return st


SPIN_FAIL_AT_ONCE = 0xFFFFFFFF


def debug_set_spin_limit(polls: int) -> None:
    """Test hook: polls per bounded device wait (0: the default bound;
    SPIN_FAIL_AT_ONCE: every bounded wait gives up before its first poll)."""
    lib.sq_debug_set_spin_limit(int(polls))


def debug_set_gemm_path(path: int) -> None:
    """0 = automatic, 1 = one-CTA tiles, 2 = CTA-pair tiles with both operands
    widened in shared memory, 3 = CTA-pair tiles with A in tensor memory,
    4 = the CUDA-core GEMV for M <= 8."""
    lib.sq_debug_set_gemm_path(int(path))
