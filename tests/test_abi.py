"""CPU checks of the C-ABI library: it loads, exports every declared symbol,
and rejects bad arguments before touching the device.  No kernel runs here.
"""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def sq():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_sq_build", os.path.join(ROOT, "rotation_ptq_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import rotation_ptq_b200 as m
    return m


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for n in ["sq_rotate_quant", "sq_swiglu_rotate_quant", "sq_w4a4_linear",
              "sq_kv4_decode_attention", "sq_kv4_decode_workspace_bytes",
              "sq_kv_rotate_quant", "sq_kv_dequant",
              "sq_kv_rotate_quant8", "sq_kv8_dequant", "sq_kv8_decode_attention",
              "sq_r2_workspace_bytes", "sq_r2_prepare", "sq_r2_loss_grad", "sq_r2_cayley_learn",
              "sq_cayley_update", "sq_cayley_workspace_bytes", "sq_orth_error",
              "sq_status_string", "sq_w4a4_workspace_bytes", "sq_device_status"]:
        assert n in names


def test_library_exports_every_declared_symbol(sq):
    lib = ctypes.CDLL(sq.library_path)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_version(sq):
    assert sq.lib.sq_status_string(0) == b"SQ_OK"
    assert sq.lib.sq_status_string(5) == b"SQ_ERR_TIMEOUT"
    assert sq.lib.sq_status_string(99) == b"SQ_ERR_UNKNOWN"
    assert sq.version() >> 16 == 1


def test_validation_happens_before_any_launch(sq):
    lib = sq.lib
    # bad dtype, bad clip, bad group, bad K: all rejected on the host
    assert lib.sq_rotate_quant(None, 7, 4, 256, 256, None, 1, 256, 1.0, None, None, None) == 1
    assert lib.sq_rotate_quant(None, 1, 4, 256, 256, None, 1, 256, 1.5, None, None, None) == 1
    assert lib.sq_rotate_quant(None, 1, 4, 256, 256, None, 1, 3, 1.0, None, None, None) == 2
    assert lib.sq_rotate_quant(None, 1, 4, 100, 100, None, 1, 4, 1.0, None, None, None) == 2
    assert lib.sq_rotate_quant(None, 1, 4, 96, 96, None, 1, 64, 1.0, None, None, None) == 2
    hs = np.zeros((12, 12), np.int8)            # not +-1
    assert lib.sq_rotate_quant(None, 1, 4, 12288, 12288, hs.ctypes.data, 12, 1024, 1.0,
                               None, None, None) == 1
    assert b"not +-1" in lib.sq_last_error()
    # fused SwiGLU: the row must hold both halves (ld >= 2K); same K and clip rules
    assert lib.sq_swiglu_rotate_quant(None, 4, 256, 300, None, 1, 256, 1.0, None, None,
                                      None) == 1
    assert lib.sq_swiglu_rotate_quant(None, 4, 256, 512, None, 1, 256, 0.0, None, None,
                                      None) == 1
    assert lib.sq_swiglu_rotate_quant(None, 4, 100, 200, None, 1, 4, 1.0, None, None,
                                      None) == 2
    assert lib.sq_swiglu_rotate_quant(None, 0, 256, 512, None, 1, 256, 1.0, None, None,
                                      None) == 0
    # GEMM shape rules: N % 16, K % 128
    assert lib.sq_w4a4_linear(None, None, None, None, 4, 24, 256, None, 0, None, 0, None) == 2
    assert lib.sq_w4a4_linear(None, None, None, None, 4, 32, 200, None, 0, None, 0, None) == 2
    assert lib.sq_w4a4_linear(None, None, None, None, 4, 32, 256, None, 9, None, 0, None) == 1
    # M == 0 is a no-op that succeeds without a device
    assert lib.sq_w4a4_linear(None, None, None, None, 0, 32, 256, None, 0, None, 0, None) == 0
    # KV: head dim must be 128, hq a multiple of hkv
    assert lib.sq_kv_rotate_quant(None, None, None, 4, 32, 8, 64, None, None, None, 0,
                                  None, None, None, None, None, None, None, None) == 2
    assert lib.sq_kv_rotate_quant(None, None, None, 4, 30, 8, 128, None, None, None, 0,
                                  None, None, None, None, None, None, None, None) == 2
    assert lib.sq_kv_dequant(None, None, None, 4, 8, 64, None, None) == 2
    assert lib.sq_rope_tables(0.5, 16, 128, None, None, None) == 1
    # decode attention: d == 128 and hq == 4 * hkv; B == 0 is a no-op
    args = [None] * 8
    assert lib.sq_kv4_decode_attention(*args, 2, 16, 32, 8, 64, None, None, 0, None) == 2
    assert lib.sq_kv4_decode_attention(*args, 2, 16, 16, 8, 128, None, None, 0, None) == 2
    assert lib.sq_kv4_decode_attention(*args, 2, 0, 32, 8, 128, None, None, 0, None) == 1
    assert lib.sq_kv4_decode_attention(*args, 0, 16, 32, 8, 128, None, None, 0, None) == 0
    # the 8-bit KV entries share the 4-bit ones' rules
    assert lib.sq_kv_rotate_quant8(None, None, None, 4, 32, 8, 64, None, None, None, 0,
                                   None, None, None, None, None, None, None, None) == 2
    assert lib.sq_kv_rotate_quant8(None, None, None, 0, 32, 8, 128, None, None, None, 0,
                                   None, None, None, None, None, None, None, None) == 0
    assert lib.sq_kv8_dequant(None, None, None, 4, 8, 64, None, None) == 2
    assert lib.sq_kv8_dequant(None, None, None, 4, 8, 128, None, None) == 1
    assert lib.sq_kv8_decode_attention(*args, 2, 16, 16, 8, 128, None, None, 0, None) == 2
    assert lib.sq_kv8_decode_attention(*args, 0, 16, 32, 8, 128, None, None, 0, None) == 0
    # Cayley R2 learner: d == 128, T and N multiples of 16; n <= 128
    assert lib.sq_r2_workspace_bytes(2048, 32, 64, 4096) == 0
    assert lib.sq_r2_prepare(None, None, 2048, 32, 64, 4096, None, 0, None) == 2
    assert lib.sq_r2_prepare(None, None, 2040, 32, 128, 4096, None, 0, None) == 2
    assert lib.sq_r2_prepare(None, None, 2048, 32, 128, 4096, None, 0, None) == 1
    assert lib.sq_r2_loss_grad(None, None, None, 2048, 32, 128, 4008, None, None, None, 0,
                               None) == 2
    assert lib.sq_r2_cayley_learn(None, None, None, 64, 4, 128, 256, 0.3, -1, None, None, None,
                                  0, None) == 1
    assert lib.sq_cayley_update(None, None, 0.1, 129, 1, None, None, None, 0, None) == 1
    assert lib.sq_cayley_update(None, None, 0.1, 16, 0, None, None, None, 0, None) == 0
    assert lib.sq_cayley_update(None, None, 0.1, 16, 1, None, None, None, 0, None) == 1
    assert lib.sq_cayley_workspace_bytes(128, 2) == 2 * 2 * 128 * 128 * 8
    assert lib.sq_orth_error(None, 0, 1, None, None) == 1
    # float64 device pointers must be 8-byte aligned (checked before any launch)
    assert lib.sq_orth_error(0x1004, 16, 1, 0x2000, None) == 3
    assert lib.sq_r2_random_hadamard(0x1000, 128, 1, 0x2004, None) == 3
    assert lib.sq_r2_random_hadamard(0x1000, 96, 1, 0x2000, None) == 1      # not a power of 2
    assert lib.sq_r2_loss_grad(0x1000, 0x2000, 0x3000, 64, 4, 128, 256, 0x4004, None,
                               0x5000, 1 << 30, None) == 3


def test_product_paley_matches_oracle():
    # Two independent constructions of the same pinned matrix.
    from oracle import oracle as O
    from rotation_ptq_b200.hadamard import paley_h12
    assert np.array_equal(paley_h12().astype(np.int64), O.paley1(11))


def test_binding_refuses_cpu_tensors(sq):
    import torch
    with pytest.raises(ValueError):
        sq.rotate_quant(torch.zeros(4, 256))
