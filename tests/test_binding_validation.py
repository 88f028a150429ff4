"""The binding rejects malformed operands before any C call (no GPU needed).

A wrong dtype, shape or layout would make a kernel read or write past the end
of a buffer on the device, so every public call checks dtype, shape,
contiguity and device of its operands (including caller-supplied outputs and
workspaces) first; these tests pass CPU tensors, so a call that got past its
checks would stop at the "no CPU path" error instead of the expected one.
"""
import pytest
import torch

import rotation_ptq_b200 as sq

u8, i8, f32, bf16, i32 = torch.uint8, torch.int8, torch.float32, torch.bfloat16, torch.int32


def z(shape, dt):
    return torch.zeros(shape, dtype=dt)


def _linear_ok(M=4, N=16, K=256):
    return dict(a_q=z((M, K // 2), u8), a_scale=z((M,), f32), w_q=z((N, K // 2), u8),
                w_scale=z((N,), f32))


@pytest.mark.parametrize("key,bad,msg", [
    ("w_q", z((16, 64), u8), "w_q must have shape"),            # short weight rows
    ("w_q", z((16, 128), i8), "w_q must be torch.uint8"),
    ("a_scale", z((3,), f32), "a_scale must have shape"),
    ("w_scale", z((16,), torch.float64), "w_scale must be torch.float32"),
    ("a_q", z((4, 256), u8)[:, ::2], "a_q must be contiguous"),
])
def test_w4a4_linear_rejects_operands(key, bad, msg):
    args = _linear_ok()
    args[key] = bad
    with pytest.raises(ValueError, match=msg):
        sq.w4a4_linear(**args)


@pytest.mark.parametrize("out_int32,out,msg", [
    (True, z((4, 16), bf16), "out must be torch.int32"),       # 4-byte sums into 2-byte slots
    (False, z((4, 16), i32), "out must be torch.bfloat16"),
    (False, z((4, 8), bf16), "out must have shape"),
])
def test_w4a4_linear_rejects_out(out_int32, out, msg):
    with pytest.raises(ValueError, match=msg):
        sq.w4a4_linear(**_linear_ok(), out_int32=out_int32, out=out)


def test_w4a4_linear_rejects_workspace_dtype():
    with pytest.raises(ValueError, match="workspace must be a contiguous uint8"):
        sq.w4a4_linear(**_linear_ok(), workspace=z((64,), f32))


def test_w4a4_linear_well_formed_reaches_device_check():
    with pytest.raises(ValueError, match="no CPU path"):
        sq.w4a4_linear(**_linear_ok())


@pytest.mark.parametrize("key,bad,msg", [
    ("a_q", z((4, 256), u8), "a_q must be torch.int8"),
    ("w_q", z((16, 64), u8), "w_q must have shape"),
    ("a_scale", z((5,), f32), "a_scale must have shape"),
])
def test_w4a8_linear_rejects_operands(key, bad, msg):
    args = dict(a_q=z((4, 256), i8), a_scale=z((4,), f32), w_q=z((16, 128), u8),
                w_scale=z((16,), f32))
    args[key] = bad
    with pytest.raises(ValueError, match=msg):
        sq.w4a8_linear(**args)


def test_w4a8_linear_rejects_out():
    with pytest.raises(ValueError, match="out must be torch.int32"):
        sq.w4a8_linear(z((4, 256), i8), z((4,), f32), z((16, 128), u8), z((16,), f32),
                       out=z((4, 16), bf16), out_i32=True)


@pytest.mark.parametrize("fn,x,aq,asc,msg", [
    (sq.rotate_quant, z((8, 256), bf16), z((8, 64), u8), None, "a_q must have shape"),
    (sq.rotate_quant, z((8, 256), bf16), z((8, 128), i8), None, "a_q must be torch.uint8"),
    (sq.rotate_quant, z((8, 256), bf16), None, z((7,), f32), "a_scale must have shape"),
    (sq.rotate_quant8, z((8, 256), bf16), z((8, 128), i8), None, "a_q must have shape"),
    (sq.rotate_quant8, z((8, 256), bf16), z((8, 256), u8), None, "a_q must be torch.int8"),
    (sq.rotate_quant8, z((8, 256), bf16), None, z((8,), torch.float16), "a_scale must be"),
    (sq.swiglu_rotate_quant, z((8, 512), bf16), z((8, 64), u8), None, "a_q must have shape"),
    (sq.swiglu_rotate_quant, z((8, 512), bf16), None, z((9,), f32), "a_scale must have shape"),
])
def test_rotate_quant_rejects_outputs(fn, x, aq, asc, msg):
    with pytest.raises(ValueError, match=msg):
        fn(x, None, 1, 1.0, a_q=aq, a_scale=asc)


def test_kv_rotate_quant_rejects_operands():
    T, hq, hkv = 4, 8, 2
    q, k, v = z((T, hq, 128), bf16), z((T, hkv, 128), bf16), z((T, hkv, 128), bf16)
    with pytest.raises(ValueError, match="pos must be torch.int32"):
        sq.kv_rotate_quant(q, k, v, z((T,), torch.int64))
    with pytest.raises(ValueError, match="v must have shape"):
        sq.kv_rotate_quant(q, k, z((T, hkv, 64), bf16), z((T,), i32))
    with pytest.raises(ValueError, match="cos must be torch.float32"):
        sq.kv_rotate_quant(q, k, v, z((T,), i32), z((16, 64), torch.float64), z((16, 64), f32))
    out = dict(q_out=z((T, hq, 128), bf16), k_cache=z((T, hkv, 32), u8),
               k_scale=z((T, hkv), f32), k_zero=z((T, hkv), u8),
               v_cache=z((T, hkv, 64), u8), v_scale=z((T, hkv), f32), v_zero=z((T, hkv), u8))
    with pytest.raises(ValueError, match=r"out\[k_cache\] must have shape"):
        sq.kv_rotate_quant(q, k, v, z((T,), i32), out=out)


def test_kv_dequant_rejects_operands():
    with pytest.raises(ValueError, match="scale must have shape"):
        sq.kv_dequant(z((4, 2, 64), u8), z((4, 3), f32), z((4, 2), u8))
    with pytest.raises(ValueError, match="out must have shape"):
        sq.kv8_dequant(z((4, 2, 128), u8), z((4, 2), f32), z((4, 2), u8), out=z((4, 2, 64), bf16))


def test_kv_decode_rejects_cache_width():
    B, S, hq, hkv = 2, 8, 8, 2
    args = [z((B, hq, 128), bf16), z((B * S, hkv, 128), u8), z((B * S, hkv), f32),
            z((B * S, hkv), u8), z((B * S, hkv, 128), u8), z((B * S, hkv), f32),
            z((B * S, hkv), u8), z((B,), i32), S]
    with pytest.raises(ValueError, match="d/2 bytes"):
        sq.kv4_decode_attention(*args)            # 8-bit rows given to the 4-bit kernel
    args[7] = z((B + 1,), i32)
    with pytest.raises(ValueError, match="lengths must have shape"):
        sq.kv8_decode_attention(*args)
