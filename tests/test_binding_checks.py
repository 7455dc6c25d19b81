"""The Python binding checks every buffer against the sizes the call touches before anything is
launched (the C ABI takes plain pointers and cannot).  CPU tensors: a mis-sized buffer raises
FluxShapeError; a well-sized one gets as far as the device-pointer check ("must be a CUDA
tensor"), which shows the size checks let it through."""
import pytest
import torch

import latent_flow_matching_b200 as F


def shape_error(fn, *args, **kw):
    with pytest.raises(F.FluxShapeError):
        fn(*args, **kw)


def passes_size_checks(fn, *args, **kw):
    with pytest.raises(ValueError) as e:
        fn(*args, **kw)
    assert not isinstance(e.value, F.FluxShapeError), e.value
    assert "CUDA" in str(e.value)


def z(*shape, dtype=torch.float32):
    return torch.zeros(*shape, dtype=dtype)


def bf(*shape):
    return z(*shape, dtype=torch.bfloat16)


def u8(*shape):
    return z(*shape, dtype=torch.uint8)


def test_shape_error_is_both_a_flux_error_and_a_value_error():
    e = F.FluxShapeError("x")
    assert isinstance(e, F.FluxError) and isinstance(e, ValueError) and e.code == F.FLUX_EINVAL


def test_latent_space_kernels():
    passes_size_checks(F.flux_pack_latents, z(32, 8, 6), z(12, 128))
    shape_error(F.flux_pack_latents, z(32, 8, 6), z(11, 128))
    shape_error(F.flux_pack_latents, z(16, 8, 6), z(6, 128))
    passes_size_checks(F.flux_unpack_latents, z(12, 128), z(32, 8, 6))
    shape_error(F.flux_unpack_latents, z(12, 64), z(32, 8, 6))
    passes_size_checks(F.flux_euler_step, z(10), z(10), 0.5)
    shape_error(F.flux_euler_step, z(10), z(9), 0.5)
    passes_size_checks(F.flux_cfg_euler_step, z(10), z(10), z(10), 2.0, 0.5)
    shape_error(F.flux_cfg_euler_step, z(10), z(10), z(5), 2.0, 0.5)
    passes_size_checks(F.flux_cfg_euler_step, z(10), z(10), z(10), 2.0, 0.5, None, z(10))
    shape_error(F.flux_cfg_euler_step, z(10), z(10), z(10), 2.0, 0.5, None, z(9))
    passes_size_checks(F.flux_blend_latents, z(4, 4), z(4, 4), 0.3, z(4, 4))
    shape_error(F.flux_blend_latents, z(4, 4), z(4, 4), 0.3, z(4, 3))


def test_attention():
    q = bf(10, 2, 128)
    passes_size_checks(F.flux_joint_attention, q, bf(10, 2, 128), bf(10, 2, 128), bf(10, 2, 128))
    shape_error(F.flux_joint_attention, q, bf(9, 2, 128), bf(10, 2, 128), bf(10, 2, 128))
    shape_error(F.flux_joint_attention, q, bf(10, 2, 128), bf(10, 2, 128), bf(10, 1, 128))
    shape_error(F.flux_joint_attention_batch, q, q, q, bf(8, 2, 128), 2)
    shape_error(F.flux_joint_attention_segments, q, q, bf(10, 2, 64), q, [4, 6])


@pytest.mark.parametrize("mode,out,gate", [
    (F.EPI_BF16_BIAS, (40, 64, torch.bfloat16), None),
    (F.EPI_F32_BIAS, (40, 64, torch.float32), None),
    (F.EPI_SWIGLU, (40, 32, torch.bfloat16), None),
    (F.EPI_RESID_GATE, (40, 64, torch.float32), 64),
])
def test_linear_output_buffers(mode, out, gate):
    a, w, b = bf(40, 128), bf(64, 128), bf(64)
    r, c, dt = out
    g = None if gate is None else z(gate)
    passes_size_checks(F.flux_linear, a, w, b, mode, z(r, c, dtype=dt), g)
    shape_error(F.flux_linear, a, w, b, mode, z(r - 1, c, dtype=dt), g)          # too few rows
    shape_error(F.flux_linear, a, w, b, mode, z(r, c - 1, dtype=dt), g)          # too few columns
    wrong = torch.float32 if dt == torch.bfloat16 else torch.bfloat16
    shape_error(F.flux_linear, a, w, b, mode, z(r, c, dtype=wrong), g)           # output dtype of another mode
    shape_error(F.flux_linear, a, bf(64, 64), b, mode, z(r, c, dtype=dt), g)     # w of another k
    shape_error(F.flux_linear, a, w, bf(32), mode, z(r, c, dtype=dt), g)         # short bias
    shape_error(F.flux_linear, z(40, 128), w, b, mode, z(r, c, dtype=dt), g)     # a not bf16
    if mode == F.EPI_RESID_GATE:
        shape_error(F.flux_linear, a, w, b, mode, z(r, c), None)
        shape_error(F.flux_linear, a, w, b, mode, z(r, c), z(63))


def test_quantisers_and_low_precision_linears():
    x = bf(40, 256)
    passes_size_checks(F.flux_quantize_rows_e4m3, x, u8(40, 256), z(40))
    shape_error(F.flux_quantize_rows_e4m3, x, u8(39, 256), z(40))
    shape_error(F.flux_quantize_rows_e4m3, x, u8(40, 256), z(39))
    shape_error(F.flux_quantize_rows_e4m3, z(40, 256), u8(40, 256), z(40))       # x not bf16
    shape_error(F.flux_quantize_rows_e4m3, x, bf(40, 256), z(40))                # q not bytes
    sfb = F.flux_nvfp4_scale_bytes(40, 256)
    passes_size_checks(F.flux_quantize_rows_nvfp4, x, u8(40, 128), u8(sfb), z(40))
    shape_error(F.flux_quantize_rows_nvfp4, x, u8(40, 127), u8(sfb), z(40))
    shape_error(F.flux_quantize_rows_nvfp4, x, u8(40, 128), u8(sfb - 1), z(40))
    xf = z(40, 1024)
    passes_size_checks(F.flux_layernorm_modulate_fp8, xf, u8(40, 1024), z(40), z(1024), z(1024))
    shape_error(F.flux_layernorm_modulate_fp8, xf, u8(40, 1000), z(40), z(1024), z(1024))
    sfl = F.flux_nvfp4_scale_bytes(40, 1024)
    passes_size_checks(F.flux_layernorm_modulate_nvfp4, xf, u8(40, 512), u8(sfl), z(40), z(1024), z(1024))
    shape_error(F.flux_layernorm_modulate_nvfp4, xf, u8(40, 512), u8(sfl), z(40), z(1023), z(1024))
    passes_size_checks(F.flux_linear_fp8, u8(40, 256), z(40), u8(64, 256), z(64), bf(64), F.EPI_F32_BIAS, z(40, 64))
    shape_error(F.flux_linear_fp8, u8(40, 256), z(39), u8(64, 256), z(64), bf(64), F.EPI_F32_BIAS, z(40, 64))
    sfa, sfw = F.flux_nvfp4_scale_bytes(40, 256), F.flux_nvfp4_scale_bytes(64, 256)
    args = (u8(40, 128), u8(sfa), z(40), u8(64, 128), u8(sfw), z(64), bf(64), F.EPI_F32_BIAS)
    passes_size_checks(F.flux_linear_nvfp4, *args, z(40, 64))
    shape_error(F.flux_linear_nvfp4, *args, z(40, 63))
    shape_error(F.flux_linear_nvfp4, bf(40, 128), *args[1:], z(40, 64))          # codes not bytes
    shape_error(F.flux_linear_nvfp4, u8(40, 128), u8(sfa - 512), *args[2:], z(40, 64))


def test_norm_rope_kernels():
    x = z(12, 256)
    passes_size_checks(F.flux_layernorm_modulate, x, bf(12, 256), z(256), z(256))
    shape_error(F.flux_layernorm_modulate, x, bf(12, 255), z(256), z(256))
    shape_error(F.flux_layernorm_modulate, x, bf(12, 256), z(255), z(256))
    passes_size_checks(F.flux_rope_table, z(7 + 12, 64, 2), 7, (3, 4))
    shape_error(F.flux_rope_table, z(7 + 11, 64, 2), 7, (3, 4))
    qkv, g, table = bf(5, 3 * 256), bf(128), z(5, 64, 2)
    passes_size_checks(F.flux_qk_rmsnorm_rope, qkv, 256, 2, g, g, table)
    shape_error(F.flux_qk_rmsnorm_rope, qkv, 600, 2, g, g, table)                 # k heads past the row
    shape_error(F.flux_qk_rmsnorm_rope, qkv, 256, 2, g, g, z(4, 64, 2))
    a, w, b = bf(5, 64), bf(3 * 256, 64), bf(3 * 256)
    passes_size_checks(F.flux_qkv_projection, a, w, b, 2, g, g, z(9, 64, 2), bf(5, 768), 4)
    shape_error(F.flux_qkv_projection, a, w, b, 2, g, g, z(8, 64, 2), bf(5, 768), 4)   # table rows 4..8
    shape_error(F.flux_qkv_projection, a, bf(3 * 256, 32), b, 2, g, g, z(9, 64, 2), bf(5, 768), 4)


def test_forward_buffers_are_checked_before_the_library():
    """The model-level shape check is a module function, so it runs without a model."""
    check = F._check_forward_shapes
    check(None, z(16, 128), (4, 4), [z(3, 64)], [(2, 2)], z(4, 128), [z(16, 128)])
    with pytest.raises(F.FluxShapeError):
        check(None, z(16, 128), (2, 4), [None], [], None, [z(16, 128)])             # grid of 8 tokens
    with pytest.raises(F.FluxShapeError):
        check(None, z(16, 128), (4, 4), [None], [], None, [z(15, 128)])             # short output
    with pytest.raises(F.FluxShapeError):
        check(None, z(16, 128), (4, 4), [None], [(2, 2)], None, [z(16, 128)])       # reference grid, no tokens
    with pytest.raises(F.FluxShapeError):
        check(None, z(16, 128), (4, 4), [z(3)], [], None, [z(16, 128)])             # text not 2-D
