"""Host-side checks of the C ABI: the library loads, exports what the header declares,
agrees with the blob generator on sizes, and rejects bad arguments with error codes.
None of these tests launches a kernel, so they run without a GPU."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import latent_flow_matching_b200 as F
from latent_flow_matching_b200 import build as fbuild
from synthetic import FluxDims, Flux3Dims, FULL_DIMS, TINY_DIMS, F3_FULL_DIMS, F3_TINY_DIMS, blob_layout
from synthetic.flux_inputs import HEADER_BYTES

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fluxdit.h")


@pytest.fixture(scope="module")
def L():
    fbuild.build()
    return F.lib()


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"FLUX_API\s+[\w\s\*]*?\b(flux3?_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ("flux_dit_create", "flux_dit_destroy", "flux_dit_forward", "flux_euler_step",
                     "flux_pack_latents", "flux_unpack_latents", "flux_joint_attention", "flux_get_error"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", F.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (flux3?_\w+)", out))
    assert set(declared_symbols()) <= exported
    assert set(F.EXPORTED) == set(declared_symbols())


@pytest.mark.parametrize("dims", [FULL_DIMS, TINY_DIMS,
                                  FluxDims(n_double=2, n_single=3, hidden=256, heads=2, mlp_hidden=512,
                                           txt_dim=192, t_freq_dim=256)])
def test_blob_size_matches_generator(L, dims):
    _, total = blob_layout(dims)
    assert F.flux_blob_expected_bytes(dims) == total


def test_full_model_parameter_count():
    layout, total = blob_layout(FULL_DIMS)
    n = sum(e[4] for e in layout)
    assert 4.8e9 < n < 4.9e9           # 5 double + 20 single blocks at width 3072
    assert total - HEADER_BYTES >= 2 * n


def test_invalid_config_gives_zero(L):
    bad = FluxDims(head_dim=64, hidden=64 * 24)
    assert F.flux_blob_expected_bytes(bad) == 0


def _tiny_blob():
    dims = FluxDims(n_double=1, n_single=1, hidden=256, heads=2, mlp_hidden=256, txt_dim=128)
    _, total = blob_layout(dims)
    from synthetic.flux_inputs import _header
    from synthetic import tensor_specs
    blob = np.zeros(total, np.uint8)
    blob[:HEADER_BYTES] = np.frombuffer(_header(dims, len(tensor_specs(dims)), total), np.uint8)
    return dims, blob


def test_create_rejects_corrupt_blob(L):
    dims, blob = _tiny_blob()
    bad = blob.copy()
    bad[0] = ord("X")
    h = L.flux_dit_create(ctypes.c_void_p(bad.ctypes.data), bad.nbytes, None, None)
    assert not h
    assert "FLUXDIT" in F.get_error()
    h = L.flux_dit_create(ctypes.c_void_p(blob.ctypes.data), blob.nbytes - 256, None, None)
    assert not h
    assert "size" in F.get_error()
    h = L.flux_dit_create(None, 0, None, None)
    assert not h
    assert L.flux_get_error_code() == F.FLUX_EINVAL          # a bad argument, not an allocation


def test_allocation_hook_needs_no_device(L):
    """Arming and disarming the out-of-memory test hook touch no device (this runs without a GPU),
    and a call rejected for its arguments while the hook is armed still reports FLUX_EINVAL."""
    L.flux_test_fail_alloc_after(0)
    h = L.flux_dit_create(None, 0, None, None)
    assert not h and L.flux_get_error_code() == F.FLUX_EINVAL
    L.flux_test_fail_alloc_after(-1)
    L.flux_test_fail_alloc_after(-5)


def test_create_rejects_config_mismatch(L):
    dims, blob = _tiny_blob()
    other = F.FluxConfig.from_dims(FluxDims(n_double=2, n_single=1, hidden=256, heads=2, mlp_hidden=256,
                                            txt_dim=128))
    h = L.flux_dit_create(ctypes.c_void_p(blob.ctypes.data), blob.nbytes, ctypes.byref(other), None)
    assert not h
    assert "config" in F.get_error()


def test_entry_points_reject_bad_arguments(L):
    p = ctypes.c_void_p(16)            # never dereferenced: validation fails first
    assert L.flux_pack_latents(None, p, 8, 8, None) == F.FLUX_EINVAL
    assert L.flux_pack_latents(p, p, 7, 8, None) == F.FLUX_EINVAL
    assert "even" in F.get_error()
    assert L.flux_unpack_latents(p, p, 8, 0, None) == F.FLUX_EINVAL
    assert L.flux_pack_latents(ctypes.c_void_p(24), p, 8, 8, None) == F.FLUX_EINVAL   # 8-byte aligned only
    assert "aligned" in F.get_error()
    assert L.flux_unpack_latents(p, ctypes.c_void_p(20), 8, 8, None) == F.FLUX_EINVAL
    assert L.flux_joint_attention(p, p, p, p, 10, 2, 64, 0.1, None) == F.FLUX_EINVAL
    assert "head_dim" in F.get_error()
    assert L.flux_joint_attention(p, p, p, p, 0, 2, 128, 0.1, None) == F.FLUX_EINVAL
    assert L.flux_linear(p, 10, 100, 100, p, 64, p, 0, p, 64, None, None) == F.FLUX_EINVAL   # k % 64
    assert L.flux_linear(p, 10, 128, 128, p, 128, p, 2, p, 64, None, None) == F.FLUX_EINVAL  # swiglu n % 256
    assert L.flux_linear(p, 10, 128, 128, p, 128, p, 3, p, 128, None, None) == F.FLUX_EINVAL  # gate missing
    assert L.flux_linear(p, 10, 128, 128, p, 128, p, 9, p, 128, None, None) == F.FLUX_EINVAL
    assert L.flux_layernorm_modulate(p, p, 4, 3, p, p, 1e-6, None) == F.FLUX_EINVAL
    assert L.flux_qk_rmsnorm_rope(p, 4, 100, 0, 1, p, p, p, 1e-6, None) == F.FLUX_EINVAL
    assert L.flux_dit_forward(None, p, 8, 8, p, 4, None, 0, 0, 1.0, p, None) == F.FLUX_EINVAL
    assert L.flux_dit_set_active_blocks(None, 1, 1) == F.FLUX_EINVAL
    assert L.flux_dit_modulation_size(None) == 0
    L.flux_dit_destroy(None)


def test_guided_update_and_wait_self_test_reject_bad_arguments(L):
    p = ctypes.c_void_p(16)            # never dereferenced: validation fails first
    assert L.flux_cfg_euler_step_out(p, p, p, None, 8, 3.5, -0.25, None) == F.FLUX_EINVAL     # no v_guided
    assert L.flux_cfg_euler_step_out(p, p, p, ctypes.c_void_p(20), 8, 3.5, -0.25, None) == F.FLUX_EINVAL
    assert "aligned" in F.get_error()
    assert L.flux_cfg_euler_step_out(p, p, p, p, 8, float("inf"), -0.25, None) == F.FLUX_EINVAL
    assert L.flux_selftest_bounded_wait(0, 0, None) == F.FLUX_EINVAL                        # no limit
    assert L.flux_selftest_bounded_wait(2_000_000_000, 0, None) == F.FLUX_EINVAL            # above 1 s
    assert L.flux_selftest_bounded_wait(1000, 2, None) == F.FLUX_EINVAL


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(4, 4)
    with pytest.raises(ValueError):
        F._ptr(x, torch.float32, "x")


def test_product_path_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "latent_flow_matching_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "oracle" not in src, f


# ---------------------------------------------------------------------------- FLUX.3 entry points
MICRO3 = Flux3Dims(n_mode=1, n_joint=2, hidden=256, heads=2, mlp_hidden=256, txt_dim=192, t_freq_dim=256,
                   flow_map=False)


@pytest.mark.parametrize("dims", [F3_FULL_DIMS, F3_TINY_DIMS, MICRO3])
def test_flux3_blob_size_matches_generator(L, dims):
    _, total = blob_layout(dims)
    assert F.flux3_blob_expected_bytes(dims) == total


def test_flux3_invalid_config_gives_zero(L):
    assert F.flux3_blob_expected_bytes(Flux3Dims(heads=3, hidden=384)) == 0          # odd head count
    assert F.flux3_blob_expected_bytes(Flux3Dims(flow_map=2)) == 0


def _micro3_blob():
    from synthetic.flux_inputs import _header
    from synthetic import tensor_specs
    _, total = blob_layout(MICRO3)
    blob = np.zeros(total, np.uint8)
    blob[:HEADER_BYTES] = np.frombuffer(_header(MICRO3, len(tensor_specs(MICRO3)), total), np.uint8)
    return blob


def test_flux3_create_rejects_corrupt_blob_and_mismatch(L):
    blob = _micro3_blob()
    bad = blob.copy()
    bad[3] = ord("Z")
    assert not L.flux3_dit_create(ctypes.c_void_p(bad.ctypes.data), bad.nbytes, None, None)
    assert "FLUX3DT" in F.get_error()
    assert not L.flux3_dit_create(ctypes.c_void_p(blob.ctypes.data), blob.nbytes - 512, None, None)
    assert "size" in F.get_error()
    other = F.Flux3Config.from_dims(Flux3Dims(n_mode=2, n_joint=2, hidden=256, heads=2, mlp_hidden=256,
                                              txt_dim=192, flow_map=False))
    assert not L.flux3_dit_create(ctypes.c_void_p(blob.ctypes.data), blob.nbytes, ctypes.byref(other), None)
    assert "config" in F.get_error()
    # a FLUX.2 blob is not a FLUX.3 blob and the other way round
    assert not L.flux_dit_create(ctypes.c_void_p(blob.ctypes.data), blob.nbytes, None, None)


def test_flux3_entry_points_reject_bad_arguments(L):
    p = ctypes.c_void_p(16)            # never dereferenced: validation fails first
    lens = (ctypes.c_int * 3)(4, 5, 6)
    assert L.flux_joint_attention_segments(p, p, p, p, 0, lens, 2, 128, 0.1, None) == F.FLUX_EINVAL
    assert L.flux_joint_attention_segments(p, p, p, p, 5, lens, 2, 128, 0.1, None) == F.FLUX_EINVAL
    assert L.flux_joint_attention_segments(p, p, p, p, 3, lens, 2, 64, 0.1, None) == F.FLUX_EINVAL
    assert "head_dim" in F.get_error()
    neg = (ctypes.c_int * 2)(4, -1)
    assert L.flux_joint_attention_segments(p, p, p, p, 2, neg, 2, 128, 0.1, None) == F.FLUX_EINVAL
    assert L.flux_joint_attention_segments(p, p, p, p, 2, None, 2, 128, 0.1, None) == F.FLUX_EINVAL
    assert L.flux3_dit_forward(None, p, 8, 8, p, 4, None, 0, None, 1.0, 0.5, p, None) == F.FLUX_EINVAL
    assert L.flux3_dit_set_active_blocks(None, 1, 1) == F.FLUX_EINVAL
    assert L.flux3_dit_modulation_size(None) == 0
    L.flux3_dit_destroy(None)


@pytest.mark.parametrize("rows,k", [(1, 64), (128, 64), (129, 3072), (4608, 12288), (0, 256), (300, 16384)])
def test_nvfp4_scale_bytes_is_whole_128_row_blocks(L, rows, k):
    """One 512-byte tile per 128 rows (rounded up) and 64 elements of the row."""
    assert F.flux_nvfp4_scale_bytes(rows, k) == -(-rows // 128) * (k // 64) * 512


def test_nvfp4_scale_bytes_rejects_bad_sizes(L):
    for rows, k in ((10, 32), (10, 100), (-1, 64), (10, 0)):
        assert F.flux_nvfp4_scale_bytes(rows, k) == 0


def test_low_precision_entry_points_reject_bad_arguments(L):
    """Shape, mode and alignment checks of the FP8 and NVFP4 entry points fail before any launch."""
    p, p8 = ctypes.c_void_p(16), ctypes.c_void_p(24)
    E = F.FLUX_EINVAL
    assert L.flux_quantize_rows_e4m3(p, 4, 12, 16, p, 16, p, None) == E                  # cols % 8
    assert L.flux_quantize_rows_e4m3(p, 4, 16, 8, p, 16, p, None) == E                   # ldx < cols
    assert L.flux_quantize_rows_e4m3(p8, 4, 16, 16, p, 16, p, None) == E                 # x 8-byte aligned
    assert L.flux_layernorm_modulate_fp8(p, p, p, 4, 3000, p, p, 1e-6, None) == E
    assert L.flux_linear_fp8(p, p, 4, 64, 64, p, p, 32, p, 1, p, 32, None, None) == E     # k % 128
    assert L.flux_linear_fp8(p, p, 4, 128, 128, p, p, 32, p, 3, p, 32, None, None) == E   # gate missing
    assert L.flux_linear_fp8(p, p, 4, 128, 128, p, p, 64, p, 2, p, 32, None, None) == E   # SwiGLU n % 256
    assert L.flux_quantize_rows_nvfp4(p, 4, 96, 96, p, 48, p, p, None) == E              # k % 64
    assert L.flux_quantize_rows_nvfp4(p, 4, 16448, 16448, p, 8224, p, p, None) == E      # k > 16384
    assert L.flux_quantize_rows_nvfp4(p, 4, 128, 128, p, 72, p, p, None) == E            # ldq % 16
    assert L.flux_layernorm_modulate_nvfp4(p, p, p, p, 4, 1536, p, p, 1e-6, None) == E
    assert "dim" in F.get_error()
    assert L.flux_linear_nvfp4(p, p, p, 4, 128, 64, p, p, p, 32, p, 1, p, 32, None, None) == E    # k % 256
    assert L.flux_linear_nvfp4(p, p, p, 4, 256, 128, p, p, p, 32, p, 4, p, 32, None, None) == E   # mode
    assert L.flux_linear_nvfp4(p8, p, p, 4, 256, 128, p, p, p, 32, p, 1, p, 32, None, None) == E  # alignment
