"""The benchmark's GEMM roofline entry: tensor-bound above the ridge point (GEMM peak / measured
copy bandwidth), HBM-bound below it, with the quantised formats' peaks at 2x / 4x the measured
sustained bf16 rate.  Pure host arithmetic on synthetic profile totals."""
import pytest

import bench

PEAKS = {"hbm_gbs": 6458.7, "bf16_tflops": 1684.5, "bf16_tflops_sustained": 1408.5}


def test_tensor_bound_above_the_ridge():
    # a 1024^2-like step: 28.28 TFLOP of linears in 20.25 ms over 17 GB of algorithmic bytes
    r = bench.gemm_roofline(20.25, 28.28e12, 17e9, PEAKS, "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(28.28e12 / 20.25e-3 / 1e12, abs=0.1)
    assert r["peak"] == pytest.approx(1408.5)
    assert r["frac"] == pytest.approx(r["achieved"] / 1408.5, abs=1e-4)
    assert r["ridge_flop_per_byte"] == pytest.approx(1408.5e12 / 6458.7e9, abs=0.1)
    assert r["flop_per_byte"] == pytest.approx(28.28e12 / 17e9, abs=0.1)
    assert set(r["frac_of"]) == {"measured_sustained", "measured_burst", "spec_2250"}


def test_hbm_bound_below_the_ridge():
    # a tiny-model-like step: 21 FLOP per byte, the weights' read bounds the launches
    r = bench.gemm_roofline(0.31, 21e9, 1e9, PEAKS, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(1e9 / 0.31e-3 / 1e9, abs=0.1)
    assert r["peak"] == pytest.approx(6458.7)
    assert r["frac"] == pytest.approx(r["achieved"] / 6458.7, abs=1e-4)
    assert r["tflops"] == pytest.approx(21e9 / 0.31e-3 / 1e12, abs=0.01)
    assert "frac_of" not in r


@pytest.mark.parametrize("fp8,fp4,mult", [(False, False, 1.0), (True, False, 2.0), (False, True, 4.0)])
def test_quantised_peaks_scale_the_ridge(fp8, fp4, mult):
    # 500 FLOP per byte: above the bf16 ridge (218), below the NVFP4 one (872)
    r = bench.gemm_roofline(1.0, 500e9, 1e9, PEAKS, "measured", fp4=fp4, fp8=fp8)
    ridge = mult * 1408.5e12 / 6458.7e9
    assert r["ridge_flop_per_byte"] == pytest.approx(ridge, abs=0.1)
    assert r["bound"] == ("hbm" if 500 < ridge else "tensor")
    if r["bound"] == "tensor":
        assert r["peak"] == pytest.approx(mult * 1408.5)
