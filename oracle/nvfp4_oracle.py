"""NVFP4 (block-scaled 4-bit) linear layers for the CPU oracle.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/`` and ``bench.py``'s CPU
legs import it; the product path never does.

Source: "FLUX.3 Image Klein in Diffusers: Architektur, Layout-Steuerung und
Systemanforderungen im Überblick" (mindverse), section "Hardwareanforderungen, Quantisierung und
Inferenzlatenz": besides fp8r the transformer ships as nvfp4, whose acceleration needs a
Blackwell GPU.  The pages name the format only.  NVFP4 as NVIDIA publishes it: 4-bit e2m1
values (1 sign, 2 exponent bits with bias 1, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3,
4, 6), one e4m3 scale per block of 16 consecutive elements along the reduction dimension, and
a second-level fp32 scale.

Readings where the pages are silent:
* the second-level scale is per row (per output row of a weight matrix and per token row of an
  activation), like the row-wise FP8 format, instead of per tensor;
* quantisation of one row x (all values rounded to float32 as below):
      amax  = max_j |x_j|,  S = amax / 2688  (2688 = 6 * 448: the largest e2m1 times the
              largest e4m3),  inv = 448 / amax;
      block b (16 elements): s_b = e4m3(amax_b * inv), round to nearest even, saturating;
      d_b = s_b * S,  r_b = 1 / d_b,  code_j = e2m1(x_j * r_b), round to nearest even
              (ties to the even mantissa), saturating at +-6;
      value_j = code_j * s_b * S;
  an all-zero row, or a block whose scale rounds to 0, has codes 0;
* y = sum over blocks of (codes_x . codes_w) s_bx s_bw, times S_x S_w, plus the bias;
* it applies where the row-wise FP8 format does: the linears inside the transformer blocks; an
  activation row is quantised from the values the layer receives (the format defines no other
  rounding before the quantiser), its scale and code decisions taken in float32 as above.
"""
from __future__ import annotations

import torch

from .fp8_oracle import round_e4m3

__all__ = ["E2M1_MAX", "BLOCK", "E2M1_VALUES", "round_e2m1", "quantize_rows_nvfp4", "dequantize_nvfp4",
           "linear_nvfp4"]

E2M1_MAX = 6.0
BLOCK = 16
E2M1_VALUES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)    # magnitude of code 0..7


def round_e2m1(x: torch.Tensor) -> torch.Tensor:
    """Nearest e2m1 value, ties to the even code (mantissa bit 0), saturating at +-6, as float64.

    e2m1 magnitudes: subnormal 0.5 (exponent field 0), normal 2^(e-1) (1 + m/2) for e = 1..3.
    In [0, 2) the spacing is 0.5, in [2, 4) it is 1, in [4, 6] it is 2."""
    x = torch.as_tensor(x, dtype=torch.float64)
    a = x.abs().clamp(max=E2M1_MAX)
    quantum = torch.where(a < 2.0, torch.full_like(a, 0.5), torch.where(a < 4.0, torch.ones_like(a),
                                                                        torch.full_like(a, 2.0)))
    r = torch.round(a / quantum) * quantum                  # half to even on the quantum grid
    return torch.copysign(r.clamp(max=E2M1_MAX), x)


def quantize_rows_nvfp4(x: torch.Tensor):
    """(codes [rows, k] as float64 e2m1 values, block scales [rows, k/16] as float64 e4m3 values,
    row scales S [rows] float32) of x [rows, k], k a multiple of 16."""
    x32 = torch.as_tensor(x).to(torch.float32)
    rows, k = x32.shape
    if k % BLOCK:
        raise ValueError("k must be a multiple of 16")
    f32 = torch.float32
    amax = x32.abs().amax(dim=1)
    S = amax / torch.tensor(6.0 * 448.0, dtype=f32)
    inv = torch.where(amax > 0, torch.tensor(448.0, dtype=f32) / amax, torch.zeros_like(amax))
    xb = x32.reshape(rows, k // BLOCK, BLOCK)
    amax_b = xb.abs().amax(dim=2)
    sb = round_e4m3((amax_b * inv[:, None]).to(torch.float64))            # e4m3 of a float32 product
    d = (sb.to(f32) * S[:, None])                                          # float32 product
    r = torch.where(d > 0, torch.tensor(1.0, dtype=f32) / d, torch.zeros_like(d))
    codes = round_e2m1((xb * r[:, :, None]).to(torch.float64)).reshape(rows, k)
    return codes, sb, S


def dequantize_nvfp4(codes: torch.Tensor, sb: torch.Tensor, S: torch.Tensor) -> torch.Tensor:
    rows, k = codes.shape
    v = codes.reshape(rows, k // BLOCK, BLOCK) * sb[:, :, None]
    return v.reshape(rows, k) * S.to(torch.float64)[:, None]


def linear_nvfp4(x: torch.Tensor, w: torch.Tensor, b: torch.Tensor | None) -> torch.Tensor:
    """x W^T + b with x (per token row) and W (per output row) quantised to NVFP4; the block
    products are summed exactly (float64) and scaled by both rows' second-level scales."""
    dtype = torch.as_tensor(x).dtype
    qx, bx, sx = quantize_rows_nvfp4(x)
    qw, bw, sw = quantize_rows_nvfp4(w)
    rx, k = qx.shape
    vx = (qx.reshape(rx, k // BLOCK, BLOCK) * bx[:, :, None]).reshape(rx, k)
    vw = (qw.reshape(qw.shape[0], k // BLOCK, BLOCK) * bw[:, :, None]).reshape(qw.shape[0], k)
    y = torch.matmul(vx, vw.t()) * sx.to(torch.float64)[:, None] * sw.to(torch.float64)[None, :]
    y = y.to(dtype)
    return y if b is None else y + b
