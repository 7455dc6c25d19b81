"""Row-wise FP8 (e4m3) block linears on the GPU (through the C ABI) against the FP8 oracle.

* quantisation of bf16 rows: codes and scales bit-exact (both sides decide each code from the same
  float32 product x * inv);
* LN-mod quantised in the same pass: within e4m3 rounding of the oracle's modulated row;
* FP8 GEMM (tcgen05 kind::f8f6f4) on the oracle's own codes: the exact sum of code products times
  both scales, up to fp32 accumulation (normalised max 1e-5 for fp32 output, 1e-2 for bf16);
* the tiny model's forward in FP8 against the oracle's FP8 forward, and the precision switch.
"""
import os

import numpy as np
import pytest
import torch

import latent_flow_matching_b200 as F
from oracle import flux_oracle as O
from oracle import fp8_oracle as Q
from synthetic import WORKLOADS, make_weights, make_inputs

pytestmark = pytest.mark.gpu
torch.set_grad_enabled(False)
DEV = "cuda"
TOL = 1e-2
FP8_V_TOL = 2e-2        # FP8 forward against the FP8 oracle: the per-step velocity bar of the bf16 path


def nmax(gpu, ref):
    gpu = torch.as_tensor(gpu).double().cpu()
    ref = torch.as_tensor(ref).double().cpu()
    return ((gpu - ref).abs().max() / ref.abs().max()).item()


def rel_l2(a, b):
    a = torch.as_tensor(a).double().cpu()
    b = torch.as_tensor(b).double().cpu()
    return ((a - b).norm() / b.norm()).item()


def rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g) * scale


def to_u8(codes):
    return codes.to(torch.float8_e4m3fn).view(torch.uint8)


def from_u8(q):
    return q.cpu().view(torch.float8_e4m3fn).to(torch.float64)


@pytest.fixture(autouse=True)
def _device_clean():
    yield
    assert F.flux_device_error() == 0


@pytest.mark.parametrize("rows,cols", [(300, 3072), (37, 12288), (5, 9216), (1, 8)])
def test_quantize_rows_bit_exact_against_oracle(rows, cols):
    x = rand((rows, cols), rows + cols) * torch.logspace(-3, 3, rows)[:, None]
    if rows > 2:
        x[2] = 0.0
    x = x.to(torch.bfloat16)
    q = torch.empty(rows, cols, dtype=torch.uint8, device=DEV)
    s = torch.empty(rows, dtype=torch.float32, device=DEV)
    F.flux_quantize_rows_e4m3(x.to(DEV), q, s)
    codes, scale = Q.quantize_rows(x.float())
    assert torch.equal(s.cpu(), scale)
    assert torch.equal(from_u8(q), codes)


@pytest.mark.parametrize("rows", [4608 + 5, 33])
def test_layernorm_modulate_fp8_within_e4m3_rounding(rows):
    x = rand((rows, 3072), 50) * 3 + 0.5
    shift, scale = rand((3072,), 51), rand((3072,), 52, 0.5)
    q = torch.empty(rows, 3072, dtype=torch.uint8, device=DEV)
    qs = torch.empty(rows, dtype=torch.float32, device=DEV)
    F.flux_layernorm_modulate_fp8(x.to(DEV), q, qs, shift.to(DEV), scale.to(DEV))
    y = O.modulate(O.layer_norm(x.double(), 1e-6), shift.double(), scale.double())
    amax = y.abs().amax(dim=1)
    assert torch.allclose(qs.cpu().double(), amax / 448.0, rtol=1e-5, atol=0)
    deq = from_u8(q) * qs.cpu().double()[:, None]
    # half an e4m3 spacing of the value (normal range) or of the scale's subnormal step, plus the
    # float32 difference of the two LayerNorm evaluations
    bound = torch.maximum(y.abs() * 2.0 ** -4, qs.cpu().double()[:, None] * 2.0 ** -10) * 1.001 + 1e-5 * amax[:, None]
    assert torch.all((deq - y).abs() <= bound)


def interleave_swiglu(w):
    """[a; b] rows -> per 128 output columns: 128 a-rows then 128 b-rows (GEMM order)."""
    f = w.shape[0] // 2
    a, b = w[:f], w[f:]
    parts = []
    for g in range(f // 128):
        parts += [a[128 * g:128 * g + 128], b[128 * g:128 * g + 128]]
    return torch.cat(parts)


@pytest.mark.parametrize("m,k,n,mode", [
    (300, 3072, 512, F.EPI_BF16_BIAS),
    (129, 128, 3072, F.EPI_F32_BIAS),
    (257, 3072, 1024, F.EPI_SWIGLU),
    (200, 9216, 384, F.EPI_RESID_GATE),
    (128 * 3 + 1, 12288, 256 + 32, F.EPI_RESID_GATE),
    (1, 128, 32, F.EPI_BF16_BIAS),
])
def test_linear_fp8_modes_on_oracle_codes(m, k, n, mode):
    a = rand((m, k), 60) * torch.logspace(-1, 1, m)[:, None]
    w = rand((n, k), 61, k ** -0.5)
    if mode == F.EPI_SWIGLU:
        w = interleave_swiglu(w)          # quantisation is per row, so row order does not matter
    b = rand((n,), 62, 0.5).to(torch.bfloat16)
    qa, sa = Q.quantize_rows(a)
    qw, sw = Q.quantize_rows(w)
    acc = torch.matmul(qa, qw.t()) * sa.double()[:, None] * sw.double()[None, :] + b.double()
    args = (to_u8(qa).to(DEV), sa.to(DEV), to_u8(qw).to(DEV), sw.to(DEV), b.to(DEV), mode)
    if mode == F.EPI_SWIGLU:
        # acc columns are in GEMM order: per 128 outputs, 128 a then 128 b
        g = acc.reshape(m, n // 256, 2, 128)
        ref = (O.silu(g[:, :, 0]) * g[:, :, 1]).reshape(m, n // 2)
        out = torch.empty(m, n // 2, device=DEV, dtype=torch.bfloat16)
        F.flux_linear_fp8(*args, out)
    elif mode == F.EPI_RESID_GATE:
        x0 = rand((m, n), 63)
        gate = rand((n,), 64)
        ref = x0.double() + gate.double() * acc
        out = x0.to(DEV)
        F.flux_linear_fp8(*args, out, gate=gate.to(DEV))
    else:
        ref = acc
        dt = torch.bfloat16 if mode == F.EPI_BF16_BIAS else torch.float32
        out = torch.empty(m, n, device=DEV, dtype=dt)
        F.flux_linear_fp8(*args, out)
    err = nmax(out, ref)
    assert err <= TOL, err
    if mode in (F.EPI_F32_BIAS, F.EPI_RESID_GATE):
        assert err < 1e-5, err            # fp32 output: the code products are exact, only summation order differs


def test_linear_fp8_full_size_sampled_rows():
    """Single-block linear1 size (4608 x 3072 -> 27648 rows of W), fp32 output, sampled rows."""
    m, k, n = 4608, 3072, 27648
    a = rand((m, k), 70).to(torch.bfloat16)
    w = rand((n, k), 71, k ** -0.5).to(torch.bfloat16)
    b = rand((n,), 72, 0.5).to(torch.bfloat16)
    qa = torch.empty(m, k, dtype=torch.uint8, device=DEV)
    sa = torch.empty(m, dtype=torch.float32, device=DEV)
    qw = torch.empty(n, k, dtype=torch.uint8, device=DEV)
    sw = torch.empty(n, dtype=torch.float32, device=DEV)
    F.flux_quantize_rows_e4m3(a.to(DEV), qa, sa)
    F.flux_quantize_rows_e4m3(w.to(DEV), qw, sw)
    out = torch.empty(m, n, device=DEV, dtype=torch.float32)
    F.flux_linear_fp8(qa, sa, qw, sw, b.to(DEV), F.EPI_F32_BIAS, out)
    rows = torch.arange(0, m, 97)
    ref = Q.linear_fp8(a[rows].float().double(), w.float().double(), b.double())
    assert nmax(out[rows], ref) < 1e-5


# ---------------------------------------------------------------------------- forward in FP8
@pytest.fixture(scope="module")
def tiny():
    w = WORKLOADS["tiny64"]
    blob, p = make_weights(w.dims, w.seed)
    model = F.FluxDiT(blob, w.dims)
    yield w, p, model
    model.close()


@pytest.mark.parametrize("n_txt,grid,refs", [(16, (4, 4), []), (131, (8, 8), [(4, 8)]), (0, (4, 6), [])])
def test_tiny_fp8_forward_against_fp8_oracle(tiny, n_txt, grid, refs):
    w, p, model = tiny
    g = torch.Generator().manual_seed(80 + n_txt)
    tok = torch.randn(grid[0] * grid[1], 128, generator=g).to(torch.bfloat16).float()
    txt = torch.randn(n_txt, 3072, generator=g).to(torch.bfloat16).float()
    ref_tok = [torch.randn(h * w_, 128, generator=g).to(torch.bfloat16).float() for h, w_ in refs]
    hq = dict(O.hyper(w.dims), fp8=True)
    want = O.forward(p, hq, tok, txt, 0.6, grid, ref_tok, refs)
    exact = O.forward(p, O.hyper(w.dims), tok, txt, 0.6, grid, ref_tok, refs)
    v = torch.empty(grid[0] * grid[1], 128, device=DEV)
    v16 = torch.empty_like(v)
    hw = refs if refs else (0, 0)
    rt = torch.cat(ref_tok).to(DEV) if refs else None
    model.forward(tok.to(DEV), grid, txt.to(DEV) if n_txt else None, 0.6, v16, rt, hw)
    model.set_precision(F.PRECISION_FP8)
    try:
        model.forward(tok.to(DEV), grid, txt.to(DEV) if n_txt else None, 0.6, v, rt, hw)
    finally:
        model.set_precision(F.PRECISION_BF16)
    err = rel_l2(v, want)
    print(f"fp8 forward vs fp8 oracle {err:.4f}, vs exact oracle {rel_l2(v, exact):.4f}, "
          f"fp8 oracle vs exact {rel_l2(want, exact):.4f}")
    assert err <= FP8_V_TOL, err
    assert rel_l2(v, exact) > rel_l2(v16, exact)           # FP8 is the coarser path
    again = torch.empty_like(v)
    model.forward(tok.to(DEV), grid, txt.to(DEV) if n_txt else None, 0.6, again, rt, hw)
    assert torch.equal(again, v16)                          # back to bf16, bit for bit


def test_tiny_fp8_sampler_against_fp8_oracle(tiny):
    w, p, model = tiny
    lat, txt, _ = make_inputs(w)
    hq = dict(O.hyper(w.dims), fp8=True)
    ref_final, ref_vs = O.sample(p, hq, torch.from_numpy(lat), torch.from_numpy(txt), 2)
    vs = []
    model.set_precision(F.PRECISION_FP8)
    try:
        final = F.flux_sample(model, torch.from_numpy(lat).to(DEV), torch.from_numpy(txt).to(DEV), 2,
                              on_step=lambda i, v: vs.append(v.cpu().clone()))
    finally:
        model.set_precision(F.PRECISION_BF16)
    for a, b in zip(vs, ref_vs):
        assert rel_l2(a, b) <= FP8_V_TOL
    assert rel_l2(final.cpu(), ref_final) <= FP8_V_TOL


def test_fp8_forward_full_size_against_bf16():
    """1024^2 workload, full model: the FP8 forward stays within a few percent of the bf16 one."""
    w = WORKLOADS["t2i1024"]
    blob, _ = make_weights(w.dims, w.seed)
    lat, txt, _ = make_inputs(w)
    model = F.FluxDiT(blob, w.dims)
    del blob
    try:
        tok = O.pack_latents(torch.from_numpy(lat)).float().to(DEV)
        tx = torch.from_numpy(txt).to(DEV)
        v16, v8 = torch.empty(w.n_img, 128, device=DEV), torch.empty(w.n_img, 128, device=DEV)
        model.forward(tok, (w.grid, w.grid), tx, 1.0, v16)
        model.set_precision(F.PRECISION_FP8)
        model.forward(tok, (w.grid, w.grid), tx, 1.0, v8)
        torch.cuda.synchronize()
        err = rel_l2(v8, v16)
        print(f"1024^2 fp8 vs bf16 forward: {err:.4f}")
        assert 1e-3 < err < 0.1, err
    finally:
        model.close()


def test_fp8_guided_batch_equals_two_single_forwards(tiny):
    """The batch-2 guided forward in FP8 returns, bit for bit, the two single-text FP8 forwards:
    every quantisation scale belongs to one row and the GEMM choice is made per sequence."""
    w, p, model = tiny
    g = torch.Generator().manual_seed(90)
    grid = (6, 4)
    tok = torch.randn(24, 128, generator=g).to(torch.bfloat16).float().to(DEV)
    tc = torch.randn(131, 3072, generator=g).to(torch.bfloat16).float().to(DEV)
    tu = torch.randn(131, 3072, generator=g).to(torch.bfloat16).float().to(DEV)
    vc, vu, a, b = (torch.empty(24, 128, device=DEV) for _ in range(4))
    model.set_precision(F.PRECISION_FP8)
    try:
        model.forward_cfg(tok, grid, tc, tu, 0.6, vc, vu)
        model.forward(tok, grid, tc, 0.6, a)
        model.forward(tok, grid, tu, 0.6, b)
    finally:
        model.set_precision(F.PRECISION_BF16)
    assert torch.equal(vc, a) and torch.equal(vu, b)
