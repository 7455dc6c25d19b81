"""NVFP4 block linears on the GPU (through the C ABI) against the NVFP4 oracle.

* quantisation of bf16 rows: codes, block scales and row scales bit-exact (both sides take every
  decision from the same float32 values), read back from the tensor-core byte layouts;
* NVFP4 GEMM (tcgen05 kind::mxf4nvf4 with block scales) on the oracle's own codes and scales:
  the exact sum of block products times both row scales, up to fp32 accumulation (normalised
  max 1e-5 for fp32 output, 1e-2 for bf16), in every epilogue mode, with ragged row counts and
  several tiles (so both overlapping accumulator buffers are used);
* full-size linear1 with sampled rows.
"""
import pytest
import torch

import latent_flow_matching_b200 as F
from oracle import flux_oracle as O
from oracle import nvfp4_oracle as Q4

pytestmark = pytest.mark.gpu
torch.set_grad_enabled(False)
DEV = "cuda"
TOL = 1e-2
# NVFP4 forward against the NVFP4 oracle.  The NVFP4 forward is not continuous in its quantiser
# inputs: a value that crosses a rounding boundary moves by a whole e2m1 step (1/4 to 1/2 of it).
# On the CPU the oracle alone moves by sigma = 2-3 % when every quantiser input is perturbed by one
# bf16 rounding, and sits eps = 3.5-6 % from the exact forward (tests/test_oracle_nvfp4_pins.py).
# The GPU path's attention runs on bf16 operands, so its quantiser inputs carry at least that
# perturbation and the bf16 path's 2e-2 is below this format's noise floor.  The bar is 3e-2, the
# top of the pinned sigma range and below the smallest eps (a path that did not quantise fails it),
# and the GPU must sit nearer the NVFP4 oracle than the exact forward by NV4_RATIO.
NV4_V_TOL = 3e-2
NV4_RATIO = 0.6


def nmax(gpu, ref):
    gpu = torch.as_tensor(gpu).double().cpu()
    ref = torch.as_tensor(ref).double().cpu()
    return ((gpu - ref).abs().max() / ref.abs().max()).item()


def rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g) * scale


# ---------------------------------------------------------------- byte layouts (test-side encode / decode)
MAGS = torch.tensor(Q4.E2M1_VALUES, dtype=torch.float64)


def encode_codes(vals):
    """e2m1 values [r, k] -> packed bytes [r, k/2] (element 2i in the low nibble)."""
    idx = (vals.abs()[..., None] == MAGS).double().argmax(dim=-1)
    nib = idx | ((vals < 0).long() << 3)
    nib = nib.to(torch.uint8)
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).contiguous()


def decode_codes(packed):
    p = packed.cpu().long()
    nib = torch.stack([p & 15, p >> 4], dim=-1).reshape(p.shape[0], -1)
    mag = MAGS[nib & 7]
    return torch.where((nib & 8) != 0, -mag, mag)


def sf_index(rows, k):
    """Byte offset of block scale (r, g) in the tensor-core layout, as a [rows, k/16] tensor."""
    r = torch.arange(rows)[:, None]
    g = torch.arange(k // 16)[None, :]
    return ((r // 128) * (k // 64) + g // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + g % 4


def encode_sf(sb, rows, k):
    out = torch.zeros(F.flux_nvfp4_scale_bytes(rows, k), dtype=torch.uint8)
    out[sf_index(rows, k).reshape(-1)] = sb.to(torch.float8_e4m3fn).view(torch.uint8).reshape(-1)
    return out


def decode_sf(buf, rows, k):
    b = buf.cpu()[sf_index(rows, k).reshape(-1)].reshape(rows, k // 16)
    return b.view(torch.float8_e4m3fn).to(torch.float64)


def quantize_gpu(x):
    rows, k = x.shape
    q = torch.empty(rows, k // 2, dtype=torch.uint8, device=DEV)
    sf = torch.zeros(F.flux_nvfp4_scale_bytes(rows, k), dtype=torch.uint8, device=DEV)
    s = torch.empty(rows, dtype=torch.float32, device=DEV)
    F.flux_quantize_rows_nvfp4(x.to(DEV), q, sf, s)
    return q, sf, s


@pytest.fixture(autouse=True)
def _device_clean():
    yield
    assert F.flux_device_error() == 0


def test_scale_layout_is_a_permutation_of_whole_blocks():
    """Host check of the layout the tests decode: every (row, block) lands on its own byte."""
    idx = sf_index(256, 512).reshape(-1)
    assert idx.unique().numel() == idx.numel() == F.flux_nvfp4_scale_bytes(256, 512)


@pytest.mark.parametrize("rows,k", [(300, 3072), (37, 12288), (5, 9216), (1, 64), (129, 16384), (3, 192)])
def test_quantize_rows_nvfp4_bit_exact_against_oracle(rows, k):
    x = (rand((rows, k), 10 + rows) * torch.logspace(-2, 2, rows)[:, None]).to(torch.bfloat16)
    x[0, :48] = 0.0                                             # zero blocks
    if rows > 2:
        x[2] = 0.0                                              # a zero row
        x[1, 16:32] = x[1].float().abs().max().to(torch.bfloat16) * 1e-7   # a block whose scale underflows
    qc, qsb, qs = Q4.quantize_rows_nvfp4(x.float())
    q, sf, s = quantize_gpu(x)
    torch.cuda.synchronize()
    assert torch.equal(s.cpu(), qs)
    assert torch.equal(decode_sf(sf, rows, k), qsb)
    assert torch.equal(decode_codes(q), qc)


@pytest.mark.parametrize("rows,dim", [(4608 + 5, 3072), (33, 3072), (70, 1024), (40, 2048), (37, 4096)])
def test_layernorm_modulate_nvfp4_against_oracle(rows, dim):
    """LN-mod quantised to NVFP4 in one pass, from the float32 modulated values: the codes, block
    scales and row scales of the oracle's quantisation of the same row, except where the two LayerNorm
    evaluations (float32 here, float64 there) land on opposite sides of a rounding boundary, which
    moves one code by one e2m1 step (or a block scale by one e4m3 step); that needs a value within a
    few float32 ulps of the boundary, so it is rare."""
    x = rand((rows, dim), 150) * 3 + 0.5
    shift, scale = rand((dim,), 151), rand((dim,), 152, 0.5)
    q = torch.empty(rows, dim // 2, dtype=torch.uint8, device=DEV)
    sf = torch.zeros(F.flux_nvfp4_scale_bytes(rows, dim), dtype=torch.uint8, device=DEV)
    s = torch.empty(rows, dtype=torch.float32, device=DEV)
    F.flux_layernorm_modulate_nvfp4(x.to(DEV), q, sf, s, shift.to(DEV), scale.to(DEV))
    y = O.modulate(O.layer_norm(x.double(), 1e-6), shift.double(), scale.double())
    qc, qsb, qs = Q4.quantize_rows_nvfp4(y)
    assert torch.allclose(s.cpu().double(), qs.double(), rtol=1e-5, atol=0)
    sb = decode_sf(sf, rows, dim)
    assert (sb != qsb).double().mean() < 1e-4
    codes = decode_codes(q)
    same_blocks = (sb == qsb).repeat_interleave(16, dim=1)
    diff = (codes != qc) & same_blocks
    assert diff.double().mean() < 1e-4
    steps = (codes - qc).abs()[diff]
    assert (steps <= 2.0).all()                             # neighbouring e2m1 values (spacing <= 2)


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
    (129, 256, 3072, F.EPI_F32_BIAS),
    (257, 3072, 1024, F.EPI_SWIGLU),
    (200, 9216, 384, F.EPI_RESID_GATE),
    (128 * 3 + 1, 12288, 256 + 32, F.EPI_RESID_GATE),
    (1, 256, 32, F.EPI_BF16_BIAS),
    (2000, 256, 8192, F.EPI_F32_BIAS),          # more tiles than CTA pairs: both accumulator buffers
    (1000, 256, 8192, F.EPI_SWIGLU),
    (1024, 512, 6144, F.EPI_RESID_GATE),
])
def test_linear_nvfp4_modes_on_oracle_codes(m, k, n, mode):
    a = rand((m, k), 60) * torch.logspace(-1, 1, m)[:, None]
    w = rand((n, k), 61, k ** -0.5)
    if mode == F.EPI_SWIGLU:
        w = interleave_swiglu(w)
    b = rand((n,), 62, 0.5).to(torch.bfloat16)
    qa, ba, sa = Q4.quantize_rows_nvfp4(a)
    qw, bw, sw = Q4.quantize_rows_nvfp4(w)
    va = (qa.reshape(m, -1, 16) * ba[:, :, None]).reshape(m, k)
    vw = (qw.reshape(n, -1, 16) * bw[:, :, None]).reshape(n, k)
    acc = (va @ vw.t()) * sa.double()[:, None] * sw.double()[None, :] + b.double()
    args = (encode_codes(qa).to(DEV), encode_sf(ba, m, k).to(DEV), sa.to(DEV),
            encode_codes(qw).to(DEV), encode_sf(bw, n, k).to(DEV), sw.to(DEV), b.to(DEV), mode)
    if mode == F.EPI_SWIGLU:
        g = acc.reshape(m, n // 256, 2, 128)
        ref = (O.silu(g[:, :, 0]) * g[:, :, 1]).reshape(m, n // 2)
        out = torch.empty(m, n // 2, device=DEV, dtype=torch.bfloat16)
        F.flux_linear_nvfp4(*args, out)
    elif mode == F.EPI_RESID_GATE:
        x0 = rand((m, n), 63)
        gate = rand((n,), 64)
        ref = x0.double() + gate.double() * acc
        out = x0.to(DEV)
        F.flux_linear_nvfp4(*args, out, gate=gate.to(DEV))
    else:
        ref = acc
        dt = torch.bfloat16 if mode == F.EPI_BF16_BIAS else torch.float32
        out = torch.empty(m, n, device=DEV, dtype=dt)
        F.flux_linear_nvfp4(*args, out)
    err = nmax(out, ref)
    assert err <= TOL, err
    if mode in (F.EPI_F32_BIAS, F.EPI_RESID_GATE):
        assert err < 1e-5, err            # fp32 output: block products are exact, only summation order differs


def test_linear_nvfp4_full_size_sampled_rows():
    """Single-block linear1 size (4608 x 3072 -> 27648 rows of W), GPU quantiser, fp32 output."""
    m, k, n = 4608, 3072, 27648
    a = rand((m, k), 70).to(torch.bfloat16)
    w = rand((n, k), 71, k ** -0.5).to(torch.bfloat16)
    b = rand((n,), 72, 0.5).to(torch.bfloat16)
    qa, sfa, sa = quantize_gpu(a)
    qw, sfw, sw = quantize_gpu(w)
    out = torch.empty(m, n, device=DEV, dtype=torch.float32)
    F.flux_linear_nvfp4(qa, sfa, sa, qw, sfw, sw, b.to(DEV), F.EPI_F32_BIAS, out)
    rows = torch.arange(0, m, 97)
    ref = Q4.linear_nvfp4(a[rows].float().double(), w.float().double(), b.double())
    assert nmax(out[rows], ref) < 1e-5
    # against the unquantised product: the 4-bit format's own error, a few percent
    full = a[rows].double() @ w.double().t() + b.double()
    rel = ((out[rows].cpu().double() - full).norm() / full.norm()).item()
    assert 0.02 < rel < 0.2, rel


# ---------------------------------------------------------------------------- forwards in NVFP4
from oracle import flux3_oracle as O3                      # noqa: E402
from synthetic import WORKLOADS, make_weights, make_inputs  # noqa: E402


def rel_l2(a, b):
    a = torch.as_tensor(a).double().cpu()
    b = torch.as_tensor(b).double().cpu()
    return ((a - b).norm() / b.norm()).item()


@pytest.fixture(scope="module")
def tiny():
    w = WORKLOADS["tiny64"]
    blob, p = make_weights(w.dims, w.seed)
    model = F.FluxDiT(blob, w.dims)
    yield w, p, model
    model.close()


@pytest.mark.parametrize("n_txt,grid,refs", [(16, (4, 4), []), (131, (8, 8), [(4, 8)]), (0, (4, 6), []),
                                             (200, (12, 12), [(12, 12)])])
def test_tiny_nvfp4_forward_against_nvfp4_oracle(tiny, n_txt, grid, refs):
    w, p, model = tiny
    g = torch.Generator().manual_seed(180 + n_txt)
    tok = torch.randn(grid[0] * grid[1], 128, generator=g).to(torch.bfloat16).float()
    txt = torch.randn(n_txt, 3072, generator=g).to(torch.bfloat16).float()
    ref_tok = [torch.randn(h * w_, 128, generator=g).to(torch.bfloat16).float() for h, w_ in refs]
    hq = dict(O.hyper(w.dims), nvfp4=True)
    want = O.forward(p, hq, tok, txt, 0.6, grid, ref_tok, refs)
    exact = O.forward(p, O.hyper(w.dims), tok, txt, 0.6, grid, ref_tok, refs)
    v = torch.empty(grid[0] * grid[1], 128, device=DEV)
    v16 = torch.empty_like(v)
    hw = refs if refs else (0, 0)
    rt = torch.cat(ref_tok).to(DEV) if refs else None
    model.forward(tok.to(DEV), grid, txt.to(DEV) if n_txt else None, 0.6, v16, rt, hw)
    model.set_precision(F.PRECISION_NVFP4)
    try:
        model.forward(tok.to(DEV), grid, txt.to(DEV) if n_txt else None, 0.6, v, rt, hw)
    finally:
        model.set_precision(F.PRECISION_BF16)
    err = rel_l2(v, want)
    print(f"nvfp4 forward vs nvfp4 oracle {err:.4f}, vs exact oracle {rel_l2(v, exact):.4f}, "
          f"nvfp4 oracle vs exact {rel_l2(want, exact):.4f}")
    assert err <= NV4_V_TOL, err
    assert err < NV4_RATIO * rel_l2(v, exact)               # it quantises the way the oracle does
    assert rel_l2(v, exact) > rel_l2(v16, exact)
    again = torch.empty_like(v)
    model.forward(tok.to(DEV), grid, txt.to(DEV) if n_txt else None, 0.6, again, rt, hw)
    assert torch.equal(again, v16)                          # back to bf16, bit for bit


def test_nvfp4_guided_batch_equals_two_single_forwards(tiny):
    w, p, model = tiny
    g = torch.Generator().manual_seed(190)
    grid = (6, 4)
    tok = torch.randn(24, 128, generator=g).to(torch.bfloat16).float().to(DEV)
    tc = torch.randn(131, 3072, generator=g).to(torch.bfloat16).float().to(DEV)
    tu = torch.randn(131, 3072, generator=g).to(torch.bfloat16).float().to(DEV)
    vc, vu, a, b = (torch.empty(24, 128, device=DEV) for _ in range(4))
    model.set_precision(F.PRECISION_NVFP4)
    try:
        model.forward_cfg(tok, grid, tc, tu, 0.6, vc, vu)
        model.forward(tok, grid, tc, 0.6, a)
        model.forward(tok, grid, tu, 0.6, b)
    finally:
        model.set_precision(F.PRECISION_BF16)
    assert torch.equal(vc, a) and torch.equal(vu, b)


def test_nvfp4_forward_full_size_against_bf16_and_fp8():
    """1024^2 workload, full model: NVFP4 is the coarser format, so it lands further from bf16 than FP8."""
    w = WORKLOADS["t2i1024"]
    blob, _ = make_weights(w.dims, w.seed)
    lat, txt, _ = make_inputs(w)
    model = F.FluxDiT(blob, w.dims)
    del blob
    try:
        tok = O.pack_latents(torch.from_numpy(lat)).float().to(DEV)
        tx = torch.from_numpy(txt).to(DEV)
        v16, v8, v4 = (torch.empty(w.n_img, 128, device=DEV) for _ in range(3))
        model.forward(tok, (w.grid, w.grid), tx, 1.0, v16)
        model.set_precision(F.PRECISION_FP8)
        model.forward(tok, (w.grid, w.grid), tx, 1.0, v8)
        model.set_precision(F.PRECISION_NVFP4)
        model.forward(tok, (w.grid, w.grid), tx, 1.0, v4)
        torch.cuda.synchronize()
        e8, e4 = rel_l2(v8, v16), rel_l2(v4, v16)
        print(f"1024^2 fp8 vs bf16 {e8:.4f}, nvfp4 vs bf16 {e4:.4f}")
        assert torch.isfinite(v4).all() and e8 < e4 < 0.5, (e8, e4)
    finally:
        model.close()


@pytest.fixture(scope="module")
def tiny3():
    w = WORKLOADS["f3tiny64"]
    blob, p = make_weights(w.dims, w.seed)
    model = F.Flux3DiT(blob, w.dims)
    yield w, p, model
    model.close()


@pytest.mark.parametrize("nt,grid,ref_grids", [(16, (4, 4), [(4, 4)]), (131, (8, 8), [(4, 8), (4, 4)]),
                                               (0, (4, 6), [])])
def test_tiny3_nvfp4_forward_and_guided_batch(tiny3, nt, grid, ref_grids):
    """FLUX.3: NVFP4 per-mode and joint linears against the NVFP4 oracle; the guided batch equals
    two single forwards bit for bit."""
    w, p, model = tiny3
    g = torch.Generator().manual_seed(500 + nt)
    tok = torch.randn(grid[0] * grid[1], 128, generator=g).to(torch.bfloat16).float()
    txt = torch.randn(nt, 20480, generator=g).to(torch.bfloat16).float()
    txt_u = torch.randn(nt, 20480, generator=g).to(torch.bfloat16).float()
    refs = [torch.randn(h * w_, 128, generator=g).to(torch.bfloat16).float() for h, w_ in ref_grids]
    want = O3.forward3(p, dict(O.hyper(w.dims), nvfp4=True), tok, txt, 0.6, grid, refs, ref_grids, t_target=0.35)
    rt = torch.cat(refs).to(DEV) if refs else None
    td = txt.to(DEV) if nt else None
    tud = txt_u.to(DEV) if nt else None
    v, vc, vu, su = (torch.empty(grid[0] * grid[1], 128, device=DEV) for _ in range(4))
    model.set_precision(F.PRECISION_NVFP4)
    try:
        model.forward(tok.to(DEV), grid, td, 0.6, v, rt, ref_grids, t_target=0.35)
        model.forward_cfg(tok.to(DEV), grid, td, tud, 0.6, vc, vu, rt, ref_grids, t_target=0.35)
        model.forward(tok.to(DEV), grid, tud, 0.6, su, rt, ref_grids, t_target=0.35)
    finally:
        model.set_precision(F.PRECISION_BF16)
    err = rel_l2(v, want)
    print(f"flux3 nvfp4 forward vs nvfp4 oracle {err:.4f}")
    assert err <= NV4_V_TOL, err
    assert torch.equal(vc, v) and torch.equal(vu, su)


def test_tiny_nvfp4_sampler_against_nvfp4_oracle(tiny):
    """Two NVFP4 sampling steps: every velocity and the final latent within the NVFP4 bar."""
    w, p, model = tiny
    lat, txt, _ = make_inputs(w)
    hq = dict(O.hyper(w.dims), nvfp4=True)
    ref_final, ref_vs = O.sample(p, hq, torch.from_numpy(lat), torch.from_numpy(txt), 2)
    vs = []
    model.set_precision(F.PRECISION_NVFP4)
    try:
        final = F.flux_sample(model, torch.from_numpy(lat).to(DEV), torch.from_numpy(txt).to(DEV), 2,
                              on_step=lambda i, v: vs.append(v.cpu().clone()))
    finally:
        model.set_precision(F.PRECISION_BF16)
    assert len(vs) == 2
    for a, b in zip(vs, ref_vs):
        print(f"nvfp4 sampler step velocity vs nvfp4 oracle {rel_l2(a, b):.4f}")
        assert rel_l2(a, b) <= NV4_V_TOL
    print(f"nvfp4 sampler final latent vs nvfp4 oracle {rel_l2(final.cpu(), ref_final):.4f}")
    assert rel_l2(final.cpu(), ref_final) <= NV4_V_TOL


def test_flux3_nvfp4_full_size_against_bf16_and_fp8():
    """FLUX.3 1024^2 workload, full model (5 + 28 blocks): NVFP4 lands further from bf16 than FP8."""
    w = WORKLOADS["f3t2i1024"]
    blob, _ = make_weights(w.dims, w.seed)
    lat, txt, _ = make_inputs(w)
    model = F.Flux3DiT(blob, w.dims)
    del blob
    try:
        tok = O.pack_latents(torch.from_numpy(lat)).float().to(DEV)
        tx = torch.from_numpy(txt).to(DEV)
        v16, v8, v4 = (torch.empty(w.n_img, 128, device=DEV) for _ in range(3))
        model.forward(tok, (w.grid, w.grid), tx, 1.0, v16, t_target=15 / 16)
        model.set_precision(F.PRECISION_FP8)
        model.forward(tok, (w.grid, w.grid), tx, 1.0, v8, t_target=15 / 16)
        model.set_precision(F.PRECISION_NVFP4)
        model.forward(tok, (w.grid, w.grid), tx, 1.0, v4, t_target=15 / 16)
        torch.cuda.synchronize()
        e8, e4 = rel_l2(v8, v16), rel_l2(v4, v16)
        print(f"FLUX.3 1024^2 fp8 vs bf16 {e8:.4f}, nvfp4 vs bf16 {e4:.4f}")
        assert torch.isfinite(v4).all() and e8 < e4 < 0.5, (e8, e4)
    finally:
        model.close()
