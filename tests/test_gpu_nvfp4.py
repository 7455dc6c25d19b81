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


@pytest.mark.parametrize("rows,k", [(300, 3072), (37, 12288), (5, 9216), (1, 64), (129, 16384)])
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
