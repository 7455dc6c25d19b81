"""FLUX.3 Image Klein on the GPU (through the C ABI) against the FLUX.3 CPU oracle.

Bars as for FLUX.2: velocity relative L2 <= 2e-2 per step, final latent <= 3e-2, modulation
and attention normalised max error <= 1e-2.
* segmented attention (the per-mode blocks' stream-local attention): bit-identical to one call
  per segment, and against the oracle's attention per segment;
* the tiny model (1 per-mode + 1 joint block, full width): live float64 oracle, block by block,
  ragged and degenerate shapes, several references, the flow-map sampler;
* 256^2 and 1024^2 workloads (+ a reference): the oracle's sampled rows, written by
  tests/golden/make_goldens.py (oracle only).
"""
import json
import os

import numpy as np
import pytest
import torch

import latent_flow_matching_b200 as F
from oracle import flux_oracle as O
from oracle import flux3_oracle as O3
from synthetic import WORKLOADS, make_weights, make_inputs, make_uncond_text

pytestmark = pytest.mark.gpu
torch.set_grad_enabled(False)
DEV = "cuda"
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
V_TOL, X_TOL, K_TOL = 2e-2, 3e-2, 1e-2


def rel_l2(a, b):
    a = torch.as_tensor(a).double().cpu()
    b = torch.as_tensor(b).double().cpu()
    return ((a - b).norm() / b.norm()).item()


def nmax(a, b):
    a = torch.as_tensor(a).double().cpu()
    b = torch.as_tensor(b).double().cpu()
    return ((a - b).abs().max() / b.abs().max()).item()


def bf16r(x):
    return x.to(torch.bfloat16).float()


# ---------------------------------------------------------------------------- segmented attention
@pytest.mark.parametrize("seg_len", [[37, 300, 0, 129], [160, 256], [1, 1, 1], [513]])
def test_segment_attention_matches_per_segment_calls_and_oracle(seg_len):
    g = torch.Generator().manual_seed(sum(seg_len))
    heads = 4
    rows = sum(seg_len)
    q, k, v = (torch.randn(rows, heads, 128, generator=g).to(torch.bfloat16) for _ in range(3))
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o = torch.empty_like(qd)
    F.flux_joint_attention_segments(qd, kd, vd, o, seg_len)
    r0 = 0
    for n in seg_len:
        if n:
            sl = slice(r0, r0 + n)
            one = torch.empty(n, heads, 128, dtype=torch.bfloat16, device=DEV)
            F.flux_joint_attention(qd[sl].contiguous(), kd[sl].contiguous(), vd[sl].contiguous(), one)
            assert torch.equal(one, o[sl]), (n, r0)
            want = O.attention(q[sl].double(), k[sl].double(), v[sl].double())
            assert nmax(o[sl].float().reshape(n, -1), want) <= K_TOL
        r0 += n
    assert F.flux_device_error() == 0


# ---------------------------------------------------------------------------- tiny model, live oracle
@pytest.fixture(scope="module")
def tiny3():
    w = WORKLOADS["f3tiny64"]
    blob, p = make_weights(w.dims, w.seed)
    model = F.Flux3DiT(blob, w.dims)
    yield w, p, model
    model.close()


def _mods_ref(p, t, t_target):
    D = p["time_in.w2"].shape[0]
    f64 = torch.float64
    s_img = O.silu(O3.time_vector(p, t, t_target, f64))
    s_ctx = O.silu(O3.time_vector(p, 0.0, t_target, f64))

    def lin(name, s):
        return O.linear(s, O.weight(p, name + ".w", f64), O.weight(p, name + ".b", f64))
    return torch.cat([lin("mode_mod.txt", s_ctx), lin("mode_mod.img", s_img), lin("mode_mod.ref", s_ctx),
                      lin("joint_mod", s_img), lin("joint_mod", s_ctx), lin("final.mod", s_img)]), D


@pytest.mark.parametrize("t,t_target", [(1.0, 0.75), (0.25, 0.0)])
def test_tiny3_modulation_vectors(tiny3, t, t_target):
    w, p, model = tiny3
    out = torch.empty(model.modulation_size(), device=DEV)
    model.modulation(t, t_target, out)
    ref, D = _mods_ref(p, t, t_target)
    assert out.numel() == ref.numel() == 17 * D
    assert nmax(out, ref) <= K_TOL
    # the context sets do not depend on t, the image sets do
    out2 = torch.empty_like(out)
    model.modulation(0.5 * t + 0.1, t_target, out2)
    ctx = torch.cat([torch.arange(0, 3 * D), torch.arange(6 * D, 9 * D), torch.arange(12 * D, 15 * D)])
    assert torch.equal(out[ctx], out2[ctx])
    assert not torch.equal(out[3 * D:6 * D], out2[3 * D:6 * D])


def _tiny_inputs(seed, nt, grid, ref_grids):
    g = torch.Generator().manual_seed(seed)
    tok = bf16r(torch.randn(grid[0] * grid[1], 128, generator=g))
    txt = bf16r(torch.randn(nt, 20480, generator=g))
    refs = [bf16r(torch.randn(h * w_, 128, generator=g)) for h, w_ in ref_grids]
    return tok, txt, refs


def _gpu_forward(model, tok, grid, txt, t, refs, ref_grids, t_target):
    v = torch.empty(grid[0] * grid[1], 128, device=DEV)
    ref_tok = torch.cat(refs).to(DEV) if refs else None
    model.forward(tok.to(DEV), grid, txt.to(DEV) if txt.shape[0] else None, t, v, ref_tok, ref_grids,
                  t_target=t_target)
    return v


@pytest.mark.parametrize("precision", [F.PRECISION_BF16, F.PRECISION_FP8, F.PRECISION_NVFP4])
def test_tiny3_profile_counts_the_algorithmic_work(tiny3, precision):
    """The profiling hook's FLOPs and bytes for a forward with a reference equal the closed forms:
    per block N 2D(4D + 3F) of linears; attention 4 D (Nt^2 + Ni^2 + Nr^2) in a per-mode block (each
    stream within itself) and 4 N^2 D in a joint block; GEMM bytes with A and W read once in the
    format that runs and each output written once (bf16 2 bytes; the SwiGLU half the columns in
    bf16; fp32 4; the gated residual's fp32 rows read and written)."""
    w, p, model = tiny3
    d = w.dims
    D, Fh, C, T = d.hidden, d.mlp_hidden, d.in_ch, d.txt_dim
    tok, txt, refs = _tiny_inputs(11, 16, (4, 4), [(4, 4)])
    nt, ni, nr = 16, 16, 16
    n = nt + ni + nr
    elt, row = {F.PRECISION_BF16: (2.0, 0.0), F.PRECISION_FP8: (1.0, 4.0),
                F.PRECISION_NVFP4: (0.5 + 1.0 / 16.0, 4.0)}[precision]

    def lb(m, k, nn, out_per_elt, e=elt, r=row):
        return e * (m * k + nn * k) + r * (m + nn) + out_per_elt * m * nn

    segs = (nt, ni, nr)
    mode_bytes = sum(lb(g, D, 3 * D, 2) + lb(g, D, 2 * Fh, 1) + lb(g, D + Fh, D, 8) for g in segs)
    joint_bytes = lb(n, D, 3 * D, 2) + lb(n, D, 2 * Fh, 1) + sum(lb(g, D + Fh, D, 8) for g in segs)
    io = lb(nt, T, D, 4, 2.0, 0.0) + lb(ni + nr, C, D, 4, 2.0, 0.0) + lb(ni, D, C, 4, 2.0, 0.0)
    want_bytes = d.n_mode * mode_bytes + d.n_joint * joint_bytes + io
    want_flops = ((d.n_mode + d.n_joint) * n * 2.0 * D * (4 * D + 3 * Fh) + 2.0 * (ni + nr) * C * D +
                  2.0 * nt * T * D + 2.0 * ni * D * C)
    want_attn = d.n_mode * 4.0 * D * sum(g * g for g in segs) + d.n_joint * 4.0 * n * n * D
    model.set_precision(precision)
    try:
        _gpu_forward(model, tok, (4, 4), txt, 0.6, refs, [(4, 4)], 0.35)
        model.profile(True)
        _gpu_forward(model, tok, (4, 4), txt, 0.6, refs, [(4, 4)], 0.35)
        prof = model.profile_read()
    finally:
        model.profile(False)
        model.set_precision(F.PRECISION_BF16)
    _, g_fl, g_by, g_n = prof["gemm"]
    _, a_fl, _, a_n = prof["attention"]
    assert g_n == 2 * (d.n_mode + d.n_joint) + 2
    assert a_n == d.n_mode + d.n_joint
    assert g_fl == pytest.approx(want_flops, rel=1e-12)
    assert a_fl == pytest.approx(want_attn, rel=1e-12)
    assert g_by == pytest.approx(want_bytes, rel=1e-12)


@pytest.mark.parametrize("precision", ["bf16", "nvfp4"])
def test_tiny3_programmatic_launches_change_nothing(tiny3, precision, monkeypatch):
    """FLUX.3 forward with a reference (segmented per-mode attention, three-region LN-mod) with and
    without programmatic dependent launches: bit-identical."""
    w, p, model = tiny3
    tok, txt, refs = _tiny_inputs(7, 16, (4, 4), [(4, 4)])
    model.set_precision(F.PRECISION_NVFP4 if precision == "nvfp4" else F.PRECISION_BF16)
    try:
        monkeypatch.setenv("FLUX_PDL", "0")
        plain = _gpu_forward(model, tok, (4, 4), txt, 0.6, refs, [(4, 4)], 0.35)
        monkeypatch.setenv("FLUX_PDL", "1")
        pdl = _gpu_forward(model, tok, (4, 4), txt, 0.6, refs, [(4, 4)], 0.35)
        torch.cuda.synchronize()
    finally:
        model.set_precision(F.PRECISION_BF16)
    assert torch.equal(plain, pdl)
    assert F.flux_device_error() == 0


@pytest.mark.parametrize("n_mode,n_joint", [(0, 0), (1, 0), (0, 1), (1, 1)])
def test_tiny3_forward_block_by_block(tiny3, n_mode, n_joint):
    w, p, model = tiny3
    keep = {k: v for k, v in p.items()
            if not ((k.startswith("mode.") and int(k.split(".")[1]) >= n_mode) or
                    (k.startswith("joint.") and int(k.split(".")[1]) >= n_joint))}
    tok, txt, refs = _tiny_inputs(3, 16, (4, 4), [(4, 4)])
    want = O3.forward3(keep, O.hyper(w.dims), tok, txt, 0.75, (4, 4), refs, [(4, 4)], t_target=0.5)
    model.set_active_blocks(n_mode, n_joint)
    try:
        v = _gpu_forward(model, tok, (4, 4), txt, 0.75, refs, [(4, 4)], 0.5)
    finally:
        model.set_active_blocks(-1, -1)
    assert rel_l2(v, want) <= V_TOL
    assert F.flux_device_error() == 0


@pytest.mark.parametrize("nt,grid,ref_grids", [(0, (4, 6), []), (5, (6, 4), [(4, 4)]), (16, (4, 4), []),
                                               (131, (8, 8), [(4, 8), (4, 4)]), (200, (12, 12), [(12, 12)])])
def test_tiny3_forward_ragged_and_degenerate_shapes(tiny3, nt, grid, ref_grids):
    """No text, no reference, several references, segments off the 128-row tiles and longer than one."""
    w, p, model = tiny3
    tok, txt, refs = _tiny_inputs(100 + nt, nt, grid, ref_grids)
    want = O3.forward3(p, O.hyper(w.dims), tok, txt, 0.6, grid, refs, ref_grids, t_target=0.35)
    v = _gpu_forward(model, tok, grid, txt, 0.6, refs, ref_grids, 0.35)
    assert rel_l2(v, want) <= V_TOL
    assert F.flux_device_error() == 0


def test_tiny3_target_time_and_reference_order_matter(tiny3):
    w, p, model = tiny3
    tok, txt, refs = _tiny_inputs(9, 7, (4, 4), [(4, 4), (6, 4)])
    grids = [(4, 4), (6, 4)]
    a = _gpu_forward(model, tok, (4, 4), txt, 0.5, refs, grids, 0.25)
    b = _gpu_forward(model, tok, (4, 4), txt, 0.5, refs, grids, 0.0)
    c = _gpu_forward(model, tok, (4, 4), txt, 0.5, refs[::-1], grids[::-1], 0.25)
    assert rel_l2(a, b) > 1e-3 and rel_l2(a, c) > 1e-3
    want = O3.forward3(p, O.hyper(w.dims), tok, txt, 0.5, (4, 4), refs[::-1], grids[::-1], t_target=0.25)
    assert rel_l2(c, want) <= V_TOL


def test_tiny3_sampler_matches_oracle(tiny3):
    """4 flow-map steps (target t_{i+1}) with a 64^2 reference: every velocity and the final latent."""
    w, p, model = tiny3
    lat, txt, ref = make_inputs(w)
    ref_final, ref_vs = O3.sample3(p, O.hyper(w.dims), torch.from_numpy(lat), torch.from_numpy(txt), 4,
                                   ref_latent=torch.from_numpy(ref))
    vs = []
    final = F.flux3_sample(model, torch.from_numpy(lat).to(DEV), torch.from_numpy(txt).to(DEV), 4,
                           ref_latent=torch.from_numpy(ref).to(DEV), on_step=lambda i, v: vs.append(v.cpu().clone()))
    assert len(vs) == 4
    for i in range(4):
        assert rel_l2(vs[i], ref_vs[i]) <= V_TOL, i
    assert rel_l2(final.cpu(), ref_final) <= X_TOL
    again = F.flux3_sample(model, torch.from_numpy(lat).to(DEV), torch.from_numpy(txt).to(DEV), 4,
                           ref_latent=torch.from_numpy(ref).to(DEV))
    assert torch.equal(final, again)                       # deterministic
    assert F.flux_device_error() == 0


def test_flux3_rejects_bad_arguments(tiny3):
    w, p, model = tiny3
    tok = torch.zeros(16, 128, device=DEV)
    v = torch.empty(16, 128, device=DEV)
    txt = torch.zeros(4, 20480, device=DEV)
    with pytest.raises(F.FluxError):
        model.forward(tok, (2, 8), txt, 1.0, v, t_target=0.5)
    with pytest.raises(F.FluxError):
        model.forward(tok, (4, 4), txt, 1.0, v, None, [(4, 4)], t_target=0.5)   # reference grid, no tokens
    with pytest.raises(F.FluxError):
        model.forward(tok, (4, 4), txt, 1.0, v, t_target=float("nan"))          # flow-map model needs t_target
    with pytest.raises(F.FluxError):
        model.forward(tok, (4, 4), txt, 1.0, v, torch.zeros(11 * 16, 128, device=DEV), [(4, 4)] * 11, t_target=0.5)


# ---------------------------------------------------------------------------- full-size workloads vs goldens
def _golden(name):
    path = os.path.join(GOLDEN, f"{name}.npz")
    if not os.path.exists(path):
        pytest.skip(f"golden {path} not generated")
    return np.load(path)


@pytest.mark.parametrize("name", ["f3t2i256", "f3i2i256", "f3t2i1024", "f3i2i1024"])
def test_flux3_workload_against_oracle_goldens(name):
    gd = _golden(name)
    w = WORKLOADS[name]
    meta = json.loads(str(gd["meta"]))
    assert meta["workload"] == name and meta["seed"] == w.seed
    k = meta["steps_run"]
    blob, _ = make_weights(w.dims, w.seed)
    lat, txt, ref = make_inputs(w)
    model = F.Flux3DiT(blob, w.dims)
    del blob
    try:
        ts = F.euler_schedule(w.n_steps)
        tok = torch.empty(w.n_img, 128, device=DEV)
        F.flux_pack_latents(torch.from_numpy(lat).to(DEV), tok)
        ref_tok, grids = None, []
        if ref is not None:
            ref_tok = O.pack_latents(torch.from_numpy(ref)).float().to(DEV)
            grids = [(w.ref_grid, w.ref_grid)]
        txt_d = torch.from_numpy(txt).to(DEV)
        v = torch.empty_like(tok)
        rows = torch.from_numpy(gd["rows"]).long()
        for i in range(k):
            model.forward(tok, (w.grid, w.grid), txt_d, ts[i], v, ref_tok, grids, t_target=ts[i + 1])
            err = rel_l2(v.cpu()[rows], gd["v"][i])
            assert err <= V_TOL, (i, err)
            F.flux_euler_step(tok, v, ts[i + 1] - ts[i])
        err = rel_l2(tok.cpu()[rows], gd["final"])
        assert err <= X_TOL, err
    finally:
        model.close()
    assert F.flux_device_error() == 0


# ---------------------------------------------------------------------------- row-wise FP8 block linears
@pytest.mark.parametrize("nt,grid,ref_grids", [(16, (4, 4), [(4, 4)]), (131, (8, 8), [(4, 8), (4, 4)]),
                                               (0, (4, 6), [])])
def test_tiny3_fp8_forward_against_fp8_oracle(tiny3, nt, grid, ref_grids):
    """FP8 per-mode and joint linears against the oracle's FP8 forward (bar 2e-2, as for FLUX.2);
    switching back to bf16 gives the bf16 result bit for bit."""
    w, p, model = tiny3
    tok, txt, refs = _tiny_inputs(300 + nt, nt, grid, ref_grids)
    hq = dict(O.hyper(w.dims), fp8=True)
    want = O3.forward3(p, hq, tok, txt, 0.6, grid, refs, ref_grids, t_target=0.35)
    v16 = _gpu_forward(model, tok, grid, txt, 0.6, refs, ref_grids, 0.35)
    model.set_precision(F.PRECISION_FP8)
    try:
        v8 = _gpu_forward(model, tok, grid, txt, 0.6, refs, ref_grids, 0.35)
    finally:
        model.set_precision(F.PRECISION_BF16)
    assert rel_l2(v8, want) <= V_TOL, rel_l2(v8, want)
    again = _gpu_forward(model, tok, grid, txt, 0.6, refs, ref_grids, 0.35)
    assert torch.equal(again, v16)
    assert F.flux_device_error() == 0


def test_flux3_fp8_full_size_against_bf16():
    """FLUX.3 1024^2 workload, full model: the FP8 forward stays within a few percent of the bf16 one."""
    w = WORKLOADS["f3t2i1024"]
    blob, _ = make_weights(w.dims, w.seed)
    lat, txt, _ = make_inputs(w)
    model = F.Flux3DiT(blob, w.dims)
    del blob
    try:
        tok = O.pack_latents(torch.from_numpy(lat)).float().to(DEV)
        tx = torch.from_numpy(txt).to(DEV)
        v16, v8 = torch.empty(w.n_img, 128, device=DEV), torch.empty(w.n_img, 128, device=DEV)
        model.forward(tok, (w.grid, w.grid), tx, 1.0, v16, t_target=15 / 16)
        model.set_precision(F.PRECISION_FP8)
        model.forward(tok, (w.grid, w.grid), tx, 1.0, v8, t_target=15 / 16)
        torch.cuda.synchronize()
        err = rel_l2(v8, v16)
        assert 1e-3 < err < 0.1, err
    finally:
        model.close()
    assert F.flux_device_error() == 0


# ---------------------------------------------------------------------------- classifier-free guidance
@pytest.fixture(scope="module")
def tiny3_base():
    """The tiny model without the flow-map embedding (the base checkpoint's structure)."""
    w = WORKLOADS["f3cfgtiny64"]
    blob, p = make_weights(w.dims, w.seed)
    model = F.Flux3DiT(blob, w.dims)
    yield w, p, model
    model.close()


def _cfg_pair(model, tok, grid, txt_c, txt_u, t, refs, ref_grids, t_target):
    vc = torch.full((grid[0] * grid[1], 128), float("nan"), device=DEV)
    vu = torch.full_like(vc, float("nan"))
    ref_tok = torch.cat(refs).to(DEV) if refs else None
    nt = txt_c.shape[0]
    model.forward_cfg(tok.to(DEV), grid, txt_c.to(DEV) if nt else None, txt_u.to(DEV) if nt else None, t, vc, vu,
                      ref_tok, ref_grids, t_target=t_target)
    return vc, vu


@pytest.mark.parametrize("which", ["flow_map", "base"])
@pytest.mark.parametrize("precision", ["bf16", "fp8"])
@pytest.mark.parametrize("nt,grid,ref_grids", [(16, (4, 4), [(4, 4)]), (131, (8, 8), [(4, 8), (4, 4)]),
                                               (0, (4, 6), []), (200, (12, 12), [(12, 12)]), (5, (6, 4), [])])
def test_tiny3_guided_batch_is_bit_identical_to_two_forwards(tiny3, tiny3_base, which, precision, nt, grid,
                                                               ref_grids):
    """The batch-2 forward (per-mode image and reference streams computed once) returns, bit for
    bit, the velocities of two single-text forwards; the base model matches the oracle."""
    w, p, model = tiny3 if which == "flow_map" else tiny3_base
    tok, txt_c, refs = _tiny_inputs(400 + nt, nt, grid, ref_grids)
    txt_u = bf16r(torch.randn(nt, 20480, generator=torch.Generator().manual_seed(401 + nt)))
    if precision == "fp8":
        model.set_precision(F.PRECISION_FP8)
    try:
        vc, vu = _cfg_pair(model, tok, grid, txt_c, txt_u, 0.7, refs, ref_grids, 0.45)
        sc = _gpu_forward(model, tok, grid, txt_c, 0.7, refs, ref_grids, 0.45)
        su = _gpu_forward(model, tok, grid, txt_u, 0.7, refs, ref_grids, 0.45)
    finally:
        model.set_precision(F.PRECISION_BF16)
    torch.cuda.synchronize()
    assert torch.equal(vc, sc) and torch.equal(vu, su)
    if nt:
        assert rel_l2(vc, vu) > 1e-4                     # the texts differ, so do the velocities
    if which == "base" and precision == "bf16":
        want = O3.forward3(p, O.hyper(w.dims), tok, txt_u, 0.7, grid, refs, ref_grids)
        assert rel_l2(vu, want) <= V_TOL
    assert F.flux_device_error() == 0


@pytest.mark.parametrize("strength", [1.0, 0.5])
def test_tiny3_base_guided_sampler_matches_oracle(tiny3_base, strength):
    """The base checkpoint's sampler: guidance 3.5, a reference image, text-to-image and image
    editing (strength 0.5 starts at step 2 from the blended latent); every guided velocity and the
    final latent against the oracle's guided sampler."""
    w, p, model = tiny3_base
    lat, txt, ref = make_inputs(w)
    txt_u = make_uncond_text(w)
    init = bf16r(torch.randn(*lat.shape, generator=torch.Generator().manual_seed(402))).numpy()
    edit = {} if strength == 1.0 else {"init_latent": torch.from_numpy(init), "strength": strength}
    ref_final, ref_vs = O3.sample3(p, O.hyper(w.dims), torch.from_numpy(lat), torch.from_numpy(txt), w.n_steps,
                                   ref_latent=torch.from_numpy(ref), txt_uncond=torch.from_numpy(txt_u),
                                   guidance=w.guidance, **edit)
    vs = []
    final = F.flux3_sample(model, torch.from_numpy(lat).to(DEV), torch.from_numpy(txt).to(DEV), w.n_steps,
                           ref_latent=torch.from_numpy(ref).to(DEV), txt_uncond=torch.from_numpy(txt_u).to(DEV),
                           guidance=w.guidance, on_step=lambda i, v: vs.append(v.cpu().clone()),
                           **{k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in edit.items()})
    assert len(vs) == len(ref_vs) == (w.n_steps if strength == 1.0 else 2)
    for i in range(len(vs)):
        assert rel_l2(vs[i], ref_vs[i]) <= V_TOL, i
    assert rel_l2(final.cpu(), ref_final) <= X_TOL
    assert F.flux_device_error() == 0


def test_flux3_guided_batch_rejects_bad_arguments(tiny3):
    w, p, model = tiny3
    tok = torch.zeros(16, 128, device=DEV)
    v = torch.empty(16, 128, device=DEV)
    v2 = torch.empty(16, 128, device=DEV)
    txt = torch.zeros(4, 20480, device=DEV)
    with pytest.raises(F.FluxError):
        model.forward_cfg(tok, (4, 4), txt, txt, 1.0, v, v, t_target=0.5)            # one buffer for both
    rc = F.lib().flux3_dit_forward_cfg(model._h, tok.data_ptr(), 4, 4, txt.data_ptr(), None, 4, None, 0, None,
                                       1.0, 0.5, v.data_ptr(), v2.data_ptr(), None)
    assert rc != 0                                                                  # NULL unconditional text
    with pytest.raises(ValueError):
        model.forward_cfg(tok, (4, 4), txt, None, 1.0, v, v2, t_target=0.5)
        model.forward_cfg(tok, (4, 4), txt, txt[:3], 1.0, v, v2, t_target=0.5)       # different token counts
    model.forward_cfg(tok, (4, 4), txt, txt, 1.0, v, v2, t_target=0.5)              # still usable afterwards
    torch.cuda.synchronize()
    assert torch.equal(v, v2)
    assert F.flux_device_error() == 0


def test_flux3_base_guided_full_size_bit_identical():
    """FLUX.3 base checkpoint at 1024^2 (4096 image + 160 text tokens, 5 + 28 blocks): the guided
    batch equals two single forwards bit for bit, in bf16 and in FP8."""
    w = WORKLOADS["f3cfg1024"]
    blob, _ = make_weights(w.dims, w.seed)
    lat, txt, _ = make_inputs(w)
    txt_u = make_uncond_text(w)
    model = F.Flux3DiT(blob, w.dims)
    del blob
    try:
        tok = O.pack_latents(torch.from_numpy(lat)).float().to(DEV)
        tc, tu = torch.from_numpy(txt).to(DEV), torch.from_numpy(txt_u).to(DEV)
        for prec in (F.PRECISION_BF16, F.PRECISION_FP8):
            model.set_precision(prec)
            vc, vu = torch.empty(w.n_img, 128, device=DEV), torch.empty(w.n_img, 128, device=DEV)
            sc, su = torch.empty_like(vc), torch.empty_like(vc)
            model.forward_cfg(tok, (w.grid, w.grid), tc, tu, 0.8, vc, vu)
            model.forward(tok, (w.grid, w.grid), tc, 0.8, sc)
            model.forward(tok, (w.grid, w.grid), tu, 0.8, su)
            torch.cuda.synchronize()
            assert torch.equal(vc, sc) and torch.equal(vu, su), prec
            assert torch.isfinite(vc).all() and rel_l2(vc, vu) > 1e-3
    finally:
        model.close()
    assert F.flux_device_error() == 0


def test_flux3_base_guided_sampler_against_oracle_golden():
    """FLUX.3 base checkpoint at 256^2 (256 image + 160 text tokens), guidance 3.5, 4 steps: every
    guided velocity and the final latent against the oracle's rows (tests/golden/f3cfg256.npz)."""
    gd = _golden("f3cfg256")
    g = WORKLOADS["f3cfg256"]
    meta = json.loads(str(gd["meta"]))
    assert meta["workload"] == "f3cfg256" and meta["seed"] == g.seed and meta["guidance"] == g.guidance
    blob, _ = make_weights(g.dims, g.seed)
    glat, gtxt, _ = make_inputs(g)
    gtxt_u = make_uncond_text(g)
    model = F.Flux3DiT(blob, g.dims)
    del blob
    try:
        ts = F.euler_schedule(g.n_steps)
        tok = O.pack_latents(torch.from_numpy(glat)).float().to(DEV)
        tc, tu = torch.from_numpy(gtxt).to(DEV), torch.from_numpy(gtxt_u).to(DEV)
        vc, vu = torch.empty(g.n_img, 128, device=DEV), torch.empty(g.n_img, 128, device=DEV)
        rows = torch.from_numpy(gd["rows"]).long()
        for i in range(g.n_steps):
            model.forward_cfg(tok, (g.grid, g.grid), tc, tu, ts[i], vc, vu)
            err = rel_l2((vu + g.guidance * (vc - vu)).cpu()[rows], gd["v"][i])
            assert err <= V_TOL, (i, err)
            F.flux_cfg_euler_step(tok, vc, vu, g.guidance, ts[i + 1] - ts[i])
        err = rel_l2(tok.cpu()[rows], gd["final"])
        assert err <= X_TOL, err
    finally:
        model.close()
    assert F.flux_device_error() == 0
