"""Pins of the FLUX.3 oracle (oracle/flux3_oracle.py) against what the pages and the pinned
FLUX.2 oracle fix.  CPU only."""
import json
import os

import numpy as np
import torch

from oracle import flux_oracle as O
from oracle import flux3_oracle as O3
from synthetic import (FluxDims, Flux3Dims, F3_FULL_DIMS, WORKLOADS, make_weights, bf16_bits_to_f32,
                       tensor_specs)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F64 = torch.float64
MICRO3 = Flux3Dims(n_mode=1, n_joint=1, hidden=64, heads=2, head_dim=32, mlp_hidden=96, in_ch=128, txt_dim=40,
                   t_freq_dim=256, flow_map=False)


def params(dims, seed):
    _, p = make_weights(dims, seed, threads=4)
    return {k: torch.from_numpy(bf16_bits_to_f32(v)).double() for k, v in p.items()}


def hp(d):
    return O.hyper(d)


def inputs(seed, nt=5, gh=3, gw=4, ref_grids=((2, 2),), txt_dim=40):
    g = torch.Generator().manual_seed(seed)
    img = torch.randn(gh * gw, 128, generator=g, dtype=F64)
    txt = torch.randn(nt, txt_dim, generator=g, dtype=F64)
    refs = [torch.randn(h * w, 128, generator=g, dtype=F64) for h, w in ref_grids]
    return img, txt, refs, list(ref_grids)


def as_flux2(p3):
    """The same weights under FLUX.2 names: joint block i -> single block i, joint_mod -> every
    single block's modulation linear (FLUX.2 evaluates it at one t for all tokens)."""
    p2 = {k: v for k, v in p3.items() if k.split(".")[0] in ("time_in", "img_in", "txt_in", "final")}
    for i in range(O3._count(p3, "joint")):
        for n in ("lin1.w", "lin1.b", "q_gain", "k_gain", "lin2.w", "lin2.b"):
            p2[f"single.{i}.{n}"] = p3[f"joint.{i}.{n}"]
        p2[f"single.{i}.mod.w"] = p3["joint_mod.w"]
        p2[f"single.{i}.mod.b"] = p3["joint_mod.b"]
    return p2


def test_page_numbers_and_shared_modulation_parameter_count():
    g = json.load(open(os.path.join(GOLDEN, "flux3.json")))
    d = F3_FULL_DIMS
    assert (d.n_mode, d.n_joint, d.hidden) == (g["per_mode_blocks"], g["joint_blocks"], g["width"])
    assert d.txt_dim == g["text_feature_layers"] * g["encoder_hidden"] == g["text_feature_dim"]
    n = sum(int(np.prod(s)) for _, s, _ in tensor_specs(d)) / 1e9
    assert abs(n - g["generator_params_billion"]) / g["generator_params_billion"] < 0.03   # shared modulation
    per_block = n + (d.n_mode * 3 + d.n_joint - 4) * 3 * d.hidden * d.hidden / 1e9
    assert per_block > 1.15 * g["generator_params_billion"]                               # per-block would not fit
    assert WORKLOADS["f3t2i1024"].n_tokens == g["tokens_per_call_t2i_1024"]
    assert WORKLOADS["f3i2i1024"].n_tokens == g["tokens_per_call_i2i_1024_one_1024_ref"]
    assert WORKLOADS["f3t2i1024"].n_steps == g["distilled_steps"]


def test_joint_blocks_with_one_time_equal_the_flux2_single_blocks():
    """ctx_time = t gives every token the same modulation: the joint phase is then the pinned
    FLUX.2 single-stream chain on the same weights, at t = 0 and at t = 0.7."""
    d = Flux3Dims(**{**MICRO3.__dict__, "n_mode": 0, "n_joint": 2})
    p3 = params(d, 1)
    p2 = as_flux2(p3)
    img, txt, refs, grids = inputs(2)
    for t in (0.0, 0.7):
        a = O3.forward3(p3, hp(d), img, txt, t, (3, 4), refs, grids, ctx_time=t)
        b = O.forward(p2, hp(d), img, txt, t, (3, 4), refs, grids)
        assert torch.allclose(a, b, atol=1e-12, rtol=0)
    # the pages' rule (text and references at t = 0) differs from one time for all tokens
    c = O3.forward3(p3, hp(d), img, txt, 0.7, (3, 4), refs, grids)
    assert (c - b).abs().max() > 1e-4
    assert torch.allclose(O3.forward3(p3, hp(d), img, txt, 0.0, (3, 4), refs, grids),
                          O.forward(p2, hp(d), img, txt, 0.0, (3, 4), refs, grids), atol=1e-12, rtol=0)


def test_per_mode_blocks_keep_the_streams_apart():
    """Without joint blocks the image velocity depends on neither the text nor the references."""
    d = Flux3Dims(**{**MICRO3.__dict__, "n_mode": 2, "n_joint": 0})
    p3 = params(d, 3)
    img, txt, refs, grids = inputs(4)
    _, txt2, refs2, _ = inputs(5)
    a = O3.forward3(p3, hp(d), img, txt, 0.4, (3, 4), refs, grids)
    b = O3.forward3(p3, hp(d), img, txt2, 0.4, (3, 4), refs2, grids)
    c = O3.forward3(p3, hp(d), img, txt2[:2], 0.4, (3, 4))
    assert torch.allclose(a, b, atol=1e-12, rtol=0) and torch.allclose(a, c, atol=1e-12, rtol=0)
    d1 = Flux3Dims(**{**MICRO3.__dict__, "n_mode": 2, "n_joint": 1})
    p3 = params(d1, 3)
    a = O3.forward3(p3, hp(d1), img, txt, 0.4, (3, 4), refs, grids)
    b = O3.forward3(p3, hp(d1), img, txt2, 0.4, (3, 4), refs, grids)
    assert (a - b).abs().max() > 1e-4


def test_per_mode_streams_use_their_own_weights():
    """Swapping the text stream's per-mode weights with the image stream's changes the image
    velocity only through the image stream (n_joint = 0 isolates it)."""
    d = Flux3Dims(**{**MICRO3.__dict__, "n_mode": 1, "n_joint": 0})
    p3 = params(d, 6)
    img, txt, refs, grids = inputs(7)
    base = O3.forward3(p3, hp(d), img, txt, 0.3, (3, 4), refs, grids)
    q = dict(p3)
    for n in ("lin1.w", "lin1.b", "q_gain", "k_gain", "lin2.w", "lin2.b"):
        q[f"mode.0.txt.{n}"], q[f"mode.0.ref.{n}"] = p3[f"mode.0.ref.{n}"], p3[f"mode.0.txt.{n}"]
    assert torch.allclose(O3.forward3(q, hp(d), img, txt, 0.3, (3, 4), refs, grids), base, atol=1e-12, rtol=0)
    q = dict(p3)
    q["mode.0.img.lin2.w"] = p3["mode.0.txt.lin2.w"]
    assert (O3.forward3(q, hp(d), img, txt, 0.3, (3, 4), refs, grids) - base).abs().max() > 1e-4


def test_flow_map_target_embedding_is_additive():
    """A target-time MLP that outputs zero leaves the base model; a nonzero one moves it, and
    the sampler passes t_{i+1}."""
    d_fm = Flux3Dims(**{**MICRO3.__dict__, "flow_map": True})
    p_fm = params(d_fm, 8)
    p_base = {k: v for k, v in p_fm.items() if not k.startswith("target_in.")}
    img, txt, refs, grids = inputs(9)
    z = dict(p_fm)
    z["target_in.w2"] = torch.zeros_like(p_fm["target_in.w2"])
    z["target_in.b2"] = torch.zeros_like(p_fm["target_in.b2"])
    base = O3.forward3(p_base, hp(d_fm), img, txt, 0.5, (3, 4), refs, grids)
    assert torch.allclose(O3.forward3(z, hp(d_fm), img, txt, 0.5, (3, 4), refs, grids, t_target=0.25), base,
                          atol=1e-12, rtol=0)
    a = O3.forward3(p_fm, hp(d_fm), img, txt, 0.5, (3, 4), refs, grids, t_target=0.25)
    b = O3.forward3(p_fm, hp(d_fm), img, txt, 0.5, (3, 4), refs, grids, t_target=0.0)
    assert (a - b).abs().max() > 1e-4
    seen = []
    orig = O3.forward3

    def spy(*args, **kw):
        seen.append((args[4], kw.get("t_target")))
        return orig(*args, **kw)

    O3.forward3 = spy
    try:
        noise = torch.randn(32, 6, 8, generator=torch.Generator().manual_seed(1), dtype=F64)
        O3.sample3(p_fm, hp(d_fm), noise, txt, 4, None)
    finally:
        O3.forward3 = orig
    assert seen == [(1.0, 0.75), (0.75, 0.5), (0.5, 0.25), (0.25, 0.0)]


def test_reference_order_is_rope_only():
    """With RoPE switched off the reference images are an unordered set (per-mode and joint)."""
    d = Flux3Dims(**{**MICRO3.__dict__, "n_mode": 1, "n_joint": 1})
    p3 = params(d, 10)
    img, txt, refs, grids = inputs(11, ref_grids=((2, 2), (2, 2)))
    n = 5 + 12 + 8
    z = torch.zeros(n, 4, dtype=F64)
    a = O3.forward3(p3, hp(d), img, txt, 0.6, (3, 4), refs, grids, positions=z)
    b = O3.forward3(p3, hp(d), img, txt, 0.6, (3, 4), refs[::-1], grids, positions=z)
    assert torch.allclose(a, b, atol=1e-11, rtol=0)
    a = O3.forward3(p3, hp(d), img, txt, 0.6, (3, 4), refs, grids)
    b = O3.forward3(p3, hp(d), img, txt, 0.6, (3, 4), refs[::-1], grids)
    assert (a - b).abs().max() > 1e-6


def test_without_context_tokens_every_row_is_an_image_row():
    """No text and no references: the joint blocks see image rows only, so the model is the
    FLUX.2 single-stream chain at t whatever time the (absent) context would get."""
    d = Flux3Dims(**{**MICRO3.__dict__, "n_mode": 0, "n_joint": 2})
    p3 = params(d, 12)
    p2 = as_flux2(p3)
    img, txt, _, _ = inputs(13)
    for t in (0.35, 0.9):
        a = O3.forward3(p3, hp(d), img, txt[:0], t, (3, 4))
        b = O.forward(p2, hp(d), img, txt[:0], t, (3, 4))
        assert torch.allclose(a, b, atol=1e-12, rtol=0)


def test_text_and_reference_streams_are_at_time_zero_throughout():
    """The page's "permanently t = 0": after the per-mode phase the text and reference streams
    are the same for any t; the image stream is not."""
    d = Flux3Dims(**{**MICRO3.__dict__, "n_mode": 2, "n_joint": 1})
    p3 = params(d, 14)
    img, txt, refs, grids = inputs(15)
    ta, tb = {}, {}
    O3.forward3(p3, hp(d), img, txt, 0.2, (3, 4), refs, grids, trace=ta)
    O3.forward3(p3, hp(d), img, txt, 0.9, (3, 4), refs, grids, trace=tb)
    assert torch.equal(ta["x_txt"], tb["x_txt"]) and torch.equal(ta["x_ref"], tb["x_ref"])
    assert (ta["x_img"] - tb["x_img"]).abs().max() > 1e-4
    tc = {}
    O3.forward3(p3, hp(d), img, txt, 0.2, (3, 4), refs, grids, trace=tc, ctx_time=0.5)
    assert (tc["x_txt"] - ta["x_txt"]).abs().max() > 1e-4


# ---------------------------------------------------------------- guidance and image editing (sampler)
def _sampler_case(seed, flow_map=False):
    d = Flux3Dims(**{**MICRO3.__dict__, "flow_map": flow_map})
    p3 = params(d, seed)
    g = torch.Generator().manual_seed(seed + 100)
    noise = torch.randn(32, 6, 8, generator=g, dtype=F64)
    txt_c = torch.randn(5, 40, generator=g, dtype=F64)
    txt_u = torch.randn(5, 40, generator=g, dtype=F64)
    return d, p3, noise, txt_c, txt_u


def test_guidance_one_and_zero_select_one_text():
    """v_u + g (v_c - v_u): g = 1 is the prompt's sampler, g = 0 the unconditional text's."""
    d, p3, noise, txt_c, txt_u = _sampler_case(21)
    plain_c, _ = O3.sample3(p3, hp(d), noise, txt_c, 3)
    plain_u, _ = O3.sample3(p3, hp(d), noise, txt_u, 3)
    g1, _ = O3.sample3(p3, hp(d), noise, txt_c, 3, txt_uncond=txt_u, guidance=1.0)
    g0, _ = O3.sample3(p3, hp(d), noise, txt_c, 3, txt_uncond=txt_u, guidance=0.0)
    assert torch.allclose(g1, plain_c, atol=1e-12, rtol=0)
    assert torch.allclose(g0, plain_u, atol=1e-12, rtol=0)
    g3, _ = O3.sample3(p3, hp(d), noise, txt_c, 3, txt_uncond=txt_u, guidance=3.5)
    assert (g3 - plain_c).abs().max() > 1e-3      # a real extrapolation moves the result


def test_guidance_with_one_text_is_the_plain_sampler():
    d, p3, noise, txt_c, _ = _sampler_case(22, flow_map=True)
    plain, _ = O3.sample3(p3, hp(d), noise, txt_c, 3)
    guided, _ = O3.sample3(p3, hp(d), noise, txt_c, 3, txt_uncond=txt_c, guidance=3.5)
    assert torch.allclose(guided, plain, atol=1e-12, rtol=0)


def test_image_and_reference_streams_leave_the_per_mode_phase_independent_of_the_text():
    """In the per-mode blocks each stream attends only to itself, so the image and reference
    streams that enter the joint blocks are the same for the prompt and the unconditional text
    (a guided batch may compute them once)."""
    d = Flux3Dims(**{**MICRO3.__dict__, "n_mode": 2})
    p3 = params(d, 23)
    img, txt, refs, grids = inputs(24)
    txt2 = torch.randn_like(txt)
    a, b = {}, {}
    va = O3.forward3(p3, hp(d), img, txt, 0.6, (3, 4), refs, grids, trace=a)
    vb = O3.forward3(p3, hp(d), img, txt2, 0.6, (3, 4), refs, grids, trace=b)
    assert torch.equal(a["x_img"], b["x_img"]) and torch.equal(a["x_ref"], b["x_ref"])
    assert (a["x_txt"] - b["x_txt"]).abs().max() > 1e-3
    assert (va - vb).abs().max() > 1e-4        # the joint blocks bring the text in


def test_image_editing_starts_late_on_the_blended_latent():
    """strength 1 is text-to-image; strength s < 1 starts at schedule step img2img_start(S, s)
    from (1 - t) init + t noise, and the flow-map target times follow the same schedule."""
    d, p3, noise, txt_c, _ = _sampler_case(25, flow_map=True)
    init = torch.randn(32, 6, 8, generator=torch.Generator().manual_seed(26), dtype=F64)
    plain, _ = O3.sample3(p3, hp(d), noise, txt_c, 4)
    full, _ = O3.sample3(p3, hp(d), noise, txt_c, 4, init_latent=init, strength=1.0)
    assert torch.allclose(full, plain, atol=1e-12, rtol=0)
    seen = []
    orig = O3.forward3

    def spy(*args, **kw):
        seen.append((args[2].clone(), args[4], kw.get("t_target")))
        return orig(*args, **kw)

    O3.forward3 = spy
    try:
        O3.sample3(p3, hp(d), noise, txt_c, 4, init_latent=init, strength=0.5)
    finally:
        O3.forward3 = orig
    assert [(t, tt) for _, t, tt in seen] == [(0.5, 0.25), (0.25, 0.0)]
    first = O.unpack_latents(seen[0][0], 6, 8)
    assert torch.allclose(first, 0.5 * init + 0.5 * noise, atol=1e-12, rtol=0)
