"""Plain CPU oracle of the FLUX.3 Image Klein denoising transformer and its sampler.

TEST INFRASTRUCTURE ONLY, like ``flux_oracle`` (whose elementary operations it reuses:
LayerNorm, RMSNorm, RoPE, attention, timestep embedding, linear layers).  Only ``tests/``
and ``bench.py``'s CPU legs may import it; the product path never does.

Source: "FLUX.3 Image Klein in Diffusers: Architektur, Layout-Steuerung und
Systemanforderungen im Überblick" (mindverse), sections
* "Zweistufiger Transformer und Tokenisierung": 2x2-packed 128-channel latent tokens; text
  features are the hidden states of 8 encoder layers (8 x 2560 = 20480) projected to the
  transformer width 3072 by one linear layer;
* "Entkoppelte Vorverarbeitung und gemeinsame Attention-Blöcke": 5 per-mode blocks in which
  the text, noisy-image and reference streams have their own weights and attend only to
  themselves, then 28 joint blocks with one weight set over the sequence text | image |
  reference; in every block attention and the SwiGLU MLP run in parallel on the same
  normalised input and are added to the residual; Q and K are RMS-normalised; only image
  tokens reach the output layers;
* "Modulation pro Token-Typ, Flow-Map-Destillation und 4D-RoPE": LayerNorm without affine,
  shift / scale / gate from a timestep embedding; image tokens are modulated with the
  current t, text and reference tokens always with t = 0; the time-distilled checkpoint
  embeds the target time of each step with its own embedding and adds it to every token's
  modulation; 4-axis RoPE as in FLUX.2 (text i at (0,0,0,i), image (r,c) at (0,r,c,0),
  reference k at (0,r,c,-(k+1))).
"FLUX.3 Image Klein: offene Gewichte ..." (kimiseek): the distilled checkpoint samples 16
steps without guidance.  we0.ai FLUX 3 Image Klein article: 5.6 B generator parameters.

Readings where the page is silent:
* modulation linears are shared by the blocks of a phase: one Linear(3072 -> 3*3072) per
  stream for the per-mode blocks, one for the joint blocks, Linear(3072 -> 2*3072) for the
  output layer.  With per-block linears the model would have 6.7 B parameters; shared, it
  has 5.49 B, next to the stated 5.6 B;
* "t = 0 for text and reference tokens" holds in the per-mode blocks as well (the page says
  they receive it permanently);
* the target-time embedding has the time embedding's shape (sinusoid 256 -> MLP 3072 ->
  3072) and is added to the time vector before SiLU and the modulation linears, for every
  token; the sampler's target time of step i is t_{i+1};
* reference tokens use the image input projection; the reference stream of the per-mode
  blocks is all reference images together (they attend to one another);
* block arithmetic (QK-RMSNorm gain per stream, biases, SwiGLU silu(a) * b, eps 1e-6) as in
  the FLUX.2 single-stream block; with ``hp["fp8"]`` its two linears are the row-wise FP8 ones
  (the fp8r format of section "Hardwareanforderungen, Quantisierung und Inferenzlatenz").
"""
from __future__ import annotations

import torch

from . import flux_oracle as O

__all__ = ["time_vector", "parallel_block", "forward3", "sample3"]


def _count(p, prefix):
    idx = {int(k.split(".")[1]) for k in p if k.startswith(prefix + ".")}
    return max(idx) + 1 if idx else 0


def _mlp2(p, name, x, dtype):
    h = O.silu(O.linear(x, O.weight(p, name + ".w1", dtype), O.weight(p, name + ".b1", dtype)))
    return O.linear(h, O.weight(p, name + ".w2", dtype), O.weight(p, name + ".b2", dtype))


def time_vector(p, t, t_target, dtype=torch.float64):
    """vec(t) = MLP_time(emb(t)) (+ MLP_target(emb(t_target)) for the flow-map checkpoint)."""
    dim = p["time_in.w1"].shape[1]
    vec = _mlp2(p, "time_in", O.timestep_embedding(float(t), dim, dtype=dtype), dtype)
    if "target_in.w1" in p:
        if t_target is None:
            raise ValueError("the flow-map model needs a target time")
        vec = vec + _mlp2(p, "target_in", O.timestep_embedding(float(t_target), dim, dtype=dtype), dtype)
    return vec


def parallel_block(p, pre, x, shift, scale, gate, ang, hp, dtype=torch.float64):
    """x + gate * W2 [attn(q, k, v) | silu(a) * b] of LN(x) (1 + scale) + shift, with per-row
    (or shared) shift / scale / gate; attention over the rows of x only."""
    D = x.shape[1]
    F = (p[pre + "lin1.w"].shape[0] - 3 * D) // 2
    y = O.modulate(O.layer_norm(x, hp["eps_ln"]), shift, scale)
    lin = O.block_linear(hp)                    # row-wise FP8 when hp["fp8"] (oracle/fp8_oracle.py)
    h = lin(y, O.weight(p, pre + "lin1.w", dtype), O.weight(p, pre + "lin1.b", dtype))
    q, k, v, a, b = h.split([D, D, D, F, F], dim=1)
    q = O.rms_norm(O._heads(q, hp["heads"], hp["head_dim"]), O.weight(p, pre + "q_gain", dtype), hp["eps_rms"])
    k = O.rms_norm(O._heads(k, hp["heads"], hp["head_dim"]), O.weight(p, pre + "k_gain", dtype), hp["eps_rms"])
    v = O._heads(v, hp["heads"], hp["head_dim"])
    o = O.attention(O.apply_rope(q, ang), O.apply_rope(k, ang), v)
    return x + gate * lin(torch.cat([o, O.silu(a) * b], dim=1),
                          O.weight(p, pre + "lin2.w", dtype), O.weight(p, pre + "lin2.b", dtype))


def forward3(p, hp, img_tok, txt, t, grid_hw, ref_tok=None, ref_hw=(), t_target=None,
             dtype=torch.float64, positions=None, ctx_time=0.0, trace=None):
    """Velocity [Ni, 128] of the image tokens.

    img_tok [Ni, 128]; txt [Nt, 20480]; ref_tok: None, one [Nr, 128] tensor with ref_hw = (h, w),
    or a list of tensors with a list of (h, w).  ``t_target``: the step's target time (flow-map
    checkpoint only).  ``ctx_time`` is the time the text and reference tokens are modulated with
    (0 on the pages; other values only serve the oracle's own pins).  ``positions`` overrides the
    RoPE coordinates of text | image | reference (zeros switch RoPE off).  ``trace``: a dict that
    receives the three streams after the per-mode phase (for the oracle's pins).
    """
    if isinstance(ref_tok, (list, tuple)):
        ref_grids = list(ref_hw)
        ref_tok = torch.cat([torch.as_tensor(r) for r in ref_tok]) if len(ref_tok) else None
    else:
        ref_grids = [tuple(ref_hw)] if ref_tok is not None else []
    img_tok = torch.as_tensor(img_tok).to(dtype)
    txt = torch.as_tensor(txt).to(dtype)
    ni, nt = img_tok.shape[0], txt.shape[0]
    nr = 0 if ref_tok is None else ref_tok.shape[0]
    D = p["time_in.w2"].shape[0]

    s_img = O.silu(time_vector(p, t, t_target, dtype))          # image tokens: current t
    s_ctx = O.silu(time_vector(p, ctx_time, t_target, dtype))   # text and reference tokens: t = 0

    x_txt = O.linear(txt, O.weight(p, "txt_in.w", dtype), O.weight(p, "txt_in.b", dtype))
    x_img = O.linear(img_tok, O.weight(p, "img_in.w", dtype), O.weight(p, "img_in.b", dtype))
    x_ref = None
    if nr:
        x_ref = O.linear(torch.as_tensor(ref_tok).to(dtype), O.weight(p, "img_in.w", dtype),
                         O.weight(p, "img_in.b", dtype))

    if positions is None:
        positions = O.token_positions(nt, grid_hw[0], grid_hw[1], dtype=dtype, ref_grids=ref_grids)
    ang = O.rope_angles(positions.to(dtype), hp["head_dim"], hp["rope_theta"])
    ang_txt, ang_img, ang_ref = ang[:nt], ang[nt:nt + ni], ang[nt + ni:]

    # phase 1: per-mode blocks, each stream on its own
    def mods(name, s):
        return O.linear(s, O.weight(p, name + ".w", dtype), O.weight(p, name + ".b", dtype)).split(D)

    m_txt, m_img, m_ref = mods("mode_mod.txt", s_ctx), mods("mode_mod.img", s_img), mods("mode_mod.ref", s_ctx)
    for i in range(_count(p, "mode")):
        if nt:
            x_txt = parallel_block(p, f"mode.{i}.txt.", x_txt, *m_txt, ang_txt, hp, dtype)
        x_img = parallel_block(p, f"mode.{i}.img.", x_img, *m_img, ang_img, hp, dtype)
        if nr:
            x_ref = parallel_block(p, f"mode.{i}.ref.", x_ref, *m_ref, ang_ref, hp, dtype)

    if trace is not None:
        trace.update(x_txt=x_txt.clone(), x_img=x_img.clone(), x_ref=None if x_ref is None else x_ref.clone())

    # phase 2: joint blocks over text | image | reference, modulation per token type
    x = torch.cat([x_txt, x_img] + ([x_ref] if nr else []))
    j_img, j_ctx = mods("joint_mod", s_img), mods("joint_mod", s_ctx)
    is_img = torch.zeros(x.shape[0], 1, dtype=torch.bool)
    is_img[nt:nt + ni] = True
    shift, scale, gate = (torch.where(is_img, a, c) for a, c in zip(j_img, j_ctx))
    for i in range(_count(p, "joint")):
        x = parallel_block(p, f"joint.{i}.", x, shift, scale, gate, ang, hp, dtype)

    x_out = x[nt:nt + ni]                                      # text and reference tokens dropped
    sh, sc = O.linear(s_img, O.weight(p, "final.mod.w", dtype), O.weight(p, "final.mod.b", dtype)).split(D)
    y = O.modulate(O.layer_norm(x_out, hp["eps_ln"]), sh, sc)
    return O.linear(y, O.weight(p, "final.out.w", dtype), O.weight(p, "final.out.b", dtype))


def sample3(p, hp, latent, txt, n_steps, ref_latent=None, dtype=torch.float64, on_step=None,
            init_latent=None, strength=1.0, txt_uncond=None, guidance=None):
    """Euler sampling with the FLUX.3 model; the flow-map checkpoint gets t_{i+1} as the target
    time of step i.  Returns (final latent [32, h8, w8], list of velocities).

    ``init_latent`` / ``strength`` (image editing) and ``guidance`` / ``txt_uncond``
    (classifier-free guidance, the base checkpoint's 50 steps at guidance 3.5 in the we0.ai
    FLUX 3 Image Klein article's checkpoint table) follow the FLUX.2 sampler's readings:
    start at schedule step img2img_start(S, strength) from blend_latents(init, noise, t_start);
    every guided step evaluates the prompt and the unconditional text on the same image and
    moves along guided_velocity (the returned velocities are the guided ones)."""
    latent = torch.as_tensor(latent).to(dtype)
    c, h8, w8 = latent.shape
    ts = O.schedule(n_steps)
    start = 0
    if init_latent is not None:
        start = O.img2img_start(n_steps, strength)
        latent = O.blend_latents(torch.as_tensor(init_latent).to(dtype), latent, ts[start])
    tok = O.pack_latents(latent)
    refs = [] if ref_latent is None else (list(ref_latent) if isinstance(ref_latent, (list, tuple)) else [ref_latent])
    ref_toks = [O.pack_latents(torch.as_tensor(r).to(dtype)) for r in refs]
    ref_grids = [(r.shape[1] // 2, r.shape[2] // 2) for r in refs]
    vs = []
    for i in range(start, n_steps):
        tt = ts[i + 1] if "target_in.w1" in p else None
        v = forward3(p, hp, tok, txt, ts[i], (h8 // 2, w8 // 2), ref_toks, ref_grids, t_target=tt, dtype=dtype)
        if guidance is not None:
            v_u = forward3(p, hp, tok, txt_uncond, ts[i], (h8 // 2, w8 // 2), ref_toks, ref_grids, t_target=tt,
                           dtype=dtype)
            v = O.guided_velocity(v, v_u, guidance)
        vs.append(v)
        if on_step is not None:
            on_step(i, v)
        tok = O.euler_update(tok, v, ts[i + 1] - ts[i])
    return O.unpack_latents(tok, h8, w8), vs
