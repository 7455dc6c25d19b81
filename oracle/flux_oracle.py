"""Plain CPU oracle of the FLUX.2-klein denoising transformer and its Euler sampler.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product path (``latent_flow_matching_b200``) never calls it and
shares no code with it.

The oracle writes the method out as its definition, one step after another, with
elementary PyTorch CPU tensor ops (matmul, exp, mean, ...) in float64 by default
(float32 when asked, which is the precision the pages' own C implementation
uses: hakusoku.com story 4662, "FLUX.2-klein-4B Pure C 実装の特徴": safetensors
read as float, no quantisation).  No blocking, fusion or reordering beyond the
definition.

Sources (web pages, by title and section):
* [P1] "Flux 2 Klein: Reine C-basierte Inferenz" (de.news.hada.io), section
  "Modellarchitektur und Leistung": 5 double + 20 single blocks, width 3072,
  24 heads; 4 sampling steps.
* [P2] hakusoku.com story 4662, "技術詳細" (same facts) and "CライブラリAPI".
* [P5] "FLUX.3 Image Klein in Diffusers: Architektur, ..." (mindverse), sections
  "Zweistufiger Transformer und Tokenisierung" (2x2 packing, 16x16 px tokens),
  "Entkoppelte Vorverarbeitung und gemeinsame Attention-Blöcke" (text|image|ref
  order, FLUX.2 joint attention from block 1, QK-RMSNorm, SwiGLU, parallel
  attention+MLP, image tokens only at the output), "Modulation pro Token-Typ,
  Flow-Map-Destillation und 4D-RoPE" (LayerNorm without affine, shift/scale/gate
  from the timestep embedding, one timestep for all tokens in FLUX.2, 4-axis
  RoPE with 32 dims per axis and its coordinate table).

Readings where the pages are silent:
* timestep embedding: 256 dims, t scaled by 1000, max period 1e4, [cos, sin];
  MLP 256 -> 3072 -> 3072 with SiLU between.
* modulation: one Linear(3072 -> k*3072) per block and stream applied to
  SiLU(vec); chunk order (shift1, scale1, gate1, shift2, scale2, gate2) for a
  double-block stream, (shift, scale, gate) for a single block, (shift, scale)
  for the output layer.  LN output is modulated as LN(x)*(1+scale)+shift.
* double block: attention then MLP, sequentially; single block: attention and
  MLP in parallel on the same modulated input.
* RoPE: axis order (t, h, w, l) in the head dim, 32 dims per axis, adjacent
  pairs (2m, 2m+1), frequency theta^(-2m/32); text token i at (0,0,0,i), image
  token (r,c) at (0,r,c,0), reference token (r,c) at (0,r,c,-1), with r, c the
  token-grid indices.
* SwiGLU: [a; b] = W_in y + bias, output W_out (silu(a) * b) + bias.
* LN and RMS eps 1e-6; RMSNorm gain of 128 values per stream, shared by heads.
* Euler: t_i = linspace(1, 0, S+1); x <- x + (t_{i+1} - t_i) v(x, t_i).
* img2img strength s: run the last floor(S s) steps, starting from
  (1 - t) x_in + t noise at the first kept t.  Several references: reference k at
  RoPE l = -(k+1), tokens appended in order after the image tokens.
* guidance g: v = v_u + g (v_c - v_u) with v_u the velocity for an unconditional text
  of the same token count (prompts are padded and the padding is attended, so both
  passes see sequences of one length).
"""
from __future__ import annotations

import math

import torch

__all__ = [
    "pack_latents", "unpack_latents", "token_positions", "rope_angles", "apply_rope",
    "layer_norm", "rms_norm", "modulate", "silu", "linear", "attention_probs",
    "attention", "timestep_embedding", "double_block", "single_block", "forward",
    "schedule", "euler_update", "img2img_start", "blend_latents", "guided_velocity", "sample", "weight",
    "block_linear",
]

CPU = torch.device("cpu")


def weight(p, name, dtype):
    """A parameter as a float tensor: bf16 bit patterns (uint16) are widened exactly."""
    w = p[name]
    if not isinstance(w, torch.Tensor):
        w = torch.from_numpy(w)
    if w.dtype in (torch.uint16, torch.int16):
        w = (w.to(torch.int32) & 0xFFFF) << 16
        w = w.view(torch.float32)
    return w.to(device=CPU, dtype=dtype)


# ----------------------------------------------------------------------------
# [P5 "Zweistufiger Transformer und Tokenisierung"] 2x2 latent packing
# ----------------------------------------------------------------------------
def pack_latents(lat: torch.Tensor) -> torch.Tensor:
    """[32, h8, w8] -> [(h8/2)(w8/2), 128].

    Token (i, j) (row-major over the token grid) holds channel c*4 + py*2 + px
    = lat[c, 2i+py, 2j+px]: one token per 2x2 latent patch, 32*4 = 128 channels.
    """
    c, h8, w8 = lat.shape
    gh, gw = h8 // 2, w8 // 2
    return lat.reshape(c, gh, 2, gw, 2).permute(1, 3, 0, 2, 4).reshape(gh * gw, c * 4)


def unpack_latents(tok: torch.Tensor, h8: int, w8: int) -> torch.Tensor:
    """Inverse of :func:`pack_latents`."""
    gh, gw = h8 // 2, w8 // 2
    c = tok.shape[1] // 4
    return tok.reshape(gh, gw, c, 2, 2).permute(2, 0, 3, 1, 4).reshape(c, h8, w8)


# ----------------------------------------------------------------------------
# [P5 "Modulation pro Token-Typ, Flow-Map-Destillation und 4D-RoPE"] positions
# ----------------------------------------------------------------------------
def token_positions(n_txt, grid_h, grid_w, ref_h=0, ref_w=0, dtype=torch.float64, ref_grids=None):
    """(t, h, w, l) coordinates of the joint sequence [text; image; reference 0; reference 1; ...].

    Reference k's token (r, c) sits at (0, r, c, -(k+1)).  ``ref_grids`` lists the (h, w) of
    every reference; without it, (ref_h, ref_w) describes a single reference (0 = none).
    """
    if ref_grids is None:
        ref_grids = [(ref_h, ref_w)] if ref_h > 0 else []
    rows = []
    for i in range(n_txt):
        rows.append((0.0, 0.0, 0.0, float(i)))
    for r in range(grid_h):
        for c in range(grid_w):
            rows.append((0.0, float(r), float(c), 0.0))
    for k, (rh, rw) in enumerate(ref_grids):
        for r in range(rh):
            for c in range(rw):
                rows.append((0.0, float(r), float(c), -float(k + 1)))
    return torch.tensor(rows, dtype=dtype).reshape(-1, 4)


def rope_angles(pos: torch.Tensor, head_dim: int, theta: float) -> torch.Tensor:
    """[N, 4] coordinates -> [N, head_dim/2] rotation angles.

    Axis a owns dims [a*head_dim/4, (a+1)*head_dim/4); its pair m turns by
    pos[a] * theta^(-2m / (head_dim/4)).
    """
    axis_dim = head_dim // 4
    m = torch.arange(axis_dim // 2, dtype=pos.dtype)
    omega = theta ** (-2.0 * m / axis_dim)                      # [axis_dim/2]
    ang = pos[:, :, None] * omega[None, None, :]                # [N, 4, axis_dim/2]
    return ang.reshape(pos.shape[0], head_dim // 2)


def apply_rope(x: torch.Tensor, ang: torch.Tensor) -> torch.Tensor:
    """Rotate adjacent pairs (2p, 2p+1) of x [N, H, d] by ang [N, d/2]."""
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    c = torch.cos(ang)[:, None, :]
    s = torch.sin(ang)[:, None, :]
    out = torch.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# ----------------------------------------------------------------------------
# norms, activations, linear
# ----------------------------------------------------------------------------
def layer_norm(x: torch.Tensor, eps: float) -> torch.Tensor:
    """LayerNorm over the last axis with no learned scale or shift [P5 modulation section]."""
    mu = x.mean(dim=-1, keepdim=True)
    var = ((x - mu) ** 2).mean(dim=-1, keepdim=True)
    return (x - mu) / torch.sqrt(var + eps)


def rms_norm(x: torch.Tensor, gain: torch.Tensor, eps: float) -> torch.Tensor:
    """x / sqrt(mean(x^2) + eps) * gain over the last axis (QK-RMSNorm, [P5 joint blocks])."""
    return x / torch.sqrt((x * x).mean(dim=-1, keepdim=True) + eps) * gain


def modulate(y: torch.Tensor, shift: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """Timestep-driven scale and shift of a normalised input [P5 modulation section]."""
    return y * (1.0 + scale) + shift


def silu(x: torch.Tensor) -> torch.Tensor:
    return x / (1.0 + torch.exp(-x))


def linear(x: torch.Tensor, w: torch.Tensor, b: torch.Tensor | None) -> torch.Tensor:
    """x W^T + b, W stored [out, in]."""
    y = torch.matmul(x, w.t())
    return y if b is None else y + b


# ----------------------------------------------------------------------------
# [P5 joint blocks] attention over the whole joint sequence, no mask
# ----------------------------------------------------------------------------
def attention_probs(q: torch.Tensor, k: torch.Tensor) -> torch.Tensor:
    """Per-head softmax(q k^T / sqrt(d)) for q, k [N, H, d] -> [H, N, N]."""
    d = q.shape[-1]
    s = torch.einsum("ihd,jhd->hij", q, k) / math.sqrt(d)
    s = s - s.max(dim=-1, keepdim=True).values
    e = torch.exp(s)
    return e / e.sum(dim=-1, keepdim=True)


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
    """softmax(q k^T / sqrt(d)) v per head; q, k, v [N, H, d] -> [N, H*d].

    Heads are processed one at a time to bound memory; each is the plain definition.
    """
    n, h, d = q.shape
    out = torch.empty(n, h, d, dtype=q.dtype)
    for hh in range(h):
        p = attention_probs(q[:, hh:hh + 1], k[:, hh:hh + 1])[0]    # [N, N]
        out[:, hh] = torch.matmul(p, v[:, hh])
    return out.reshape(n, h * d)


# ----------------------------------------------------------------------------
# [P5 modulation section] timestep embedding -> vec
# ----------------------------------------------------------------------------
def timestep_embedding(t: float, dim: int = 256, max_period: float = 10000.0,
                       t_scale: float = 1000.0, dtype=torch.float64) -> torch.Tensor:
    """[cos(t*1000*f_j), sin(t*1000*f_j)], f_j = max_period^(-j/(dim/2)), j < dim/2."""
    half = dim // 2
    j = torch.arange(half, dtype=dtype)
    f = torch.exp(-math.log(max_period) * j / half)
    a = (t * t_scale) * f
    return torch.cat([torch.cos(a), torch.sin(a)])


def block_linear(hp):
    """The linear layer used inside the transformer blocks: the plain definition, the row-wise
    FP8 one (``oracle/fp8_oracle.py``) when ``hp["fp8"]`` is set, or the NVFP4 one
    (``oracle/nvfp4_oracle.py``) when ``hp["nvfp4"]`` is set."""
    if hp.get("fp8"):
        from .fp8_oracle import linear_fp8
        return linear_fp8
    if hp.get("nvfp4"):
        from .nvfp4_oracle import linear_nvfp4
        return linear_nvfp4
    return linear


def _heads(x, heads, head_dim):
    return x.reshape(x.shape[0], heads, head_dim)


def _pre_attention(p, prefix, x, s, hp, dtype):
    """One stream's modulated LN -> QKV -> QK-RMSNorm (double block)."""
    D = x.shape[1]
    m = linear(s, weight(p, prefix + "mod.w", dtype), weight(p, prefix + "mod.b", dtype))
    sh1, sc1, g1, sh2, sc2, g2 = m.split(D)
    y = modulate(layer_norm(x, hp["eps_ln"]), sh1, sc1)
    qkv = block_linear(hp)(y, weight(p, prefix + "qkv.w", dtype), weight(p, prefix + "qkv.b", dtype))
    q, k, v = (_heads(z, hp["heads"], hp["head_dim"]) for z in qkv.split(D, dim=1))
    q = rms_norm(q, weight(p, prefix + "q_gain", dtype), hp["eps_rms"])
    k = rms_norm(k, weight(p, prefix + "k_gain", dtype), hp["eps_rms"])
    return q, k, v, (g1, sh2, sc2, g2)


def _mlp(p, prefix, y, dtype, lin_in="mlp_in", lin_out="mlp_out", hp=None):
    lin = block_linear(hp or {})
    h = lin(y, weight(p, prefix + lin_in + ".w", dtype), weight(p, prefix + lin_in + ".b", dtype))
    a, b = h.chunk(2, dim=1)
    return lin(silu(a) * b, weight(p, prefix + lin_out + ".w", dtype), weight(p, prefix + lin_out + ".b", dtype))


def double_block(p, i, x_txt, x_img, s, ang, hp, dtype=torch.float64):
    """Double-stream block i: separate text / image weights, joint attention [P1, P5]."""
    pt, pi = f"double.{i}.txt.", f"double.{i}.img."
    qt, kt, vt, mt = _pre_attention(p, pt, x_txt, s, hp, dtype)
    qi, ki, vi, mi = _pre_attention(p, pi, x_img, s, hp, dtype)
    q = apply_rope(torch.cat([qt, qi]), ang)
    k = apply_rope(torch.cat([kt, ki]), ang)
    v = torch.cat([vt, vi])
    o = attention(q, k, v)
    nt = x_txt.shape[0]
    outs = []
    for x, o_s, (g1, sh2, sc2, g2), pre in ((x_txt, o[:nt], mt, pt), (x_img, o[nt:], mi, pi)):
        x = x + g1 * block_linear(hp)(o_s, weight(p, pre + "proj.w", dtype), weight(p, pre + "proj.b", dtype))
        y = modulate(layer_norm(x, hp["eps_ln"]), sh2, sc2)
        x = x + g2 * _mlp(p, pre, y, dtype, hp=hp)
        outs.append(x)
    return outs[0], outs[1]


def single_block(p, i, x, s, ang, hp, dtype=torch.float64):
    """Single-stream block i: shared weights, attention and SwiGLU MLP in parallel [P5]."""
    pre = f"single.{i}."
    D = x.shape[1]
    F = (p[pre + "lin1.w"].shape[0] - 3 * D) // 2
    sh, sc, g = linear(s, weight(p, pre + "mod.w", dtype), weight(p, pre + "mod.b", dtype)).split(D)
    y = modulate(layer_norm(x, hp["eps_ln"]), sh, sc)
    h = block_linear(hp)(y, weight(p, pre + "lin1.w", dtype), weight(p, pre + "lin1.b", dtype))
    q, k, v, a, b = h.split([D, D, D, F, F], dim=1)
    q = rms_norm(_heads(q, hp["heads"], hp["head_dim"]), weight(p, pre + "q_gain", dtype), hp["eps_rms"])
    k = rms_norm(_heads(k, hp["heads"], hp["head_dim"]), weight(p, pre + "k_gain", dtype), hp["eps_rms"])
    v = _heads(v, hp["heads"], hp["head_dim"])
    o = attention(apply_rope(q, ang), apply_rope(k, ang), v)
    return x + g * block_linear(hp)(torch.cat([o, silu(a) * b], dim=1),
                                    weight(p, pre + "lin2.w", dtype), weight(p, pre + "lin2.b", dtype))


def _count(p, kind):
    idx = {int(k.split(".")[1]) for k in p if k.startswith(kind + ".")}
    return max(idx) + 1 if idx else 0


def forward(p, hp, img_tok, txt, t, grid_hw, ref_tok=None, ref_hw=(0, 0),
            dtype=torch.float64, positions=None):
    """Velocity v [Ni, 128] of the image tokens at time t.

    img_tok [Ni, 128], txt [Nt, txt_dim].  References: ref_tok [Nr, 128] with
    ref_hw = (h, w) for one, or a list of token tensors with a list of (h, w)
    for several (reference k at RoPE l = -(k+1) [P5]).  The joint sequence is
    ordered text | image | references [P5]; reference tokens go through the
    image-stream weights and the same t (one timestep for every token in
    FLUX.2 [P5]).  ``positions`` overrides the RoPE coordinates (all zeros
    switches RoPE off).
    """
    if isinstance(ref_tok, (list, tuple)):
        ref_grids = list(ref_hw)
        ref_tok = torch.cat([torch.as_tensor(r) for r in ref_tok]) if ref_tok else None
    else:
        ref_grids = [tuple(ref_hw)] if ref_tok is not None else []
    img_tok = torch.as_tensor(img_tok).to(dtype)
    txt = torch.as_tensor(txt).to(dtype)
    ni, nt = img_tok.shape[0], txt.shape[0]
    temb = timestep_embedding(float(t), p["time_in.w1"].shape[1], dtype=dtype)
    h = silu(linear(temb, weight(p, "time_in.w1", dtype), weight(p, "time_in.b1", dtype)))
    vec = linear(h, weight(p, "time_in.w2", dtype), weight(p, "time_in.b2", dtype))
    s = silu(vec)

    tok = img_tok
    if ref_tok is not None:
        tok = torch.cat([img_tok, torch.as_tensor(ref_tok).to(dtype)])
    x_img = linear(tok, weight(p, "img_in.w", dtype), weight(p, "img_in.b", dtype))
    x_txt = linear(txt, weight(p, "txt_in.w", dtype), weight(p, "txt_in.b", dtype))

    if positions is None:
        positions = token_positions(nt, grid_hw[0], grid_hw[1], dtype=dtype, ref_grids=ref_grids)
    ang = rope_angles(positions.to(dtype), hp["head_dim"], hp["rope_theta"])

    for i in range(_count(p, "double")):
        x_txt, x_img = double_block(p, i, x_txt, x_img, s, ang, hp, dtype)
    x = torch.cat([x_txt, x_img])
    for i in range(_count(p, "single")):
        x = single_block(p, i, x, s, ang, hp, dtype)

    x_out = x[nt:nt + ni]                          # text and reference tokens dropped [P5]
    D = x.shape[1]
    sh, sc = linear(s, weight(p, "final.mod.w", dtype), weight(p, "final.mod.b", dtype)).split(D)
    y = modulate(layer_norm(x_out, hp["eps_ln"]), sh, sc)
    return linear(y, weight(p, "final.out.w", dtype), weight(p, "final.out.b", dtype))


# ----------------------------------------------------------------------------
# [P1 "Modellarchitektur und Leistung": 4 sampling steps] Euler flow matching
# ----------------------------------------------------------------------------
def schedule(n_steps: int) -> list[float]:
    """t_0 = 1, ..., t_S = 0, evenly spaced, as float32 values."""
    return [float(torch.tensor(1.0 - i / n_steps, dtype=torch.float32)) for i in range(n_steps + 1)]


def euler_update(x: torch.Tensor, v: torch.Tensor, dt: float) -> torch.Tensor:
    return x + dt * v


# ----------------------------------------------------------------------------
# img2img strength ["Flux 2 Klein: Reine C-basierte Inferenz", "Nutzungsbeispiele":
# -t 0.0 keeps the input, 1.0 regenerates it; hakusoku "コマンドラインオプション": default 0.75]
# ----------------------------------------------------------------------------
def img2img_start(n_steps: int, strength: float) -> int:
    """Index of the first schedule step run for a given strength.

    Reading (the pages give only the two end points): run the last floor(S * strength)
    steps of the S-step schedule; strength 1 runs them all, 0 runs none.
    """
    k = min(int(n_steps * strength), n_steps)
    return n_steps - k


def blend_latents(x: torch.Tensor, noise: torch.Tensor, t: float) -> torch.Tensor:
    """The flow-matching state at time t between data x (t = 0) and noise (t = 1)."""
    return (1.0 - t) * x + t * noise


# ----------------------------------------------------------------------------
# Classifier-free guidance [hakusoku.com story 4662, "CライブラリAPI": the parameter
# struct carries guidance_scale, the CFG scale; "FLUX.3 Image Klein: offene Gewichte
# ..." (kimiseek), opening section: the base checkpoint samples 50 steps with guidance,
# the distilled one 16 steps without; we0.ai article on FLUX 3 Image Klein, checkpoint
# table: Klein Base, 50 steps, guidance 3.5]
# ----------------------------------------------------------------------------
def guided_velocity(v_cond: torch.Tensor, v_uncond: torch.Tensor, g: float) -> torch.Tensor:
    """Reading (the pages name the scale, not the formula): extrapolate from the velocity of
    the unconditional text towards that of the prompt, v_u + g (v_c - v_u)."""
    return v_uncond + g * (v_cond - v_uncond)


def sample(p, hp, latent, txt, n_steps, ref_latent=None, dtype=torch.float64, on_step=None,
           init_latent=None, strength=1.0, txt_uncond=None, guidance=None):
    """Run the sampler; returns (final latent [32, h8, w8], list of velocities [Ni, 128]).

    ``latent`` is the noise.  ``ref_latent`` is one reference latent or a list of them
    (context tokens, never updated).  With ``init_latent`` (the latent of an image to
    edit) and ``strength`` < 1 the run starts at schedule step img2img_start(S, strength)
    from blend_latents(init_latent, latent, t_start).  With ``guidance`` g, every step
    runs the forward once with ``txt`` and once with ``txt_uncond`` (same image and
    references) and moves along guided_velocity; the returned velocities are the guided
    ones.  ``on_step(i, v)`` is called after every step if given.
    """
    latent = torch.as_tensor(latent).to(dtype)
    c, h8, w8 = latent.shape
    ts = schedule(n_steps)
    start = 0
    if init_latent is not None:
        start = img2img_start(n_steps, strength)
        latent = blend_latents(torch.as_tensor(init_latent).to(dtype), latent, ts[start])
    tok = pack_latents(latent)
    refs = [] if ref_latent is None else (list(ref_latent) if isinstance(ref_latent, (list, tuple)) else [ref_latent])
    ref_toks, ref_grids = [], []
    for r in refs:
        r = torch.as_tensor(r).to(dtype)
        ref_toks.append(pack_latents(r))
        ref_grids.append((r.shape[1] // 2, r.shape[2] // 2))
    vs = []
    for i in range(start, n_steps):
        v = forward(p, hp, tok, txt, ts[i], (h8 // 2, w8 // 2), ref_toks, ref_grids, dtype)
        if guidance is not None:
            v_u = forward(p, hp, tok, txt_uncond, ts[i], (h8 // 2, w8 // 2), ref_toks, ref_grids, dtype)
            v = guided_velocity(v, v_u, guidance)
        vs.append(v)
        if on_step is not None:
            on_step(i, v)
        tok = euler_update(tok, v, ts[i + 1] - ts[i])
    return unpack_latents(tok, h8, w8), vs


def hyper(dims) -> dict:
    """The scalar hyper-parameters the oracle needs, from any object with the dims fields."""
    return {k: getattr(dims, k) for k in ("heads", "head_dim", "rope_theta", "eps_ln", "eps_rms")}
