"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks the oracle against what the pages fix (token counts, the RoPE
coordinate table), a closed form, an invariant, brute force on a tiny input, or
a special case that reduces to a PyTorch library routine (F.layer_norm,
F.rms_norm, F.silu, F.scaled_dot_product_attention).  The library-based special
cases are written with different primitives than the oracle, so a dropped term,
a wrong sign, a wrong index or a transposed operand in the oracle fails one of
them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import flux_oracle as O
from synthetic import FluxDims, Workload, WORKLOADS, make_weights, make_inputs, bf16_bits_to_f32

torch.set_grad_enabled(False)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F64 = torch.float64

MICRO = FluxDims(n_double=1, n_single=1, hidden=64, heads=2, head_dim=32, mlp_hidden=96,
                 in_ch=128, txt_dim=48, t_freq_dim=256)


def micro_params(seed=0, dims=MICRO):
    _, p = make_weights(dims, seed, threads=4)
    return {k: torch.from_numpy(bf16_bits_to_f32(v)).double() for k, v in p.items()}


def hp_of(d):
    return O.hyper(d)


# ---------------------------------------------------------------------------- tokens
def test_token_counts_match_pages():
    g = json.load(open(os.path.join(GOLDEN, "token_counts.json")))
    lat = torch.zeros(g["latent_channels"], 1024 // 8, 1024 // 8)
    tok = O.pack_latents(lat)
    assert tok.shape == (g["tokens_1024x1024"], g["token_channels"])
    assert 1024 // g["pixels_per_token_side"] == g["grid_1024x1024"][0]
    for name, n_img in (("tiny64", 16), ("t2i256", 256), ("t2i512", 1024), ("t2i1024", 4096)):
        w = WORKLOADS[name]
        assert w.n_img == n_img
        assert O.pack_latents(torch.zeros(32, w.image // 8, w.image // 8)).shape[0] == n_img
    w = WORKLOADS["i2i1024"]
    assert w.n_ref == g["reference_1024x1024_extra_tokens"]
    assert w.n_tokens == 512 + 4096 + 4096
    assert WORKLOADS["t2i1024"].n_tokens == 4608


def test_pack_brute_force_and_round_trip():
    g = torch.Generator().manual_seed(1)
    for c, h8, w8 in ((32, 6, 10), (32, 2, 2), (3, 4, 8)):
        lat = torch.randn(c, h8, w8, generator=g)
        tok = O.pack_latents(lat)
        gw = w8 // 2
        assert tok.shape == ((h8 // 2) * gw, 4 * c)
        for i in range(h8 // 2):
            for j in range(gw):
                for ch in range(c):
                    for py in range(2):
                        for px in range(2):
                            assert tok[i * gw + j, ch * 4 + py * 2 + px] == lat[ch, 2 * i + py, 2 * j + px]
        back = O.unpack_latents(tok, h8, w8)
        assert torch.equal(back, lat)


# ---------------------------------------------------------------------------- attention
def _qkv(n, h, d, seed=0, dtype=F64):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(n, h, d, generator=g, dtype=dtype) for _ in range(3))


def test_attention_rows_sum_to_one():
    q, k, _ = _qkv(37, 3, 16)
    p = O.attention_probs(q * 3, k)
    assert torch.allclose(p.sum(-1), torch.ones(3, 37, dtype=F64), atol=1e-12, rtol=0)
    assert (p >= 0).all()


def test_attention_naive_triple_loop():
    n, h, d = 6, 2, 4
    q, k, v = _qkv(n, h, d, seed=3)
    out = O.attention(q, k, v).reshape(n, h, d)
    for hh in range(h):
        for i in range(n):
            s = [sum(float(q[i, hh, c]) * float(k[j, hh, c]) for c in range(d)) / math.sqrt(d)
                 for j in range(n)]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = sum(e)
            for c in range(d):
                ref = sum(e[j] / z * float(v[j, hh, c]) for j in range(n))
                assert abs(float(out[i, hh, c]) - ref) < 1e-12


def test_attention_matches_library_sdpa():
    n, h, d = 50, 4, 32
    q, k, v = _qkv(n, h, d, seed=4)
    ref = F.scaled_dot_product_attention(q.permute(1, 0, 2), k.permute(1, 0, 2), v.permute(1, 0, 2))
    out = O.attention(q, k, v).reshape(n, h, d).permute(1, 0, 2)
    assert torch.allclose(out, ref, atol=1e-12, rtol=0)


def test_attention_zero_query_gives_mean_value():
    n, h, d = 9, 2, 8
    _, k, v = _qkv(n, h, d, seed=5)
    out = O.attention(torch.zeros(n, h, d, dtype=F64), k, v).reshape(n, h, d)
    assert torch.allclose(out, v.mean(0, keepdim=True).expand(n, h, d), atol=1e-14, rtol=0)


def test_attention_permutation_equivariant():
    n, h, d = 21, 2, 8
    q, k, v = _qkv(n, h, d, seed=6)
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(0))
    out = O.attention(q, k, v)
    outp = O.attention(q[perm], k[perm], v[perm])
    assert torch.allclose(outp, out[perm], atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------- norms
def test_layer_norm_matches_library_and_invariants():
    x = torch.randn(7, 3072, dtype=F64) * 3 + 1.5
    y = O.layer_norm(x, 1e-6)
    assert torch.allclose(y, F.layer_norm(x, (3072,), eps=1e-6), atol=1e-12, rtol=0)
    assert torch.allclose(y.mean(-1), torch.zeros(7, dtype=F64), atol=1e-12)
    assert torch.allclose(y.var(-1, unbiased=False), torch.ones(7, dtype=F64), atol=1e-6)


def test_rms_norm_matches_library_and_unit_rms():
    x = torch.randn(5, 4, 128, dtype=F64) * 2
    gain = torch.randn(128, dtype=F64)
    y = O.rms_norm(x, gain, 1e-6)
    assert torch.allclose(y, F.rms_norm(x, (128,), gain, eps=1e-6), atol=1e-12, rtol=0)
    y1 = O.rms_norm(x, torch.ones(128, dtype=F64), 1e-6)
    assert torch.allclose(y1.pow(2).mean(-1).sqrt(), torch.ones(5, 4, dtype=F64), atol=1e-6)


def test_modulate_closed_form():
    y = torch.tensor([[1.0, -2.0]], dtype=F64)
    out = O.modulate(y, torch.tensor([0.5, 0.25], dtype=F64), torch.tensor([1.0, -0.5], dtype=F64))
    assert torch.equal(out, torch.tensor([[2.5, -0.75]], dtype=F64))


def test_silu_closed_form():
    x = torch.tensor([0.0, 1.0, -1.0, 20.0, -40.0], dtype=F64)
    y = O.silu(x)
    assert y[0] == 0
    assert abs(float(y[1]) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(float(y[2]) + math.exp(-1.0) / (1.0 + math.exp(-1.0))) < 1e-15
    assert torch.allclose(y, F.silu(x), atol=1e-15, rtol=0)


# ---------------------------------------------------------------------------- RoPE
def test_rope_coordinate_table_from_pages():
    g = json.load(open(os.path.join(GOLDEN, "rope_coordinates.json")))
    n_txt, gh, gw, rh, rw = 6, 3, 4, 2, 3
    pos = O.token_positions(n_txt, gh, gw, ref_grids=[(rh, rw), (rh, rw)])
    assert pos.shape == (n_txt + gh * gw + 2 * rh * rw, 4)
    assert torch.equal(O.token_positions(n_txt, gh, gw, rh, rw), pos[:n_txt + gh * gw + rh * rw])
    for c in g["cases"]:
        if c["kind"] == "text":
            row = c["index"]
        elif c["kind"] == "image":
            row = n_txt + c["row"] * gw + c["col"]
        else:
            row = n_txt + gh * gw + c["k"] * rh * rw + c["row"] * rw + c["col"]
        assert pos[row].tolist() == [float(v) for v in c["coord"]]
    # several references of different sizes follow one another, reference k at l = -(k+1)
    pos2 = O.token_positions(n_txt, gh, gw, ref_grids=[(rh, rw), (rh, rw), (1, 2)])
    assert pos2.shape[0] == n_txt + gh * gw + 2 * rh * rw + 2
    assert pos2[-1].tolist() == [0.0, 0.0, 1.0, -3.0]
    assert torch.equal(pos2[:pos.shape[0]], pos)


def test_rope_unit_vector_closed_form():
    """e_(2p) at a position with only axis a set turns to (cos, sin)(pos * theta^(-2m/32))."""
    theta, d = 10000.0, 128
    for a, m, posval in ((0, 0, 3.0), (1, 5, 7.0), (2, 15, 63.0), (3, 1, -1.0), (3, 9, 511.0)):
        pos = torch.zeros(1, 4, dtype=F64)
        pos[0, a] = posval
        ang = O.rope_angles(pos, d, theta)
        x = torch.zeros(1, 1, d, dtype=F64)
        pair = a * 16 + m
        x[0, 0, 2 * pair] = 1.0
        y = O.apply_rope(x, ang)
        w = posval * theta ** (-2.0 * m / 32.0)
        expect = torch.zeros(d, dtype=F64)
        expect[2 * pair] = math.cos(w)
        expect[2 * pair + 1] = math.sin(w)
        assert torch.allclose(y[0, 0], expect, atol=1e-12, rtol=0)


def test_rope_matches_complex_rotation():
    """Same rotation written with complex numbers (a different formulation)."""
    g = torch.Generator().manual_seed(2)
    n, h, d = 11, 3, 128
    x = torch.randn(n, h, d, generator=g, dtype=F64)
    pos = O.token_positions(3, 2, 4)
    ang = O.rope_angles(pos, d, 10000.0)
    z = torch.view_as_complex(x.reshape(n, h, d // 2, 2).contiguous())
    rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]
    ref = torch.view_as_real(z * rot).reshape(n, h, d)
    assert torch.allclose(O.apply_rope(x, ang), ref, atol=1e-12, rtol=0)


def test_rope_invariants():
    g = torch.Generator().manual_seed(3)
    n, h, d = 8, 2, 128
    q = torch.randn(n, h, d, generator=g, dtype=F64)
    k = torch.randn(n, h, d, generator=g, dtype=F64)
    pos = torch.randint(-20, 60, (n, 4), generator=g).to(F64)
    zero = O.apply_rope(q, O.rope_angles(torch.zeros(n, 4, dtype=F64), d, 1e4))
    assert torch.equal(zero, q)
    qr = O.apply_rope(q, O.rope_angles(pos, d, 1e4))
    assert torch.allclose(qr.norm(dim=-1), q.norm(dim=-1), atol=1e-12, rtol=0)
    shift = torch.tensor([[1.0, -3.0, 5.0, 17.0]], dtype=F64)
    kr = O.apply_rope(k, O.rope_angles(pos, d, 1e4))
    qs = O.apply_rope(q, O.rope_angles(pos + shift, d, 1e4))
    ks = O.apply_rope(k, O.rope_angles(pos + shift, d, 1e4))
    dots = torch.einsum("ihd,jhd->hij", qr, kr)
    dots_s = torch.einsum("ihd,jhd->hij", qs, ks)
    assert torch.allclose(dots, dots_s, atol=1e-9, rtol=0)


# ---------------------------------------------------------------------------- timestep
def test_timestep_embedding_closed_forms():
    e0 = O.timestep_embedding(0.0)
    assert torch.equal(e0, torch.cat([torch.ones(128, dtype=F64), torch.zeros(128, dtype=F64)]))
    e = O.timestep_embedding(math.pi / 2000.0)       # first frequency is 1: angle pi/2
    assert abs(float(e[0])) < 1e-12 and abs(float(e[128]) - 1.0) < 1e-12
    # frequencies are geometric from 1 down to 1e4^(-127/128)
    t = 1e-3 / 1000.0                                 # small angle: sin(a) ~ a
    s = O.timestep_embedding(t)[128:] / 1e-3
    f = torch.tensor([1e4 ** (-j / 128.0) for j in range(128)], dtype=F64)
    assert torch.allclose(s, f, rtol=1e-6, atol=0)


# ---------------------------------------------------------------------------- blocks
def _library_vec(p, t):
    temb = O.timestep_embedding(t)
    h = F.silu(F.linear(temb, p["time_in.w1"], p["time_in.b1"]))
    return F.linear(h, p["time_in.w2"], p["time_in.b2"])


def _micro_inputs(seed=0, n_txt=5, gh=3, gw=4):
    g = torch.Generator().manual_seed(seed)
    img = torch.randn(gh * gw, MICRO.in_ch, generator=g, dtype=F64)
    txt = torch.randn(n_txt, MICRO.txt_dim, generator=g, dtype=F64)
    return img, txt


def _zero_gates(p):
    D = MICRO.hidden
    q = dict(p)
    for k in list(q):
        if k.endswith("mod.w") or k.endswith("mod.b"):
            v = q[k].clone()
            chunks = 6 if k.startswith("double") else 3 if k.startswith("single") else 0
            gate_chunks = (2, 5) if chunks == 6 else (2,) if chunks == 3 else ()
            for c in gate_chunks:
                v[c * D:(c + 1) * D] = 0
            q[k] = v
    return q


def test_zero_gates_make_blocks_identity():
    """With every gate 0 the velocity is output(LN(img_in(x))), built here from library ops."""
    p = _zero_gates(micro_params(1))
    img, txt = _micro_inputs(1)
    t = 0.6
    v = O.forward(p, hp_of(MICRO), img, txt, t, (3, 4))
    s = F.silu(_library_vec(p, t))
    D = MICRO.hidden
    m = F.linear(s, p["final.mod.w"], p["final.mod.b"])
    shift, scale = m[:D], m[D:]
    x = F.linear(img, p["img_in.w"], p["img_in.b"])
    y = F.layer_norm(x, (D,), eps=1e-6) * (1 + scale) + shift
    ref = F.linear(y, p["final.out.w"], p["final.out.b"])
    assert torch.allclose(v, ref, atol=1e-10, rtol=0)


def _library_rope(x, pos, theta=1e4):
    """Complex-number RoPE built from the pages' axis layout, independent of the oracle."""
    n, h, d = x.shape
    ad = d // 4
    omega = torch.tensor([theta ** (-2.0 * m / ad) for m in range(ad // 2)], dtype=F64)
    ang = torch.cat([pos[:, a:a + 1] * omega[None, :] for a in range(4)], dim=1)
    z = torch.view_as_complex(x.reshape(n, h, d // 2, 2).contiguous())
    return torch.view_as_real(z * torch.polar(torch.ones_like(ang), ang)[:, None, :]).reshape(n, h, d)


def _library_attention(q, k, v):
    o = F.scaled_dot_product_attention(q.permute(1, 0, 2), k.permute(1, 0, 2), v.permute(1, 0, 2))
    return o.permute(1, 0, 2).reshape(q.shape[0], -1)


def test_single_block_mlp_branch_alone():
    """q, k, v rows of the fused linear zeroed: the block reduces to x + g*(W2 [0; silu(a) b] + b2)."""
    p = micro_params(2)
    D, Fh = MICRO.hidden, MICRO.mlp_hidden
    p["single.0.lin1.w"][:3 * D] = 0
    p["single.0.lin1.b"][:3 * D] = 0
    g = torch.Generator().manual_seed(4)
    x = torch.randn(10, D, generator=g, dtype=F64)
    s = F.silu(torch.randn(D, generator=g, dtype=F64))
    ang = O.rope_angles(O.token_positions(4, 2, 3), MICRO.head_dim, 1e4)
    out = O.single_block(p, 0, x, s, ang, hp_of(MICRO))
    sh, sc, gate = F.linear(s, p["single.0.mod.w"], p["single.0.mod.b"]).split(D)
    y = F.layer_norm(x, (D,), eps=1e-6) * (1 + sc) + sh
    h = F.linear(y, p["single.0.lin1.w"][3 * D:], p["single.0.lin1.b"][3 * D:])
    a, b = h[:, :Fh], h[:, Fh:]
    ref = x + gate * F.linear(F.silu(a) * b, p["single.0.lin2.w"][:, D:], p["single.0.lin2.b"])
    assert torch.allclose(out, ref, atol=1e-10, rtol=0)


def test_single_block_attention_branch_alone():
    """a, b rows zeroed: the block reduces to x + g*(W2[:, :D] attn(rope(rms(q)), rope(rms(k)), v) + b2)."""
    p = micro_params(3)
    D, H, hd = MICRO.hidden, MICRO.heads, MICRO.head_dim
    p["single.0.lin1.w"][3 * D:] = 0
    p["single.0.lin1.b"][3 * D:] = 0
    g = torch.Generator().manual_seed(5)
    x = torch.randn(10, D, generator=g, dtype=F64)
    s = F.silu(torch.randn(D, generator=g, dtype=F64))
    pos = O.token_positions(4, 2, 3)
    ang = O.rope_angles(pos, hd, 1e4)
    out = O.single_block(p, 0, x, s, ang, hp_of(MICRO))
    sh, sc, gate = F.linear(s, p["single.0.mod.w"], p["single.0.mod.b"]).split(D)
    y = F.layer_norm(x, (D,), eps=1e-6) * (1 + sc) + sh
    qkv = F.linear(y, p["single.0.lin1.w"][:3 * D], p["single.0.lin1.b"][:3 * D])
    q, k, v = (z.reshape(10, H, hd) for z in qkv.split(D, dim=1))
    q = _library_rope(F.rms_norm(q, (hd,), p["single.0.q_gain"], eps=1e-6), pos)
    k = _library_rope(F.rms_norm(k, (hd,), p["single.0.k_gain"], eps=1e-6), pos)
    o = _library_attention(q, k, v)
    ref = x + gate * F.linear(o, p["single.0.lin2.w"][:, :D], p["single.0.lin2.b"])
    assert torch.allclose(out, ref, atol=1e-10, rtol=0)


def test_double_block_matches_library_composition():
    """Per-stream weights, joint attention over [text; image], then the MLP on the updated residual."""
    p = micro_params(4)
    D, H, hd, Fh = MICRO.hidden, MICRO.heads, MICRO.head_dim, MICRO.mlp_hidden
    g = torch.Generator().manual_seed(6)
    nt, ni = 4, 6
    xt = torch.randn(nt, D, generator=g, dtype=F64)
    xi = torch.randn(ni, D, generator=g, dtype=F64)
    s = F.silu(torch.randn(D, generator=g, dtype=F64))
    pos = O.token_positions(nt, 2, 3)
    ot, oi = O.double_block(p, 0, xt, xi, s, O.rope_angles(pos, hd, 1e4), hp_of(MICRO))

    def pre(x, st):
        m = F.linear(s, p[f"double.0.{st}.mod.w"], p[f"double.0.{st}.mod.b"]).split(D)
        y = F.layer_norm(x, (D,), eps=1e-6) * (1 + m[1]) + m[0]
        q, k, v = (z.reshape(len(x), H, hd) for z in
                   F.linear(y, p[f"double.0.{st}.qkv.w"], p[f"double.0.{st}.qkv.b"]).split(D, 1))
        q = F.rms_norm(q, (hd,), p[f"double.0.{st}.q_gain"], eps=1e-6)
        k = F.rms_norm(k, (hd,), p[f"double.0.{st}.k_gain"], eps=1e-6)
        return q, k, v, m

    qt, kt, vt, mt = pre(xt, "txt")
    qi, ki, vi, mi = pre(xi, "img")
    o = _library_attention(_library_rope(torch.cat([qt, qi]), pos), _library_rope(torch.cat([kt, ki]), pos),
                           torch.cat([vt, vi]))
    refs = []
    for x, os_, m, st in ((xt, o[:nt], mt, "txt"), (xi, o[nt:], mi, "img")):
        x = x + m[2] * F.linear(os_, p[f"double.0.{st}.proj.w"], p[f"double.0.{st}.proj.b"])
        y = F.layer_norm(x, (D,), eps=1e-6) * (1 + m[4]) + m[3]
        h = F.linear(y, p[f"double.0.{st}.mlp_in.w"], p[f"double.0.{st}.mlp_in.b"])
        x = x + m[5] * F.linear(F.silu(h[:, :Fh]) * h[:, Fh:], p[f"double.0.{st}.mlp_out.w"],
                                p[f"double.0.{st}.mlp_out.b"])
        refs.append(x)
    assert torch.allclose(ot, refs[0], atol=1e-10, rtol=0)
    assert torch.allclose(oi, refs[1], atol=1e-10, rtol=0)


def test_double_block_attention_is_joint_from_first_block():
    """Changing one text token changes image outputs of block 0 (joint attention [P5])."""
    p = micro_params(5)
    D, hd = MICRO.hidden, MICRO.head_dim
    g = torch.Generator().manual_seed(7)
    xt = torch.randn(3, D, generator=g, dtype=F64)
    xi = torch.randn(4, D, generator=g, dtype=F64)
    s = F.silu(torch.randn(D, generator=g, dtype=F64))
    ang = O.rope_angles(O.token_positions(3, 2, 2), hd, 1e4)
    _, oi = O.double_block(p, 0, xt, xi, s, ang, hp_of(MICRO))
    xt2 = xt.clone()
    xt2[1] += torch.randn(D, generator=g, dtype=F64)   # a constant shift would vanish in LN
    _, oi2 = O.double_block(p, 0, xt2, xi, s, ang, hp_of(MICRO))
    assert (oi - oi2).abs().max() > 1e-6
    # the text stream's MLP weights never reach the image rows
    p2 = dict(p)
    p2["double.0.txt.mlp_out.w"] = p["double.0.txt.mlp_out.w"] * 3
    _, oi3 = O.double_block(p2, 0, xt, xi, s, ang, hp_of(MICRO))
    assert torch.equal(oi3, oi)


def test_model_permutation_equivariant_without_rope():
    p = micro_params(6)
    img, txt = _micro_inputs(2, n_txt=3, gh=3, gw=3)
    n = 3 + 9
    zero_pos = torch.zeros(n, 4, dtype=F64)
    v = O.forward(p, hp_of(MICRO), img, txt, 0.3, (3, 3), positions=zero_pos)
    perm = torch.randperm(9, generator=torch.Generator().manual_seed(1))
    vp = O.forward(p, hp_of(MICRO), img[perm], txt, 0.3, (3, 3), positions=zero_pos)
    assert torch.allclose(vp, v[perm], atol=1e-10, rtol=0)
    # with RoPE the image grid positions matter
    v_rope = O.forward(p, hp_of(MICRO), img, txt, 0.3, (3, 3))
    assert (v_rope - v).abs().max() > 1e-6


def test_reference_tokens_are_context_only():
    p = micro_params(7)
    img, txt = _micro_inputs(3, gh=2, gw=2)
    ref = torch.randn(4, MICRO.in_ch, generator=torch.Generator().manual_seed(9), dtype=F64)
    v0 = O.forward(p, hp_of(MICRO), img, txt, 0.5, (2, 2))
    v1 = O.forward(p, hp_of(MICRO), img, txt, 0.5, (2, 2), ref_tok=ref, ref_hw=(2, 2))
    assert v1.shape == v0.shape == (4, MICRO.in_ch)
    assert (v1 - v0).abs().max() > 1e-6


# ---------------------------------------------------------------------------- sampler
def test_schedule_and_constant_velocity_euler():
    assert O.schedule(4) == [1.0, 0.75, 0.5, 0.25, 0.0]
    assert O.schedule(1) == [1.0, 0.0]
    x = torch.randn(16, 128, dtype=torch.float32)
    v = torch.randn(16, 128, dtype=torch.float32).to(torch.bfloat16).float()
    ts = O.schedule(4)
    y = x.clone()
    for i in range(4):
        y = O.euler_update(y, v, ts[i + 1] - ts[i])
    assert torch.allclose(y, x - v, atol=1e-6, rtol=0)
    # dt are exact binary fractions: the fp64 sum of the steps is exactly -1
    assert sum(ts[i + 1] - ts[i] for i in range(4)) == -1.0


def test_sampler_uses_schedule_times():
    """The sampler calls forward at t_0..t_{S-1} and never updates reference tokens."""
    p = micro_params(8)
    lat = torch.randn(32, 4, 4, generator=torch.Generator().manual_seed(3), dtype=F64)
    txt = torch.randn(2, MICRO.txt_dim, generator=torch.Generator().manual_seed(4), dtype=F64)
    final, vs = O.sample(p, hp_of(MICRO), lat, txt, 2)
    tok = O.pack_latents(lat)
    v0 = O.forward(p, hp_of(MICRO), tok, txt, 1.0, (2, 2))
    assert torch.allclose(vs[0], v0, atol=0, rtol=0)
    tok1 = tok - 0.5 * v0
    v1 = O.forward(p, hp_of(MICRO), tok1, txt, 0.5, (2, 2))
    assert torch.allclose(vs[1], v1, atol=1e-12, rtol=0)
    assert torch.allclose(final, O.unpack_latents(tok1 - 0.5 * v1, 4, 4), atol=1e-12, rtol=0)


def test_img2img_strength_end_points_from_pages():
    """strength 0 keeps the input latent unchanged; strength 1 equals sampling from pure noise."""
    g = json.load(open(os.path.join(GOLDEN, "img2img_and_references.json")))
    p = micro_params(9)
    gen = torch.Generator().manual_seed(11)
    noise = torch.randn(32, 4, 4, generator=gen, dtype=F64)
    init = torch.randn(32, 4, 4, generator=gen, dtype=F64)
    txt = torch.randn(3, MICRO.txt_dim, generator=gen, dtype=F64)
    kept, vs = O.sample(p, hp_of(MICRO), noise, txt, 4, init_latent=init, strength=g["strength_keeps_original"])
    assert vs == [] and torch.equal(kept, init)
    full, _ = O.sample(p, hp_of(MICRO), noise, txt, 4, init_latent=init, strength=g["strength_regenerates"])
    plain, _ = O.sample(p, hp_of(MICRO), noise, txt, 4)
    assert torch.equal(full, plain)
    # the default strength runs the last 3 of 4 steps, from t = 0.75
    assert O.img2img_start(4, g["strength_default"]) == 1 and O.schedule(4)[1] == 0.75
    part, vs = O.sample(p, hp_of(MICRO), noise, txt, 4, init_latent=init, strength=0.75)
    assert len(vs) == 3


def test_blend_latents_closed_forms():
    x = torch.randn(5, dtype=F64)
    n = torch.randn(5, dtype=F64)
    assert torch.equal(O.blend_latents(x, n, 0.0), x)
    assert torch.equal(O.blend_latents(x, n, 1.0), n)
    assert torch.allclose(O.blend_latents(x, n, 0.5), (x + n) / 2, atol=1e-15, rtol=0)


def test_multiple_references_are_ordered_and_distinguished():
    """Reference order matters (l = -1 vs -2); a one-element list equals the single-reference call."""
    g = json.load(open(os.path.join(GOLDEN, "img2img_and_references.json")))
    p = micro_params(10)
    img, txt = _micro_inputs(4, gh=2, gw=2)
    gen = torch.Generator().manual_seed(12)
    r0 = torch.randn(4, MICRO.in_ch, generator=gen, dtype=F64)
    r1 = torch.randn(4, MICRO.in_ch, generator=gen, dtype=F64)
    one = O.forward(p, hp_of(MICRO), img, txt, 0.5, (2, 2), r0, (2, 2))
    one_list = O.forward(p, hp_of(MICRO), img, txt, 0.5, (2, 2), [r0], [(2, 2)])
    assert torch.equal(one, one_list)
    a = O.forward(p, hp_of(MICRO), img, txt, 0.5, (2, 2), [r0, r1], [(2, 2), (2, 2)])
    b = O.forward(p, hp_of(MICRO), img, txt, 0.5, (2, 2), [r1, r0], [(2, 2), (2, 2)])
    assert (a - b).abs().max() > 1e-6
    # with RoPE off the two references are interchangeable context
    n = 5 + 4 + 8
    z = torch.zeros(n, 4, dtype=F64)
    az = O.forward(p, hp_of(MICRO), img, txt, 0.5, (2, 2), [r0, r1], [(2, 2), (2, 2)], positions=z)
    bz = O.forward(p, hp_of(MICRO), img, txt, 0.5, (2, 2), [r1, r0], [(2, 2), (2, 2)], positions=z)
    assert torch.allclose(az, bz, atol=1e-10, rtol=0)
    assert g["max_reference_images"] == 10


@pytest.mark.slow
def test_fp32_oracle_close_to_fp64_on_tiny_workload():
    w = WORKLOADS["tiny64"]
    _, p = make_weights(w.dims, w.seed)
    lat, txt, _ = make_inputs(w)
    hp = O.hyper(w.dims)
    tok = O.pack_latents(torch.from_numpy(lat))
    v64 = O.forward(p, hp, tok, torch.from_numpy(txt), 1.0, (w.grid, w.grid), dtype=F64)
    v32 = O.forward(p, hp, tok, torch.from_numpy(txt), 1.0, (w.grid, w.grid), dtype=torch.float32)
    rel = ((v32.double() - v64).norm() / v64.norm()).item()
    assert rel < 1e-5


def test_weight_widening_is_exact():
    bits = np.array([0x3F80, 0xBF80, 0x0000, 0x4049, 0x7F7F, 0x0001], dtype=np.uint16)
    w = O.weight({"w": bits}, "w", F64)
    ref = [1.0, -1.0, 0.0, 3.140625, 3.3895313892515355e38, 9.183549615799121e-41]
    assert w.tolist() == ref


# ---------------------------------------------------------------------------- classifier-free guidance
def _guidance_case(seed):
    p = micro_params(seed)
    gen = torch.Generator().manual_seed(100 + seed)
    noise = torch.randn(32, 4, 6, generator=gen, dtype=F64)
    txt_c = torch.randn(5, MICRO.txt_dim, generator=gen, dtype=F64)
    txt_u = torch.randn(5, MICRO.txt_dim, generator=gen, dtype=F64)
    return p, noise, txt_c, txt_u


def test_guidance_one_and_zero_select_one_text():
    """g = 1 follows the prompt alone, g = 0 the unconditional text alone (which side is which)."""
    p, noise, txt_c, txt_u = _guidance_case(13)
    cond, vc = O.sample(p, hp_of(MICRO), noise, txt_c, 3)
    uncond, vu = O.sample(p, hp_of(MICRO), noise, txt_u, 3)
    g1, v1 = O.sample(p, hp_of(MICRO), noise, txt_c, 3, txt_uncond=txt_u, guidance=1.0)
    g0, v0 = O.sample(p, hp_of(MICRO), noise, txt_c, 3, txt_uncond=txt_u, guidance=0.0)
    assert torch.allclose(g1, cond, atol=1e-12, rtol=0) and torch.allclose(g0, uncond, atol=1e-12, rtol=0)
    for a, b in zip(v1, vc):
        assert torch.allclose(a, b, atol=1e-12, rtol=0)
    assert (cond - uncond).abs().max() > 1e-3          # the two texts do steer differently


def test_guidance_with_identical_texts_is_unguided():
    p, noise, txt_c, _ = _guidance_case(14)
    g = json.load(open(os.path.join(GOLDEN, "guidance.json")))
    plain, _ = O.sample(p, hp_of(MICRO), noise, txt_c, 2)
    guided, _ = O.sample(p, hp_of(MICRO), noise, txt_c, 2, txt_uncond=txt_c.clone(), guidance=g["base_guidance"])
    assert torch.allclose(guided, plain, atol=1e-12, rtol=0)


def test_guided_velocity_is_affine_in_the_scale():
    """One step from the same state: v(g) = (1 - g) v(0) + g v(1) also outside [0, 1] (no clamping)."""
    p, noise, txt_c, txt_u = _guidance_case(15)
    g = json.load(open(os.path.join(GOLDEN, "guidance.json")))["base_guidance"]
    vs = {}
    for s in (0.0, 1.0, g):
        _, v = O.sample(p, hp_of(MICRO), noise, txt_c, 1, txt_uncond=txt_u, guidance=s)
        vs[s] = v[0]
    assert torch.allclose(vs[g], (1 - g) * vs[0.0] + g * vs[1.0], atol=1e-12, rtol=0)
    assert (vs[g] - vs[1.0]).abs().max() > 1e-3


def test_guidance_settings_from_pages():
    g = json.load(open(os.path.join(GOLDEN, "guidance.json")))
    assert g["base_steps"] == 50 and g["base_guidance"] == 3.5
    assert g["distilled_steps"] == 16 and g["distilled_guidance"] is None
    # the base schedule: 51 evenly spaced times from 1 to 0
    ts = O.schedule(g["base_steps"])
    assert len(ts) == 51 and ts[0] == 1.0 and ts[-1] == 0.0 and abs(ts[25] - 0.5) < 1e-7
