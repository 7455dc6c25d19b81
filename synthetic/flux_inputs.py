"""Seeded synthetic inputs for the FLUX.2-klein denoising transformer.

This module only draws random numbers and lays bytes out.  It holds none of
the model's arithmetic: both the CPU oracle (``oracle/``) and the CUDA path
(``latent_flow_matching_b200``) receive the same arrays from here and compute
independently.

Recipe (every value is a bf16 number, stored as its 16 raw bits):

* Each weight tensor ``i`` (index in blob order) is filled chunk by chunk; chunk
  ``c`` (``CHUNK`` elements) comes from ``numpy.random.default_rng([seed, i, c])``
  (PCG64 seeded through SeedSequence), ``standard_normal(float32)``, multiplied
  by ``1/sqrt(fan_in)`` in float32, then rounded to bf16 (nearest, ties to even).
  Gains of the QK-RMSNorm have ``fan_in = 1``; a bias uses its layer's fan-in.
  Chunking keeps the values independent of the number of worker threads.
* The latent ``[32, H/8, W/8]``, the text features ``[Nt, txt_dim]`` and the
  reference latent come from ``default_rng([seed, INPUT_KEY + k])`` with
  k = 0, 1, 2 respectively, N(0,1) rounded to bf16.

Architecture facts behind the shapes: 5 double-stream and 20 single-stream
blocks, width 3072, 24 heads of 128 (antirez flux pages, "Modellarchitektur und
Leistung"; hakusoku "技術詳細"); 32-channel latent packed 2x2 into 128-channel
tokens (mindverse FLUX.3 write-up, "Zweistufiger Transformer und Tokenisierung").
"""
from __future__ import annotations

import dataclasses
import struct
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

CHUNK = 1 << 22           # elements per independently seeded chunk
INPUT_KEY = 1_000_000     # seed-key offset of the latent / text / reference draws
BLOB_MAGIC = b"FLUXDIT\0"
BLOB3_MAGIC = b"FLUX3DT\0"
BLOB_VERSION = 1
HEADER_BYTES = 256
ALIGN = 256


@dataclasses.dataclass(frozen=True)
class FluxDims:
    n_double: int = 5
    n_single: int = 20
    hidden: int = 3072
    heads: int = 24
    head_dim: int = 128
    mlp_hidden: int = 9216
    in_ch: int = 128
    txt_dim: int = 3072
    t_freq_dim: int = 256
    rope_theta: float = 10000.0
    eps_ln: float = 1e-6
    eps_rms: float = 1e-6


@dataclasses.dataclass(frozen=True)
class Flux3Dims:
    """FLUX.3 Image Klein ("FLUX.3 Image Klein in Diffusers: ..." (mindverse), sections
    "Zweistufiger Transformer und Tokenisierung" and "Entkoppelte Vorverarbeitung und
    gemeinsame Attention-Blöcke"): 5 per-mode blocks (own weights for the text, image and
    reference streams, attention within a stream) then 28 joint blocks (one weight set,
    attention over text | image | reference), every block in the parallel attention + SwiGLU
    form; text features are 8 stacked encoder layers of 2560 (20480) projected to 3072.
    ``flow_map``: the time-distilled checkpoint's extra embedding of the target time
    (section "Modulation pro Token-Typ, Flow-Map-Destillation und 4D-RoPE")."""
    n_mode: int = 5
    n_joint: int = 28
    hidden: int = 3072
    heads: int = 24
    head_dim: int = 128
    mlp_hidden: int = 9216
    in_ch: int = 128
    txt_dim: int = 20480
    t_freq_dim: int = 256
    rope_theta: float = 10000.0
    eps_ln: float = 1e-6
    eps_rms: float = 1e-6
    flow_map: bool = True


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic generation problem (batch 1)."""
    name: str
    seed: int
    image: int            # square image side in pixels
    n_txt: int
    ref_image: int        # 0 = no reference image
    n_steps: int
    dims: FluxDims
    extra_refs: tuple = ()  # sides of further reference images, after ref_image
    guidance: float | None = None   # classifier-free guidance scale (None: unguided)

    @property
    def grid(self) -> int:       # image tokens per side (16 px per token)
        return self.image // 16

    @property
    def ref_grid(self) -> int:
        return self.ref_image // 16

    @property
    def ref_images(self) -> tuple:
        return ((self.ref_image,) if self.ref_image else ()) + tuple(self.extra_refs)

    @property
    def ref_grids(self) -> list:
        return [(r // 16, r // 16) for r in self.ref_images]

    @property
    def n_img(self) -> int:
        return self.grid * self.grid

    @property
    def n_ref(self) -> int:
        return sum(h * w for h, w in self.ref_grids)

    @property
    def n_tokens(self) -> int:
        return self.n_txt + self.n_img + self.n_ref


TINY_DIMS = FluxDims(n_double=1, n_single=1)
FULL_DIMS = FluxDims()
F3_TINY_DIMS = Flux3Dims(n_mode=1, n_joint=1)
F3_FULL_DIMS = Flux3Dims()
F3_BASE_DIMS = Flux3Dims(flow_map=False)
F3_TINY_BASE_DIMS = Flux3Dims(n_mode=1, n_joint=1, flow_map=False)

WORKLOADS = {
    "tiny64": Workload("tiny64", 0, 64, 16, 0, 1, TINY_DIMS),
    "t2i256": Workload("t2i256", 1, 256, 512, 0, 4, FULL_DIMS),
    "t2i512": Workload("t2i512", 2, 512, 512, 0, 4, FULL_DIMS),
    "t2i1024": Workload("t2i1024", 3, 1024, 512, 0, 4, FULL_DIMS),
    "i2i1024": Workload("i2i1024", 4, 1024, 512, 1024, 4, FULL_DIMS),
    "mref1024": Workload("mref1024", 5, 1024, 512, 512, 4, FULL_DIMS, extra_refs=(512,)),
    # guided sampling: the base checkpoint's 3.5 (its 50 steps on the 1024^2 workload; the
    # 256^2 golden case keeps 4 steps so the oracle finishes in minutes)
    "cfg256": Workload("cfg256", 6, 256, 512, 0, 4, FULL_DIMS, guidance=3.5),
    "cfg1024": Workload("cfg1024", 7, 1024, 512, 0, 50, FULL_DIMS, guidance=3.5),
    # FLUX.3 Image Klein, time-distilled checkpoint (16 steps, flow-map target time).  Text token
    # counts from the pages' per-call totals: 4256 = 4096 + 160 at 1024^2, 8272 = 4096 + 4096 + 80
    # with one 1024^2 reference (mindverse, "Einfluss von Referenzbildern auf die Sequenzlänge").
    "f3tiny64": Workload("f3tiny64", 20, 64, 16, 64, 1, F3_TINY_DIMS),
    "f3t2i256": Workload("f3t2i256", 21, 256, 160, 0, 4, F3_FULL_DIMS),
    "f3i2i256": Workload("f3i2i256", 22, 256, 80, 256, 4, F3_FULL_DIMS),
    "f3t2i1024": Workload("f3t2i1024", 23, 1024, 160, 0, 16, F3_FULL_DIMS),
    "f3i2i1024": Workload("f3i2i1024", 24, 1024, 80, 1024, 16, F3_FULL_DIMS),
    # FLUX.3 Image Klein base checkpoint (no flow-map embedding): 50 steps at guidance 3.5 (we0.ai
    # FLUX 3 Image Klein article, checkpoint table); the 256^2 golden case keeps 4 steps
    "f3cfgtiny64": Workload("f3cfgtiny64", 26, 64, 16, 64, 4, F3_TINY_BASE_DIMS, guidance=3.5),
    "f3cfg256": Workload("f3cfg256", 27, 256, 160, 0, 4, F3_BASE_DIMS, guidance=3.5),
    "f3cfg1024": Workload("f3cfg1024", 28, 1024, 160, 0, 50, F3_BASE_DIMS, guidance=3.5),
}


def _parallel_block_specs(p, D, F, hd):
    return [
        (p + "lin1.w", (3 * D + 2 * F, D), D), (p + "lin1.b", (3 * D + 2 * F,), D),
        (p + "q_gain", (hd,), 1), (p + "k_gain", (hd,), 1),
        (p + "lin2.w", (D, D + F), D + F), (p + "lin2.b", (D,), D + F),
    ]


def tensor_specs3(d: Flux3Dims):
    """FLUX.3 blob order: list of (name, shape, fan_in).  Modulation linears are shared by the
    blocks of a phase: one per stream for the per-mode blocks, one for the joint blocks."""
    D, F, hd = d.hidden, d.mlp_hidden, d.head_dim
    specs = [
        ("time_in.w1", (D, d.t_freq_dim), d.t_freq_dim), ("time_in.b1", (D,), d.t_freq_dim),
        ("time_in.w2", (D, D), D), ("time_in.b2", (D,), D),
    ]
    if d.flow_map:
        specs += [
            ("target_in.w1", (D, d.t_freq_dim), d.t_freq_dim), ("target_in.b1", (D,), d.t_freq_dim),
            ("target_in.w2", (D, D), D), ("target_in.b2", (D,), D),
        ]
    specs += [
        ("img_in.w", (D, d.in_ch), d.in_ch), ("img_in.b", (D,), d.in_ch),
        ("txt_in.w", (D, d.txt_dim), d.txt_dim), ("txt_in.b", (D,), d.txt_dim),
    ]
    for s in ("txt", "img", "ref"):
        specs += [(f"mode_mod.{s}.w", (3 * D, D), D), (f"mode_mod.{s}.b", (3 * D,), D)]
    for i in range(d.n_mode):
        for s in ("txt", "img", "ref"):
            specs += _parallel_block_specs(f"mode.{i}.{s}.", D, F, hd)
    specs += [("joint_mod.w", (3 * D, D), D), ("joint_mod.b", (3 * D,), D)]
    for i in range(d.n_joint):
        specs += _parallel_block_specs(f"joint.{i}.", D, F, hd)
    specs += [
        ("final.mod.w", (2 * D, D), D), ("final.mod.b", (2 * D,), D),
        ("final.out.w", (d.in_ch, D), D), ("final.out.b", (d.in_ch,), D),
    ]
    return specs


def tensor_specs(d):
    """Blob order: list of (name, shape, fan_in)."""
    if isinstance(d, Flux3Dims):
        return tensor_specs3(d)
    D, F, hd = d.hidden, d.mlp_hidden, d.head_dim
    specs = [
        ("time_in.w1", (D, d.t_freq_dim), d.t_freq_dim), ("time_in.b1", (D,), d.t_freq_dim),
        ("time_in.w2", (D, D), D), ("time_in.b2", (D,), D),
        ("img_in.w", (D, d.in_ch), d.in_ch), ("img_in.b", (D,), d.in_ch),
        ("txt_in.w", (D, d.txt_dim), d.txt_dim), ("txt_in.b", (D,), d.txt_dim),
    ]
    for i in range(d.n_double):
        for s in ("img", "txt"):
            p = f"double.{i}.{s}."
            specs += [
                (p + "mod.w", (6 * D, D), D), (p + "mod.b", (6 * D,), D),
                (p + "qkv.w", (3 * D, D), D), (p + "qkv.b", (3 * D,), D),
                (p + "q_gain", (hd,), 1), (p + "k_gain", (hd,), 1),
                (p + "proj.w", (D, D), D), (p + "proj.b", (D,), D),
                (p + "mlp_in.w", (2 * F, D), D), (p + "mlp_in.b", (2 * F,), D),
                (p + "mlp_out.w", (D, F), F), (p + "mlp_out.b", (D,), F),
            ]
    for i in range(d.n_single):
        p = f"single.{i}."
        specs += [
            (p + "mod.w", (3 * D, D), D), (p + "mod.b", (3 * D,), D),
            (p + "lin1.w", (3 * D + 2 * F, D), D), (p + "lin1.b", (3 * D + 2 * F,), D),
            (p + "q_gain", (hd,), 1), (p + "k_gain", (hd,), 1),
            (p + "lin2.w", (D, D + F), D + F), (p + "lin2.b", (D,), D + F),
        ]
    specs += [
        ("final.mod.w", (2 * D, D), D), ("final.mod.b", (2 * D,), D),
        ("final.out.w", (d.in_ch, D), D), ("final.out.b", (d.in_ch,), D),
    ]
    return specs


def _align(x: int) -> int:
    return (x + ALIGN - 1) // ALIGN * ALIGN


def blob_layout(d):
    """Byte offset (from the start of the blob) of every tensor, and total size."""
    off = HEADER_BYTES
    layout = []
    for name, shape, fan_in in tensor_specs(d):
        n = int(np.prod(shape))
        layout.append((name, shape, fan_in, off, n))
        off = _align(off + 2 * n)
    return layout, off


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _header(d, n_tensors: int, total: int) -> bytes:
    if isinstance(d, Flux3Dims):
        h = BLOB3_MAGIC + struct.pack(
            "<II10i3fQQ", BLOB_VERSION, n_tensors,
            d.n_mode, d.n_joint, d.hidden, d.heads, d.head_dim, d.mlp_hidden,
            d.in_ch, d.txt_dim, d.t_freq_dim, 1 if d.flow_map else 0, d.rope_theta, d.eps_ln, d.eps_rms,
            HEADER_BYTES, total - HEADER_BYTES)
        return h + b"\0" * (HEADER_BYTES - len(h))
    h = BLOB_MAGIC + struct.pack(
        "<II9i3fQQ", BLOB_VERSION, n_tensors,
        d.n_double, d.n_single, d.hidden, d.heads, d.head_dim, d.mlp_hidden,
        d.in_ch, d.txt_dim, d.t_freq_dim, d.rope_theta, d.eps_ln, d.eps_rms,
        HEADER_BYTES, total - HEADER_BYTES)
    return h + b"\0" * (HEADER_BYTES - len(h))


def _fill(dst_u16: np.ndarray, seed: int, idx: int, chunk: int, scale: np.float32):
    lo = chunk * CHUNK
    hi = min(lo + CHUNK, dst_u16.size)
    g = np.random.default_rng([seed, idx, chunk])
    x = g.standard_normal(hi - lo, dtype=np.float32)
    if scale != 1:
        x *= scale
    dst_u16[lo:hi] = round_to_bf16_bits(x)


def make_weights(d, seed: int, threads: int | None = None):
    """Return (blob: uint8 array, params: dict name -> uint16 view of bf16 bits)."""
    layout, total = blob_layout(d)
    blob = np.zeros(total, dtype=np.uint8)
    blob[:HEADER_BYTES] = np.frombuffer(_header(d, len(layout), total), dtype=np.uint8)
    params = {}
    jobs = []
    for idx, (name, shape, fan_in, off, n) in enumerate(layout):
        view = blob[off:off + 2 * n].view(np.uint16)
        params[name] = view.reshape(shape)
        scale = np.float32(1.0 / np.sqrt(np.float32(fan_in)))
        for c in range((n + CHUNK - 1) // CHUNK):
            jobs.append((view, seed, idx, c, scale))
    threads = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(lambda j: _fill(*j), jobs))
    return blob, params


def make_inputs(w: Workload):
    """Latent, text and reference latent(s) as float32 arrays holding bf16 values.

    The reference is None, one array, or (several references) a list of arrays drawn
    with keys INPUT_KEY + 2, + 3, ...
    """
    def draw(k, shape):
        g = np.random.default_rng([w.seed, INPUT_KEY + k])
        x = g.standard_normal(int(np.prod(shape)), dtype=np.float32)
        return bf16_bits_to_f32(round_to_bf16_bits(x)).reshape(shape)

    h8 = w.image // 8
    latent = draw(0, (32, h8, h8))
    txt = draw(1, (w.n_txt, w.dims.txt_dim))
    refs = [draw(2 + k, (32, r // 8, r // 8)) for k, r in enumerate(w.ref_images)]
    ref = None if not refs else (refs[0] if len(refs) == 1 else refs)
    return latent, txt, ref


UNCOND_KEY = 100


def make_uncond_text(w: Workload):
    """The unconditional text of a guided workload: same token count as the prompt (prompts
    are padded to one length), N(0,1) features rounded to bf16, its own generator stream."""
    g = np.random.default_rng([w.seed, INPUT_KEY + UNCOND_KEY])
    x = g.standard_normal(w.n_txt * w.dims.txt_dim, dtype=np.float32)
    return bf16_bits_to_f32(round_to_bf16_bits(x)).reshape(w.n_txt, w.dims.txt_dim)

