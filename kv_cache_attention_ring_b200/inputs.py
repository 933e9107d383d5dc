"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no arithmetic of the method: it only draws random tensors and names
the workload shapes.  Both the CUDA path (through the tests and the benchmark) and the
CPU oracle receive exactly the tensors made here.

Workload sources:
  * "Runway Characters: Serving a 57B Video Diffusion Transformer for Real-Time
    Conversation", abstract: 240 attention calls per chunk step, a 5,788-slot cache,
    757 new tokens per call, four denoising passes.
  * "Stream LTX", section "Training": 1 s blocks of 3 video latent frames (4 in the first
    block) and 25 audio latents (26 in the first block).
  * The Wan-style, tiny and long-stream shapes are synthetic cases of the same method.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BIG = 1 << 30  # a block length that puts a whole chunk into one block


@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    D: int
    C: int               # ring capacity (slots)
    n: int               # new tokens per chunk (= queries per call for self paths)
    in_dtype: str        # "fp32" | "bf16"
    dist: str            # "normal" | "student_t4"
    in_scale: float      # inputs are multiplied by this after drawing
    mask: tuple          # (q_first_len, q_block_len, k_first_len, k_block_len)
    biases: tuple = (0.0,)
    passes: int = 1
    note: str = ""
    extra: dict = field(default_factory=dict)


TINY = Workload("tiny", H=2, D=64, C=256, n=32, in_dtype="fp32", dist="normal", in_scale=1.0,
                mask=(32, 32, 32, 32), biases=(0.0, -2.0), passes=1,
                note="12 chunks of 32 (ring wraps after chunk 8), reset delta=-128 after chunk 8",
                extra=dict(chunks=12, reset_after=8, delta=-128))

RUNWAY = Workload("runway_5788x757", H=40, D=128, C=5788, n=757, in_dtype="bf16",
                  dist="normal", in_scale=1.0 / math.sqrt(128.0), mask=(1, 1, 1, 1),
                  biases=(0.0,), passes=4,
                  note="60 rings x 4 passes = 240 write+attention calls per chunk step; "
                       "token-causal inside the new block",
                  extra=dict(rings=60))

WAN = Workload("wan_4680x23400", H=40, D=128, C=23400, n=4680, in_dtype="bf16",
               dist="normal", in_scale=1.0 / math.sqrt(128.0),
               mask=(1560, 1560, 1560, 1560), biases=(-3.0, -2.0, -1.0, 0.0), passes=4,
               note="3 latent frames x 1,560 tokens per chunk, 4 prior chunks (18,720 slots) "
                    "of history, block-causal per frame, bias swept -3..0")

AV_VIDEO = Workload("av_video", H=32, D=128, C=21 * 1152, n=1152, in_dtype="bf16",
                    dist="normal", in_scale=1.0 / math.sqrt(128.0), mask=(BIG, BIG, BIG, BIG),
                    passes=4, note="3 frames x 384 tokens per 1 s block (first block 4 frames)",
                    extra=dict(first_n=1536, history_blocks=20))
AV_AUDIO = Workload("av_audio", H=32, D=128, C=21 * 25, n=25, in_dtype="bf16",
                    dist="normal", in_scale=1.0 / math.sqrt(128.0), mask=(BIG, BIG, BIG, BIG),
                    passes=4, note="25 audio latents per 1 s block (first block 26)",
                    extra=dict(first_n=26, history_blocks=20))

STRESS = Workload("stress_32768", H=40, D=128, C=32768, n=1024, in_dtype="bf16",
                  dist="student_t4", in_scale=1.0, mask=(BIG, BIG, BIG, BIG),
                  biases=(0.0, -4.0), passes=1,
                  note="600 chunks of 1,024, reset every 50 chunks, bias 0<->-4 every 10 "
                       "chunks, K/V Student-t(4), Q N(0,1)",
                  extra=dict(chunks=600, reset_every=50, bias_every=10))

WORKLOADS = {w.name: w for w in (TINY, RUNWAY, WAN, AV_VIDEO, AV_AUDIO, STRESS)}


def seed_of(*parts: int) -> int:
    """A stable 63-bit seed from small integers (workload id, chunk, pass, tensor)."""
    s = 0x9E3779B97F4A7C15
    for p in parts:
        s = (s ^ (int(p) & 0xFFFFFFFFFFFF)) * 0x100000001B3 & 0xFFFFFFFFFFFFFFFF
    return s >> 1


def draw(seed: int, shape, dist: str = "normal", scale: float = 1.0,
         dtype: str = "bf16") -> torch.Tensor:
    """One seeded CPU tensor of the given distribution, rounded to the input dtype."""
    rng = np.random.default_rng(seed)
    if dist == "normal":
        x = rng.standard_normal(shape, dtype=np.float32)
    elif dist == "student_t4":
        x = rng.standard_t(4.0, size=shape).astype(np.float32)
    else:
        raise ValueError(dist)
    t = torch.from_numpy(x)
    if scale != 1.0:
        t = t * scale
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "fp32":
        return t.contiguous()
    raise ValueError(dtype)


def chunk_qkv(w: Workload, chunk: int, pss: int = 0, n: int | None = None, stream: int = 0):
    """(q, k, v) of one chunk/pass: [n][H][D] CPU tensors in the workload's input dtype.

    Queries are always N(0,1)-based; keys and values follow the workload's distribution."""
    n = w.n if n is None else n
    wid = sum(map(ord, w.name))
    shape = (n, w.H, w.D)
    q = draw(seed_of(wid, stream, chunk, pss, 1), shape, "normal", w.in_scale, w.in_dtype)
    k = draw(seed_of(wid, stream, chunk, pss, 2), shape, w.dist, w.in_scale, w.in_dtype)
    v = draw(seed_of(wid, stream, chunk, pss, 3), shape, w.dist, w.in_scale, w.in_dtype)
    return q, k, v


def as_f32(t: torch.Tensor) -> np.ndarray:
    """Exact binary32 view of an input tensor (bf16 widens exactly)."""
    return t.to(torch.float32).numpy()


def draw_torch(seed: int, shape, dist: str = "normal", scale: float = 1.0, dtype: str = "bf16",
               device="cuda") -> torch.Tensor:
    """Seeded tensor drawn by torch on `device` (fast for long streams).  Student-t(4) is
    z0 / sqrt((z1^2 + z2^2 + z3^2 + z4^2) / 4) with independent normals z.  The same seed
    on the same device gives the same tensor; copy it to the host for the oracle."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    if dist == "normal":
        x = torch.randn(shape, generator=g, device=device)
    elif dist == "student_t4":
        z = torch.randn((5, *shape), generator=g, device=device)
        x = z[0] / torch.sqrt((z[1:] ** 2).sum(0) / 4.0)
    else:
        raise ValueError(dist)
    if scale != 1.0:
        x = x * scale
    return x.to(torch.bfloat16) if dtype == "bf16" else x.contiguous()


def chunk_qkv_torch(w: Workload, chunk: int, pss: int = 0, device="cuda"):
    """(q, k, v) of one chunk drawn on `device` with torch (see draw_torch)."""
    wid = sum(map(ord, w.name))
    shape = (w.n, w.H, w.D)
    q = draw_torch(seed_of(wid, 7, chunk, pss, 1), shape, "normal", w.in_scale, w.in_dtype, device)
    k = draw_torch(seed_of(wid, 7, chunk, pss, 2), shape, w.dist, w.in_scale, w.in_dtype, device)
    v = draw_torch(seed_of(wid, 7, chunk, pss, 3), shape, w.dist, w.in_scale, w.in_dtype, device)
    return q, k, v
