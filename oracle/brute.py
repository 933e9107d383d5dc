"""Brute-force second implementation for tiny inputs (numpy + torch dtype casts).

TEST INFRASTRUCTURE ONLY.  It pins the C oracle: it shares no code with it and uses
different primitives for every step --

* the ring is a plain Python list of every token ever written (a linear buffer); the
  window is its last C entries and a token's slot is its global index mod C;
* binary32 arithmetic is numpy float32 arithmetic (IEEE, one rounding per op, no FMA);
* e4m3 and bf16 rounding are torch's own dtype casts (``float8_e4m3fn``, ``bfloat16``);
* angles come from Python's ``math`` module;
* attention builds the full score matrix with a dense block mask from ``searchsorted``
  over block boundaries and takes a softmax over it.

Definitions followed: the ring KV cache with RoPE + FP8 applied once per write and a
delta rotation on position reset ("Runway Characters: Serving a 57B Video Diffusion
Transformer for Real-Time Conversation", abstract); the additive cache bias of the
"Plastic Windows" section ("KREA Real-Time 14B / video-conductor"); block-causal masking
("Stream LTX", section "Training").
"""
from __future__ import annotations

import math

import numpy as np
import torch

F32 = np.float32


def e4m3_codes(x32: np.ndarray) -> np.ndarray:
    """binary32 values -> e4m3fn bytes through torch's RNE cast (saturated to +-448 first)."""
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32))
    t = torch.where(torch.isnan(t), t, t.clamp(-448.0, 448.0))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()


def e4m3_values(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def bf16(x32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def angles(p: int, D: int, base: float, rope3d=None):
    """(cos, sin) per pair of token position p.  rope3d = (pairs_t, pairs_h, pairs_w,
    grid_h, grid_w): pair i belongs to the time, height or width run; its coordinate is
    the token's frame, row or column in a raster-ordered grid_h x grid_w frame, and its
    frequency counts within its own run."""
    if rope3d is None:
        coord = [p] * (D // 2)
        freq = [base ** (-(2.0 * i) / D) for i in range(D // 2)]
    else:
        pt, ph, pw, gh, gw = rope3d
        frame, rest = divmod(p, gh * gw)          # floor division, rest >= 0
        row, col = divmod(rest, gw)
        coord, freq = [], []
        for n, cval in ((pt, frame), (ph, row), (pw, col)):
            coord += [cval] * n
            freq += [base ** (-(2.0 * k) / (2 * n)) for k in range(n)]
    c = np.array([math.cos(coord[i] * freq[i]) for i in range(D // 2)], F32)
    s = np.array([math.sin(coord[i] * freq[i]) for i in range(D // 2)], F32)
    return c, s


def rope32(x: np.ndarray, p: int, base: float, rope3d=None) -> np.ndarray:
    """x: [..., D] float32, one position for all leading rows."""
    c, s = angles(p, x.shape[-1], base, rope3d)
    x0, x1 = x[..., 0::2].astype(F32), x[..., 1::2].astype(F32)
    y = np.empty(x.shape, F32)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


def quant(y: np.ndarray):
    """Per-row (last axis) quantisation in numpy float32 -> (codes, scales)."""
    y = y.astype(F32)
    rows = y.reshape(-1, y.shape[-1])
    codes = np.zeros(rows.shape, np.uint8)
    scales = np.zeros(rows.shape[0], F32)
    for r in range(rows.shape[0]):
        row = rows[r]
        if not np.all(np.isfinite(row)):
            codes[r] = 0x7F
            scales[r] = np.frombuffer(np.uint32(0x7FC00000).tobytes(), F32)[0]
            continue
        amax = F32(np.max(np.abs(row)))
        if amax == 0:
            continue
        with np.errstate(over="ignore", divide="ignore"):
            inv = F32(448.0) / amax
        if not np.isfinite(inv):
            continue
        scales[r] = amax / F32(448.0)
        codes[r] = e4m3_codes(row * inv)
    return codes.reshape(y.shape), scales.reshape(y.shape[:-1])


class BruteRing:
    """The ring as a linear list of token records."""

    def __init__(self, C: int, H: int, D: int, base: float = 10000.0, next_pos: int = 0,
                 rope3d=None):
        self.C, self.H, self.D, self.base = C, H, D, base
        self.rope3d = rope3d
        self.tokens: list[dict] = []   # committed tokens, oldest first
        self.pending: list[dict] = []
        self.next_pos = next_pos

    def write(self, k, v, commit=False):
        k, v = np.asarray(k, F32), np.asarray(v, F32)
        g0 = len(self.tokens)
        self.pending = []
        for t in range(k.shape[0]):
            pos = self.next_pos + t
            kc, ks = quant(rope32(k[t], pos, self.base, self.rope3d))
            vc, vs = quant(v[t])
            self.pending.append(dict(g=g0 + t, pos=pos, kc=kc, ks=ks, vc=vc, vs=vs))
        if commit:
            self.commit()

    def commit(self):
        self.tokens.extend(self.pending)
        self.next_pos += len(self.pending)
        self.pending = []

    def window(self) -> list[dict]:
        return (self.tokens + self.pending)[-self.C:]

    def state(self):
        """(write_slot, live, pending, next_pos) as a ring would report them."""
        return (len(self.tokens) % self.C, min(len(self.tokens), self.C), len(self.pending),
                self.next_pos)

    def delta_rotate(self, delta: int):
        if self.rope3d is not None and delta % (self.rope3d[3] * self.rope3d[4]) != 0:
            raise ValueError("3-D resets move whole frames")
        for tok in self.window():
            # binary32 product: both factors are binary32, numpy rounds once
            x = (e4m3_values(tok["kc"]).astype(F32) * tok["ks"][:, None]).astype(F32)
            tok["kc"], tok["ks"] = quant(rope32(x, delta, self.base, self.rope3d))
            tok["pos"] += delta
        self.next_pos += delta

    def arrays(self):
        """Scatter the window into ring arrays (slot = global index mod C)."""
        C, H, D = self.C, self.H, self.D
        kc = np.zeros((H, C, D), np.uint8)
        vc = np.zeros((H, C, D), np.uint8)
        ks = np.zeros((H, C), F32)
        vs = np.zeros((H, C), F32)
        sp = np.zeros(C, np.int32)
        for tok in self.window():
            s = tok["g"] % C
            kc[:, s], vc[:, s], ks[:, s], vs[:, s] = tok["kc"], tok["vc"], tok["ks"], tok["vs"]
            sp[s] = tok["pos"]
        return kc, vc, ks, vs, sp

    def attention(self, q, q_pos0, n_current, mask, cache_bias, softmax_scale, mode_b=False):
        """Dense attention of every query row over the window; returns (out, lse).

        mode_b: the rotated bf16 query is also quantised per row to e4m3 and dequantised."""
        q = np.asarray(q, F32)
        n_q, H, D = q.shape
        win = self.window()
        n_k = len(win)
        qf, qb, kf, kb = mask
        # block boundaries of a chunk: first, first+len, first+2len, ...
        def ids(n, first, blen):
            bounds = np.arange(first, max(n, first) + blen, blen)
            return np.searchsorted(bounds, np.arange(n), side="right")
        q_ids = ids(n_q, qf, qb)
        cur = min(n_current, n_k)
        k_cur_ids = ids(cur, kf, kb)
        visible = np.ones((n_q, n_k), bool)
        bias = np.zeros(n_k)
        bias[: n_k - cur] = cache_bias
        if cur:
            visible[:, n_k - cur:] = k_cur_ids[None, :] <= q_ids[:, None]
        out = np.zeros((n_q, H, D))
        lse = np.full((H, n_q), -np.inf)
        if n_k == 0:
            return out, lse
        K = np.stack([e4m3_values(t["kc"]) * t["ks"][:, None].astype(np.float64) for t in win], 1)
        V = np.stack([e4m3_values(t["vc"]) * t["vs"][:, None].astype(np.float64) for t in win], 1)
        for h in range(H):
            Q = np.stack([bf16(rope32(q[i, h], q_pos0 + i, self.base, self.rope3d))
                          for i in range(n_q)])
            if mode_b:
                qc, qs = quant(Q)
                Q = e4m3_values(qc) * qs[:, None].astype(np.float64)
            S = float(softmax_scale) * (Q.astype(np.float64) @ K[h].T) + bias[None, :]
            S = np.where(visible, S, -np.inf)
            m = S.max(axis=1, keepdims=True)
            live = np.isfinite(m[:, 0])          # rows with at least one finite score
            P = np.exp(S[live] - m[live])
            l = P.sum(axis=1, keepdims=True)
            out[live, h] = (P @ V[h]) / l
            lse[h, live] = (m[live] + np.log(l))[:, 0]
        return out, lse


class BruteAnchoredRing(BruteRing):
    """A persistent anchor beside the sliding window ("Why Live Video Generation Still
    Struggles With Timing", Transcript: recent history plus the first chunk kept as an
    anchor).  The first ``A`` committed tokens stay for good; the window holds the last
    ``C`` tokens after them, the pending chunk included.  Keys are ordered anchor first,
    so the current chunk is still the newest ``n_current`` of them; a reset re-rotates
    every cached key, the anchor's too."""

    def __init__(self, A: int, C: int, H: int, D: int, base: float = 10000.0,
                 next_pos: int = 0):
        super().__init__(C, H, D, base, next_pos)
        self.A = A

    def window(self) -> list[dict]:
        return self.tokens[: self.A] + (self.tokens[self.A:] + self.pending)[-self.C:]

    def fifo_arrays(self):
        """The FIFO part scattered into ring arrays (slot = (global index - A) mod C)."""
        C, H, D = self.C, self.H, self.D
        kc = np.zeros((H, C, D), np.uint8)
        ks = np.zeros((H, C), F32)
        sp = np.zeros(C, np.int32)
        for tok in self.window()[min(self.A, len(self.tokens)):]:
            s = (tok["g"] - self.A) % C
            kc[:, s], ks[:, s], sp[s] = tok["kc"], tok["ks"], tok["pos"]
        return kc, ks, sp
