"""Chunk attention parity (CUDA path through the C ABI vs the fp64 oracle on the same
dequantised FP8 cache): max-abs <= 2e-2 and relative L2 <= 5e-3 on bf16 outputs."""
import math

import numpy as np
import pytest
import torch

import kv_cache_attention_ring_b200 as kv
from kv_cache_attention_ring_b200 import inputs
from helpers import assert_attention_close, assert_ring_equal, sample_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_attention_ring_b200 import build
    build.build()
    kv.lib()


def _q_bf16(q):
    return q.to(torch.bfloat16)


def test_tiny_stream_all_rows(orc):
    """The tiny workload end to end: every chunk's last pass is attended with the
    per-32-token block mask and finer masks, at cache bias 0 and -2."""
    w = inputs.TINY
    ring = kv.KvRing(w.C, w.H, w.D, pos_min=-256, pos_max=1024)
    o = orc.OracleRing(w.C, w.H, w.D)
    worst = (0.0, 0.0)
    for ch in range(w.extra["chunks"]):
        for p in range(4):
            q, k, v = inputs.chunk_qkv(w, ch, p)
            kv.kv_ring_write(ring, to_dev(k), to_dev(v))
            o.write(inputs.as_f32(k), inputs.as_f32(v))
        qb = _q_bf16(q)
        for bias in w.biases:
            for mask in (w.mask, (8, 8, 8, 8), (1, 1, 1, 1), (5, 9, 3, 7)):
                out, lse = kv.chunk_attention(ring, to_dev(qb), ring.next_pos, w.n, mask, bias)
                ro, rl = o.attention(inputs.as_f32(qb), o.next_pos, w.n, mask, bias)
                e = assert_attention_close(out, lse, ro, rl, what=f"chunk {ch} {mask} {bias}")
                worst = (max(worst[0], e[0]), max(worst[1], e[1]))
        kv.kv_ring_commit(ring)
        o.commit()
        if ch == w.extra["reset_after"]:
            kv.kv_ring_delta_rotate(ring, w.extra["delta"])
            o.delta_rotate(w.extra["delta"])
    assert_ring_equal(ring, o, what="after stream")
    print("tiny worst max-abs %.3e rel-L2 %.3e" % worst)


def _runway_ring(orc, with_oracle=True, start_slot=1234):
    """Full 5,788-slot ring: 7 committed chunks of 757 (wraps) + the pending chunk."""
    w = inputs.RUNWAY
    ring = kv.KvRing(w.C, w.H, w.D, pos_min=0, pos_max=20000)
    o = orc.OracleRing(w.C, w.H, w.D) if with_oracle else None
    ring.s.write_slot = start_slot
    if o is not None:
        o._s.write_slot = start_slot
    for ch in range(8):
        _, k, v = inputs.chunk_qkv(w, ch)
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=(ch < 7))
        if o is not None:
            o.write(inputs.as_f32(k), inputs.as_f32(v), commit=(ch < 7))
    q, _, _ = inputs.chunk_qkv(w, 7)
    return ring, o, q


@pytest.mark.parametrize("mask", [(1, 1, 1, 1), (inputs.BIG,) * 4])
def test_runway_shape_all_rows(orc, mask):
    """H=40, D=128, 757 new tokens over a full 5,788-slot FP8 ring, bias 0: token-causal
    inside the new chunk, and the whole-chunk block variant; every row and head."""
    w = inputs.RUNWAY
    ring, o, q = _runway_ring(orc)
    assert ring.n_valid == w.C
    out, lse = kv.chunk_attention(ring, to_dev(q), ring.next_pos, w.n, mask, 0.0)
    ro, rl = o.attention(inputs.as_f32(q), o.next_pos, w.n, mask, 0.0)
    e, r = assert_attention_close(out, lse, ro, rl, what=f"runway {mask}")
    print(f"runway {mask}: max-abs {e:.3e} rel-L2 {r:.3e}")


@pytest.mark.parametrize("n_q", [1, 127, 129, 300])
@pytest.mark.parametrize("bias", [0.0, -3.0, -math.inf])
def test_ragged_queries_partial_ring(orc, n_q, bias):
    """Partial ring (valid < C), valid range wrapping the end of the ring, ragged query
    counts; bias -inf leaves only the current chunk."""
    C, H, D = 700, 2, 128
    ring = kv.KvRing(C, H, D, pos_min=0, pos_max=4000)
    o = orc.OracleRing(C, H, D)
    ring.s.write_slot = o._s.write_slot = 610
    for i, n in enumerate((150, 200)):
        k = inputs.draw(inputs.seed_of(11, i, 1), (n, H, D), "normal", 1.0, "bf16")
        v = inputs.draw(inputs.seed_of(11, i, 2), (n, H, D), "normal", 1.0, "bf16")
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=True)
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=True)
    k = inputs.draw(inputs.seed_of(11, 9, 1), (n_q, H, D), "normal", 1.0, "bf16")
    v = inputs.draw(inputs.seed_of(11, 9, 2), (n_q, H, D), "normal", 1.0, "bf16")
    q = inputs.draw(inputs.seed_of(11, 9, 3), (n_q, H, D), "normal", 1.0, "bf16")
    kv.kv_ring_write(ring, to_dev(k), to_dev(v))
    o.write(inputs.as_f32(k), inputs.as_f32(v))
    for mask in ((1, 1, 1, 1), (16, 32, 16, 32)):
        out, lse = kv.chunk_attention(ring, to_dev(q), ring.next_pos, n_q, mask, bias)
        ro, rl = o.attention(inputs.as_f32(q), o.next_pos, n_q, mask, bias)
        assert_attention_close(out, lse, ro, rl, what=f"n_q={n_q} bias={bias} {mask}")


def test_empty_and_history_only(orc):
    C, H, D = 256, 2, 64
    ring = kv.KvRing(C, H, D, pos_min=0, pos_max=1000)
    o = orc.OracleRing(C, H, D)
    q = inputs.draw(1, (40, H, D), "normal", 1.0, "bf16")
    out, lse = kv.chunk_attention(ring, to_dev(q), 0, 0)
    torch.cuda.synchronize()
    assert (out.float() == 0).all() and torch.isneginf(lse).all()
    k = inputs.draw(2, (100, H, D), "normal", 1.0, "bf16")
    kv.kv_ring_write(ring, to_dev(k), to_dev(k), commit=True)
    o.write(inputs.as_f32(k), inputs.as_f32(k), commit=True)
    for bias in (0.0, -1.5):
        out, lse = kv.chunk_attention(ring, to_dev(q), ring.next_pos, 0, None, bias)
        ro, rl = o.attention(inputs.as_f32(q), o.next_pos, 0, cache_bias=bias)
        assert_attention_close(out, lse, ro, rl, what=f"history only {bias}")
    out, lse = kv.chunk_attention(ring, to_dev(q), ring.next_pos, 0, None, -math.inf)
    torch.cuda.synchronize()
    assert (out.float() == 0).all() and torch.isneginf(lse).all()


def test_future_block_perturbation_is_bit_identical(orc):
    """Changing the keys, values and queries of later blocks leaves the outputs of
    earlier blocks bit-identical on the GPU."""
    w = inputs.RUNWAY
    ring, _, q = _runway_ring(orc, with_oracle=False)
    mask = (200, 200, 200, 200)
    out1, lse1 = kv.chunk_attention(ring, to_dev(q), ring.next_pos, w.n, mask, -1.0)
    out1, lse1 = out1.clone(), lse1.clone()
    _, k, v = inputs.chunk_qkv(w, 7)
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    g = torch.Generator().manual_seed(0)
    for t in (q2, k2, v2):
        t[400:] = torch.randn(t[400:].shape, generator=g).to(t.dtype)
    kv.kv_ring_write(ring, to_dev(k2), to_dev(v2))
    out2, lse2 = kv.chunk_attention(ring, to_dev(q2), ring.next_pos, w.n, mask, -1.0)
    torch.cuda.synchronize()
    assert torch.equal(out1[:400], out2[:400]) and torch.equal(lse1[:, :400], lse2[:, :400])
    assert not torch.equal(out1[400:], out2[400:])


def test_deterministic_and_wrap_placement(orc):
    w = inputs.RUNWAY
    ring_a, _, q = _runway_ring(orc, with_oracle=False, start_slot=0)
    ring_b, _, _ = _runway_ring(orc, with_oracle=False, start_slot=4321)
    qd = to_dev(q)
    a1, la1 = kv.chunk_attention(ring_a, qd, ring_a.next_pos, w.n, (1, 1, 1, 1), 0.0)
    a1, la1 = a1.clone(), la1.clone()
    a2, la2 = kv.chunk_attention(ring_a, qd, ring_a.next_pos, w.n, (1, 1, 1, 1), 0.0)
    b, lb = kv.chunk_attention(ring_b, qd, ring_b.next_pos, w.n, (1, 1, 1, 1), 0.0)
    torch.cuda.synchronize()
    assert torch.equal(a1, a2) and torch.equal(la1, la2)
    assert (a1.float() - b.float()).abs().max().item() < 2e-2
    assert kv.kv_wait_timeout_count() == 0
