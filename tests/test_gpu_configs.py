"""Full-size parity of the Wan-style, joint audio+video and long-stream workloads.

The whole stream runs on the GPU through the C ABI and is replayed by the oracle.  Ring
state (codes, scales, slot positions, head integers) is compared bit for bit at sampled
points; attention is compared on 64 seeded query rows x all heads (the oracle computes rows
independently) plus the tile edges and the last row, at every bias value and checkpoint."""
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


def test_wan_chunk_four_passes_bias_sweep(orc):
    """40 heads x 128, 3 frames x 1,560 = 4,680 queries per chunk over 4 prior chunks
    (18,720 slots), block-causal per frame, 4 denoising passes with bias -3, -2, -1, 0."""
    w = inputs.WAN
    ring = kv.KvRing(w.C, w.H, w.D, 0, 6 * w.n)
    o = orc.OracleRing(w.C, w.H, w.D)
    for ch in range(4):
        _, k, v = inputs.chunk_qkv(w, ch)
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=True)
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=True)
    rows = sample_rows(w.n, 64, seed=3)
    rows = np.unique(np.concatenate([rows, [1559, 1560, 3119, 3120]])).astype(np.int32)
    for p, bias in enumerate(w.biases):
        q, k, v = inputs.chunk_qkv(w, 4, p)
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=False)
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=False)
        out, lse = kv.chunk_attention(ring, to_dev(q), ring.next_pos, w.n, w.mask, bias)
        ro, rl = o.attention(inputs.as_f32(q), o.next_pos, w.n, w.mask, bias, rows=rows)
        assert_attention_close(out, lse, ro, rl, rows=rows, what=f"wan pass {p} bias {bias}")
    assert_ring_equal(ring, o, what="wan ring after 4 passes")


def _av_stream(orc, w, blocks):
    # both modalities share one position range: cross-modal queries keep their own
    ring = kv.KvRing(w.C, w.H, w.D, 0, 4 * inputs.AV_VIDEO.C)
    o = orc.OracleRing(w.C, w.H, w.D)
    for b in range(blocks):
        n = w.extra["first_n"] if b == 0 else w.n
        _, k, v = inputs.chunk_qkv(w, b, n=n)
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=True)
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=True)
    q, k, v = inputs.chunk_qkv(w, blocks, n=w.n)
    kv.kv_ring_write(ring, to_dev(k), to_dev(v))
    o.write(inputs.as_f32(k), inputs.as_f32(v))
    return ring, o, q


def test_joint_audio_video_four_paths(orc):
    """1 s blocks (3 video frames x 384 + 25 audio latents; the first block 4 frames + 26),
    32 heads x 128, 20 prior blocks in each ring: v->v, a->a, v->a, a->v."""
    wv, wa = inputs.AV_VIDEO, inputs.AV_AUDIO
    rv, ov, qv = _av_stream(orc, wv, 21)
    ra, oa, qa = _av_stream(orc, wa, 21)
    assert rv.n_valid == wv.C and ra.n_valid == wa.C
    assert_ring_equal(rv, ov, what="video ring")
    assert_ring_equal(ra, oa, what="audio ring")
    rows_v = sample_rows(wv.n, 64, seed=4)
    # v->v and a->a: self paths; one block per chunk, so bidirectional inside it
    out, lse = kv.chunk_attention(rv, to_dev(qv), rv.next_pos, wv.n, None, 0.0)
    ro, rl = ov.attention(inputs.as_f32(qv), ov.next_pos, wv.n, rows=rows_v)
    assert_attention_close(out, lse, ro, rl, rows=rows_v, what="v->v")
    out, lse = kv.chunk_attention(ra, to_dev(qa), ra.next_pos, wa.n, None, 0.0)
    ro, rl = oa.attention(inputs.as_f32(qa), oa.next_pos, wa.n)
    assert_attention_close(out, lse, ro, rl, what="a->a")
    # cross-modal paths read the other modality's ring; queries keep their own positions
    out, lse = kv.chunk_attention(ra, to_dev(qv), rv.next_pos, wa.n, None, -1.0)
    ro, rl = oa.attention(inputs.as_f32(qv), ov.next_pos, wa.n, cache_bias=-1.0, rows=rows_v)
    assert_attention_close(out, lse, ro, rl, rows=rows_v, what="v->a")
    out, lse = kv.chunk_attention(rv, to_dev(qa), ra.next_pos, wv.n, None, -1.0)
    ro, rl = ov.attention(inputs.as_f32(qa), oa.next_pos, wv.n, cache_bias=-1.0)
    assert_attention_close(out, lse, ro, rl, what="a->v")


def test_long_stream_resets_and_bias_toggle(orc):
    """32,768-slot ring, 600 chunks of 1,024 (many wraparounds), a delta re-rotation of the
    whole cache every 50 chunks (positions return to 0..C-1), cache bias 0 <-> -4 every 10
    chunks, Student-t(4) keys and values.  The GPU runs the whole stream.  At checkpoints the
    oracle replays the last 40 chunks from the recorded ring head: 40 x 1,024 slots cover
    the ring, so the replayed state equals the full stream's (including the resets in the
    window); attention and ring state are compared there."""
    w = inputs.STRESS
    chunks, every = w.extra["chunks"], w.extra["reset_every"]
    window = 40
    assert window * w.n > w.C
    max_pos = w.C + every * w.n + w.n
    ring = kv.KvRing(w.C, w.H, w.D, 0, max_pos)
    checked = (49, 50, 51, 299, 599)
    rows = sample_rows(w.n, 64, seed=6)
    heads = []          # ring head (write_slot, next_pos) before each chunk's write
    resets = {}         # chunk -> delta applied after that chunk's commit
    for ch in range(chunks):
        heads.append((ring.s.write_slot, ring.s.next_pos))
        q, k, v = inputs.chunk_qkv_torch(w, ch)
        kv.kv_ring_write(ring, k, v)
        if ch in checked:
            bias = w.biases[(ch // w.extra["bias_every"]) % 2]
            out, lse = kv.chunk_attention(ring, q, ring.next_pos, w.n, None, bias)
            o = orc.OracleRing(w.C, w.H, w.D)
            first = max(0, ch - window)
            o._s.write_slot, o._s.next_pos = heads[first]
            for c2 in range(first, ch + 1):
                _, k2, v2 = inputs.chunk_qkv_torch(w, c2)
                o.write(inputs.as_f32(k2.cpu()), inputs.as_f32(v2.cpu()), commit=c2 < ch)
                if c2 < ch and c2 in resets:
                    o.delta_rotate(resets[c2])
            assert (o.write_slot, o.next_pos) == (ring.s.write_slot, ring.s.next_pos)
            slots = [o.slot_of_age(a) for a in range(w.C)]
            assert_ring_equal(ring, o, slots=slots, what=f"stress ring at chunk {ch}")
            ro, rl = o.attention(inputs.as_f32(q.cpu()), o.next_pos, w.n, cache_bias=bias,
                                 rows=rows)
            assert_attention_close(out, lse, ro, rl, rows=rows, what=f"stress chunk {ch}")
        kv.kv_ring_commit(ring)
        if (ch + 1) % every == 0:
            oldest = int(ring.slot_pos[(ring.s.write_slot) % w.C].item())   # ring is full
            kv.kv_ring_delta_rotate(ring, -oldest)
            resets[ch] = -oldest
            assert int(ring.slot_pos.min().item()) == 0
    assert kv.kv_wait_timeout_count() == 0
