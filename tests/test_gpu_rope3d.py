"""3-D (time, height, width) RoPE on the GPU path: the ring write, the whole-frame delta
rotation and the attention's query rotation read a 3-D table (kv_rope3d_table_build);
codes, scales, slot positions and state bit-exact against the oracle's 3-D form, and
attention within the tolerance."""
import numpy as np
import pytest

import kv_cache_attention_ring_b200 as kv
from kv_cache_attention_ring_b200 import inputs
from helpers import assert_attention_close, assert_ring_equal, sample_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_attention_ring_b200 import build
    build.build()
    kv.lib()


def _stream(orc, r3, H, C, frames_per_chunk, chunks, reset_after, reset_frames, seed, attend,
            dist="normal", scale=0.09):
    hw = r3[3] * r3[4]
    n = frames_per_chunk * hw
    ring = kv.KvRing(C, H, 128, -8 * C, 8 * C, rope3d=r3)
    o = orc.OracleRing(C, H, 128, rope3d=r3)
    checked = 0
    for ch in range(chunks):
        k = inputs.draw(inputs.seed_of(seed, ch, 1), (n, H, 128), dist, scale, "bf16")
        v = inputs.draw(inputs.seed_of(seed, ch, 2), (n, H, 128), dist, 1.0, "bf16")
        kv.kv_ring_write(ring, to_dev(k), to_dev(v))
        o.write(inputs.as_f32(k), inputs.as_f32(v))
        if ch in attend:
            q = inputs.draw(inputs.seed_of(seed, ch, 3), (n, H, 128), "normal", 1.0, "bf16")
            mask = (hw, hw, hw, hw)                    # block-causal per frame
            out, lse = kv.chunk_attention(ring, to_dev(q), ring.next_pos, n, mask, -0.5)
            rows = sample_rows(n, 64, seed=ch) if n > 256 else None
            ro, rl = o.attention(inputs.as_f32(q), o.next_pos, n, mask, -0.5, rows=rows)
            assert_attention_close(out, lse, ro, rl, rows=rows, what=f"3-D chunk {ch}")
            checked += 1
        kv.kv_ring_commit(ring)
        o.commit()
        if ch == reset_after:
            kv.kv_ring_delta_rotate(ring, -reset_frames * hw)
            o.delta_rotate(-reset_frames * hw)
            assert_ring_equal(ring, o, what=f"after the reset at chunk {ch}")
    assert_ring_equal(ring, o, what="end of stream")
    assert checked == len(attend)


def test_rope3d_small_grid_stream_wraps_and_resets(orc):
    """4 x 6 frames, 2 frames per chunk, a 480-slot ring (wraps), a reset of -4 frames."""
    _stream(orc, (22, 21, 21, 4, 6), H=2, C=480, frames_per_chunk=2, chunks=14,
            reset_after=9, reset_frames=4, seed=71, attend=(3, 10, 13))


def test_rope3d_latent_frame_grid(orc):
    """16 x 24 latent frames (384 tokens), 3 frames per chunk, 6 chunks of ring, a reset
    of -6 frames, Student-t keys and values."""
    _stream(orc, (22, 21, 21, 16, 24), H=4, C=6 * 1152, frames_per_chunk=3, chunks=8,
            reset_after=5, reset_frames=6, seed=72, attend=(6, 7), dist="student_t4", scale=1.0)


def test_rope3d_rejects_partial_frame_reset():
    ring = kv.KvRing(96, 1, 128, -1000, 1000, rope3d=(22, 21, 21, 4, 6))
    k = inputs.draw(1, (48, 1, 128), "normal", 1.0, "bf16")
    kv.kv_ring_write(ring, to_dev(k), to_dev(k), commit=True)
    with pytest.raises(kv.KvError):
        kv.kv_ring_delta_rotate(ring, -25)
    kv.kv_ring_delta_rotate(ring, -24)
    assert ring.next_pos == 24
    assert kv.kv_wait_timeout_count() == 0
