"""Mode B (KV_QK_FP8): the rotated bf16 query row is quantised to e4m3 by the write's row
rule and Q.K^T runs as one e4m3 MMA set.  Checked against the oracle evaluated on the
same quantised-then-dequantised query, with the attention tolerance."""
import numpy as np
import pytest
import torch

import kv_cache_attention_ring_b200 as kv
from kv_cache_attention_ring_b200 import inputs
from helpers import assert_attention_close, sample_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_attention_ring_b200 import build
    build.build()
    kv.lib()


def _ring(orc, C, H, n_hist, n_new, seed, start=0, k_scale=0.09, v_scale=1.0):
    ring = kv.KvRing(C, H, 128, 0, 4 * C + 4096)
    o = orc.OracleRing(C, H, 128)
    ring.s.write_slot = o._s.write_slot = start
    done, i = 0, 0
    while done < n_hist:
        n = min(1024, n_hist - done)
        k = inputs.draw(inputs.seed_of(seed, i, 1), (n, H, 128), "normal", k_scale, "bf16")
        v = inputs.draw(inputs.seed_of(seed, i, 2), (n, H, 128), "normal", v_scale, "bf16")
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=True)
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=True)
        done += n
        i += 1
    k = inputs.draw(inputs.seed_of(seed, 99, 1), (n_new, H, 128), "normal", k_scale, "bf16")
    v = inputs.draw(inputs.seed_of(seed, 99, 2), (n_new, H, 128), "normal", v_scale, "bf16")
    kv.kv_ring_write(ring, to_dev(k), to_dev(v))
    o.write(inputs.as_f32(k), inputs.as_f32(v))
    return ring, o


def test_mode_b_wrapped_ring_block_mask_bias(orc):
    """All rows: partial wrapped ring, block mask, history bias, a zero query row."""
    ring, o = _ring(orc, 1000, 3, 700, 200, seed=51, start=900)
    q = inputs.draw(71, (200, 3, 128), "normal", 1.0, "bf16")
    q[17] = 0                                                    # zero row: scale 0
    mask = (50, 50, 50, 50)
    out, lse = kv.chunk_attention(ring, to_dev(q), ring.next_pos, 200, mask, -0.75, mode_b=True)
    ro, rl = o.attention(inputs.as_f32(q), o.next_pos, 200, mask, -0.75, mode_b=True)
    assert_attention_close(out, lse, ro, rl, what="mode B")
    # it is a different (quantised) query: not the mode A result
    ra, _ = o.attention(inputs.as_f32(q), o.next_pos, 200, mask, -0.75)
    assert np.abs(ro - ra).max() > 1e-4


def test_mode_b_runway_chunk_and_split(orc):
    """Runway shape, sampled rows; also split over keys."""
    w = inputs.RUNWAY
    ring, o = _ring(orc, w.C, w.H, 7 * 757 - 757, 757, seed=52, start=77,
                    k_scale=w.in_scale, v_scale=w.in_scale)
    q = inputs.draw(72, (w.n, w.H, w.D), "normal", w.in_scale, "bf16")
    out, lse = kv.chunk_attention(ring, to_dev(q), ring.next_pos, w.n, w.mask, 0.0, mode_b=True)
    rows = sample_rows(w.n, 16, seed=11)
    ro, rl = o.attention(inputs.as_f32(q), o.next_pos, w.n, w.mask, rows=rows, mode_b=True)
    assert_attention_close(out, lse, ro, rl, rows=rows, what="mode B runway")
    ws = torch.empty(kv.chunk_attention_workspace_size(w.n, w.H, w.D, 4), dtype=torch.uint8,
                     device="cuda")
    o4, l4 = kv.chunk_attention_split(ring, to_dev(q), ring.next_pos, w.n, 4, ws, mask=w.mask,
                                      mode_b=True)
    assert_attention_close(o4, l4, ro, rl, rows=rows, what="mode B runway split")
    assert kv.kv_wait_timeout_count() == 0
