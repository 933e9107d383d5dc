"""Attention split over keys (partials in a caller workspace, then merged): parity with
the oracle and with the unsplit kernel, for few queries over long rings."""
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


def _ring(orc, C, H, n_hist, n_new, seed, start=0):
    ring = kv.KvRing(C, H, 128, 0, 4 * C + 4096)
    o = orc.OracleRing(C, H, 128)
    ring.s.write_slot = o._s.write_slot = start
    done = 0
    i = 0
    while done < n_hist:
        n = min(1024, n_hist - done)
        k = inputs.draw(inputs.seed_of(seed, i, 1), (n, H, 128), "normal", 0.09, "bf16")
        v = inputs.draw(inputs.seed_of(seed, i, 2), (n, H, 128), "normal", 1.0, "bf16")
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=True)
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=True)
        done += n
        i += 1
    k = inputs.draw(inputs.seed_of(seed, 99, 1), (n_new, H, 128), "normal", 0.09, "bf16")
    v = inputs.draw(inputs.seed_of(seed, 99, 2), (n_new, H, 128), "normal", 1.0, "bf16")
    kv.kv_ring_write(ring, to_dev(k), to_dev(v))
    o.write(inputs.as_f32(k), inputs.as_f32(v))
    return ring, o


@pytest.mark.parametrize("n_splits", [1, 3, 8, 64])
def test_audio_queries_over_video_ring(orc, n_splits):
    """25 audio queries over a 24,192-slot video ring (32 heads), cache bias -1."""
    C, H = 21 * 1152, 32
    ring, o = _ring(orc, C, H, 20 * 1152, 1152, seed=31, start=5000)
    q = inputs.draw(77, (25, H, 128), "normal", 0.09, "bf16")
    ws = torch.empty(kv.chunk_attention_workspace_size(25, H, 128, n_splits), dtype=torch.uint8,
                     device="cuda")
    out, lse = kv.chunk_attention_split(ring, to_dev(q), 3000, 1152, n_splits, ws,
                                        cache_bias=-1.0)
    ro, rl = o.attention(inputs.as_f32(q), 3000, 1152, cache_bias=-1.0)
    assert_attention_close(out, lse, ro, rl, what=f"a->v split {n_splits}")
    ref, rlse = kv.chunk_attention(ring, to_dev(q), 3000, 1152, None, -1.0)
    torch.cuda.synchronize()
    # same arithmetic, another summation order: at most a one-ulp bf16 flip
    diff = (out.float() - ref.float()).abs()
    assert (diff <= 2e-3 + ref.float().abs() / 128).all(), diff.max().item()
    assert (lse - rlse).abs().max().item() < 1e-4


def test_split_with_masks_ragged_and_empty_splits(orc):
    """757 queries, token-causal current chunk, partial wrapped ring; more splits than
    tiles leaves some splits empty."""
    C, H = 1500, 4
    ring, o = _ring(orc, C, H, 600, 757, seed=5, start=1200)
    q = inputs.draw(78, (757, H, 128), "normal", 1.0, "bf16")
    for n_splits in (2, 64):
        ws = torch.empty(kv.chunk_attention_workspace_size(757, H, 128, n_splits),
                         dtype=torch.uint8, device="cuda")
        out, lse = kv.chunk_attention_split(ring, to_dev(q), ring.next_pos, 757, n_splits, ws,
                                            mask=(1, 1, 1, 1), cache_bias=0.5)
        rows = sample_rows(757, 40, seed=n_splits)
        ro, rl = o.attention(inputs.as_f32(q), o.next_pos, 757, (1, 1, 1, 1), 0.5, rows=rows)
        assert_attention_close(out, lse, ro, rl, rows=rows, what=f"split {n_splits}")


def test_split_empty_ring_gives_zero_and_minus_inf(orc):
    ring = kv.KvRing(512, 2, 128, 0, 1000)
    q = inputs.draw(1, (10, 2, 128), "normal", 1.0, "bf16")
    ws = torch.empty(kv.chunk_attention_workspace_size(10, 2, 128, 4), dtype=torch.uint8,
                     device="cuda")
    out, lse = kv.chunk_attention_split(ring, to_dev(q), 0, 0, 4, ws)
    torch.cuda.synchronize()
    assert (out.float() == 0).all() and torch.isneginf(lse).all()
    assert kv.kv_wait_timeout_count() == 0
