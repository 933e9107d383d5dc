"""chunk_attention_multi (the stream's ring plus history-only rings, e.g. the first chunk
kept as a persistent anchor beside the sliding window): parity with the oracle's
multi-ring attention, with the rings' codes checked bit for bit first."""
import pytest
import torch

import kv_cache_attention_ring_b200 as kv
from kv_cache_attention_ring_b200 import inputs
from helpers import assert_attention_close, assert_ring_equal, to_dev

pytestmark = pytest.mark.gpu

H, D, A, W, N = 4, 128, 192, 1024, 192


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_attention_ring_b200 import build
    build.build()
    kv.lib()


def _chunk(seed, i, n=N):
    k = inputs.draw(inputs.seed_of(seed, i, 1), (n, H, D), "normal", 0.09, "bf16")
    v = inputs.draw(inputs.seed_of(seed, i, 2), (n, H, D), "normal", 1.0, "bf16")
    return k, v


def _anchored_stream(orc, seed):
    """First chunk into the anchor ring; seven more into a 1,024-slot window ring (it
    wraps), the last one pending; a reset of -300 on both rings after the fifth."""
    anchor = kv.KvRing(A, H, D, -2048, 4096)
    win = kv.KvRing(W, H, D, -2048, 4096, next_pos=A)
    oa, ow = orc.OracleRing(A, H, D), orc.OracleRing(W, H, D, next_pos=A)
    k, v = _chunk(seed, 0)
    kv.kv_ring_write(anchor, to_dev(k), to_dev(v), commit=True)
    oa.write(inputs.as_f32(k), inputs.as_f32(v), commit=True)
    for i in range(1, 8):
        k, v = _chunk(seed, i)
        last = i == 7
        kv.kv_ring_write(win, to_dev(k), to_dev(v), commit=not last)
        ow.write(inputs.as_f32(k), inputs.as_f32(v), commit=not last)
        if i == 5:
            for r in (anchor, win):
                kv.kv_ring_delta_rotate(r, -300)
            oa.delta_rotate(-300)
            ow.delta_rotate(-300)
    assert_ring_equal(anchor, oa, what="anchor")
    assert_ring_equal(win, ow, what="window")
    return (win, anchor), (ow, oa)


@pytest.mark.parametrize("n_splits", [1, 3])
def test_anchor_beside_wrapped_window(orc, n_splits):
    (win, anchor), (ow, oa) = _anchored_stream(orc, seed=61)
    q = inputs.draw(62, (N, H, D), "normal", 1.0, "bf16")
    ws = torch.empty(kv.chunk_attention_workspace_size(N, H, D, 2 * n_splits),
                     dtype=torch.uint8, device="cuda")
    out, lse = kv.chunk_attention_multi([win, anchor], to_dev(q), win.next_pos, N, n_splits, ws,
                                        mask=(64, 64, 64, 64), cache_bias=-0.7)
    ro, rl = orc.attention_multi(ow, [oa], inputs.as_f32(q), ow.next_pos, N, (64, 64, 64, 64),
                                 -0.7)
    assert_attention_close(out, lse, ro, rl, what=f"anchor + window, {n_splits} splits")


def test_three_rings_with_an_empty_one_mode_b(orc):
    (win, anchor), (ow, oa) = _anchored_stream(orc, seed=63)
    empty, oe = kv.KvRing(256, H, D, -2048, 4096), orc.OracleRing(256, H, D)
    q = inputs.draw(64, (N, H, D), "normal", 1.0, "bf16")
    ws = torch.empty(kv.chunk_attention_workspace_size(N, H, D, 3 * 4), dtype=torch.uint8,
                     device="cuda")
    for mode_b in (False, True):
        out, lse = kv.chunk_attention_multi([win, anchor, empty], to_dev(q), win.next_pos, N, 4,
                                            ws, mask=(1, 1, 1, 1), cache_bias=0.0,
                                            mode_b=mode_b)
        ro, rl = orc.attention_multi(ow, [oa, oe], inputs.as_f32(q), ow.next_pos, N,
                                     (1, 1, 1, 1), 0.0, mode_b=mode_b)
        assert_attention_close(out, lse, ro, rl, what=f"three rings, mode B {mode_b}")
