"""chunk_attention_split_noalloc (the library's static per-device scratch instead of a
caller workspace) against chunk_attention_split with a workspace, on two calls in a
row of different shapes, within the attention tolerance.  Collected last on purpose:
it must pass alone and after every other test."""
import numpy as np
import pytest
import torch

import kv_cache_attention_ring_b200 as kv
from kv_cache_attention_ring_b200 import inputs
from helpers import assert_attention_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_attention_ring_b200 import build
    build.build()
    kv.lib()


def _ring(C=4096, H=8):
    ring = kv.KvRing(C, H, 128, 0, 4 * C)
    for i in range(5):                       # 5 x 1,000 tokens: the ring wraps
        k = inputs.draw(inputs.seed_of(41, i, 1), (1000, H, 128), "normal", 0.09, "bf16")
        v = inputs.draw(inputs.seed_of(41, i, 2), (1000, H, 128), "normal", 1.0, "bf16")
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=True)
    k = inputs.draw(inputs.seed_of(41, 9, 1), (300, H, 128), "normal", 0.09, "bf16")
    v = inputs.draw(inputs.seed_of(41, 9, 2), (300, H, 128), "normal", 1.0, "bf16")
    kv.kv_ring_write(ring, to_dev(k), to_dev(v))
    return ring


def _as_ref(out, lse):
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def test_noalloc_matches_workspace_split_on_two_calls_in_a_row():
    ring = _ring()
    H = ring.H
    calls = [  # (queries, q_pos0, n_current, mask, bias, n_splits)
        (25, 2000, 300, None, -1.0, 8),
        (300, ring.next_pos, 300, (1, 1, 1, 1), 0.0, 4),
    ]
    for i, (n_q, q_pos0, n_cur, mask, bias, splits) in enumerate(calls):
        q = to_dev(inputs.draw(inputs.seed_of(42, i), (n_q, H, 128), "normal", 1.0, "bf16"))
        assert kv.chunk_attention_workspace_size(n_q, H, 128, splits) <= kv.KV_NOALLOC_SCRATCH_BYTES
        out = torch.empty_like(q)
        lse = torch.empty((H, n_q), dtype=torch.float32, device="cuda")
        kv.chunk_attention_split_noalloc(ring, q, q_pos0, n_cur, splits, out, lse, mask=mask,
                                         cache_bias=bias)
        ws = torch.empty(kv.chunk_attention_workspace_size(n_q, H, 128, splits),
                         dtype=torch.uint8, device="cuda")
        ref_o, ref_l = kv.chunk_attention_split(ring, q, q_pos0, n_cur, splits, ws, mask=mask,
                                                cache_bias=bias)
        ro, rl = _as_ref(ref_o, ref_l)
        assert_attention_close(out, lse, ro, rl, what=f"no-alloc call {i}")
    assert kv.kv_wait_timeout_count() == 0
