"""Attention for a gathered subset of query rows (edited regions recomputed, the rest of
the chunk's outputs kept): parity with the oracle's gathered rows, bit-identity with the
full call's rows, untouched rows left as they were."""
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


def _ring(orc, C=1500, H=4, n_new=757, seed=61):
    ring = kv.KvRing(C, H, 128, 0, 8 * C)
    o = orc.OracleRing(C, H, 128)
    ring.s.write_slot = o._s.write_slot = 1100
    for i, n in enumerate((600, 500)):
        k = inputs.draw(inputs.seed_of(seed, i, 1), (n, H, 128), "normal", 0.09, "bf16")
        v = inputs.draw(inputs.seed_of(seed, i, 2), (n, H, 128), "normal", 1.0, "bf16")
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=True)
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=True)
    k = inputs.draw(inputs.seed_of(seed, 9, 1), (n_new, H, 128), "normal", 0.09, "bf16")
    v = inputs.draw(inputs.seed_of(seed, 9, 2), (n_new, H, 128), "normal", 1.0, "bf16")
    kv.kv_ring_write(ring, to_dev(k), to_dev(v))
    o.write(inputs.as_f32(k), inputs.as_f32(v))
    q = inputs.draw(inputs.seed_of(seed, 9, 3), (n_new, H, 128), "normal", 1.0, "bf16")
    return ring, o, q


SENTINEL = 7.0


@pytest.mark.parametrize("mode_b", [False, True])
@pytest.mark.parametrize("mask,bias", [((1, 1, 1, 1), 0.0), ((100, 64, 100, 64), -1.5)])
def test_gathered_rows_match_oracle_and_full_call(orc, mask, bias, mode_b):
    ring, o, q = _ring(orc)
    n_q, H = q.shape[0], ring.H
    rng = np.random.default_rng(5)
    # tile edges, the last row, a seeded scatter, duplicates, unsorted
    listed = np.concatenate([[0, 127, 128, 255, 256, 511, 512, 756, 300, 300, 5],
                             rng.choice(n_q, 150, replace=False), [756, 0]]).astype(np.int32)
    rng.shuffle(listed)
    qd = to_dev(q)
    out = torch.full_like(qd, SENTINEL)
    lse = torch.full((H, n_q), 123.0, dtype=torch.float32, device="cuda")
    kv.chunk_attention_rows(ring, qd, ring.next_pos, n_q, to_dev(torch.from_numpy(listed)), out,
                            lse, mask=mask, cache_bias=bias, mode_b=mode_b)
    full_o, full_l = kv.chunk_attention(ring, qd, ring.next_pos, n_q, mask, bias, mode_b=mode_b)
    torch.cuda.synchronize()
    uniq = np.unique(listed)
    rest = np.setdiff1d(np.arange(n_q), uniq)
    # untouched rows keep what the caller left there
    assert (out[torch.from_numpy(rest)].float() == SENTINEL).all()
    assert (lse[:, torch.from_numpy(rest)] == 123.0).all()
    # listed rows: the very values the full call writes (rows are computed independently)
    u = torch.from_numpy(uniq)
    assert torch.equal(out[u], full_o[u]) and torch.equal(lse[:, u], full_l[:, u])
    ro, rl = o.attention(inputs.as_f32(q), o.next_pos, n_q, mask, bias, rows=uniq,
                         mode_b=mode_b)
    assert_attention_close(out, lse, ro, rl, rows=uniq, what=f"rows {mask} {bias} {mode_b}")


def test_out_of_range_indices_are_skipped_and_empty_list_is_a_no_op(orc):
    ring, o, q = _ring(orc, n_new=200)
    n_q, H = q.shape[0], ring.H
    listed = torch.tensor([3, -1, 200, 199, 1 << 30, 3], dtype=torch.int32)
    qd = to_dev(q)
    out = torch.full_like(qd, SENTINEL)
    lse = torch.full((H, n_q), 123.0, dtype=torch.float32, device="cuda")
    kv.chunk_attention_rows(ring, qd, ring.next_pos, n_q, to_dev(listed[:0]), out, lse)
    kv.chunk_attention_rows(ring, qd, ring.next_pos, n_q, to_dev(listed), out, lse,
                            mask=(1, 1, 1, 1))
    torch.cuda.synchronize()
    rest = [i for i in range(n_q) if i not in (3, 199)]
    assert (out[rest].float() == SENTINEL).all() and (lse[:, rest] == 123.0).all()
    ro, rl = o.attention(inputs.as_f32(q), o.next_pos, n_q, (1, 1, 1, 1), rows=[3, 199])
    assert_attention_close(out, lse, ro, rl, rows=[3, 199], what="rows in range")
    assert kv.kv_wait_timeout_count() == 0


@pytest.mark.parametrize("n_splits", [2, 5])
def test_gathered_rows_with_key_splits(orc, n_splits):
    """The rows path with the keys split over CTAs: partials per list entry, one merge.
    Listed rows match the oracle (the merge adds in another order, so not bit for bit),
    out-of-range entries are skipped, every other row is left as it was."""
    ring, o, q = _ring(orc, seed=67)
    n_q, H = q.shape[0], ring.H
    rng = np.random.default_rng(9)
    listed = np.concatenate([[0, 255, 256, 756, 40, 40, -3, n_q, 1 << 29],
                             rng.choice(n_q, 90, replace=False)]).astype(np.int32)
    rng.shuffle(listed)
    qd = to_dev(q)
    out = torch.full_like(qd, SENTINEL)
    lse = torch.full((H, n_q), 123.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(kv.chunk_attention_workspace_size(len(listed), H, 128, n_splits),
                     dtype=torch.uint8, device="cuda")
    kv.chunk_attention_rows(ring, qd, ring.next_pos, n_q, to_dev(torch.from_numpy(listed)), out,
                            lse, mask=(1, 1, 1, 1), cache_bias=-0.5, n_splits=n_splits,
                            workspace=ws)
    torch.cuda.synchronize()
    uniq = np.unique(listed[(listed >= 0) & (listed < n_q)])
    rest = np.setdiff1d(np.arange(n_q), uniq)
    assert (out[torch.from_numpy(rest)].float() == SENTINEL).all()
    assert (lse[:, torch.from_numpy(rest)] == 123.0).all()
    ro, rl = o.attention(inputs.as_f32(q), o.next_pos, n_q, (1, 1, 1, 1), -0.5, rows=uniq)
    assert_attention_close(out, lse, ro, rl, rows=uniq, what=f"rows, {n_splits} key splits")
    assert kv.kv_wait_timeout_count() == 0
