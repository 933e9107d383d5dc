"""Bit-exact parity of the ring write and the delta rotation (CUDA path through the C ABI
vs the fp64 oracle): e4m3 codes, fp32 scale bit patterns, slot positions, ring state."""
import numpy as np
import pytest
import torch

import kv_cache_attention_ring_b200 as kv
from kv_cache_attention_ring_b200 import inputs
from helpers import assert_ring_equal, to_dev, valid_slots

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_attention_ring_b200 import build
    build.build()
    kv.lib()


def test_tiny_stream_every_pass(orc):
    """12 chunks of 32 into 256 slots (wraps after chunk 8), 4 passes per chunk, reset
    by -128 after chunk 8; fp32 inputs, D=64."""
    w = inputs.TINY
    ring = kv.KvRing(w.C, w.H, w.D, pos_min=-256, pos_max=1024)
    o = orc.OracleRing(w.C, w.H, w.D)
    for ch in range(w.extra["chunks"]):
        for p in range(4):
            _, k, v = inputs.chunk_qkv(w, ch, p)
            kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=(p == 3))
            o.write(inputs.as_f32(k), inputs.as_f32(v), commit=(p == 3))
            assert_ring_equal(ring, o, what=f"chunk {ch} pass {p}")
        if ch == w.extra["reset_after"]:
            kv.kv_ring_delta_rotate(ring, w.extra["delta"])
            o.delta_rotate(w.extra["delta"])
            assert_ring_equal(ring, o, what=f"reset after chunk {ch}")


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("D", [64, 128])
def test_write_wraps_and_commits(orc, dtype, D):
    C, H = 300, 3
    ring = kv.KvRing(C, H, D, pos_min=0, pos_max=2000)
    o = orc.OracleRing(C, H, D)
    for i, n in enumerate((257, 1, 128, 300, 77)):
        k = inputs.draw(inputs.seed_of(D, i, 1), (n, H, D), "student_t4", 1.0, dtype)
        v = inputs.draw(inputs.seed_of(D, i, 2), (n, H, D), "normal", 0.3, dtype)
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=True)
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=True)
        assert_ring_equal(ring, o, what=f"write {i} n={n}")


def test_write_degenerate_rows(orc):
    """Zero rows, rows with inf/NaN, rows so small that 448/amax overflows, huge rows,
    subnormal inputs and signed zeros."""
    C, H, D = 64, 4, 128
    n = 8
    k = np.random.default_rng(3).standard_normal((n, H, D)).astype(np.float32)
    v = k.copy()
    k[0, 0] = 0.0
    v[0, 1] = -0.0
    k[1, 2, 5] = np.inf
    v[1, 3, 7] = np.nan
    k[2, 1] = 1e-37
    v[2, 0] = -3e-39                         # binary32 subnormals
    k[3, 3] = 1e38
    v[3, 2] = np.float32(3.0e38)
    k[4, 0, ::2] = -0.0
    k[4, 0, 1::2] = 1e-45
    ring = kv.KvRing(C, H, D, pos_min=0, pos_max=100)
    o = orc.OracleRing(C, H, D)
    kv.kv_ring_write(ring, to_dev(torch.from_numpy(k)), to_dev(torch.from_numpy(v)), commit=True)
    o.write(k, v, commit=True)
    assert_ring_equal(ring, o, what="degenerate rows")
    # bf16 inputs with extreme exponents
    kb = torch.from_numpy(k * 1e-20).to(torch.bfloat16)
    vb = torch.from_numpy(v).to(torch.bfloat16)
    kv.kv_ring_write(ring, to_dev(kb), to_dev(vb), commit=True)
    o.write(inputs.as_f32(kb), inputs.as_f32(vb), commit=True)
    assert_ring_equal(ring, o, what="degenerate rows bf16")
    # rotating rows that hold NaN scales or zero scales keeps them as they are
    kv.kv_ring_delta_rotate(ring, 37)
    o.delta_rotate(37)
    assert_ring_equal(ring, o, what="degenerate rows rotated")


def test_runway_shape_write_wrapping(orc):
    """H=40, D=128, C=5,788, 757 bf16 tokens per call, started near the end of the ring
    so the chunk wraps; three committed chunks and a pending one."""
    w = inputs.RUNWAY
    ring = kv.KvRing(w.C, w.H, w.D, pos_min=0, pos_max=10000)
    o = orc.OracleRing(w.C, w.H, w.D)
    ring.s.write_slot = o._s.write_slot = 5000
    for ch in range(4):
        _, k, v = inputs.chunk_qkv(w, ch)
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=(ch < 3))
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=(ch < 3))
    assert_ring_equal(ring, o, what="runway write")


def test_rotate_full_stress_shape(orc):
    """C=32,768 slots x 40 heads, Student-t(4) keys, whole-cache reset by -18,432
    (the stress stream's first reset: positions return to 0..C-1)."""
    w = inputs.STRESS
    ring = kv.KvRing(w.C, w.H, w.D, pos_min=-20000, pos_max=60000, next_pos=18432)
    o = orc.OracleRing(w.C, w.H, w.D, next_pos=18432)
    for ch in range(w.C // w.n):
        _, k, v = inputs.chunk_qkv(w, ch)
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=True)
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=True)
    assert_ring_equal(ring, o, what="stress fill")
    kv.kv_ring_delta_rotate(ring, -18432)
    o.delta_rotate(-18432)
    assert_ring_equal(ring, o, what="stress rotate")
    assert ring.slot_pos.min().item() == 0 and ring.slot_pos.max().item() == w.C - 1


def test_rotate_partial_and_wrapped_valid_range(orc):
    C, H, D = 200, 2, 128
    ring = kv.KvRing(C, H, D, pos_min=-500, pos_max=2000)
    o = orc.OracleRing(C, H, D)
    ring.s.write_slot = o._s.write_slot = 150
    for i, (n, commit) in enumerate(((90, True), (40, False))):
        k = inputs.draw(inputs.seed_of(7, i, 1), (n, H, D), "normal", 1.0, "bf16")
        v = inputs.draw(inputs.seed_of(7, i, 2), (n, H, D), "normal", 1.0, "bf16")
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=commit)
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=commit)
    for delta in (-100, 3, 0, 1999):
        kv.kv_ring_delta_rotate(ring, delta)
        o.delta_rotate(delta)
        assert_ring_equal(ring, o, slots=valid_slots(o), what=f"delta {delta}")
