"""Pins of the fp64 CPU oracle against things other than itself (CPU only).

Each test checks the oracle against a library routine (torch's e4m3/bf16 casts, numpy
float32 arithmetic, Python's math module), a closed form, an invariant of the method, or
the independent brute-force implementation in ``oracle/brute.py`` on tiny inputs.
"""
import math

import numpy as np
import pytest
import torch

from oracle import brute

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------- e4m3 / bf16 rounding

def test_e4m3_decode_exhaustive(orc):
    codes = np.arange(256, dtype=np.uint8)
    got = orc.e4m3_decode(codes)
    want = brute.e4m3_values(codes)
    nan = np.isnan(want)
    assert (np.isnan(got) == nan).all()
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert (got[~nan] == want[~nan]).all()
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def _e4m3_sweep():
    vals = brute.e4m3_values(np.arange(256, dtype=np.uint8))
    fin = np.sort(np.unique(vals[np.isfinite(vals)]))
    mids = (fin[1:] + fin[:-1]) / 2                      # exact ties
    nudged = np.concatenate([np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
                             np.nextafter(mids.astype(np.float32), np.float32(-np.inf))])
    rng = np.random.default_rng(7)
    rand = np.concatenate([rng.uniform(-460, 460, 20000), rng.uniform(-0.02, 0.02, 20000),
                           rng.standard_normal(20000) * 10.0 ** rng.uniform(-6, 2, 20000)])
    edge = np.array([0.0, -0.0, 448.0, -448.0, 449.0, 463.9, 464.0, 470.0, 1e30, -1e30,
                     2.0 ** -10, -(2.0 ** -10), 2.0 ** -11, 3 * 2.0 ** -10, 1e-40])
    return np.concatenate([fin, mids, nudged, rand, edge]).astype(np.float32)


def test_e4m3_encode_matches_torch_cast(orc):
    x = _e4m3_sweep()
    got = orc.e4m3_encode(x)
    want = brute.e4m3_codes(x)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(x[i]), int(got[i]), int(want[i])) for i in bad[:10]]
    assert orc.e4m3_encode([np.nan])[0] == 0x7F


def test_e4m3_encode_roundtrip_and_saturation(orc):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = orc.e4m3_decode(codes).astype(np.float32)
    assert (orc.e4m3_encode(vals) == codes).all()
    assert (orc.e4m3_encode([449.0, 500.0, 1e38, np.inf]) == 0x7E).all()
    assert (orc.e4m3_encode([-449.0, -1e38, -np.inf]) == 0xFE).all()


def test_bf16_round_matches_torch_cast(orc):
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 2 ** 32, 200000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    ties = (np.arange(1, 5000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    sub = (rng.integers(1, 2 ** 23, 5000, dtype=np.uint64).astype(np.uint32)).view(np.float32)
    edge = np.array([3.3895313e38, 3.3961776e38, 3.4e38, -3.4e38, 1e-45, 1.0, 1.00390625,
                     1.01171875], np.float32)
    x = np.concatenate([x, ties, -ties, sub, edge])
    got = orc.bf16_round(x)
    want = brute.bf16(x)
    assert (got.view(np.uint32) == want.view(np.uint32)).all()


# ---------------------------------------------------------------- RoPE

@pytest.mark.parametrize("p", [0, 1, 7, 31, 255, -128, -1, 4096, 83968, -51200])
def test_rope_cs_matches_math_module(orc, p):
    for D in (64, 128):
        c, s = orc.rope_cs(p, D)
        bc, bs = brute.angles(p, D, 10000.0)
        assert (c.view(np.uint32) == bc.view(np.uint32)).all()
        assert (s.view(np.uint32) == bs.view(np.uint32)).all()
    c, s = orc.rope_cs(p, 64)
    assert c[0] == np.float32(math.cos(p)) and s[0] == np.float32(math.sin(p))


@pytest.mark.parametrize("p", [0, 3, 257, -128, 40000])
def test_rope_binary32_ops_match_numpy_float32(orc, p):
    rng = np.random.default_rng(11 + abs(p))
    x = (rng.standard_normal((16, 128)) * 10.0 ** rng.uniform(-3, 3, (16, 1))).astype(np.float32)
    got = np.stack([orc.rope_apply(r, p) for r in x])
    want = brute.rope32(x, p, 10000.0)
    assert (got.view(np.uint32) == want.view(np.uint32)).all()


def test_rope_is_a_rotation_and_composes(orc):
    rng = np.random.default_rng(5)
    x = rng.standard_normal(128)
    for p, d in [(0, 5), (17, -17), (1000, -999), (5787, 3), (-128, 300)]:
        y = orc.rope_apply_f64(x, p)
        assert abs(np.linalg.norm(y) / np.linalg.norm(x) - 1) < 1e-14
        z = orc.rope_apply_f64(y, d)
        w = orc.rope_apply_f64(x, p + d)
        assert np.abs(z - w).max() < 1e-12 * np.abs(x).max() * (1 + abs(p) + abs(d)) ** 0.5
    # relative-position invariance of the dot product
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    base = orc.rope_apply_f64(q, 40) @ orc.rope_apply_f64(k, 13)
    for a in (-13, 1, 977, 20000):
        sh = orc.rope_apply_f64(q, 40 + a) @ orc.rope_apply_f64(k, 13 + a)
        assert abs(sh - base) < 1e-10
    # binary32 path composes up to binary32 rounding
    x32 = x.astype(np.float32)
    z = orc.rope_apply(orc.rope_apply(x32, 300), -128)
    w = orc.rope_apply(x32, 172)
    assert np.abs(z - w).max() < 1e-5 * np.abs(x).max()


# ---------------------------------------------------------------- per-row quantisation

def test_quant_rows_match_brute_and_bound(orc):
    rng = np.random.default_rng(21)
    y = np.concatenate([
        rng.standard_normal((200, 128)),
        rng.standard_t(4.0, (200, 128)),
        rng.standard_normal((50, 128)) * 1e-30,
        rng.standard_normal((50, 128)) * 1e30,
    ]).astype(np.float32)
    codes, scales = orc.quant_rows(y)
    bc, bs = brute.quant(y)
    assert (codes == bc).all() and (scales.view(np.uint32) == bs.view(np.uint32)).all()
    deq = orc.e4m3_decode(codes) * scales[:, None].astype(np.float64)
    err = np.abs(deq - y.astype(np.float64))
    bound = (2.0 ** -4 * np.abs(y) + scales[:, None] * 2.0 ** -10) * (1 + 1e-6)
    assert (err <= bound).all()
    # the largest element of every row maps to +-448 exactly
    arg = np.abs(y).argmax(1)
    assert set(np.unique(codes[np.arange(len(y)), arg] & 0x7F).tolist()) == {0x7E}


def test_quant_degenerate_rows(orc):
    D = 64
    rows = np.zeros((5, D), np.float32)
    rows[1, 3] = np.inf
    rows[2, 0] = np.nan
    rows[3, :] = 1e-37            # 448/amax overflows binary32
    rows[4, :] = -0.0
    codes, scales = orc.quant_rows(rows)
    bc, bs = brute.quant(rows)
    assert (codes == bc).all() and (scales.view(np.uint32) == bs.view(np.uint32)).all()
    assert scales[0] == 0 and (codes[0] == 0).all()
    assert scales[1].view(np.uint32) == 0x7FC00000 and (codes[1] == 0x7F).all()
    assert scales[2].view(np.uint32) == 0x7FC00000 and (codes[2] == 0x7F).all()
    assert scales[3] == 0 and (codes[3] == 0).all()
    assert scales[4] == 0 and (codes[4] == 0).all()


# ---------------------------------------------------------------- ring == linear buffer

def _tiny_stream(orc, check_every_pass=True, mode_b=False, rope3d=None):
    """The tiny workload: 12 chunks of 32 into 256 slots, 4 passes per chunk (3 pending
    rewrites and a commit), reset by -128 after chunk 8; attention on every last pass."""
    C, H, D, n = 256, 2, 64, 32
    rng = np.random.default_rng(1)
    o = orc.OracleRing(C, H, D, rope3d=rope3d)
    b = brute.BruteRing(C, H, D, rope3d=rope3d)
    sm = float(np.float32(1 / np.sqrt(D)))
    worst = 0.0
    for ch in range(12):
        q = rng.standard_normal((n, H, D)).astype(np.float32)
        for p in range(4):
            k = rng.standard_normal((n, H, D)).astype(np.float32)
            v = rng.standard_normal((n, H, D)).astype(np.float32)
            o.write(k, v)
            b.write(k, v)
            if p == 3:
                for bias in (0.0, -2.0):
                    for mask in ((32, 32, 32, 32), (8, 8, 8, 8), (1, 1, 1, 1)):
                        oo, ol = o.attention(q, o.next_pos, n, mask, bias, mode_b=mode_b)
                        bo, bl = b.attention(q, b.next_pos, n, mask, bias, sm, mode_b=mode_b)
                        worst = max(worst, np.abs(oo - bo).max(), np.abs(ol - bl).max())
            if check_every_pass or p == 3:
                kc, vc, ks, vs, sp = b.arrays()
                assert o.state() == b.state()
                for age in range(min(o.live + o.pending, C)):
                    assert o.slot_of_age(age) == (len(b.tokens) + len(b.pending) - 1 - age) % C
                assert (o.kc == kc).all() and (o.vc == vc).all(), (ch, p)
                assert (o.ks.view(np.uint32) == ks.view(np.uint32)).all()
                assert (o.vs.view(np.uint32) == vs.view(np.uint32)).all()
                assert (o.slot_pos == sp).all()
        o.commit()
        b.commit()
        if ch == 8:
            o.delta_rotate(-128)
            b.delta_rotate(-128)
            kc, vc, ks, vs, sp = b.arrays()
            assert o.state() == b.state() and (o.kc == kc).all() and (o.slot_pos == sp).all()
    return worst


def test_ring_matches_linear_buffer_tiny(orc):
    worst = _tiny_stream(orc)
    assert worst < 1e-12


def test_mode_b_matches_brute_tiny(orc):
    assert _tiny_stream(orc, check_every_pass=False, mode_b=True) < 1e-12


# ---------------------------------------------------------------- attention invariants

def _ring_with_history(orc, C=96, H=2, D=32, hist=64, n=16, seed=9, start_slot=0):
    rng = np.random.default_rng(seed)
    o = orc.OracleRing(C, H, D)
    o._s.write_slot = start_slot
    for ch in range(hist // n):
        o.write(rng.standard_normal((n, H, D)), rng.standard_normal((n, H, D)), commit=True)
    k, v = rng.standard_normal((n, H, D)), rng.standard_normal((n, H, D))
    q = rng.standard_normal((n, H, D)).astype(np.float32)
    o.write(k, v)
    return o, q, (k, v)


def test_bias_zero_is_plain_softmax_attention(orc):
    o, q, _ = _ring_with_history(orc)
    n, H, D = q.shape
    out, _ = o.attention(q, o.next_pos, n, (4, 4, 4, 4), 0.0)
    nv = o.live + o.pending
    slots = [o.slot_of_age(a) for a in range(nv)][::-1]        # oldest first
    K = torch.from_numpy(orc.e4m3_decode(o.kc[:, slots]) * o.ks[:, slots, None])
    V = torch.from_numpy(orc.e4m3_decode(o.vc[:, slots]) * o.vs[:, slots, None])
    Q = torch.from_numpy(np.stack([[orc.bf16_round(orc.rope_apply(q[i, h], o.next_pos + i))
                                    for h in range(H)] for i in range(n)]).astype(np.float64))
    blk_q = torch.tensor([0 if i < 4 else 1 + (i - 4) // 4 for i in range(n)])
    allowed = torch.ones(n, nv, dtype=torch.bool)
    allowed[:, nv - n:] = blk_q[None, :] <= blk_q[:, None]
    sm = float(np.float32(1 / np.sqrt(D)))
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.permute(1, 0, 2), K, V, attn_mask=allowed, scale=sm).permute(1, 0, 2)
    assert np.abs(out - ref.numpy()).max() < 1e-12


def test_bias_minus_inf_keeps_only_the_current_chunk(orc):
    o, q, (k, v) = _ring_with_history(orc)
    n, H, D = q.shape
    got, _ = o.attention(q, o.next_pos, n, (4, 4, 4, 4), -1e30)
    fresh = orc.OracleRing(o.C, H, D, next_pos=o.next_pos)
    fresh.write(k, v)
    want, _ = fresh.attention(q, o.next_pos, n, (4, 4, 4, 4), 0.0)
    assert np.abs(got - want).max() < 1e-13


def test_bias_is_an_additive_logit_closed_form(orc):
    """exp(lse(b)) = e^b L_h + L_c and o(b) = (e^b N_h + N_c) / (e^b L_h + L_c)."""
    o, q, _ = _ring_with_history(orc)
    n = q.shape[0]
    b1, b2, b3 = 0.0, -2.0, -0.75
    o1, l1 = o.attention(q, o.next_pos, n, (1, 1, 1, 1), b1)
    o2, l2 = o.attention(q, o.next_pos, n, (1, 1, 1, 1), b2)
    o3, l3 = o.attention(q, o.next_pos, n, (1, 1, 1, 1), b3)
    E1, E2 = np.exp(l1), np.exp(l2)                              # [H][n]
    Lh = (E1 - E2) / (np.exp(b1) - np.exp(b2))
    Lc = E1 - np.exp(b1) * Lh
    assert np.allclose(np.log(np.exp(b3) * Lh + Lc), l3, rtol=0, atol=1e-10)
    T1, T2 = o1 * E1.T[:, :, None], o2 * E2.T[:, :, None]        # [n][H][D]
    Nh = (T1 - T2) / (np.exp(b1) - np.exp(b2))
    Nc = T1 - np.exp(b1) * Nh
    pred = (np.exp(b3) * Nh + Nc) / (np.exp(b3) * Lh + Lc).T[:, :, None]
    assert np.abs(pred - o3).max() < 1e-9


def test_future_block_perturbation_leaves_earlier_blocks_unchanged(orc):
    o, q, (k, v) = _ring_with_history(orc)
    n = q.shape[0]
    mask = (4, 4, 4, 4)                                           # blocks 0..3 of 4 tokens
    before, lb = o.attention(q, o.next_pos, n, mask, -1.0)
    k2, v2, q2 = k.copy(), v.copy(), q.copy()
    rng = np.random.default_rng(99)
    k2[8:], v2[8:], q2[8:] = (rng.standard_normal(k2[8:].shape) for _ in range(3))
    o.write(k2, v2)                                               # rewrite the pending chunk
    after, la = o.attention(q2, o.next_pos, n, mask, -1.0)
    assert (before[:8] == after[:8]).all() and (lb[:, :8] == la[:, :8]).all()
    assert np.abs(before[8:] - after[8:]).max() > 1e-3


def test_ring_wrap_placement_does_not_change_attention(orc):
    outs = []
    for start in (0, 37, 95):
        o, q, _ = _ring_with_history(orc, start_slot=start)
        outs.append(o.attention(q, o.next_pos, q.shape[0], (2, 3, 2, 3), -0.5))
    for out, lse in outs[1:]:
        assert np.abs(out - outs[0][0]).max() < 1e-13 and np.abs(lse - outs[0][1]).max() < 1e-13


def test_empty_ring_gives_zero_output_and_minus_inf_lse(orc):
    o = orc.OracleRing(64, 2, 32)
    q = np.ones((3, 2, 32), np.float32)
    out, lse = o.attention(q, 0, 0)
    assert (out == 0).all() and np.isneginf(lse).all()


def test_minus_inf_bias_without_current_keys_attends_nothing(orc):
    o, q, _ = _ring_with_history(orc)
    o.commit()
    out, lse = o.attention(q, o.next_pos, 0, cache_bias=-np.inf)
    assert (out == 0).all() and np.isneginf(lse).all()
    b = brute.BruteRing(o.C, o.H, o.D)
    bo, bl = b.attention(q, 0, 0, (1, 1, 1, 1), -np.inf, 0.125)
    assert (bo == 0).all() and np.isneginf(bl).all()


# ---------------------------------------------------------------- persistent anchor

def _lse_merge(parts):
    """Merge (out [n][H][D], lse [H][n]) results over disjoint key sets: the softmax over
    the union, written in closed form from the parts."""
    lses = np.stack([l for _, l in parts])                        # [P][H][n]
    top = lses.max(0)
    safe = np.where(np.isfinite(top), top, 0.0)
    w = np.exp(lses - safe)                                       # [P][H][n]
    tot = w.sum(0)
    out = sum(wp.T[:, :, None] * o for wp, (o, _) in zip(w, parts))
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where(tot.T[:, :, None] > 0, out / tot.T[:, :, None], 0.0)
        lse = np.where(tot > 0, safe + np.log(tot), -np.inf)
    return out, lse


def test_anchor_beside_window_matches_brute_tiny(orc):
    """First chunk kept as a persistent anchor ring, later chunks in a 128-slot window ring
    that wraps twice; a reset re-rotates both.  The oracle's multi-ring attention equals the
    brute model's dense attention over anchor + window, the rings equal the brute arrays bit
    for bit, and the anchor is never evicted."""
    A, W, H, D, n = 32, 128, 2, 64, 32
    rng = np.random.default_rng(17)
    anchor = orc.OracleRing(A, H, D)
    win = orc.OracleRing(W, H, D, next_pos=A)
    b = brute.BruteAnchoredRing(A, W, H, D)
    sm = float(np.float32(1 / np.sqrt(D)))
    worst, worst_merge = 0.0, 0.0
    for ch in range(10):
        main, hist = (anchor, [win]) if ch == 0 else (win, [anchor])
        q = rng.standard_normal((n, H, D)).astype(np.float32)
        for p in range(2):
            k = rng.standard_normal((n, H, D)).astype(np.float32)
            v = rng.standard_normal((n, H, D)).astype(np.float32)
            main.write(k, v)
            b.write(k, v)
            for bias in (0.0, -2.0):
                for mask in ((32, 32, 32, 32), (8, 8, 8, 8)):
                    oo, ol = orc.attention_multi(main, hist, q, main.next_pos, n, mask, bias)
                    bo, bl = b.attention(q, b.next_pos, n, mask, bias, sm)
                    worst = max(worst, np.abs(oo - bo).max(), np.abs(ol - bl).max())
                    # the union of disjoint key sets: the closed-form merge of the parts
                    parts = [orc.attention_multi(main, [], q, main.next_pos, n, mask, bias)]
                    parts += [orc.attention_multi(r, [], q, main.next_pos, 0, mask, bias)
                              for r in hist]
                    mo, ml = _lse_merge(parts)
                    worst_merge = max(worst_merge, np.abs(mo - oo).max(),
                                      np.abs(ml - ol).max())
        main.commit()
        b.commit()
        if ch == 6:
            for r in (anchor, win):
                r.delta_rotate(-96)
            b.delta_rotate(-96)
        # the anchor holds the first chunk for good; the window the last W tokens after it
        kc, ks, sp = b.fifo_arrays()
        assert (win.kc == kc).all() and (win.ks.view(np.uint32) == ks.view(np.uint32)).all()
        assert (win.slot_pos == sp).all()
        assert b.next_pos == win.next_pos
        for s, tok in enumerate(b.window()[:A]):
            assert (anchor.kc[:, s] == tok["kc"]).all() and anchor.slot_pos[s] == tok["pos"]
            assert (anchor.ks[:, s].view(np.uint32) == tok["ks"].view(np.uint32)).all()
    assert (anchor.slot_pos == np.arange(A) - 96).all()      # first chunk, shifted once
    assert worst < 1e-12 and worst_merge < 1e-12


def test_empty_anchor_is_the_plain_ring(orc):
    o, q, _ = _ring_with_history(orc)
    empty = orc.OracleRing(16, o.H, o.D)
    n = q.shape[0]
    a = o.attention(q, o.next_pos, n, (4, 4, 4, 4), -0.5)
    m = orc.attention_multi(o, [empty], q, o.next_pos, n, (4, 4, 4, 4), -0.5)
    assert np.array_equal(a[0], m[0]) and np.array_equal(a[1], m[1])


def test_gathered_rows_equal_the_full_rows(orc):
    """The sampled-row form the full-size parity tests use: attention of a gathered subset
    of query rows equals those rows of the full result exactly (rows are independent)."""
    o, q, _ = _ring_with_history(orc, n=16)
    n = q.shape[0]
    full, lse = o.attention(q, o.next_pos, n, (3, 5, 3, 5), -1.5)
    rows = [15, 0, 7, 7, 3]
    part, lp = o.attention(q, o.next_pos, n, (3, 5, 3, 5), -1.5, rows=rows)
    assert np.array_equal(part, full[rows]) and np.array_equal(lp, lse[:, rows])
