"""Pins of the oracle's 3-D RoPE form (time, height and width runs of the head dimension,
temporal-only resets).  The reading follows "Why Live Video Generation Still Struggles
With Timing", Transcript (positions of long video streams calibrated and reset along
time); the frame grid and the run split are the usual video-DiT layout.

What pins it, besides the oracle itself:
  * with one run and a 1 x 1 grid it is the 1-D rule, bit for bit;
  * a second implementation (``oracle/brute.py``: Python divmod coordinates, math-module
    angles, numpy float32 rotation, torch casts) gives the same ring, bit for bit, and the
    same attention to 1e-12, through a stream that wraps and resets;
  * rotation by whole frames composes on the time run and leaves the height and width
    runs untouched; scores depend only on the frame/row/column offsets."""
import math

import numpy as np
import pytest

from oracle import brute

R3_TINY = (12, 10, 10, 4, 8)        # D = 64: 12 + 10 + 10 pairs; 4 x 8 = 32 tokens per frame
R3_VIDEO = (22, 21, 21, 16, 24)     # D = 128, a 16 x 24 latent frame (384 tokens)


def test_one_run_and_unit_grid_is_the_1d_rule(orc):
    plain = orc.OracleRing(16, 1, 64)
    one = orc.OracleRing(16, 1, 64, rope3d=(32, 0, 0, 1, 1))
    for p in (-4097, -1, 0, 1, 37, 12345, 2 ** 20):
        a, b = plain.rope_cs(p), one.rope_cs(p)
        assert (a[0].view(np.uint32) == b[0].view(np.uint32)).all()
        assert (a[1].view(np.uint32) == b[1].view(np.uint32)).all()


@pytest.mark.parametrize("p", [-1000, -385, -384, -1, 0, 1, 23, 24, 383, 384, 385, 9999])
def test_angles_match_the_brute_force_rule(orc, p):
    for r3, D in ((R3_TINY, 64), (R3_VIDEO, 128)):
        o = orc.OracleRing(8, 1, D, rope3d=r3)
        c, s = o.rope_cs(p)
        bc, bs = brute.angles(p, D, 10000.0, r3)
        assert (c.view(np.uint32) == bc.view(np.uint32)).all(), (r3, p)
        assert (s.view(np.uint32) == bs.view(np.uint32)).all(), (r3, p)


def test_ring_and_attention_match_the_brute_force_ring_3d(orc):
    """The tiny stream (wraps twice, a reset of -4 frames after chunk 8) under 3-D RoPE:
    every slot, scale, position and state integer equal; attention to 1e-12."""
    from test_oracle_pins import _tiny_stream
    assert _tiny_stream(orc, rope3d=R3_TINY) < 1e-12


def _cs64(o, p):
    c, s = o.rope_cs(p)
    return c.astype(np.float64), s.astype(np.float64)


def test_whole_frame_rotation_composes_on_time_and_spares_height_width(orc):
    pt, ph, pw, gh, gw = R3_VIDEO
    o = orc.OracleRing(8, 1, 128, rope3d=R3_VIDEO)
    hw = gh * gw
    for p in (0, 5, 383, 384 * 7 + 100, -384 * 3 + 17):
        for frames in (-9, -1, 1, 4):
            d = frames * hw
            c_d, s_d = _cs64(o, d)
            # a whole-frame delta turns the height and width runs by exactly nothing
            assert (c_d[pt:] == 1.0).all() and (s_d[pt:] == 0.0).all()
            c_p, s_p = _cs64(o, p)
            c_q, s_q = _cs64(o, p + d)
            # angle addition on every pair, to binary32 rounding of the tabled values
            assert np.abs(c_q - (c_p * c_d - s_p * s_d)).max() < 4e-7
            assert np.abs(s_q - (s_p * c_d + c_p * s_d)).max() < 4e-7
            assert (c_q[pt:] == c_p[pt:]).all() and (s_q[pt:] == s_p[pt:]).all()


def _rot64(x, c, s):
    z = (x[0::2] + 1j * x[1::2]) * (c + 1j * s)     # interleaved pairs as complex numbers
    out = np.empty_like(x)
    out[0::2], out[1::2] = z.real, z.imag
    return out


def test_scores_depend_only_on_frame_row_column_offsets(orc):
    """<R(P1) q, R(P2) k> is unchanged when both tokens move by whole frames, and it
    changes when one token moves by a row (so the height run is live)."""
    pt, ph, pw, gh, gw = R3_VIDEO
    o = orc.OracleRing(8, 1, 128, rope3d=R3_VIDEO)
    hw = gh * gw
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(128), rng.standard_normal(128)

    def score(p1, p2):
        # angles recomputed in fp64 from the frame/row/column coordinates
        def cs(p):
            f, rest = divmod(p, hw)
            y, x = divmod(rest, gw)
            coord = [f] * pt + [y] * ph + [x] * pw
            freq = [10000.0 ** (-(2.0 * kk) / (2 * n)) for n in (pt, ph, pw) for kk in range(n)]
            ang = np.array(coord, np.float64) * np.array(freq)
            return np.cos(ang), np.sin(ang)
        return _rot64(q, *cs(p1)) @ _rot64(k, *cs(p2))

    for p1, p2 in ((5, 900), (383, 384), (10000, 777)):
        for frames in (-3, 2, 11):
            assert abs(score(p1 + frames * hw, p2 + frames * hw) - score(p1, p2)) < 1e-9
        assert abs(score(p1 + gw, p2) - score(p1, p2)) > 1e-6
    # and the oracle's binary32 table is that fp64 rule, rounded
    for p in (7, 385, -2000):
        c, s = o.rope_cs(p)
        f, rest = divmod(p, hw)
        y, x = divmod(rest, gw)
        coord = [f] * pt + [y] * ph + [x] * pw
        freq = [10000.0 ** (-(2.0 * kk) / (2 * n)) for n in (pt, ph, pw) for kk in range(n)]
        ang = np.array(coord, np.float64) * np.array(freq)
        assert np.abs(c - np.cos(ang)).max() < 6e-8 and np.abs(s - np.sin(ang)).max() < 6e-8


def test_a_reset_that_is_not_a_whole_frame_is_refused(orc):
    o = orc.OracleRing(64, 1, 64, rope3d=R3_TINY)
    rng = np.random.default_rng(0)
    o.write(rng.standard_normal((32, 1, 64)), rng.standard_normal((32, 1, 64)), commit=True)
    before = (o.kc.copy(), o.ks.copy(), o.state())
    with pytest.raises(ValueError):
        o.delta_rotate(-5)
    assert (o.kc == before[0]).all() and (o.ks == before[1]).all() and o.state() == before[2]
    o.delta_rotate(-32)                                   # one frame: fine
    assert o.next_pos == 0


def test_planted_height_width_swap_is_caught(orc):
    """A plausible mistake (height and width coordinates swapped) changes the angles: the
    brute-force rule with a transposed grid disagrees with the oracle."""
    pt, ph, pw, gh, gw = R3_TINY
    o = orc.OracleRing(8, 1, 64, rope3d=R3_TINY)
    bad = 0
    for p in range(0, 64):
        c, _ = o.rope_cs(p)
        f, rest = divmod(p, gh * gw)
        col, row = divmod(rest, gh)                       # the swapped reading
        coord = [f] * pt + [row] * ph + [col] * pw
        freq = [10000.0 ** (-(2.0 * kk) / (2 * n)) for n in (pt, ph, pw) for kk in range(n)]
        cw = np.array([math.cos(a * b) for a, b in zip(coord, freq)], np.float32)
        bad += int((cw != c).any())
    assert bad > 40
