"""Pins of the oracle's content-memory pieces ("Stream LTX", Inference: keys scored on
attention quality and temporal diversity, evicted down to a top-M budget):

  * key mass: the probability mass every history key receives sums, over all keys of all
    rings, to (rows with a visible key) x heads; it equals the column sums of the dense
    brute-force softmax of ``oracle/brute.py``;
  * selection: equal to an independent greedy implementation (pick the best remaining
    score; every kept key of a frame halves the scores of that frame's other keys), to
    plain top-M when gamma = 1, and to one key per frame first when gamma is tiny."""
import numpy as np
import pytest

from oracle import brute


def _stream(orc, C=96, H=2, D=32, n=16, chunks=9, seed=3):
    rng = np.random.default_rng(seed)
    o, b = orc.OracleRing(C, H, D), brute.BruteRing(C, H, D)
    for ch in range(chunks):
        k = rng.standard_normal((n, H, D)).astype(np.float32)
        v = rng.standard_normal((n, H, D)).astype(np.float32)
        o.write(k, v, commit=True)
        b.write(k, v, commit=True)
    q = rng.standard_normal((n, H, D)).astype(np.float32)
    return o, b, q


def test_key_mass_sums_to_one_per_row_and_head(orc):
    o, _, q = _stream(orc)
    ages = np.arange(o.C)
    anchor = orc.OracleRing(24, 2, 32)
    rng = np.random.default_rng(8)
    anchor.write(rng.standard_normal((24, 2, 32)), rng.standard_normal((24, 2, 32)), commit=True)
    for bias in (0.0, -1.5):
        m0 = orc.key_mass(o, [anchor], q, o.next_pos, 0, 0, ages, cache_bias=bias)
        m1 = orc.key_mass(o, [anchor], q, o.next_pos, 0, 1, np.arange(24), cache_bias=bias)
        assert (m0 > 0).all() and (m1 > 0).all()
        assert abs(m0.sum() + m1.sum() - q.shape[0] * 2) < 1e-9


def test_key_mass_equals_brute_force_column_sums(orc):
    o, b, q = _stream(orc)
    n, H = q.shape[0], 2
    sm = float(np.float32(1 / np.sqrt(32)))
    # brute: dense softmax over the window (all history: n_current = 0), column sums
    win = b.window()
    K = np.stack([brute.e4m3_values(t["kc"]) * t["ks"][:, None].astype(np.float64) for t in win], 1)
    want = np.zeros(len(win))
    for h in range(H):
        Q = np.stack([brute.bf16(brute.rope32(q[i, h], b.next_pos + i, 10000.0))
                      for i in range(n)]).astype(np.float64)
        S = sm * (Q @ K[h].T) - 0.75
        P = np.exp(S - S.max(1, keepdims=True))
        want += (P / P.sum(1, keepdims=True)).sum(0)
    # window entry w is the (len(win) - 1 - w)-th newest slot
    ages = np.arange(len(win))[::-1]
    got = orc.key_mass(o, [], q, o.next_pos, 0, 0, ages, cache_bias=-0.75)
    assert np.abs(got - want).max() < 1e-10


def _greedy(quality, frame, pos, M, gamma):
    """Independent restatement: repeatedly keep the best remaining effective score."""
    n = len(quality)
    kept_per_frame = {}
    left = set(range(n))
    out = []
    while left and len(out) < M:
        def eff(i):
            return quality[i] * gamma ** kept_per_frame.get(frame[i], 0)
        best = min(left, key=lambda i: (-eff(i), pos[i], i))
        out.append(best)
        left.remove(best)
        kept_per_frame[frame[best]] = kept_per_frame.get(frame[best], 0) + 1
    return sorted(out)


@pytest.mark.parametrize("seed", range(6))
def test_selection_equals_independent_greedy(orc, seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 300))
    quality = rng.random(n) ** 3
    quality[rng.integers(0, n, n // 10)] = 0.5                 # exact ties on purpose
    pos = rng.permutation(4 * n)[:n]
    frame = pos // 24
    M = int(rng.integers(1, n + 10))
    for gamma in (0.5, 1.0, 0.25):
        got = orc.memory_select(quality, frame, pos, M, gamma)
        assert got.tolist() == _greedy(quality, frame, pos, M, gamma), (seed, gamma)


@pytest.mark.parametrize("seed", range(4))
def test_selection_ties_on_quality_and_position(orc, seed):
    """Quality from four values and positions from a narrow range around zero: most
    candidates tie on quality, many share a position (the candidate index decides), and
    negative positions fall in negative frames (floor division)."""
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 250))
    quality = rng.choice([0.0, 0.25, 0.5, 1.0], size=n)
    pos = rng.integers(-60, 60, size=n)
    frame = np.floor_divide(pos, 24)
    M = int(rng.integers(1, n + 3))
    for gamma in (0.5, 0.25, 1.0):
        got = orc.memory_select(quality, frame, pos, M, gamma)
        assert got.tolist() == _greedy(quality, frame, pos, M, gamma), (seed, gamma)


def test_selection_limits(orc):
    rng = np.random.default_rng(11)
    quality = rng.random(200)
    pos = np.arange(200)
    frame = pos // 10                                          # 20 frames of 10
    top = orc.memory_select(quality, frame, pos, 37, 1.0)
    assert top.tolist() == sorted(np.argsort(-quality, kind="stable")[:37].tolist())
    one_each = orc.memory_select(quality, frame, pos, 20, 1e-300)
    best = [f * 10 + int(np.argmax(quality[f * 10:(f + 1) * 10])) for f in range(20)]
    assert one_each.tolist() == sorted(best)
    assert orc.memory_select(quality, frame, pos, 500, 0.5).tolist() == list(range(200))
