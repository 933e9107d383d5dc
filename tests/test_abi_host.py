"""Host-side checks of the C ABI that need no GPU: exports, status strings, the RoPE
table, and argument/state validation that returns before anything is enqueued."""
import ctypes
import re

import numpy as np
import pytest

import kv_cache_attention_ring_b200 as kv
from kv_cache_attention_ring_b200 import build

MAGIC = 0x6B7672696E673031


@pytest.fixture(scope="module")
def L():
    build.build()
    return kv.lib()


def _declared():
    src = open(build.os.path.join(build.HERE, "..", "include", "kvring.h")).read()
    return re.findall(r"^KV_API\s+[\w\s\*]+?\b(\w+)\(", src, re.M)


def test_library_exports_every_declared_symbol(L):
    names = _declared()
    assert sorted(names) == sorted(kv.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, -5):
        assert kv.kv_status_string(code) and "unknown" not in kv.kv_status_string(code)
    assert "unknown" in kv.kv_status_string(-99)


def test_rope_table_matches_oracle_angles(L, orc):
    tab = kv.kv_rope_table_build(-130, 300, 64)
    for p in (-130, -1, 0, 1, 255, 300):
        c, s = orc.rope_cs(p, 64)
        assert (tab[p + 130, :, 0].view(np.uint32) == c.view(np.uint32)).all()
        assert (tab[p + 130, :, 1].view(np.uint32) == s.view(np.uint32)).all()
    with pytest.raises(kv.KvError):
        kv.kv_rope_table_build(5, 4, 64)


@pytest.mark.parametrize("r3,D", [((12, 10, 10, 4, 8), 64), ((22, 21, 21, 16, 24), 128),
                                   ((64, 0, 0, 1, 1), 128)])
def test_rope3d_table_matches_oracle_angles(L, orc, r3, D):
    """The library's 3-D table equals the oracle's 3-D angles bit for bit (negative
    positions, frame and row boundaries included); one run on a 1 x 1 grid is the 1-D
    table."""
    tab = kv.kv_rope3d_table_build(-800, 1200, D, r3)
    o = orc.OracleRing(4, 1, D, rope3d=r3)
    hw = r3[3] * r3[4]
    for p in sorted({-800, -hw - 1, -hw, -1, 0, 1, r3[4] - 1, r3[4], hw - 1, hw, hw + 1, 1200}):
        c, s_ = o.rope_cs(p)
        assert (tab[p + 800, :, 0].view(np.uint32) == c.view(np.uint32)).all(), p
        assert (tab[p + 800, :, 1].view(np.uint32) == s_.view(np.uint32)).all(), p
    if r3[1] == r3[2] == 0:
        one = kv.kv_rope_table_build(-800, 1200, D)
        assert (one.view(np.uint32) == tab.view(np.uint32)).all()


def test_rope3d_validation(L):
    out = np.empty((4, 32, 2), np.float32)
    ptr = ctypes.c_void_p(out.ctypes.data)
    assert L.kv_rope3d_table_build(ptr, 0, 3, 64, 10000.0, 12, 10, 10, 4, 8) == kv.KV_OK
    assert L.kv_rope3d_table_build(ptr, 0, 3, 64, 10000.0, 12, 10, 11, 4, 8) == kv.KV_EINVAL
    assert L.kv_rope3d_table_build(ptr, 0, 3, 64, 10000.0, -1, 23, 10, 4, 8) == kv.KV_EINVAL
    assert L.kv_rope3d_table_build(ptr, 0, 3, 64, 10000.0, 12, 10, 10, 0, 8) == kv.KV_EINVAL
    assert L.kv_rope3d_table_build(None, 0, 3, 64, 10000.0, 12, 10, 10, 4, 8) == kv.KV_EINVAL
    s = _fake_ring()
    s.initialized = 0
    s.rope_pairs_t, s.rope_pairs_h, s.rope_pairs_w, s.rope_grid_h, s.rope_grid_w = 12, 10, 9, 4, 8
    assert L.kv_ring_init(ctypes.byref(s)) == kv.KV_EINVAL            # pairs sum 31 != 32
    s.rope_pairs_w, s.rope_grid_w = 10, 0
    assert L.kv_ring_init(ctypes.byref(s)) == kv.KV_EINVAL            # empty grid
    # a reset moves whole frames: 32 tokens per frame here
    s = _fake_ring()
    s.rope_pairs_t, s.rope_pairs_h, s.rope_pairs_w, s.rope_grid_h, s.rope_grid_w = 12, 10, 10, 4, 8
    s.next_pos = 500
    r = ctypes.byref(s)
    assert L.kv_ring_delta_rotate(r, -33, None) == kv.KV_EINVAL
    assert s.next_pos == 500
    assert L.kv_ring_delta_rotate(r, -64, None) == kv.KV_OK             # empty ring: no launch
    assert s.next_pos == 436


def _fake_ring(C=256, H=2, D=64, pmin=0, pmax=4096):
    s = kv.kv_ring_t()
    s.capacity, s.n_heads, s.head_dim = C, H, D
    for f in ("k_codes", "v_codes", "k_scale", "v_scale", "slot_pos", "rope_table"):
        setattr(s, f, 0x100000)             # never dereferenced on these paths
    s.rope_pos_min, s.rope_pos_max, s.rope_base = pmin, pmax, 10000.0
    s.initialized = 1
    s.opaque[64] = MAGIC
    return s


def test_init_validation_without_gpu(L):
    s = kv.kv_ring_t()
    assert L.kv_ring_init(None) == kv.KV_EINVAL
    assert L.kv_ring_init(ctypes.byref(s)) == kv.KV_EINVAL          # zero capacity
    s = _fake_ring(D=96)
    assert L.kv_ring_init(ctypes.byref(s)) == kv.KV_EUNSUPPORTED
    s = _fake_ring()
    s.k_codes = 0
    assert L.kv_ring_init(ctypes.byref(s)) == kv.KV_EINVAL
    s = _fake_ring()
    s.k_codes = 0x100001                                             # misaligned
    assert L.kv_ring_init(ctypes.byref(s)) == kv.KV_EINVAL
    s = _fake_ring()
    assert L.kv_ring_init(ctypes.byref(s)) in (kv.KV_ECUDA, kv.KV_EUNSUPPORTED)  # no GPU here
    assert s.initialized == 0


def test_calls_on_uninitialised_ring_are_refused(L):
    s = kv.kv_ring_t()
    assert L.kv_ring_commit(ctypes.byref(s)) == kv.KV_ESTATE
    assert L.kv_ring_write(ctypes.byref(s), 16, 16, 1, 1, 0, None) == kv.KV_ESTATE
    assert L.kv_ring_delta_rotate(ctypes.byref(s), 3, None) == kv.KV_ESTATE
    assert L.chunk_attention(ctypes.byref(s), 16, 1, 0, 0, None, None, 1.0, 16, None, 0,
                             None) == kv.KV_ESTATE


def test_write_validation_before_launch(L):
    s = _fake_ring()
    r = ctypes.byref(s)
    assert L.kv_ring_write(r, 16, 16, 1, 257, 0, None) == kv.KV_ERANGE   # n > C
    assert L.kv_ring_write(r, 16, 16, 1, 0, 0, None) == kv.KV_ERANGE
    assert L.kv_ring_write(r, 16, 16, 3, 8, 0, None) == kv.KV_EINVAL     # dtype
    assert L.kv_ring_write(r, 16, 16, 1, 8, 4, None) == kv.KV_EINVAL     # flag
    assert L.kv_ring_write(r, 17, 16, 1, 8, 0, None) == kv.KV_EINVAL     # misaligned
    assert L.kv_ring_write(r, None, 16, 1, 8, 0, None) == kv.KV_EINVAL
    s.next_pos = 4090                                                    # past the table
    assert L.kv_ring_write(r, 16, 16, 1, 8, 0, None) == kv.KV_ERANGE
    s.next_pos = 0
    s.pending = 32
    assert L.kv_ring_write(r, 16, 16, 1, 16, 0, None) == kv.KV_ESTATE    # shorter rewrite
    assert s.pending == 32


def test_commit_matches_the_oracle_ring_arithmetic(L, orc):
    s = _fake_ring(C=100)
    o = orc.OracleRing(100, 1, 64)
    for n in (30, 30, 30, 30, 7, 100, 1, 99):
        s.pending = n
        o._s.pending = n
        assert L.kv_ring_commit(ctypes.byref(s)) == kv.KV_OK
        o.commit()
        assert (s.write_slot, s.live, s.pending, s.next_pos) == o.state()
    s.live = 101
    assert L.kv_ring_commit(ctypes.byref(s)) == kv.KV_ESTATE


def test_delta_rotate_host_logic(L):
    s = _fake_ring()
    r = ctypes.byref(s)
    s.next_pos = 500
    assert L.kv_ring_delta_rotate(r, -128, None) == kv.KV_OK           # empty ring: no launch
    assert s.next_pos == 372
    assert L.kv_ring_delta_rotate(r, 2 ** 31, None) == kv.KV_ERANGE
    assert L.kv_ring_delta_rotate(r, -(2 ** 31) - 400, None) == kv.KV_ERANGE
    assert s.next_pos == 372


def test_attention_validation_before_launch(L):
    s = _fake_ring()
    s.live = 64
    r = ctypes.byref(s)
    ok_args = (r, 16, 8, 0, 8, None, None, 0.125, 16, None)
    assert L.chunk_attention(*ok_args[:1], 16, 0, 0, 0, None, None, 0.125, 16, None, 0,
                             None) == kv.KV_OK                            # n_q = 0: no launch
    assert L.chunk_attention(*ok_args, 4, None) == kv.KV_EINVAL           # unknown flag
    assert L.chunk_attention(*ok_args, kv.KV_PV_FP8, None) == kv.KV_EUNSUPPORTED  # e4m3 P, D 64
    assert L.chunk_attention(*ok_args, kv.KV_QK_FP8, None) == kv.KV_EUNSUPPORTED  # mode B, D 64
    assert L.chunk_attention(r, 16, 8, 0, 65, None, None, 0.125, 16, None, 0,
                             None) == kv.KV_ERANGE                        # n_current > valid
    assert L.chunk_attention(r, 16, 8, 4090, 8, None, None, 0.125, 16, None, 0,
                             None) == kv.KV_ERANGE                        # q positions
    assert L.chunk_attention(r, 16, 8, 0, 8, None, None, 0.0, 16, None, 0,
                             None) == kv.KV_EINVAL                        # scale
    bad = kv.kv_cache_bias_t(float("nan"))
    assert L.chunk_attention(r, 16, 8, 0, 8, None, ctypes.byref(bad), 0.125, 16, None, 0,
                             None) == kv.KV_EINVAL
    m = kv.kv_block_mask_t(0, 1, 1, 1)
    assert L.chunk_attention(r, 16, 8, 0, 8, ctypes.byref(m), None, 0.125, 16, None, 0,
                             None) == kv.KV_EINVAL


def test_rows_validation_before_launch(L):
    """chunk_attention_rows refuses bad row lists on the host; an empty list enqueues
    nothing.  No call here reaches a launch except the last, which needs a device."""
    s = _fake_ring(D=128)
    s.live = 64
    r = ctypes.byref(s)

    def call(rows=16, n_rows=4, n_q=8, flags=0, ring=r, splits=1, ws=None, ws_bytes=0):
        return L.chunk_attention_rows(ring, 16, n_q, 0, 8, rows, n_rows, None, None, 0.125, 16,
                                      None, splits, ws, ws_bytes, flags, None)

    need = kv.lib().chunk_attention_workspace_size(4, s.n_heads, 128, 3)
    assert need == 3 * 4 * s.n_heads * (4 * 128 + 8)
    assert call(splits=0) == kv.KV_EINVAL
    assert call(splits=65) == kv.KV_EINVAL
    assert call(splits=3) == kv.KV_EINVAL              # no workspace
    assert call(splits=3, ws=24, ws_bytes=need) == kv.KV_EINVAL      # not 16-byte aligned
    assert call(splits=3, ws=32, ws_bytes=need - 1) == kv.KV_ERANGE
    assert call(n_rows=-1) == kv.KV_EINVAL
    assert call(n_rows=0) == kv.KV_OK                  # nothing to do
    assert call(n_q=0) == kv.KV_OK
    assert call(rows=None) == kv.KV_EINVAL
    assert call(rows=18) == kv.KV_EINVAL               # not 4-byte aligned
    assert call(flags=4) == kv.KV_EINVAL
    s64 = _fake_ring(D=64)
    s64.live = 64
    assert call(ring=ctypes.byref(s64)) == kv.KV_EUNSUPPORTED
    assert call() == kv.KV_ECUDA                       # valid: reaches the device (none here)


def test_content_memory_validation(L):
    main, cand = _fake_ring(D=128), _fake_ring(C=64, D=128)
    main.live, cand.live = 64, 64
    rm, rc = ctypes.byref(main), ctypes.byref(cand)

    def mass(n_q=8, slot_first=0, n_cand=16, scale=0.125, ring=rc, lse=16, m=16):
        return L.chunk_key_mass(rm, ring, 16, n_q, 0, lse, None, scale, slot_first, n_cand, m,
                                None)

    assert mass(n_cand=0) == kv.KV_OK and mass(n_q=0) == kv.KV_OK     # nothing to do
    assert mass(n_cand=65) == kv.KV_EINVAL
    assert mass(slot_first=64) == kv.KV_EINVAL
    assert mass(scale=0.0) == kv.KV_EINVAL
    assert mass(lse=None) == kv.KV_EINVAL and mass(m=18) == kv.KV_EINVAL
    wide = _fake_ring(C=64, H=4, D=128)
    assert mass(ring=ctypes.byref(wide)) == kv.KV_EINVAL
    assert mass() == kv.KV_ECUDA                                        # reaches the device
    out = _fake_ring(C=32, D=128)
    out.k_codes = 0x200000

    def sel(memory=None, n_fifo=16, budget=32, frame=8, gamma=0.5, dst=None, kept=16):
        return L.kv_memory_select(memory, 16, rc, 16, 0, n_fifo, budget, frame, gamma,
                                  ctypes.byref(out) if dst is None else dst, kept, None)

    assert sel(budget=0) == kv.KV_EINVAL and sel(frame=0) == kv.KV_EINVAL
    assert sel(gamma=0.0) == kv.KV_EINVAL and sel(gamma=1.5) == kv.KV_EINVAL
    assert sel(budget=33) == kv.KV_ERANGE                              # memory_out too small
    assert sel(n_fifo=65) == kv.KV_ERANGE
    assert sel(dst=rc) == kv.KV_EINVAL                                 # aliases the FIFO
    assert sel(kept=None) == kv.KV_EINVAL
    assert out.live == 0
    big = _fake_ring(C=8192, D=128)
    big.live = 8192
    assert sel(memory=ctypes.byref(big)) == kv.KV_ERANGE               # > 8,192 candidates


def test_key_mass_multi_validation(L):
    main, c1, c2 = _fake_ring(D=128), _fake_ring(C=64, D=128), _fake_ring(C=32, D=128)
    main.live, c1.live, c2.live = 64, 64, 32
    rm = ctypes.byref(main)

    def multi(rings=(c1, c2), firsts=(0, 0), counts=(16, 8), outs=(16, 32), n_sets=None,
              n_q=8, lse=16, scale=0.125, ws=None, ws_bytes=0):
        n = len(rings) if n_sets is None else n_sets
        k = max(1, len(rings))
        ra = (ctypes.c_void_p * k)(*[None if r is None else ctypes.addressof(r) for r in rings])
        fa = (ctypes.c_int64 * k)(*firsts)
        ca = (ctypes.c_int * k)(*counts)
        oa = (ctypes.c_void_p * k)(*outs)
        return L.chunk_key_mass_multi(rm, n, ra, 16, n_q, 0, lse, None, scale, fa, ca, oa, ws,
                                      ws_bytes, None)

    assert multi(n_sets=0) == kv.KV_EINVAL
    five = (c1,) * 5
    assert multi(rings=five, firsts=(0,) * 5, counts=(1,) * 5, outs=(16,) * 5) == kv.KV_EINVAL
    assert L.chunk_key_mass_multi(rm, 1, None, 16, 8, 0, 16, None, 0.125, None, None, None,
                                  None, 0, None) == kv.KV_EINVAL         # null arrays
    assert multi(rings=(c1, None)) == kv.KV_EINVAL
    wide = _fake_ring(C=64, H=4, D=128)
    assert multi(rings=(c1, wide)) == kv.KV_EINVAL                       # heads differ
    assert multi(counts=(16, 33)) == kv.KV_EINVAL                        # > capacity of set 1
    assert multi(firsts=(0, 32)) == kv.KV_EINVAL
    assert multi(outs=(16, 34)) == kv.KV_EINVAL                          # misaligned mass
    assert multi(outs=(16, None)) == kv.KV_EINVAL
    assert multi(counts=(0, 0)) == kv.KV_OK                              # nothing to score
    assert multi(counts=(0, 8), outs=(None, 32)) == kv.KV_ECUDA          # an empty set's
    assert multi(n_q=0) == kv.KV_OK                                      # mass is not read
    assert multi() == kv.KV_ECUDA                                        # reaches the device
    need = kv.chunk_key_mass_workspace_size(8, 2)
    assert need == 2 * 1 * 16896 and kv.chunk_key_mass_workspace_size(65, 40) == 40 * 2 * 16896
    assert kv.chunk_key_mass_workspace_size(-1, 2) == 0
    assert multi(ws=24, ws_bytes=need) == kv.KV_EINVAL                   # misaligned
    assert multi(ws=256, ws_bytes=need - 16) == kv.KV_ERANGE             # too small
    assert multi(ws=256, ws_bytes=need) == kv.KV_ECUDA
    m64 = _fake_ring(D=64)
    m64.live = 64
    c64 = _fake_ring(C=64, D=64)
    c64.live = 64
    ra = (ctypes.c_void_p * 1)(ctypes.addressof(c64))
    assert L.chunk_key_mass_multi(ctypes.byref(m64), 1, ra, 16, 8, 0, 16, None, 0.125,
                                  (ctypes.c_int64 * 1)(0), (ctypes.c_int * 1)(8),
                                  (ctypes.c_void_p * 1)(16), None, 0, None) == kv.KV_EUNSUPPORTED


def test_split_workspace_size_and_validation(L):
    assert kv.chunk_attention_workspace_size(25, 32, 128, 8) == 8 * 25 * 32 * (4 * 128 + 8)
    assert kv.chunk_attention_workspace_size(25, 32, 128, 0) == 0
    s = _fake_ring(D=128)
    s.live = 64
    r = ctypes.byref(s)
    args = (r, 16, 8, 0, 8, None, None, 0.125, 16, None)
    need = kv.chunk_attention_workspace_size(8, 2, 128, 4)
    assert L.chunk_attention_split(*args, 0, 16, need, 0, None) == kv.KV_EINVAL     # splits
    assert L.chunk_attention_split(*args, 65, 16, need, 0, None) == kv.KV_EINVAL
    assert L.chunk_attention_split(*args, 4, None, need, 0, None) == kv.KV_EINVAL   # workspace
    assert L.chunk_attention_split(*args, 4, 17, need, 0, None) == kv.KV_EINVAL     # misaligned
    assert L.chunk_attention_split(*args, 4, 16, need - 1, 0, None) == kv.KV_ERANGE
    s64 = _fake_ring(D=64)
    s64.live = 64
    assert L.chunk_attention_split(ctypes.byref(s64), 16, 8, 0, 8, None, None, 0.125, 16, None,
                                   4, 16, need, 0, None) in (kv.KV_EUNSUPPORTED, kv.KV_ECUDA)


def _waves_cost(n_q, n_heads, n_keys, n_sms, z):
    """One wave-filling cost, counted CTA by CTA: the SMs take the CTAs in waves of n_sms,
    each CTA costs its key tiles plus a fixed 10."""
    n_cta = -(-n_q // 256) * n_heads * z
    tiles = -(-n_keys // 64)
    waves = 0
    left = n_cta
    while left > 0:
        waves += 1
        left -= n_sms
    return waves * (tiles / z + 10.0)


@pytest.mark.parametrize("n_q,n_heads,n_keys,n_sms", [
    (757, 40, 5788, 148), (4680, 40, 23400, 148), (1152, 32, 24192, 148),
    (1024, 40, 32768, 148), (25, 32, 24192, 148), (189, 40, 5788, 148), (256, 1, 1024, 148),
    (4096, 8, 200000, 132), (1, 1, 100000, 1)])
def test_suggest_splits_minimises_the_wave_cost(n_q, n_heads, n_keys, n_sms):
    z = kv.chunk_attention_suggest_splits(n_q, n_heads, n_keys, n_sms)
    tiles = -(-n_keys // 64)
    z_max = max(1, min(16, tiles // 4))
    assert 1 <= z <= z_max
    costs = {c: _waves_cost(n_q, n_heads, n_keys, n_sms, c) for c in range(1, z_max + 1)}
    best = min(costs.values())
    if best > 0.9 * costs[1]:                       # less than a 10% gain: not split
        assert z == 1
        return
    assert costs[z] <= best * (1 + 1e-12)
    assert all(costs[c] > best * (1 + 1e-12) for c in range(1, z))       # ties: fewest splits


def test_suggest_splits_special_cases():
    # a chunk whose CTAs already fill less than one wave over a short ring is not split
    assert kv.chunk_attention_suggest_splits(757, 40, 5788, 148) == 1
    # 760 CTAs over 366 key tiles: 3 splits would gain about 6%, under the 10% margin
    assert kv.chunk_attention_suggest_splits(4680, 40, 23400, 148) == 1
    # 160 CTAs on 148 SMs (a second wave of 12): split
    assert kv.chunk_attention_suggest_splits(1152, 32, 24192, 148) == 6
    # fewer than 8 key tiles never split; out-of-range arguments give 1
    assert kv.chunk_attention_suggest_splits(1, 1, 448, 148) == 1
    assert kv.chunk_attention_suggest_splits(1, 1, 512, 148) == 2
    for bad in [(0, 1, 100, 148), (1, 0, 100, 148), (1, 1, 0, 148), (1, 1, 100, 0),
                (-5, 1, 100, 148)]:
        assert kv.chunk_attention_suggest_splits(*bad) == 1
    # one query tile, one head, a long ring and a large GPU: the cap of 16 holds
    assert kv.chunk_attention_suggest_splits(1, 1, 10 ** 7, 148) == 16


def test_noalloc_rejects_oversize_before_any_cuda_call(L):
    s = _fake_ring(C=4096, D=128)
    s.live = 2048
    r = ctypes.byref(s)
    assert kv.KV_NOALLOC_SCRATCH_BYTES == 16 << 20
    # 1,024 queries x 2 heads x 128 x 9 splits = 9.6 MB fits; 17 splits (18.1 MB) do not
    assert kv.chunk_attention_workspace_size(1024, 2, 128, 17) > kv.KV_NOALLOC_SCRATCH_BYTES
    assert L.chunk_attention_split_noalloc(r, 16, 1024, 0, 8, None, None, 0.125, 16, None,
                                           17, 0, None) == kv.KV_ERANGE
    assert L.chunk_attention_split_noalloc(r, 16, 1024, 0, 8, None, None, 0.125, 16, None,
                                           0, 0, None) == kv.KV_EINVAL
    assert L.chunk_attention_split_noalloc(r, 16, 0, 0, 8, None, None, 0.125, 16, None,
                                           4, 0, None) == kv.KV_OK          # nothing to do
    # within the limit the call reaches the device (none here)
    assert L.chunk_attention_split_noalloc(r, 16, 1024, 0, 8, None, None, 0.125, 16, None,
                                           9, 0, None) == kv.KV_ECUDA


def test_multi_ring_validation_before_launch(L):
    """chunk_attention_multi refuses bad ring lists, splits and workspaces on the host.
    Every call here is invalid, so none reaches a launch (the rings are fakes)."""
    main, anchor = _fake_ring(D=128), _fake_ring(C=64, D=128)
    main.live, anchor.live = 64, 32
    arr = lambda *rs: (ctypes.c_void_p * len(rs))(*[ctypes.addressof(r) for r in rs])
    need = kv.chunk_attention_workspace_size(8, 2, 128, 2 * 4)

    def call(rings, n_rings, n_current=8, n_splits=4, ws=16, nbytes=need, flags=0):
        return L.chunk_attention_multi(rings, n_rings, 16, 8, 0, n_current, None, None, 0.125,
                                       16, None, n_splits, ws, nbytes, flags, None)

    two = arr(main, anchor)
    assert call(None, 2) == kv.KV_EINVAL
    assert call(two, 0) == kv.KV_EINVAL
    assert call(arr(*([main] * 9)), 9) == kv.KV_EINVAL                  # > KV_MAX_RINGS
    assert call((ctypes.c_void_p * 2)(ctypes.addressof(main), None), 2) == kv.KV_EINVAL
    assert call(two, 2, n_splits=0) == kv.KV_EINVAL
    assert call(two, 2, n_splits=33) == kv.KV_EINVAL                    # 2 x 33 > 64 splits
    assert call(two, 2, ws=None) == kv.KV_EINVAL
    assert call(two, 2, ws=17) == kv.KV_EINVAL                          # misaligned
    assert call(two, 2, nbytes=need - 1) == kv.KV_ERANGE                # sized for 8 splits
    assert call(two, 2, n_current=65) == kv.KV_ERANGE                   # main ring: 64 valid
    assert call(two, 2, flags=4) == kv.KV_EINVAL
    wide = _fake_ring(C=64, H=4, D=128)
    assert call(arr(main, wide), 2) == kv.KV_EINVAL                     # heads differ
    other_base = _fake_ring(C=64, D=128)
    other_base.rope_base = 500000.0
    assert call(arr(main, other_base), 2) == kv.KV_EINVAL
    short_table = _fake_ring(C=64, D=128, pmax=4)
    assert call(arr(main, short_table), 2) == kv.KV_ERANGE              # q positions 0..7
    assert call(arr(main, kv.kv_ring_t()), 2) == kv.KV_ESTATE
    m64, a64 = _fake_ring(D=64), _fake_ring(C=64, D=64)
    m64.live = 64
    assert call(arr(m64, a64), 2) == kv.KV_EUNSUPPORTED
    assert kv.KV_MAX_RINGS == 8
