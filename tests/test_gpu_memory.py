"""Content memory on the GPU ("Stream LTX", Inference: anchor + content memory + FIFO of
recent blocks; keys scored on attention quality and temporal diversity, evicted down to a
top-M budget).  A stream of chunks runs through a FIFO ring with a persistent anchor and a
double-buffered memory ring; at every eviction the block the next write overwrites and
the memory's keys are scored (chunk_key_mass) and the best M kept (kv_memory_select).
Checked against the oracle: masses within tolerance, the kept set exactly (the oracle's
rule applied to the GPU's binary32 masses, so both take the decision in the same
precision), the new memory ring bit for bit, and attention over the three rings."""
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


def _copy_kept(orc_dst, kept, n_mem, srcs):
    """Oracle side of the gather: kept candidate r goes to slot r of orc_dst."""
    mem, mem_first, fifo, fifo_first = srcs
    for r, idx in enumerate(kept):
        if idx < n_mem:
            src, slot = mem, (mem_first + idx) % mem.C
        else:
            src, slot = fifo, (fifo_first + idx - n_mem) % fifo.C
        orc_dst.kc[:, r], orc_dst.vc[:, r] = src.kc[:, slot], src.vc[:, slot]
        orc_dst.ks[:, r], orc_dst.vs[:, r] = src.ks[:, slot], src.vs[:, slot]
        orc_dst.slot_pos[r] = src.slot_pos[slot]
    orc_dst._s.write_slot = len(kept) % orc_dst.C
    orc_dst._s.live = len(kept)
    orc_dst._s.pending = 0


def test_fifo_anchor_memory_stream(orc):
    H, D, n, C_fifo, M, frame_len = 4, 128, 96, 384, 160, 48      # 2 frames per chunk
    fifo = kv.KvRing(C_fifo, H, D, 0, 8192)
    anchor = kv.KvRing(n, H, D, 0, 8192, rope_table=fifo.rope_table)
    mems = [kv.KvRing(M, H, D, 0, 8192, rope_table=fifo.rope_table) for _ in range(2)]
    o_fifo, o_anchor = orc.OracleRing(C_fifo, H, D), orc.OracleRing(n, H, D)
    o_mems = [orc.OracleRing(M, H, D) for _ in range(2)]
    cur = 0
    events = 0
    for ch in range(11):
        q, k, v = (inputs.draw(inputs.seed_of(51, ch, t), (n, H, D), "normal", s, "bf16")
                   for t, s in ((1, 1.0), (2, 0.09), (3, 1.0)))
        if ch == 0:                                  # the first chunk is also the anchor
            kv.kv_ring_write(anchor, to_dev(k), to_dev(v), commit=True)
            o_anchor.write(inputs.as_f32(k), inputs.as_f32(v), commit=True)
        kv.kv_ring_write(fifo, to_dev(k), to_dev(v))
        o_fifo.write(inputs.as_f32(k), inputs.as_f32(v))
        rings = [fifo, anchor] + ([mems[cur]] if mems[cur].n_valid else [])
        o_rings = [o_anchor] + ([o_mems[cur]] if o_mems[cur].live else [])
        ws = torch.empty(kv.chunk_attention_workspace_size(n, H, D, 2 * len(rings)),
                         dtype=torch.uint8, device="cuda")
        qd = to_dev(q)
        out, lse = kv.chunk_attention_multi(rings, qd, fifo.next_pos, n, 2, ws,
                                            mask=(frame_len,) * 4, cache_bias=-0.25)
        ro, rl = orc.attention_multi(o_fifo, o_rings, inputs.as_f32(q), o_fifo.next_pos, n,
                                     (frame_len,) * 4, -0.25)
        assert_attention_close(out, lse, ro, rl, what=f"three rings, chunk {ch}")
        if fifo.s.live + n >= C_fifo:
            # eviction: the next write overwrites the block after this chunk
            first = (fifo.s.write_slot + n) % C_fifo
            mf = kv.chunk_key_mass(fifo, fifo, qd, fifo.next_pos, lse, first, n,
                                   cache_bias=-0.25)
            mem, o_mem = mems[cur], o_mems[cur]
            n_mem = mem.n_valid
            mem_first = (mem.s.write_slot + mem.s.pending - n_mem) % M
            mm = (kv.chunk_key_mass(fifo, mem, qd, fifo.next_pos, lse, mem_first, n_mem,
                                    cache_bias=-0.25) if n_mem else None)
            # the same two sets in one launch: bit for bit the separate calls
            # (and with the workspace: queries split once, streamed into the scoring CTAs)
            if n_mem:
                both = kv.chunk_key_mass_multi(fifo, [fifo, mem], qd, fifo.next_pos, lse,
                                               [first, mem_first], [n, n_mem], cache_bias=-0.25)
                assert torch.equal(both[0], mf) and torch.equal(both[1], mm)
                wsm = torch.empty(kv.chunk_key_mass_workspace_size(n, H), dtype=torch.uint8,
                                  device="cuda")
                piped = kv.chunk_key_mass_multi(fifo, [fifo, mem], qd, fifo.next_pos, lse,
                                                [first, mem_first], [n, n_mem],
                                                cache_bias=-0.25, workspace=wsm)
                assert torch.equal(piped[0], mf) and torch.equal(piped[1], mm)
            torch.cuda.synchronize()
            # masses against the oracle's definition (ages of the scored slots)
            newest = (o_fifo.write_slot + o_fifo.pending - 1) % C_fifo
            ages = [(newest - (first + c)) % C_fifo for c in range(n)]
            want = orc.key_mass(o_fifo, o_rings, inputs.as_f32(q), o_fifo.next_pos, n, 0, ages,
                                (frame_len,) * 4, -0.25)
            got = mf.double().sum(0).cpu().numpy()
            assert np.abs(got - want).max() <= 1e-3 * want.max() + 1e-6
            if n_mem:
                newest_m = (o_mem.write_slot + o_mem.pending - 1) % M
                ages_m = [(newest_m - (mem_first + c)) % M for c in range(n_mem)]
                want_m = orc.key_mass(o_fifo, o_rings, inputs.as_f32(q), o_fifo.next_pos, n,
                                      len(o_rings), ages_m, (frame_len,) * 4, -0.25)
                got_m = mm.double().sum(0).cpu().numpy()
                assert np.abs(got_m - want_m).max() <= 1e-3 * want_m.max() + 1e-6
            # selection: the oracle's rule on the GPU's binary32 qualities
            dst, o_dst = mems[1 - cur], o_mems[1 - cur]
            kept = kv.kv_memory_select(mem if n_mem else None, mm, fifo, mf, first, n, M,
                                       frame_len, dst)
            torch.cuda.synchronize()
            qual = []
            for m_t, cnt in ((mm, n_mem), (mf, n)):
                if cnt:
                    acc = np.zeros(cnt, np.float32)
                    for h in range(H):                          # heads in order, binary32
                        acc = acc + m_t[h].cpu().numpy()
                    qual.append(acc)
            qual = np.concatenate(qual).astype(np.float64)
            pos = np.concatenate([o_mem.slot_pos[(mem_first + np.arange(n_mem)) % M],
                                  o_fifo.slot_pos[(first + np.arange(n)) % C_fifo]]).astype(np.int64)
            want_kept = orc.memory_select(qual, np.floor_divide(pos, frame_len), pos, M, 0.5)
            assert kept.cpu().numpy().tolist() == want_kept.tolist()
            _copy_kept(o_dst, want_kept, n_mem, (o_mem, mem_first, o_fifo, first))
            assert dst.state()[:3] == o_dst.state()[:3]
            m_live = len(want_kept)
            for name in ("k_codes", "v_codes"):
                a = getattr(dst, name)[:, :m_live].cpu().numpy()
                b = (o_dst.kc if name == "k_codes" else o_dst.vc)[:, :m_live]
                assert (a == b).all(), name
            assert (dst.k_scale[:, :m_live].cpu().numpy().view(np.uint32)
                    == o_dst.ks[:, :m_live].view(np.uint32)).all()
            assert (dst.slot_pos[:m_live].cpu().numpy() == o_dst.slot_pos[:m_live]).all()
            cur = 1 - cur
            events += 1
        kv.kv_ring_commit(fifo)
        o_fifo.commit()
    assert events >= 5
    assert kv.kv_wait_timeout_count() == 0


def test_key_mass_multi_sets_match_single_calls():
    """Four sets in one launch (several CTAs each, a range that wraps the ring's end, an
    empty set, a second ring): every set's masses equal its own chunk_key_mass call, with
    and without the workspace (300 queries: four whole 64-row tiles and a ragged one)."""
    H, D, C, n = 4, 128, 1500, 300
    ring = kv.KvRing(C, H, D, 0, 1 << 14)
    other = kv.KvRing(700, H, D, 0, 1 << 14, rope_table=ring.rope_table)
    for ch in range(6):
        k, v = (inputs.draw(inputs.seed_of(57, ch, t), (n, H, D), "normal", 1.0, "bf16")
                for t in (1, 2))
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=True)
        if ch < 2:
            kv.kv_ring_write(other, to_dev(k), to_dev(v), commit=True)
    q = to_dev(inputs.draw(inputs.seed_of(57, 9, 3), (n, H, D), "normal", 1.0, "bf16"))
    k, v = (to_dev(inputs.draw(inputs.seed_of(57, 9, t), (n, H, D), "normal", 1.0, "bf16"))
            for t in (1, 2))
    kv.kv_ring_write(ring, k, v)
    _, lse = kv.chunk_attention(ring, q, ring.next_pos, n, None, -0.5)
    # history: the pending chunk is slots 300 .. 599; 1,300 .. 299 wraps the end
    sets = [(ring, 600, 700), (ring, 1300, 500), (ring, 0, 0), (other, 50, 550)]
    multi = kv.chunk_key_mass_multi(ring, [r for r, _, _ in sets], q, ring.next_pos, lse,
                                    [f for _, f, _ in sets], [c for _, _, c in sets],
                                    cache_bias=-0.5)
    ws = torch.empty(kv.chunk_key_mass_workspace_size(n, H), dtype=torch.uint8, device="cuda")
    piped = kv.chunk_key_mass_multi(ring, [r for r, _, _ in sets], q, ring.next_pos, lse,
                                    [f for _, f, _ in sets], [c for _, _, c in sets],
                                    cache_bias=-0.5, workspace=ws)
    for (r, f, c), m, p in zip(sets, multi, piped):
        if c == 0:
            continue
        one = kv.chunk_key_mass(ring, r, q, ring.next_pos, lse, f, c, cache_bias=-0.5)
        torch.cuda.synchronize()
        assert torch.isfinite(one).all()
        assert torch.equal(one, m), (f, c)
        assert torch.equal(one, p), (f, c, (one - p).abs().max().item())


def _select_case(orc, H, C_mem, n_mem_fill, C_fifo, n_fifo, M, frame_len, masses, positions,
                 seed):
    """One kv_memory_select call on engineered masses and slot positions; the kept list
    must equal the oracle's rule applied to the GPU's binary32 qualities."""
    D = 128
    fifo = kv.KvRing(C_fifo, H, D, -(1 << 20), 1 << 20)
    mem = kv.KvRing(C_mem, H, D, -(1 << 20), 1 << 20, rope_table=fifo.rope_table) if C_mem else None
    for ring, fill in ((mem, n_mem_fill), (fifo, C_fifo)):
        if ring is None:
            continue
        done = 0
        while done < fill:
            n = min(256, fill - done)
            k, v = (inputs.draw(inputs.seed_of(seed, done, t), (n, H, D), "normal", 1.0, "bf16")
                    for t in (1, 2))
            kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=True)
            done += n
    n_mem = mem.n_valid if mem is not None else 0
    mem_first = (mem.s.write_slot + mem.s.pending - n_mem) % C_mem if mem is not None else 0
    first = (fifo.s.write_slot + 7) % C_fifo
    n = n_mem + n_fifo
    pos_mem, pos_fifo = positions[:n_mem], positions[n_mem:n]
    if mem is not None:
        mem.slot_pos[(mem_first + torch.arange(n_mem)) % C_mem] = torch.as_tensor(
            pos_mem, dtype=torch.int32, device="cuda")
    fifo.slot_pos[(first + torch.arange(n_fifo)) % C_fifo] = torch.as_tensor(
        pos_fifo, dtype=torch.int32, device="cuda")
    mm = torch.as_tensor(masses[:, :n_mem], dtype=torch.float32, device="cuda").contiguous()
    mf = torch.as_tensor(masses[:, n_mem:n], dtype=torch.float32, device="cuda").contiguous()
    dst = kv.KvRing(max(M, 1), H, D, -(1 << 20), 1 << 20, rope_table=fifo.rope_table)
    kept = kv.kv_memory_select(mem, mm if n_mem else None, fifo, mf, first, n_fifo, M,
                               frame_len, dst)
    torch.cuda.synchronize()
    qual = np.zeros(n, np.float32)
    for h in range(H):                                   # heads in order, binary32
        qual = qual + masses[h, :n].astype(np.float32)
    pos = np.asarray(positions[:n], np.int64)
    want = orc.memory_select(qual.astype(np.float64), np.floor_divide(pos, frame_len), pos, M,
                             0.5)
    assert kept.cpu().numpy().tolist() == want.tolist()
    assert dst.n_valid == len(want)


@pytest.mark.parametrize("case", ["ties_max", "all_kept", "one_kept", "zeros", "fifo_only"])
def test_memory_select_ties_and_edges(orc, case):
    """Selection on engineered candidates: qualities from a few small integers (most
    scores tie, so position and then index decide), repeated and negative positions, the
    largest candidate count (8,192), budgets of all and of one, all-zero masses, and no
    memory ring."""
    rng = np.random.default_rng(71)
    H = 2
    if case == "fifo_only":
        C_mem, n_mem_fill, C_fifo, n_fifo, M = 0, 0, 300, 5, 3
    else:
        C_mem, n_mem_fill, C_fifo, n_fifo = 3000, 3000, 5200, 5192
        M = {"ties_max": 4000, "all_kept": 8192, "one_kept": 1, "zeros": 100}[case]
    n = n_mem_fill + n_fifo
    masses = rng.integers(0, 4, size=(H, n)).astype(np.float32) * 0.25
    if case == "zeros":
        masses[:] = 0.0
    # spread positions, plus about 50 candidates at one position (one deep frame: ranks up
    # to ~55, so quality * 2^-rank stays a normal binary32, as exact as the oracle's fp64)
    positions = rng.integers(-200000, 200000, size=n)
    positions[::160] = positions[0]
    _select_case(orc, H, C_mem, n_mem_fill, C_fifo, n_fifo, M, 64, masses, positions, 72)
