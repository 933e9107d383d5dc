"""The path shards across processes with no exchange: heads of a ring are independent.
Two gloo ranks on CPU each run the oracle on their own head shard; the concatenation
equals the single-process result bit for bit, and the timing reduction takes the max."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from kv_cache_attention_ring_b200 import multirank

C, H, D, N = 96, 5, 32, 16


def _stream(orc, heads):
    """A small stream on the given heads: 5 committed chunks, a pending one, a reset."""
    rng = np.random.default_rng(123)
    k_all = [rng.standard_normal((N, H, D)).astype(np.float32) for _ in range(7)]
    v_all = [rng.standard_normal((N, H, D)).astype(np.float32) for _ in range(7)]
    q = rng.standard_normal((N, H, D)).astype(np.float32)
    o = orc.OracleRing(C, len(heads), D)
    for i in range(5):
        o.write(k_all[i][:, heads], v_all[i][:, heads], commit=True)
    o.delta_rotate(-7)
    o.write(k_all[5][:, heads], v_all[5][:, heads])
    out, lse = o.attention(q[:, heads], o.next_pos, N, (4, 4, 4, 4), -1.5)
    return o.kc.copy(), o.ks.copy(), out, lse


def _worker(rank, world, port, result_dir):
    import torch.distributed as dist
    from oracle import oracle as orc
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    heads = list(multirank.shard(H, rank, world))
    kc, ks, out, lse = _stream(orc, heads)
    np.savez(os.path.join(result_dir, f"r{rank}.npz"), heads=heads, kc=kc, ks=ks, out=out, lse=lse)
    t = multirank.max_over_ranks(float(rank + 1))
    assert t == float(world)
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_tiles_exactly():
    for n in (0, 1, 5, 40, 757):
        for w in (1, 2, 3, 8):
            parts = [multirank.shard(n, r, w) for r in range(w)]
            assert [i for p in parts for i in p] == list(range(n))
            assert max(map(len, parts)) - min(map(len, parts)) <= 1
    with pytest.raises(ValueError):
        multirank.shard(4, 2, 2)


def test_two_gloo_ranks_head_shards_match_single_process(orc, tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    kc, ks, out, lse = _stream(orc, list(range(H)))
    got = [np.load(tmp_path / f"r{r}.npz") for r in range(world)]
    heads = np.concatenate([g["heads"] for g in got])
    assert (heads == np.arange(H)).all()
    assert (np.concatenate([g["kc"] for g in got]) == kc).all()
    assert (np.concatenate([g["ks"] for g in got]).view(np.uint32) == ks.view(np.uint32)).all()
    assert (np.concatenate([g["out"] for g in got], axis=1) == out).all()
    assert (np.concatenate([g["lse"] for g in got], axis=0) == lse).all()
