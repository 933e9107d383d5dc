"""The benchmark's arithmetic, checked on the CPU: unmasked-pair counts against a brute
count of the mask, FLOP and byte figures against their closed forms, and the traffic
record's source-hash rule."""
import hashlib
import importlib.util
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_token_causal_pairs_match_a_brute_count():
    b = _bench()
    for n_new, C in ((1, 1), (5, 9), (32, 256), (100, 100), (757, 5788)):
        # query i (of the new chunk) sees all C - n_new history slots and new tokens 0..i
        brute = sum((C - n_new) + (i + 1) for i in range(n_new))
        assert b.attn_pairs_token_causal(n_new, C) == brute


def test_runway_flops_and_bytes_closed_forms():
    b = _bench()
    pairs = b.attn_pairs_token_causal(757, 5788)
    flop = 4 * 128 * pairs * 40
    assert abs(flop / 1e9 - 83.8731776) < 1e-9            # 83.87 GFLOP per call
    assert b.write_bytes(757, 40, 128) == 757 * 40 * 776   # 776 B per (token, head), bf16
    assert b.write_bytes(757, 40, 128, in_bytes=4) == 757 * 40 * (2 * 128 * 4 + 2 * 128 + 8)
    assert b.rotate_bytes(32768, 40, 128) == 32768 * 40 * 264   # 264 B per (slot, head)


def test_traffic_record_follows_the_source_hash(tmp_path, monkeypatch):
    b = _bench()
    src = tmp_path / "k.cu"
    src.write_bytes(b"kernel v1")
    rec = tmp_path / "traffic.txt"
    h = hashlib.sha256(b"kernel v1").hexdigest()[:16]
    rec.write_text(f"# comment\nsource_sha256_16={h}\ndram_bytes_per_launch=123\n")
    monkeypatch.setattr(b, "TRAFFIC_FILE", str(rec))
    assert b.traffic_for(str(src)) == 123.0
    src.write_bytes(b"kernel v2")                          # kernel changed: no traffic
    assert b.traffic_for(str(src)) is None


def test_committed_traffic_record_matches_the_attention_source():
    b = _bench()
    src = os.path.join(ROOT, "kv_cache_attention_ring_b200", "csrc", "chunk_attn_sm100.cu")
    t = b.traffic_for(src)
    assert t is not None and 60e6 < t < 100e6              # about the 76.6 MB algorithmic
