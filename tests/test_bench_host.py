"""The benchmark's arithmetic, checked on the CPU: unmasked-pair counts against a brute
count of the mask, FLOP and byte figures against their closed forms, the traffic
record's source-hash rule, and the reference arm's output line."""
import hashlib
import importlib.util
import json
import os
import subprocess
import sys

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


def test_traffic_record_is_used_only_for_the_source_it_was_taken_on(tmp_path):
    """The committed ncu traffic record is well formed; bench.py reports it only while the
    attention source hash matches (else null), and a matching record is plausible."""
    b = _bench()
    with open(b.TRAFFIC_FILE) as f:
        rec = dict(line.split("=", 1) for line in f.read().split("\n") if "=" in line)
    assert len(rec["source_sha256_16"].strip()) == 16
    assert 60e6 < float(rec["dram_bytes_per_launch"]) < 100e6   # about the 76.6 MB algorithmic
    src = os.path.join(ROOT, "kv_cache_attention_ring_b200", "csrc", "chunk_attn_sm100.cu")
    t = b.traffic_for(src)
    assert t is None or t == float(rec["dram_bytes_per_launch"])
    other = tmp_path / "other.cu"
    other.write_text("// not the captured source\n")
    assert b.traffic_for(str(other)) is None


def _run_bench(env_extra, *args):
    env = dict(os.environ, OMP_NUM_THREADS="4", **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_one_contract_line():
    """The reference arm (the oracle on the host cores) prints exactly one JSON line with
    the contract's keys, on rank 0; other ranks exit 0 without output or work."""
    r = _run_bench({}, "--impl", "reference", "--steps", "1", "--warmup", "0")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "us/call" and d["higher_is_better"] is False
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("runway_chunk_step")
    r1 = _run_bench({"RANK": "1", "WORLD_SIZE": "2"}, "--impl", "reference", "--steps", "1",
                    "--warmup", "0")
    assert r1.returncode == 0 and r1.stdout.strip() == ""


def test_block_mask_pair_counts_match_the_closed_forms():
    """attn_pairs (used for the Wan and other extra configs) equals the token-causal closed
    form, the whole-chunk block count, and the Wan chunk's 102.2 M pairs per head."""
    b = _bench()
    n, C = 757, 5788
    assert b.attn_pairs(n, C - n, 1, 1, 1, 1, n) == b.attn_pairs_token_causal(n, C)
    assert b.attn_pairs(n, C - n, 1 << 30, 1 << 30, 1 << 30, 1 << 30, n) == n * C
    wan = b.attn_pairs(4680, 18720, 1560, 1560, 1560, 1560, 4680)
    assert wan == 4680 * 18720 + 1560 * 1560 * (1 + 2 + 3)
    assert abs(4 * 128 * 40 * wan / 1e12 - 2.093) < 1e-3
    # brute force on a small ragged block mask
    qf, qb, kf, kb, nq, nc = 5, 3, 2, 4, 17, 13
    bid = lambda t, f, l: 0 if t < f else 1 + (t - f) // l
    brute = sum(1 for i in range(nq) for t in range(nc) if bid(t, kf, kb) <= bid(i, qf, qb))
    assert b.attn_pairs(nq, 0, qf, qb, kf, kb, nc) == brute
