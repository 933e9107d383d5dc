"""The fast e4m3 P.V mode (KV_PV_FP8): P (times the key's V scale) rounded to e4m3 and
P.V run on the raw V codes.  Its error against the oracle is measured and printed on the
Runway chunk shape ("KREA Real-Time 14B / video-conductor", "What didn't": FP8 by default
cost quality, so the cost is reported, not hidden).  It is not held to the acceptance
tolerance, only to a loose bound that catches a broken kernel.  A partial ring whose
invalid slots hold NaN codes checks that stale memory never reaches the e4m3 MMA."""
import numpy as np
import pytest
import torch

import kv_cache_attention_ring_b200 as kv
from kv_cache_attention_ring_b200 import inputs
from helpers import LSE_ATOL, sample_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_attention_ring_b200 import build
    build.build()
    kv.lib()


def _errors(out, lse, ro, rl, rows):
    torch.cuda.synchronize()
    o = out.float().cpu().numpy().astype(np.float64)[rows]
    l = lse.cpu().numpy().astype(np.float64)[:, rows]
    assert np.isfinite(o).all()
    rel = np.linalg.norm(o - ro) / np.linalg.norm(ro)
    return float(np.abs(o - ro).max()), float(rel), float(np.abs(l - rl).max())


def test_pv_fp8_error_on_the_runway_chunk(orc):
    from test_gpu_attention import _runway_ring
    w = inputs.RUNWAY
    ring, o, q = _runway_ring(orc)
    rows = sample_rows(w.n, 128, seed=9)
    ro, rl = o.attention(inputs.as_f32(q), o.next_pos, w.n, (1, 1, 1, 1), 0.0, rows=rows)
    report = {}
    for name, kw in (("mode A", {}), ("e4m3 P.V", {"pv_fp8": True}),
                     ("mode B + e4m3 P.V", {"pv_fp8": True, "mode_b": True})):
        out, lse = kv.chunk_attention(ring, to_dev(q), ring.next_pos, w.n, (1, 1, 1, 1), 0.0,
                                      **kw)
        report[name] = _errors(out, lse, ro, rl, rows)
    for name, (e, r, le) in report.items():
        print(f"{name:18s}: max-abs {e:.3e}  rel-L2 {r:.3e}  lse {le:.2e}")
    e, r, le = report["e4m3 P.V"]
    assert r < 5e-2 and e < 0.5                     # broken kernels land far above
    assert le <= LSE_ATOL                           # the row sums stay exact (fp32)
    assert r > report["mode A"][1]                  # it is the less exact mode


def test_pv_fp8_split_and_stale_nan_codes_in_invalid_slots(orc):
    C, H = 1500, 4
    ring = kv.KvRing(C, H, 128, 0, 8000)
    ring.k_codes.fill_(0x7F)                        # NaN codes everywhere before any write
    ring.v_codes.fill_(0x7F)
    ring.k_scale.fill_(float("nan"))
    ring.v_scale.fill_(float("nan"))
    o = orc.OracleRing(C, H, 128)
    ring.s.write_slot = o._s.write_slot = 1200
    for i, n in enumerate((400, 333)):              # a partial ring that wraps
        k = inputs.draw(inputs.seed_of(91, i, 1), (n, H, 128), "normal", 0.09, "bf16")
        v = inputs.draw(inputs.seed_of(91, i, 2), (n, H, 128), "normal", 1.0, "bf16")
        kv.kv_ring_write(ring, to_dev(k), to_dev(v), commit=(i == 0))
        o.write(inputs.as_f32(k), inputs.as_f32(v), commit=(i == 0))
    q = inputs.draw(inputs.seed_of(91, 9, 3), (333, H, 128), "normal", 1.0, "bf16")
    rows = np.arange(333)
    ro, rl = o.attention(inputs.as_f32(q), o.next_pos, 333, (1, 1, 1, 1), -0.5)
    out, lse = kv.chunk_attention(ring, to_dev(q), ring.next_pos, 333, (1, 1, 1, 1), -0.5,
                                  pv_fp8=True)
    e1, r1, l1 = _errors(out, lse, ro, rl, rows)
    ws = torch.empty(kv.chunk_attention_workspace_size(333, H, 128, 5), dtype=torch.uint8,
                     device="cuda")
    out5, lse5 = kv.chunk_attention_split(ring, to_dev(q), ring.next_pos, 333, 5, ws,
                                          mask=(1, 1, 1, 1), cache_bias=-0.5, pv_fp8=True)
    e5, r5, l5 = _errors(out5, lse5, ro, rl, rows)
    print(f"partial ring e4m3 P.V: rel-L2 {r1:.3e} (unsplit), {r5:.3e} (5 splits)")
    assert r1 < 5e-2 and r5 < 5e-2 and l1 <= LSE_ATOL and l5 <= LSE_ATOL
    assert kv.kv_wait_timeout_count() == 0
