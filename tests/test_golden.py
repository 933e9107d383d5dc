"""Values printed on the pages (and in the OCP FP8 definition) as fixtures."""
import json
import math
import os

import numpy as np

from kv_cache_attention_ring_b200 import inputs

G = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(G, name)) as f:
        return json.load(f)


def test_runway_workload_matches_the_abstract():
    g = _load("runway_workload.json")
    w = inputs.RUNWAY
    assert w.C == g["cache_slots"] and w.n == g["new_tokens_per_call"]
    assert w.passes == g["denoising_passes_per_chunk"]
    assert w.extra["rings"] * w.passes == g["attention_calls_per_chunk"]
    # the real-time budget printed on the page is four frames at 24 fps
    assert abs(1000 * g["frames_per_chunk"] / g["fps"] - g["budget_ms_per_chunk"]) < 0.05
    # 1.51x and 1.63x are the printed speed-ups
    s = g["step_ms"]
    assert round(s["original"] / s["without_fused_kernel"], 2) == 1.51
    assert round(s["original"] / s["with_fused_kernel"], 2) == 1.63


def test_stream_ltx_block_shape():
    g = _load("stream_ltx_blocks.json")
    assert inputs.AV_VIDEO.n == g["later_block"]["video_frames"] * 384
    assert inputs.AV_VIDEO.extra["first_n"] == g["first_block"]["video_frames"] * 384
    assert inputs.AV_AUDIO.n == g["later_block"]["audio_latents"]
    assert inputs.AV_AUDIO.extra["first_n"] == g["first_block"]["audio_latents"]


def test_e4m3_named_values(orc):
    g = _load("e4m3_named_values.json")
    for code, val in g["values"].items():
        got = orc.e4m3_decode([int(code, 16)])[0]
        assert got == val and math.copysign(1, got) == math.copysign(1, val)
        assert orc.e4m3_encode([val])[0] == int(code, 16)
    for code in g["nan_codes"]:
        assert np.isnan(orc.e4m3_decode([int(code, 16)])[0])
