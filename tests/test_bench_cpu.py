"""bench.py's host-side paths on the CPU (no GPU): the reference arm (the fp64 oracle timed on
this host's cores) prints exactly one JSON line with the fields the contract asks for, and the
algorithmic work per frame counts the keys the page table makes visible."""

import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--config", "0"], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "frames/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["n_gpus"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "frames/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_frame_work_follows_retained_key_count():
    """The key count per frame bench.py divides by matches what the oracle's page table makes
    visible (patch pages x patches + special tokens), frame by frame."""
    import bench
    from oracle import retention
    from rope_paged_kv_02_b200 import workloads
    for cid in (1, 2):                               # every frame a keyframe; every 5th
        cfg = workloads.CONFIGS[cid]
        flops, nbytes, keys = bench.frame_work(cfg)
        r = retention.PagedRetention(cfg.scale_frames, cfg.sliding_window, cfg.n_keyframes)
        for f, key in enumerate(cfg.keyframes):
            r.append(f, key)
            vis = r.visible()
            nk = len(vis.patch_pages) * cfg.patches + vis.n_special
            r.finish()
            assert keys[f] == nk
            assert flops[f] == 4.0 * cfg.tokens * nk * cfg.heads * cfg.head_dim
        assert np.all(nbytes == 6.0 * cfg.tokens * cfg.heads * cfg.head_dim * 2)


@pytest.mark.parametrize("content,expect", [
    ('{"hbm_gbs": 7000, "bf16_tflops": 1600, "bf16_tflops_sustained": 1380}',
     (7000.0, 1600.0, 1380.0, "measured")),
    ('{"hbm_gbs": {"value": 7100}, "bf16_tflops": {"median": 1610}}',
     (7100.0, 1610.0, 1610.0, "measured")),
    ('{"gpu0": {"hbm_gbs": 7050, "bf16_tflops": 1620, "bf16_tflops_sustained": 1390}}',
     (7050.0, 1620.0, 1390.0, "measured")),
    ('{"hbm_gbs": 7000}', (7000.0, 1590.0, 1400.0, "measured (fallback for bf16_tflops)")),
    ("not json", (6650.0, 1590.0, 1400.0, "fallback (MEASURED_PEAKS.json unreadable")),
])
def test_peaks_file_shapes(tmp_path, content, expect):
    """The roofline denominators are read from the peaks file whatever its nesting; a figure
    it lacks, or an unreadable file, falls back to the recipe's figures and says so."""
    import bench
    p = tmp_path / "MEASURED_PEAKS.json"
    p.write_text(content)
    got = bench._peaks(str(p))
    assert (got["hbm_gbs"], got["bf16_tflops"], got["bf16_tflops_sustained"]) == expect[:3]
    assert got["source"].startswith(expect[3])


def test_peaks_fallback_without_file(tmp_path):
    import bench
    got = bench._peaks(str(tmp_path / "absent.json"))
    assert got["source"] == "fallback" and got["hbm_gbs"] == 6650.0
