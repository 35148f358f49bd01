"""bench.py's JSON line (CPU): the reference arm on a tiny workload, and the
host-side helpers the GPU arm uses. The GPU arm itself runs on a B200 only."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
             "vs_baseline", "dtype", "data", "config"}


def test_reference_arm_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "c1", "--steps", "2",
                          "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert BASE_KEYS <= set(d), BASE_KEYS - set(d)
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["metric"] == bench.METRIC
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0
    assert "workload" in d["config"]


@pytest.mark.parametrize("world", [1, 2, 3, 8])
@pytest.mark.parametrize("batch", [1, 2, 7, 16])
def test_rank_batch_slices_cover_the_batch(world, batch):
    spans = [bench.rank_batch_slice(batch, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == batch
    for (a, b), (c, _) in zip(spans, spans[1:]):
        assert b == c
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_kernel_source_hash_ignores_comments():
    text = "int a; // one\n/* two */ int b;\n"
    assert bench._code_only(text) == bench._code_only("int a;\n  int b;  // three\n")
    assert bench._code_only(text) != bench._code_only("int a; int c;")
    for k in bench.KERNEL_SOURCES:
        h = bench.kernel_source_hash(k)
        assert len(h) == 16 and int(h, 16) >= 0


def test_traffic_entries_name_known_kernels():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        tr = json.load(f)
    assert set(k for k in tr if k != "about") == {"fa_bwd", "fa_fwd_kernel", "fa_fwd_kernel_e4m3"}
    assert sum(tr["fa_bwd"]["parts"].values()) == tr["fa_bwd"]["bytes_per_launch"]
    for k, ent in tr.items():
        if k != "about":
            assert ent["bytes_per_launch"] > 0 and len(ent["source_hash"]) == 16
