"""bench.py's reference arm on the CPU: the oracle timed on a bounded sample of a
statement prints one JSON line with the contract's keys; the MoE layer's sample is
made of the layer's own sites."""

import json
import subprocess
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parent.parent


def test_reference_arm_prints_one_line():
    out = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1", "--config", "1"], cwd=ROOT, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["nproc"] >= 1 and "cpu_model" in d["cpu_baseline"]


def test_moe_sample_is_sites_of_the_layer():
    sys.path.insert(0, str(ROOT))
    import bench
    import workloads
    wl, label = bench.cpu_sample(5, 0, 3)
    assert [s.name for s in wl.sites] == ["e3.gate", "e3.up", "e3.down"] and "expert 3" in label
    # the same tensors as in a layer built with more experts (each expert's draws have their own seeds)
    wide = workloads.build(5, 0, experts=[2, 3, 4], shared=False)
    for a, b in zip(wl.sites, [s for s in wide.sites if s.name.startswith("e3.")]):
        assert a.name == b.name and (a.w == b.w).all() and (a.xt == b.xt).all()
