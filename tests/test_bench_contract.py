"""CPU: the reference arm of bench.py (the oracle on the host cores) prints one
JSON line with the keys the benchmark contract requires, in the same metric,
unit and workload description as the native arm."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    env.pop("RANK", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny_chain64"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ["impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"]:
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == "atom-steps/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["value"] > 0
    assert d["config"]["workload"] == "tiny_chain64" and d["config"]["atoms"] == 64
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "atom-steps/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    import bench
    assert d["metric"] == bench.METRIC


def test_traffic_figure_is_keyed_to_the_kernel_sources(tmp_path, monkeypatch):
    """The DRAM traffic in the roofline object is reported only while the kernel
    sources hash to the value recorded beside the capture; an edit voids it.
    Checked on copies of the sources with a record written for them, so the
    mechanism is tested whether or not the committed capture is current."""
    import hashlib
    import shutil
    import bench
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    h = hashlib.sha256()
    for src in d["sources"]:
        os.makedirs(tmp_path / os.path.dirname(src), exist_ok=True)
        shutil.copy(os.path.join(ROOT, src), tmp_path / src)
        h.update(open(tmp_path / src, "rb").read())
    rec = dict(d, sources_sha256_16=h.hexdigest()[:16])
    os.makedirs(tmp_path / "profiles")
    json.dump(rec, open(tmp_path / "profiles" / "traffic.json", "w"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("k_cfconv_bwd") == d["k_cfconv_bwd"]
    with open(tmp_path / d["sources"][0], "a") as f:
        f.write("\n// edited\n")
    assert bench._traffic("k_cfconv_bwd") is None
    # and the committed record is honoured only if it matches the committed sources
    monkeypatch.setattr(bench, "ROOT", ROOT)
    h = hashlib.sha256()
    for src in d["sources"]:
        h.update(open(os.path.join(ROOT, src), "rb").read())
    current = h.hexdigest()[:16] == d["sources_sha256_16"]
    assert (bench._traffic("k_cfconv_bwd") is not None) == current
