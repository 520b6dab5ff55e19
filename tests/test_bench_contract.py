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


def test_fused_work_model_from_the_filter_shape():
    """The roofline's algorithmic work: the filter network K -> F -> F costs 2 (K F + F^2)
    FLOP per evaluation (45,568 for K = 50, F = 128); per step the forward kernel evaluates it
    L E_cut times in the forwards and (L - 1) E_cut / 2 times in the dE/dh launches over the
    complementary list, and the pair kernel forms value and derivative once per unordered pair
    (2 L E_cut / 2 evaluations).  MUFU operations: K Gaussian exponentials per evaluation, per
    feature an exponential and a logarithm for the softplus (a quarter of the exponentials on the
    FMA pipe), and in the pair kernel one more exponential per feature for the logistic."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    K, F, L, E = 50, 128, 3, 1_000_000
    assert b.mufu_per_edge(K, F) == {"fwd": 50 + 256 - 32, "bwd": 50 + 384 - 32}
    work = b.fused_work_per_step(K, F, L, E)
    per_eval = 2 * (50 * 128 + 128 * 128)
    assert per_eval == 45_568
    assert work["k_cfconv_fwd"]["flop_step"] == per_eval * (3 * E + 2 * E / 2)
    assert work["k_cfconv_bwd"]["flop_step"] == per_eval * 2 * 3 * E / 2
    assert work["k_cfconv_fwd"]["mufu_step"] == 274 * (3 * E + 2 * E / 2)
    assert work["k_cfconv_bwd"]["mufu_step"] == 402 * 3 * E / 2
    # one interaction: no dE/dh launch at all
    assert b.fused_work_per_step(K, F, 1, E)["k_cfconv_fwd"]["flop_step"] == per_eval * E
