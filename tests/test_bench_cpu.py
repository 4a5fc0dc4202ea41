"""bench.py's host-side contract, without a GPU: the reference arm's JSON line, its
behaviour on ranks other than 0, the CPU baseline's fallback, and the rule that the
committed ncu traffic figure is used only while the kernel sources are unchanged."""
import json
import os
import subprocess
import sys

import bench
import dsgen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, *args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, env=env, timeout=300, cwd=ROOT)


def test_reference_arm_prints_one_contract_line():
    p = _run({}, "--impl", "reference", "--steps", "1", "--warmup", "0", "--cpu-seconds", "1")
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 0
    assert d["config"]["workload"] == "llama2-7b-B8-H32-T4K"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == os.cpu_count() and cb["value"] == d["value"]
    assert "C++" in cb["sample"] and "std::thread" in cb["sample"]
    # the same configuration as the GPU arm reports
    assert d["config"]["path"] == "step" and "l2" in d["config"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_without_work():
    p = _run({"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"}, "--impl", "reference",
             "--steps", "1", "--warmup", "0", "--cpu-seconds", "1")
    assert p.returncode == 0 and p.stdout.strip() == ""


def test_cpu_baseline_falls_back_to_the_numpy_oracle(monkeypatch):
    import oracle.cxx

    def no_compiler(force=False):
        raise OSError("no C++ compiler")

    monkeypatch.setattr(oracle.cxx, "build", no_compiler)
    r = bench.time_oracle(dsgen.workload("tiny-B1-H4-T1K"), 0.2)
    assert r["kind"] == "oracle" and r["value"] > 0 and "numpy" in r["sample"]


def test_traffic_profile_used_only_for_the_profiled_sources(tmp_path, monkeypatch):
    f = tmp_path / "traffic.txt"
    f.write_text("# comment: not a value\n"
                 f"kernel_source_hash: {bench.kernel_source_hash()}\n"
                 "dram_bytes_per_launch[k_step]: 12345\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(f))
    assert bench.profiled_traffic("k_step") == 12345.0
    assert bench.profiled_traffic("k_attend") is None
    f.write_text("kernel_source_hash: 0000000000000000\n"
                 "dram_bytes_per_launch[k_step]: 12345\n")
    assert bench.profiled_traffic("k_step") is None
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(tmp_path / "missing.txt"))
    assert bench.profiled_traffic("k_step") is None


def test_cpu_baseline_bounded_sample_on_every_core():
    """A workload too large for the byte budget is timed on a seeded sample of its
    heads, every host core running the C++ oracle; the dense oracle beside it."""
    w = dsgen.workload("sweep-B32-H32-T32K-r8-k512")
    per_head = w.T * w.d * 2 * 2 + w.T * w.r * 2
    r = bench.time_oracle(w, 0.5, with_dense=True, max_bytes=3 * per_head)
    assert "over 3 of the 1024 heads" in r["sample"] and r["value"] > 0
    assert r["us_per_step"] > 0 and r["cores"] == os.cpu_count()
    assert r["dense_us_per_step"] > 0 and r["dense_gbs"] > 0


def test_committed_profiles_are_consistent():
    """The committed summaries parse, name the commands that made them, and agree with
    the algorithmic bytes bench.py reports for the same kernel and workload."""
    prof = os.path.join(ROOT, "profiles")
    w = dsgen.workload(bench.HEADLINE)
    ks = open(os.path.join(prof, f"k_step_{w.name}.txt")).read()
    assert "ncu --set full --clock-control none" in ks
    kv = dict(l.split(":", 1) for l in ks.splitlines() if ":" in l and not l.startswith("#"))
    alg = int(kv["algorithmic_bytes_per_launch"].split()[0])
    assert alg == bench.stage_bytes(w)["decode_step"]
    total = float(kv["dram_bytes_total"])
    assert 0.9 < total / alg < 1.2  # no large re-reads
    tr = open(os.path.join(prof, f"traffic_{w.name}.txt")).read()
    assert f"dram_bytes_per_launch[k_step]: {total:.0f}" in tr
    ls = open(os.path.join(prof, f"launches_{w.name}.txt")).read()
    assert "--clock-control none" in ls and "ds::k_step" in ls
