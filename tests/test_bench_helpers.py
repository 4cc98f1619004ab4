"""Host helpers of bench.py: the kernel-source hash that keys the committed DRAM
captures, and the lookup of those captures."""
import os

import bench


def test_code_tokens_ignore_comments_and_layout():
    a = "int f(int x) {  // the doubling\n  return 2 * x; /* twice */ }\n"
    b = "int f(int x) {\n\n    return 2 * x;\n}"
    assert bench._code_tokens(a) == bench._code_tokens(b)
    assert bench._code_tokens(a) != bench._code_tokens(a.replace("2 *", "3 *"))


def test_code_tokens_keep_string_literals():
    src = 'asm volatile("ld.shared // not a comment /* nor this */ [%0];" ::"r"(a)); // gone'
    t = bench._code_tokens(src)
    assert "// not a comment /* nor this */" in t and "gone" not in t
    assert bench._code_tokens('s = "a\\"//b"; x') == 's = "a\\"//b"; x'


def test_source_hash_is_stable_and_tracks_code(tmp_path, monkeypatch):
    csrc = tmp_path / "adapter_pregate_router_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("__global__ void k() { }\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    (csrc / "k.cu").write_text("// a comment\n__global__ void k()\n{\n}\n")
    assert bench.kernel_source_hash() == h0
    (csrc / "k.cu").write_text("__global__ void k() { int a; }\n")
    assert bench.kernel_source_hash() != h0


def test_measured_traffic_needs_the_matching_hash(tmp_path, monkeypatch):
    csrc = tmp_path / "adapter_pregate_router_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("__global__ void k() { }\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("decode") is None       # no data file
    # an ncu --csv launch capture with two kernels' DRAM bytes, ingested as bytes per call
    csv = tmp_path / "cap.csv"
    csv.write_text('==PROF== noise\n'
                   '"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"\n'
                   '"0","k1","dram__bytes_read.sum","Mbyte","1.50"\n'
                   '"0","k1","dram__bytes_write.sum","Kbyte","500"\n'
                   '"0","k1","gpu__time_duration.sum","usecond","9.5"\n'
                   '"1","k2","dram__bytes_read.sum","byte","1,000"\n')
    assert bench.ingest_traffic(str(csv), "decode", 2, "ncu ...") == (1.5e6 + 5e5 + 1000) / 2
    assert bench.measured_traffic("decode") == (1.5e6 + 5e5 + 1000) / 2
    assert bench.measured_traffic("prefill") is None      # not captured
    (csrc / "k.cu").write_text("__global__ void k() { int changed; }\n")
    assert bench.measured_traffic("decode") is None       # captured on other kernels


def _run_bench(args, env_extra=None):
    import subprocess
    import sys
    env = dict(os.environ)
    env.update(env_extra or {})
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    return subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], cwd=root, env=env,
                          capture_output=True, text=True, timeout=240)


def test_reference_arm_prints_the_contract_line():
    import json
    r = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3",
                    "--ref-budget", "0.5"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["n_gpus"] == 1
    assert d["config"]["workload"].startswith("tiny") and "model" not in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                   {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_bench_rejects_short_warmup():
    r = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "2"])
    assert r.returncode != 0 and "--warmup" in r.stderr
