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
    h = bench.kernel_source_hash()
    (tmp_path / "profiles" / "dram_traffic.md").write_text(
        f"text\n\ntraffic: decode 1234 {h}\ntraffic: prefill 99 0000000000000000\n")
    assert bench.measured_traffic("decode") == 1234.0
    assert bench.measured_traffic("prefill") is None      # captured on other kernels
    assert bench.measured_traffic("merge") is None        # no line
    os.remove(tmp_path / "profiles" / "dram_traffic.md")
    assert bench.measured_traffic("decode") is None
