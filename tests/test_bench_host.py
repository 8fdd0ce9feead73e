"""Host logic of bench.py that needs no GPU: the DRAM traffic of a committed
ncu summary is reported only while the kernel's source files still hash to the
value recorded with it, and the committed summaries name the kernel they were
taken on."""
import importlib.util
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_host", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_traffic_only_for_the_captured_source(tmp_path):
    b = _bench()
    src = tmp_path / "kernel.cu"
    src.write_text("__global__ void k() {}\n")
    digest = b.kernel_source_hash([str(src)])
    prof = tmp_path / "profile.md"
    prof.write_text(f"kernel_source_sha256: {digest}\n\ndram_bytes_per_launch_full: 3356569088\n")
    assert b.profile_traffic([str(src)], str(prof)) == 3356569088.0
    src.write_text("__global__ void k() { /* changed */ }\n")
    assert b.profile_traffic([str(src)], str(prof)) is None
    assert b.profile_traffic([str(src)], str(tmp_path / "missing.md")) is None


def test_committed_attention_summaries_are_parseable():
    b = _bench()
    for layout, path in b.PROFILES.items():
        text = open(path).read()
        assert re.search(r"kernel_source_sha256:\s*[0-9a-f]{64}", text), layout
        m = re.search(r"dram_bytes_per_launch_full:\s*([0-9]+)", text)
        assert m and int(m.group(1)) > 3.3e9, layout       # at least Q, K, V and O once
