"""Host logic of bench.py that needs no GPU: the DRAM traffic of a kernel is
reported from the traffic record only while the kernel's source files still
hash to the value recorded with the capture."""
import importlib.util
import json
import os

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
    rec = tmp_path / "traffic.json"
    rec.write_text(json.dumps({"kernels": {"k<1>": {"source_sha256": digest,
                                                     "dram_bytes_per_launch": 3356569088}}}))
    assert b.profile_traffic("k<1>", [str(src)], str(rec)) == 3356569088.0
    assert b.profile_traffic("k<2>", [str(src)], str(rec)) is None
    src.write_text("__global__ void k() { /* changed */ }\n")
    assert b.profile_traffic("k<1>", [str(src)], str(rec)) is None
    assert b.profile_traffic("k<1>", [str(src)], str(tmp_path / "missing.json")) is None


def test_committed_traffic_record_is_well_formed():
    b = _bench()
    if not os.path.exists(b.TRAFFIC_RECORD):
        return
    with open(b.TRAFFIC_RECORD) as f:
        rec = json.load(f)
    for name, entry in rec["kernels"].items():
        assert len(entry["source_sha256"]) == 64, name
        assert entry["dram_bytes_per_launch"] > 0, name
        assert entry["command"], name


def test_head_slices_partition_the_layer():
    b = _bench()
    for heads in (1, 7, 24, 40):
        for world in (1, 2, 3, 4, 8):
            got = [b.head_slice(heads, r, world) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == heads
            assert all(got[i][1] == got[i + 1][0] for i in range(world - 1))
            sizes = [h1 - h0 for h0, h1 in got]
            assert max(sizes) - min(sizes) <= 1


def test_job_time_by_sharding():
    b = _bench()
    assert b.job_ms_per_layer(12.0, 4) == 3.0              # replicas: 4 layers per 12 ms
    assert b.job_ms_per_layer(12.0, 4, "heads") == 12.0    # one layer split four ways
