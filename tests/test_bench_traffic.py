"""bench.py's DRAM-traffic record (profiles/traffic.json) on CPU: a kernel's bytes per launch
are reported only while its source file still has the hash recorded with the capture, so a
changed kernel reports no traffic rather than stale counters."""
import hashlib
import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_traffic_under_test",
                                                  os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _tree(tmp_path, src_text, recorded_hash):
    csrc = tmp_path / "longlora_shifted_sparse_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "kern.cu").write_text(src_text)
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"k": {"source": "kern.cu", "sha256_16": recorded_hash, "bytes_per_launch": 1234,
               "how": "test"}}))


def test_traffic_follows_the_source_hash(tmp_path):
    bench = _bench()
    src = "__global__ void k() {}\n"
    _tree(tmp_path, src, hashlib.sha256(src.encode()).hexdigest()[:16])
    bench.ROOT = str(tmp_path)
    assert bench._traffic("k") == 1234
    assert bench._traffic("other") is None                 # no record for that kernel
    (tmp_path / "longlora_shifted_sparse_b200" / "csrc" / "kern.cu").write_text(src + "// x\n")
    assert bench._traffic("k") is None                     # the source changed since


def test_committed_records_name_existing_sources():
    # every record points at a kernel source of this tree and carries a 16-digit hash
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    assert set(rec) <= {"fwd_tc", "bwd_dkdv_tc", "bwd_dq_tc"}
    for name, r in rec.items():
        assert os.path.exists(os.path.join(ROOT, "longlora_shifted_sparse_b200", "csrc",
                                           r["source"])), name
        assert len(r["sha256_16"]) == 16 and int(r["sha256_16"], 16) >= 0
        assert r["bytes_per_launch"] > 0
