"""Host-side helpers of bench.py on CPU: the clock-sample summary (median SM clock, throttle
reasons seen) and the lookup of a kernel's profiled DRAM traffic, which is dropped once the
kernel's source no longer matches the one the counters were taken on."""

import hashlib
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test_host", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_clock_summary():
    bench = _bench()
    c = bench.ClockSampler(0)
    c.lines = ["1965, 1965, Not Active, Not Active, Not Active, Not Active",
               "1800, 1965, Not Active, Not Active, Not Active, Active",
               "1900, 1965, Not Active, Not Active, Not Active, Not Active",
               "[N/A], 1965, Not Active, Not Active, Not Active, Not Active",   # unreadable sample: skipped
               "garbage"]
    s = c.summary()
    assert s == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    c.lines = []
    assert c.summary()["samples"] == 0 and c.summary()["sm_mhz"] is None


def test_profiled_traffic_follows_the_source(tmp_path):
    bench = _bench()
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "block_sparse_attention_attngate_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k.cu").write_bytes(b"kernel source v1\n")
    (src / "k.cuh").write_bytes(b"header v1\n")
    sha = hashlib.sha256(b"kernel source v1\n").hexdigest()
    sha2 = hashlib.sha256(b"kernel source v1\nheader v1\n").hexdigest()
    (tmp_path / "profiles" / "k.md").write_text(f"# k\n\ntraffic_bytes_per_launch: 12345\nsource_sha256: {sha}\n")
    (tmp_path / "profiles" / "k2.md").write_text(f"# k\n\ntraffic_bytes_per_launch: 777\nsource_sha256: {sha2}\n")
    bench.ROOT = str(tmp_path)
    assert bench._profiled_traffic("k.md", ["k.cu"]) == 12345
    assert bench._profiled_traffic("k2.md", ["k.cu", "k.cuh"]) == 777     # every source of the kernel, in order
    (src / "k.cuh").write_bytes(b"header v2\n")                        # a header of the kernel changed
    assert bench._profiled_traffic("k2.md", ["k.cu", "k.cuh"]) is None
    (src / "k.cu").write_bytes(b"kernel source v2\n")                  # the kernel changed since the capture
    assert bench._profiled_traffic("k.md", ["k.cu"]) is None
    assert bench._profiled_traffic("missing.md", ["k.cu"]) is None


def test_committed_profiles_carry_traffic_and_hash():
    for name in ("sparse_decode_kernel.qwen3-8b-32k-decode.md", "truth_kernel.qwen3-8b-32k-ground-truth.md"):
        with open(os.path.join(ROOT, "profiles", name)) as f:
            text = f.read()
        keys = dict(ln.split(": ", 1) for ln in text.splitlines() if ": " in ln)
        assert int(keys["traffic_bytes_per_launch"]) > 0, name
        assert len(keys["source_sha256"].strip()) == 64, name
