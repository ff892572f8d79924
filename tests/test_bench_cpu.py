"""Host helpers of bench.py, on CPU: the DRAM-traffic lookup tied to the
kernel source, the L2 note, and the whole-job throughput arithmetic."""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _src_sha():
    with open(os.path.join(ROOT, "kv_cache_vector_04_b200", "csrc", "attend_impl.cuh"), "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()


def test_profiled_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    # the committed summary carries the hash of the source it was taken on
    fields = {}
    with open(os.path.join(ROOT, "profiles", "attend_split_llama70b_32k.md"), encoding="utf-8") as f:
        for line in f:
            if ":" in line and line.split(":", 1)[0].strip() in ("kernel_source_sha1",
                                                                 "dram_bytes_per_launch"):
                k, v = line.split(":", 1)
                fields[k.strip()] = v.split()[0]
    got = bench.profiled_traffic(bench.DEFAULT_WORKLOAD)
    if fields.get("kernel_source_sha1") == _src_sha():
        assert got == int(fields["dram_bytes_per_launch"])
    else:
        assert got is None
    # another workload never borrows the figure
    assert bench.profiled_traffic("qwen2.5-3b_decode_8k") is None
    # a summary taken on other source is ignored
    fake_root = tmp_path
    (fake_root / "profiles").mkdir()
    (fake_root / "kv_cache_vector_04_b200" / "csrc").mkdir(parents=True)
    (fake_root / "kv_cache_vector_04_b200" / "csrc" / "attend_impl.cuh").write_bytes(b"other source")
    (fake_root / "profiles" / "attend_split_llama70b_32k.md").write_text(
        "kernel_source_sha1: %s\ndram_bytes_per_launch: 123\n" % _src_sha())
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    assert bench.profiled_traffic(bench.DEFAULT_WORKLOAD) is None
    sha_other = hashlib.sha1(b"other source").hexdigest()
    (fake_root / "profiles" / "attend_split_llama70b_32k.md").write_text(
        "kernel_source_sha1: %s\ndram_bytes_per_launch: 123\n" % sha_other)
    assert bench.profiled_traffic(bench.DEFAULT_WORKLOAD) == 123


def test_l2_note():
    assert "larger than L2" in bench.l2_note(45e9, 562e6)
    assert "fit in L2" in bench.l2_note(26e6, 26e6)
    assert "fit in L2" in bench.l2_note(bench.L2_BYTES, bench.L2_BYTES)


def test_whole_job_gbs():
    # 2 ranks x 562 MB in a 0.2 ms slowest step: 5620 GB/s
    assert abs(bench.whole_job_gbs(2 * 562e6, 0.2) - 5620.0) < 1e-9
