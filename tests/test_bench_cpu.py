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
    # the committed record carries the hash of the source it was taken on
    import json
    got = bench.profiled_traffic(bench.DEFAULT_WORKLOAD)
    if os.path.exists(bench.TRAFFIC_FILE):
        rec = json.load(open(bench.TRAFFIC_FILE))
        if rec.get("kernel_source_sha1") == _src_sha() and rec.get("workload") == bench.DEFAULT_WORKLOAD:
            assert got == int(rec["dram_bytes_per_launch"])
        else:
            assert got is None
    else:
        assert got is None
    # another workload never borrows the figure
    assert bench.profiled_traffic("qwen2.5-3b_decode_8k") is None
    # a record taken on other source is ignored
    fake_root = tmp_path
    (fake_root / "profiles").mkdir()
    (fake_root / "kv_cache_vector_04_b200" / "csrc").mkdir(parents=True)
    (fake_root / "kv_cache_vector_04_b200" / "csrc" / "attend_impl.cuh").write_bytes(b"other source")
    rec_path = fake_root / "profiles" / "attend_split_llama70b_32k.json"
    rec_path.write_text(json.dumps({"workload": bench.DEFAULT_WORKLOAD, "kernel_source_sha1": _src_sha(),
                                    "dram_bytes_per_launch": 123}))
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec_path))
    assert bench.profiled_traffic(bench.DEFAULT_WORKLOAD) is None
    sha_other = hashlib.sha1(b"other source").hexdigest()
    rec_path.write_text(json.dumps({"workload": bench.DEFAULT_WORKLOAD, "kernel_source_sha1": sha_other,
                                    "dram_bytes_per_launch": 123}))
    assert bench.profiled_traffic(bench.DEFAULT_WORKLOAD) == 123


def test_bytes_per_head_token_match_the_oracle_tiles():
    # the bench's byte count per (token, kv head) is the packed tile layout's
    from kv_cache_vector_04_b200 import inputs
    from oracle import oracle as O
    for w in list(inputs.WORKLOADS.values()) + inputs.sweep_workloads() + inputs.format_workloads():
        fmt = bench.fmt_of(w)
        assert bench.bytes_per_head_token(w) * 16 == O.tile_bytes(w.d, fmt), w.name


def test_reference_arm_reports_the_gpu_arms_config():
    # both arms describe the same workload (context N + 1: the decode step's token included)
    from kv_cache_vector_04_b200 import inputs
    w = inputs.WORKLOADS[bench.DEFAULT_WORKLOAD]
    cfg = bench.workload_config(w, w.layers, 1)
    assert cfg["context"] == w.N + 1 and cfg["format"] == [3, 4, 1] and cfg["layers"] == 80
    assert cfg["packed_cache_gb"] == round(80 * 16 * 8 * (w.N + 16) * 134 / 1e9, 2)


def test_l2_note():
    assert "larger than L2" in bench.l2_note(45e9, 562e6)
    assert "fit in L2" in bench.l2_note(26e6, 26e6)
    assert "fit in L2" in bench.l2_note(bench.L2_BYTES, bench.L2_BYTES)


def test_whole_job_gbs():
    # 2 ranks x 562 MB in a 0.2 ms slowest step: 5620 GB/s
    assert abs(bench.whole_job_gbs(2 * 562e6, 0.2) - 5620.0) < 1e-9


def test_reference_arm_inputs_do_not_map_the_cuda_library():
    # The reference arm takes its workload and seeded inputs from inputs.py
    # without importing the package, whose __init__ loads libtq.so.
    import subprocess
    code = ("import sys; sys.path.insert(0, %r); import bench; "
            "w = bench.workload_by_name(bench.DEFAULT_WORKLOAD); "
            "q = bench.load_inputs().queries(w, B=1, Hq=8); "
            "assert q.shape == (1, 8, w.d), q.shape; "
            "assert 'kv_cache_vector_04_b200' not in sys.modules; "
            "assert 'libtq' not in open('/proc/self/maps').read(); print('ok')" % ROOT)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr[-2000:]
