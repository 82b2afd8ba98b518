"""The roofline "traffic" field of bench.py comes from a committed ncu
summary only when that summary was taken on the current kernel source (a
hash over the tensor-core kernel's files) and on the benchmarked workload;
a capture on fewer heads is scaled to the workload.  Host logic only."""

import bench

W = "bf16_b1_h8_s262144_d128_causal_striped_n16_p16"


def write(tmp_path, **kv):
    lines = ["# comment: ignored", "# key: ignored too"]
    lines += [f"{k}: {v}" for k, v in kv.items()]
    p = tmp_path / "traffic.txt"
    p.write_text("\n".join(lines) + "\n")
    return str(p)


def test_current_source_and_workload_give_scaled_bytes(tmp_path):
    h = bench.source_hash(bench.TC_SOURCES)
    p = write(tmp_path, workload=W, source_sha256_16=h, dram_bytes_per_launch=1000,
              scale_to_workload=8)
    assert bench.profiled_traffic(W, p) == 8000.0


def test_unscaled_capture_defaults_to_one(tmp_path):
    h = bench.source_hash(bench.TC_SOURCES)
    p = write(tmp_path, workload=W, source_sha256_16=h, dram_bytes_per_launch=1234)
    assert bench.profiled_traffic(W, p) == 1234.0


def test_other_source_or_workload_or_missing_file_give_none(tmp_path):
    h = bench.source_hash(bench.TC_SOURCES)
    stale = "0" * 16 if h != "0" * 16 else "1" * 16
    assert bench.profiled_traffic(W, write(tmp_path, workload=W, source_sha256_16=stale,
                                           dram_bytes_per_launch=1)) is None
    assert bench.profiled_traffic("other", write(tmp_path, workload=W, source_sha256_16=h,
                                                 dram_bytes_per_launch=1)) is None
    assert bench.profiled_traffic(W, str(tmp_path / "absent.txt")) is None
    assert bench.profiled_traffic(W, write(tmp_path, workload=W, source_sha256_16=h,
                                           dram_bytes_per_launch="n/a")) is None


def test_source_hash_is_stable_and_covers_every_listed_file():
    h = bench.source_hash(bench.TC_SOURCES)
    assert h == bench.source_hash(list(bench.TC_SOURCES)) and len(h) == 16
    assert all(bench.source_hash(bench.TC_SOURCES[:i] + bench.TC_SOURCES[i + 1:]) != h
               for i in range(len(bench.TC_SOURCES)))


def test_committed_summary_parses():
    # the committed file names the headline workload; its traffic is either
    # current (a positive byte count) or flagged stale (None), never garbage
    t = bench.profiled_traffic(W)
    assert t is None or t > 0
