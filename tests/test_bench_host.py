"""Host logic of bench.py that needs no GPU: the algorithmic byte counts the
GB/s figures divide by, and the DRAM-traffic record, which is reported only
while the decode kernel's source matches the capture."""
import hashlib

import bench


def test_decode_bytes_closed_forms():
    # codes N K / 2 + fp16 scales N K / 128 * 2 (+ zeros) + X 2 M K + Y 2 M N
    assert bench.decode_bytes(4096, 4096, 1) - 2 * 4096 - 2 * 4096 == 8_650_752
    assert bench.decode_bytes(11008, 4096, 1) - 2 * 4096 - 2 * 11008 == 23_248_896
    assert bench.decode_bytes(4096, 11008, 1) - 2 * 11008 - 2 * 4096 == 23_248_896
    asym = bench.decode_bytes(28672, 8192, 1, asym=True) - 2 * 8192 - 2 * 28672
    assert asym == 117_440_512 + 2 * 3_670_016
    step = sum(bench.decode_bytes(N, K, 1) for N, K in [(4096, 4096), (11008, 4096), (4096, 11008)])
    assert step == 55_225_344


def test_traffic_record_follows_the_kernel_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_bytes(b"__global__ void k() {}\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    rec = tmp_path / "profile.txt"
    rec.write_text(f"kernel_source_sha256: {sha}\ndram_bytes_per_step: 55349760\n")
    monkeypatch.setattr(bench, "DECODE_SRC", str(src))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.recorded_traffic() == 55349760
    src.write_bytes(b"__global__ void k() { /* changed */ }\n")
    assert bench.recorded_traffic() is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.txt"))
    assert bench.recorded_traffic() is None


def test_committed_traffic_record_matches_the_committed_kernel():
    assert bench.recorded_traffic() == 55349760


def test_whole_job_throughput_counts_every_replica():
    one = bench.job_throughput_gbs(1, 100, 55_225_344, 5.0)
    assert bench.job_throughput_gbs(4, 100, 55_225_344, 5.0) == 4 * one
    assert one == 100 * 55_225_344 / 5e-3 / 1e9
