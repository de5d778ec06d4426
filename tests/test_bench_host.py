"""Host logic of bench.py that needs no GPU: the algorithmic byte counts the
GB/s figures divide by, the tokens/s-equivalent, the DRAM-traffic records
(reported only while the decode kernel's source matches the capture) and the
CPU oracle leg's row sharding."""
import hashlib

import numpy as np

import bench
from workloads import WORKLOADS


def test_decode_bytes_closed_forms():
    # codes N K / 2 + fp16 scales N K / 128 * 2 (+ zeros) + X 2 M K + Y 2 M N
    assert bench.decode_bytes(4096, 4096, 1) - 2 * 4096 - 2 * 4096 == 8_650_752
    assert bench.decode_bytes(11008, 4096, 1) - 2 * 4096 - 2 * 11008 == 23_248_896
    assert bench.decode_bytes(4096, 11008, 1) - 2 * 11008 - 2 * 4096 == 23_248_896
    asym = bench.decode_bytes(28672, 8192, 1, asym=True) - 2 * 8192 - 2 * 28672
    assert asym == 117_440_512 + 2 * 3_670_016
    step = sum(bench.decode_bytes(N, K, 1) for N, K in [(4096, 4096), (11008, 4096), (4096, 11008)])
    assert step == 55_225_344
    step70 = sum(bench.decode_bytes(N, K, 1, asym=True) for N, K in [(28672, 8192), (8192, 28672)])
    assert step70 == 2 * (117_440_512 + 2 * 3_670_016) + 2 * (2 * 8192 + 2 * 28672)


def test_tokens_per_s_equivalent():
    # 70B at INT4 g128 with fp16 scale and zero: 0.5 + 4/128 bytes per weight
    assert bench.bytes_per_param(True) == 0.53125
    assert bench.bytes_per_param(False) == 0.515625
    t = bench.tokens_per_s_equiv(5000.0, 1, "70b-decode", True)
    assert abs(t - 5000e9 / (70e9 * 0.53125)) < 1e-9
    assert bench.tokens_per_s_equiv(5000.0, 8, "70b-decode", True) == 8 * t


def test_traffic_record_follows_the_kernel_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_bytes(b"__global__ void k() {}\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    rec = tmp_path / "profile.txt"
    rec.write_text(f"kernel_source_sha256: {sha}\ndram_bytes_per_step: 55349760\n")
    monkeypatch.setattr(bench, "DECODE_SRC", str(src))
    assert bench.recorded_traffic(str(rec)) == 55349760
    src.write_bytes(b"__global__ void k() { /* changed */ }\n")
    assert bench.recorded_traffic(str(rec)) is None
    assert bench.recorded_traffic(str(tmp_path / "missing.txt")) is None


def test_whole_job_throughput_counts_every_replica():
    one = bench.job_throughput_gbs(1, 100, 55_225_344, 5.0)
    assert bench.job_throughput_gbs(4, 100, 55_225_344, 5.0) == 4 * one
    assert one == 100 * 55_225_344 / 5e-3 / 1e9


def test_oracle_leg_sharding_matches_one_thread():
    """The CPU leg shards row blocks over threads; the sharded step computes
    the same rows (bytes) as the single-threaded one, and the row-block
    products equal the whole product."""
    import concurrent.futures as cf
    import oracle
    wl = WORKLOADS["7b-decode"]
    prepared = bench.prepare_oracle(wl, None, 1, 1 / 128)
    b1 = bench.oracle_step(prepared, True, 1)
    with cf.ThreadPoolExecutor(4) as pool:
        b4 = bench.oracle_step(prepared, True, 4, pool)
    assert b1 == b4 == sum(bench.decode_bytes(n, K, 1) for _, _, _, _, n, K in prepared)
    x, c, s, z, n, K = prepared[0]
    whole, _ = oracle.gemm_w4a16(x, c, s, z, 128, True)
    parts = np.concatenate([oracle.gemm_w4a16(x, c, s, z, 128, True, a, min(n, a + 8))[0]
                            for a in range(0, n, 8)], axis=1)
    assert np.array_equal(whole, parts)


def test_committed_traffic_records_match_the_committed_kernel():
    """Each step's DRAM traffic was captured on the decode kernel as committed
    (the record names its source hash), and it is within 2% of the
    algorithmic bytes (no re-reads)."""
    for name, path in bench.TRAFFIC.items():
        t = bench.recorded_traffic(path)
        assert t is not None, path
        wl = WORKLOADS[name]
        alg = sum(bench.decode_bytes(N, K, 1, not wl.sym) for N, K in wl.shapes)
        assert alg <= t <= 1.02 * alg, (name, t, alg)
