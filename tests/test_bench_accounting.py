"""bench.py's byte accounting and roofline denominators, on the CPU: the chunk sizes it
counts are the library's and the oracle's, the algorithmic bytes of the batched step
are the ones its JSON line reports, the whole-job throughput sums the ranks, and
the peak comes from the measured-peaks file."""
import json
import os

import pytest

import bench
from kv_cache_vector_02_b200 import workloads as W


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_02_b200 import tq as _tq
    return _tq


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_chunk_bytes_agree_with_the_library_and_the_oracle(tq, orc, bits):
    ctx = tq.tq_init_host(128, bits, 0, tq.ROT_HAAR, tq.KEY_PROD)
    o = orc.Oracle(128, bits, 0)
    for kind in (0, 1):
        assert bench.chunk_bytes(bits, kind) == tq.tq_chunk_bytes(ctx, kind) == o.chunk_bytes(kind)
    tq.tq_destroy(ctx)


def test_batched_step_bytes():
    w = W.WORKLOADS["batched"]
    comp, dec = bench.step_bytes(w)
    vec = 32 * 4096 * 8
    # compress: fp16 K and V in (2 x 256 B) + 88 B key and 68 B value packed out, per vector
    assert comp == vec * (512 + 88 + 68) == 700448768
    # decode: every packed byte of the context once, q in and out (fp16), the block
    # table and the sequence lengths
    assert dec == vec * (88 + 68) + 2 * 32 * 32 * 128 * 2 + 32 * 256 * 4 + 32 * 4 == 164135040


def test_whole_job_throughput_sums_the_ranks():
    one = bench.whole_job_gbs(1, 1e9, 1.0)
    assert one == pytest.approx(1000.0)
    assert bench.whole_job_gbs(4, 1e9, 1.0) == pytest.approx(4 * one)
    assert bench.whole_job_gbs(4, 1e9, 2.0) == pytest.approx(2 * one)


def test_peak_is_the_measured_copy_bandwidth():
    p = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(p):   # a checkout without the measured file: the stated fallback
        assert bench.measured_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
        return
    with open(p) as f:
        want = float(json.load(f)["hbm_gbs"])
    assert bench.measured_peak() == (want, "measured")


def test_traffic_records_name_their_sources():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for k, r in rec.items():
        assert os.path.exists(os.path.join(bench.ROOT, r["profile"])), (k, r["profile"])
        for src in r["sources"]:
            assert os.path.exists(os.path.join(bench.ROOT, src)), (k, src)
        got = bench.traffic_record(k)
        # a record is used only while its sources hash as they did at the capture
        assert got is None or got["sha256"] == r["sha256"]
