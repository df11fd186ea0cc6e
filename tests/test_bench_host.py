"""Host-side arithmetic of the benchmark (no GPU).

The throughput the benchmark reports is algorithmic bytes over time. The
numerator is pinned here to the byte count the operator's definition fixes:
per row, x1 and x2 read and xOut written (16-bit each), plus codes (1 or 1/2
byte per element) and one binary32 scale for every produced output; once per
call, each parameter vector present.  The expected totals are worked out by
hand for each workload's shapes and options; they do not call the benchmark.
"""
import pytest

import bench
from int4_quant_b200 import workloads as wl


def _outputs(w):
    on1 = w.mask is None or w.mask[0]
    on2 = (w.mask is not None and w.mask[1]) or (
        w.mask is None and w.smooth1 is not None and w.smooth2 is not None)
    return on1, on2


# rows x n; 6 bytes per element of x1, x2, xOut; codes + 4-byte scale per output; 2n bytes per
# parameter vector.
EXPECTED = {
    # gamma only; one INT8 output: 64 * (6*1024 + 1024 + 4) + 2*1024
    "c1": 64 * (6 * 1024 + 1024 + 4) + 2 * 1024,
    # gamma, beta, smooth1; one INT8 output
    "c2": 8192 * (6 * 4096 + 4096 + 4) + 3 * 2 * 4096,
    # gamma, smooth1, smooth2; two INT8 outputs
    "c3": 4096 * (6 * 7168 + 2 * (7168 + 4)) + 3 * 2 * 7168,
    # gamma, beta (zeros, passed); one packed INT4 output
    "c4": 16384 * (6 * 5120 + 5120 // 2 + 4) + 2 * 2 * 5120,
    # gamma, beta, smooth1; one INT8 output
    "c5a": 1 * (6 * 16384 + 16384 + 4) + 3 * 2 * 16384,
    "c5b": 8 * (6 * 16384 + 16384 + 4) + 3 * 2 * 16384,
    "c5c": 128 * (6 * 16384 + 16384 + 4) + 3 * 2 * 16384,
    "c5d": 2048 * (6 * 16384 + 16384 + 4) + 3 * 2 * 16384,
}


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_algorithmic_bytes_of_each_workload(name, monkeypatch):
    # the byte count needs only the shapes and which tensors are present:
    # avoid drawing the full-size random inputs
    calls = {}

    def fake_random_case(rows, n, **kw):
        calls.update(kw)
        z = None
        return wl.Workload(name=name, rows=rows, n=n, dtype=kw.get("dtype", "bf16"),
                           qdtype=kw.get("qdtype", "int8"), eps=1e-6, mask=kw.get("mask"),
                           x1=z, x2=z, gamma=z,
                           beta=(0 if kw.get("beta") is not None and kw.get("beta") is not False
                                 else None),
                           smooth1=0 if kw.get("smooth1") else None,
                           smooth2=0 if kw.get("smooth2") else None)

    monkeypatch.setattr(wl, "random_case", fake_random_case)
    w = wl.CONFIGS[name]()
    on1, on2 = _outputs(w)
    assert bench.workload_bytes(w, on1, on2) == EXPECTED[name]


def test_bench_workload_floor():
    # 234.94 MB per call on the 8192 x 4096 workload: 35.84 us at 6554.6 GB/s
    nbytes = EXPECTED["c2"]
    assert nbytes == 234_938_368
    assert abs(nbytes / 6554.6e9 * 1e6 - 35.84) < 0.01


def test_algorithmic_bytes_of_the_no_add_operator():
    # rms_norm_dynamic_quant on the 8192 x 4096 workload's x1 and parameters:
    # per row x read (2 B/element), INT8 codes written (1 B/element) and one
    # fp32 scale; no x2, no xOut; gamma, beta, smooth1 read once
    per_row = 4096 * 2 + 4096 + 4
    assert bench.algorithmic_bytes(8192, 4096, "bf16", "int8", True, True, False, True, False,
                                   has_x2=False, x_out=False) == 8192 * per_row + 3 * 4096 * 2
    assert 8192 * per_row + 3 * 4096 * 2 == 100_720_640


def test_launches_per_call():
    # one kernel per call, whether a row has one CTA or a cluster
    class P:
        cluster = 1
    assert bench.launches_per_call(P) == 1
    P.cluster = 4
    assert bench.launches_per_call(P) == 1


def test_rotated_sets_cover_twice_the_l2():
    class W:  # 64 x 1024 bf16, gamma only, one INT8 output: 461,056 bytes a call
        rows, n, dtype, qdtype = 64, 1024, "bf16", "int8"
        beta = smooth1 = smooth2 = None
    assert bench.sets_for(W, True, False) == 3
    k = bench.sets_for(W, True, False, min_bytes=300 << 20)
    assert k == -(-(300 << 20) // 461_056) and k * 461_056 >= 300 << 20
    assert bench.sets_for(W, True, False, min_bytes=1 << 40) == 2048


def test_job_throughput_counts_every_rank():
    # weak scaling: every rank moves the same bytes per step
    one = bench.job_gbs(1e9, 10, 1, 1000.0)
    assert abs(one - 10.0) < 1e-9
    assert abs(bench.job_gbs(1e9, 10, 4, 1000.0) - 4 * one) < 1e-9
