"""bench.py's recorded DRAM traffic (MEASURED_TRAFFIC: ncu's dram__bytes_read.sum
+ dram__bytes_write.sum per launch, summarised in profiles/) belongs to the
kernels as committed: each record's source digest matches the current sources,
so the bench line reports it rather than null, and each recorded byte count
sits close to the bytes bench.py's own model says the kernel must move on the
headline workload (each token tensor once, each state once, the walks' state
cache; LASP paper, section 3.4). A kernel edited without a new capture fails
the first test; a capture of the wrong kernel or size fails the second."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def _records():
    return sorted(_bench().MEASURED_TRAFFIC)


@pytest.mark.parametrize("kernel", _records())
def test_record_matches_the_committed_kernel_sources(kernel):
    bench = _bench()
    files, _, nbytes = bench.MEASURED_TRAFFIC[kernel]
    for f in files:
        assert os.path.isfile(os.path.join(ROOT, "sequence_linear_attention_b200", "csrc", f)), f
    assert bench.measured_traffic(kernel, bench.DEFAULT_WORKLOAD) == nbytes, \
        f"{kernel}: its sources changed since the traffic capture"


@pytest.mark.parametrize("kernel", _records())
def test_recorded_bytes_are_close_to_the_byte_model(kernel):
    bench = _bench()
    from sequence_linear_attention_b200 import inputs as lasp_inputs
    w = lasp_inputs.WORKLOADS[bench.DEFAULT_WORKLOAD]
    tokens_heads = w["B"] * w["N"] * w["H"]
    G = 1024  # the segment length the headline workload walks with (lasp_segment_tokens)
    model = bench.algorithmic_bytes(kernel, tokens_heads, w["d"], w["C"], G, 2 if w["bf16"] else 4)
    measured = bench.MEASURED_TRAFFIC[kernel][2]
    # DRAM traffic may fall a little below the model (writes still in L2 when
    # the kernel ends) and rise above it by re-reads; outside this window the
    # record is not of this kernel at this size
    assert 0.85 * model <= measured <= 1.25 * model, (kernel, measured, model, measured / model)
