"""The decode-step trace (hca_step_trace): every CTA of the step's kernels
leaves one record with ordered times and a valid SM id, and nothing is
recorded once the trace is off."""
import pytest
import torch

import bench
from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import workloads

pytestmark = pytest.mark.gpu


def test_step_trace_records_every_cta(cuda):
    wl = workloads.HYBRID_DECODE_128K.with_(B=4, pos=8192)
    b = bench.DecodeBench(wl)
    b.step()
    torch.cuda.synchronize()
    buf = torch.zeros(1 + 4 * 16384, dtype=torch.int64, device=cuda)
    hb.step_trace(buf)
    try:
        b.step()
        torch.cuda.synchronize()
    finally:
        hb.step_trace(None)
    recs = hb.step_trace_records(buf)
    assert int(buf[0].item()) == len(recs) > 0
    kinds = {r["kernel"] for r in recs}
    assert kinds == {"ingest", "indexer", "top-k", "attend CSA", "attend HCA"}, kinds
    # ingest: one CTA per sequence and part (CSA: main, indexer, ring; HCA: main, ring)
    assert sum(r["kernel"] == "ingest" for r in recs) == 5 * wl.B
    n_sm = torch.cuda.get_device_properties(cuda).multi_processor_count
    for r in recs:
        assert r["entry"] <= r["ready"] <= r["exit"], r
        assert 0 <= r["sm"] < n_sm, r
    # off: another step adds nothing
    n = int(buf[0].item())
    b.step()
    torch.cuda.synchronize()
    assert int(buf[0].item()) == n
