"""Timeline of one decode step: which kernel occupies which SMs when.

    python -m long_context_compressed_hca_b200.microbench.step_trace [128k|1m]

Replays the step's CUDA graph (the bench's stream, priority and budget
settings) with the library's step trace on and prints, per kernel, its CTA
count, when its CTAs entered, became ready (after the dependent-launch wait)
and left, relative to the step's first entry; then the number of SMs each
kernel holds in 4 us slices of the step."""
import sys

import torch

import bench
from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import workloads


def main():
    wl = workloads.HYBRID_DECODE_1M if (len(sys.argv) > 1 and sys.argv[1] == "1m") else workloads.HYBRID_DECODE_128K
    b = bench.DecodeBench(wl)
    stream = torch.cuda.Stream()
    flush = torch.empty(bench.L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    g = bench.capture_graph(b.step, stream)
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize()
    buf = torch.zeros(1 + 4 * 65536, dtype=torch.int64, device="cuda")
    hb.step_trace(buf)
    with torch.cuda.stream(stream):
        flush.fill_(1)
        g.replay()
    torch.cuda.synchronize()
    hb.step_trace(None)
    recs = hb.step_trace_records(buf)
    t0 = min(r["entry"] for r in recs)
    t1 = max(r["exit"] for r in recs)
    print(f"{wl.name}: {len(recs)} CTA records, first entry -> last exit {(t1 - t0) / 1e3:.1f} us")
    kernels = sorted({r["kernel"] for r in recs}, key=lambda k: min(r["entry"] for r in recs if r["kernel"] == k))
    for k in kernels:
        rs = [r for r in recs if r["kernel"] == k]
        f = lambda key, agg: (agg(r[key] for r in rs) - t0) / 1e3
        print(f"  {k:11s} {len(rs):5d} CTAs on {len({r['sm'] for r in rs}):3d} SMs  entry {f('entry', min):6.1f}-"
              f"{f('entry', max):6.1f}  ready {f('ready', min):6.1f}-{f('ready', max):6.1f}  "
              f"exit {f('exit', min):6.1f}-{f('exit', max):6.1f} us")
    step = 4000
    print("  SMs held per 4 us slice (entry..exit of each CTA):")
    print("  " + " ".join(f"{k[:8]:>8s}" for k in kernels))
    for s in range(t0, t1, step):
        row = []
        for k in kernels:
            sms = {r["sm"] for r in recs if r["kernel"] == k and r["entry"] < s + step and r["exit"] > s}
            row.append(f"{len(sms):8d}")
        print(f"  {(s - t0) / 1e3:6.0f} " + " ".join(row))


if __name__ == "__main__":
    main()
