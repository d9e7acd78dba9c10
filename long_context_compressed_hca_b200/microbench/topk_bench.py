"""Time the index score + top-k call on a slice of a long prefill (each query
row holds about start_pos/m visible entries) or on a decode batch.

    python -m long_context_compressed_hca_b200.microbench.topk_bench [n_q] [start_pos] [B] [kernel]

kernel: the top-k kernel (hca_topk_kernel mode: 0 by shape, 1 a CTA per row,
2 a warp per row, 3 segmented clusters, 4 a cluster per row).

Inputs are seeded N(0,1); per-kernel device times come from CUDA-graph
replays with the library's event profiler on."""
import sys

import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth


def main():
    n_q = int(sys.argv[1]) if len(sys.argv) > 1 else 2048
    start_pos = int(sys.argv[2]) if len(sys.argv) > 2 else 63488
    B = int(sys.argv[3]) if len(sys.argv) > 3 else 1
    hb.topk_kernel(int(sys.argv[4]) if len(sys.argv) > 4 else 0)
    m, k, n_hI, c_I = 4, 512, 8, 64
    E = (start_pos + n_q) // m
    dev = "cuda"
    qI = synth.normal_on(dev, (B, n_q, n_hI, c_I), 9, 1, dtype=torch.bfloat16)
    wI = synth.normal_on(dev, (B, n_q, n_hI), 9, 2, std=c_I ** -0.5 * n_hI ** -0.5)
    KI = synth.normal_on(dev, (B, E + 1, c_I), 9, 3, dtype=torch.bfloat16)
    d = hb.attn_desc(B, 64, 512, 64, 128, m, k=k, n_hI=n_hI, c_I=c_I, rd_I=64, dtype=hb.HCA_BF16,
                     idx_key_dtype=hb.HCA_BF16)
    ws = torch.empty(hb.csa_index_topk_workspace_size(d, n_q, start_pos), dtype=torch.uint8, device=dev)
    idx = torch.empty(B, n_q, k, dtype=torch.int32, device=dev)

    def run():
        hb.csa_index_topk(d, qI, wI, KI, None, E + 1, n_q, start_pos, idx, None, 0, ws)

    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        hb.profile_enable(True)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            run()
        # the captured graph records the profiler's events on every replay
        for _ in range(10):
            g.replay()
            torch.cuda.synchronize()
            hb.profile_sample()
        prof = hb.profile_collect()
        hb.profile_enable(False)
    rows = B * n_q
    for name, (n, ms) in prof.items():
        print(f"{name}: {ms / n * 1e3:.1f} us per launch, {ms / n * 1e6 / rows:.1f} ns per row ({n} launches)")


if __name__ == "__main__":
    main()
