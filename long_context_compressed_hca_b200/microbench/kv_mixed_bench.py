"""Time the mixed-precision KV row kernels on a cache-sized batch of rows.

    python -m long_context_compressed_hca_b200.microbench.kv_mixed_bench [rows] [c] [rd]

Default: 1048576 rows of c = 512 with rd = 64 (the 128K batch-32 CSA cache).
Inputs are seeded N(0,1) bf16 rows; device time per call from CUDA events over
10 calls after 3 warm-up calls; bytes = rows read + records written (quant),
records read + rows written (dequant)."""
import sys

import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth


def main():
    rows = int(sys.argv[1]) if len(sys.argv) > 1 else 1 << 20
    c = int(sys.argv[2]) if len(sys.argv) > 2 else 512
    rd = int(sys.argv[3]) if len(sys.argv) > 3 else 64
    rec = hb.kv_mixed_row_bytes(c, rd)
    x = synth.normal_on("cuda", (rows, c), 7, 1, dtype=torch.bfloat16)
    out = torch.empty(rows, rec, dtype=torch.uint8, device="cuda")
    back = torch.empty(rows, c, dtype=torch.bfloat16, device="cuda")
    for name, fn, nbytes in (("kv_quant_mixed", lambda: hb.kv_quant_mixed(x, hb.HCA_BF16, rows, c, rd, out),
                              rows * (2 * c + rec)),
                             ("kv_dequant_mixed", lambda: hb.kv_dequant_mixed(out, rows, c, rd, back),
                              rows * (2 * c + rec))):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 10
        print(f"{name}: {rows} rows of c={c} (record {rec} B): {ms * 1e3:.1f} us per call, "
              f"{nbytes / (ms * 1e-3) / 1e9:.0f} GB/s", flush=True)


if __name__ == "__main__":
    main()
