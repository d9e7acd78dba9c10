"""Run the CSA prefill layer of the 64K workload's shapes (d_model 4096, 64
heads x 512, indexer 8 x 64, top-512, window 128) -- or, with `hca`, the HCA
prefill layer (batch 2, d_model 1024, 16 heads x 128, m' = 128) -- at a
chosen length, a few times, and print the library's per-kernel device times.
Sized for kernel captures of the prefill kernels (compression, tensor-core
GEMMs, indexer, top-k on prefill rows, attention) on a case of a few GB.

    python -m long_context_compressed_hca_b200.microbench.prefill_layer [n] [reps] [csa|hca]

Inputs are seeded N(0,1) hidden states and N(0, 1/d_in) weights (bf16)."""
import sys

import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth, workloads
from long_context_compressed_hca_b200.layer import LayerHandle


def main():
    n = int(sys.argv[1]) if len(sys.argv) > 1 else 16384
    reps = int(sys.argv[2]) if len(sys.argv) > 2 else 3
    kind = sys.argv[3] if len(sys.argv) > 3 else "csa"
    wl = (workloads.HCA_PREFILL if kind == "hca" else workloads.CSA_PREFILL).with_(n=n)
    L = wl.layers[0]
    W = synth.layer_weights_on("cuda", L, wl.d, wl.d_c, wl.seed, torch.bfloat16)
    lh = LayerHandle(L, W, wl.d, wl.d_c, torch.bfloat16, wl.B)
    H = synth.normal_on("cuda", (wl.B, n, wl.d), wl.seed, synth.STREAMS["H"], dtype=torch.bfloat16)
    o = torch.empty(wl.B, n, L.n_h, L.c, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(hb.layer_workspace_size(lh.struct, n), dtype=torch.uint8, device="cuda")
    hb.hybrid_layer_forward(lh.struct, H, n, None, o, ws)
    torch.cuda.synchronize()
    hb.profile_enable(True)
    hb.profile_collect()
    for _ in range(reps):
        hb.hybrid_layer_forward(lh.struct, H, n, None, o, ws)
        torch.cuda.synchronize()
        hb.profile_sample()
    prof = hb.profile_collect()
    hb.profile_enable(False)
    print(f"{kind.upper()} prefill layer, batch {wl.B} x {n} tokens, workspace {ws.numel() / 2**30:.2f} GiB")
    for name, (cnt, ms) in sorted(prof.items()):
        print(f"  {name}: {ms / reps:.3f} ms per layer ({cnt // reps} launches)")
    print("device status", hb.device_status())


if __name__ == "__main__":
    main()
