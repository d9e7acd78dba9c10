"""Time the tensor-core attention kernel alone on a synthetic prefill batch and
print the per-role wait-cycle trace.

    python -m long_context_compressed_hca_b200.microbench.attend_bench <n_q> <csa|hca> [c] [n_h] [B] [m]
    python -m long_context_compressed_hca_b200.microbench.attend_bench decode <csa|hca> [B] [pos] [max_ctas] [mixed]

Inputs are seeded N(0,1) (bf16); CSA index lists take one random visible entry
per equal-width bucket (valid, sorted, no repeats)."""
import sys

import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth


def decode_main():
    """One decode token per sequence over a ring window and a compressed cache
    (the 128K decode workload's attention call), split-KV included."""
    kind = sys.argv[2] if len(sys.argv) > 2 else "csa"
    B = int(sys.argv[3]) if len(sys.argv) > 3 else 32
    pos = int(sys.argv[4]) if len(sys.argv) > 4 else 131072
    max_ctas = int(sys.argv[5]) if len(sys.argv) > 5 else 0
    mixed = len(sys.argv) > 6 and sys.argv[6] == "mixed"   # mixed-precision KV records
    n_h, c, rd, w = 64, 512, 64, 128
    m, k = (4, 512) if kind == "csa" else (128, 0)
    V = (pos + 1) // m
    cap = V + 8
    dev = "cuda"
    q = synth.normal_on(dev, (B, 1, n_h, c), 2, 1, dtype=torch.bfloat16)
    kv = synth.normal_on(dev, (B, cap, c), 2, 2, dtype=torch.bfloat16)
    ring = synth.normal_on(dev, (B, w, c), 2, 3, dtype=torch.bfloat16)
    if mixed:
        rec = hb.kv_mixed_row_bytes(c, rd)
        kvr = torch.empty(B * cap * rec, dtype=torch.uint8, device=dev)
        rr = torch.empty(B * w * rec, dtype=torch.uint8, device=dev)
        hb.kv_quant_mixed(kv, hb.HCA_BF16, B * cap, c, rd, kvr)
        hb.kv_quant_mixed(ring, hb.HCA_BF16, B * w, c, rd, rr)
        kv, ring = kvr, rr
    sink = synth.normal_on(dev, (n_h,), 2, 4)
    idx = None
    if kind == "csa":
        g = torch.Generator(device=dev)
        g.manual_seed(4)
        j = torch.arange(k, device=dev)
        u = torch.rand(B, k, device=dev, generator=g)
        idx = torch.floor((j[None] + u) * (V / k)).long().clamp(max=V - 1).int()[:, None].contiguous()
    o = torch.empty(B, 1, n_h, c, dtype=torch.bfloat16, device=dev)
    d = hb.attn_desc(B, n_h, c, rd, w, m, k=max(k, 1), dtype=hb.HCA_BF16, max_ctas=max_ctas, kv_mixed=int(mixed))
    wsz = (hb.csa_attend_workspace_size if kind == "csa" else hb.hca_attend_workspace_size)(d, 1, pos)
    ws = torch.empty(max(wsz, 16), dtype=torch.uint8, device=dev)

    def run(use_ws=True):
        w = ws if use_ws else None
        if kind == "csa":
            hb.csa_attend(d, q, kv, cap, idx, ring, 1, sink, 1, pos, o, w)
        else:
            hb.hca_attend(d, q, kv, cap, ring, 1, sink, 1, pos, o, w)

    # device time per call from CUDA-graph replays (no host work in the interval):
    # with the workspace (fp32 partials + combine kernel) and without it (cluster merge)
    outs = {}
    for use_ws in (True, False):
        st = torch.cuda.Stream()
        with torch.cuda.stream(st):
            for _ in range(3):
                run(use_ws)
            torch.cuda.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=st):
                for _ in range(10):
                    run(use_ws)
            gr.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            for _ in range(5):
                gr.replay()
            e1.record(st)
            torch.cuda.synchronize()
            outs[use_ws] = o.clone()
        print(f"{'workspace + combine' if use_ws else 'cluster merge'}: {e0.elapsed_time(e1) / 50 * 1e3:.2f} us per call")
    print("max |workspace - cluster| =", (outs[True].float() - outs[False].float()).abs().max().item())
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    hb.profile_enable(True)
    hb.profile_collect()
    for _ in range(10):
        run()
        torch.cuda.synchronize()
        hb.profile_sample()
        hb.profile_collect() if False else None
    prof = hb.profile_collect()
    hb.profile_enable(False)
    keys = min(w, pos + 1) + (min(k, V) if kind == "csa" else V)
    byts = B * (keys * (hb.kv_mixed_row_bytes(c, rd) if mixed else c * 2) + 2 * n_h * c * 2)
    for name, (n, ms) in prof.items():
        print(f"{name}: {ms / n * 1e3:.1f} us per launch ({n} launches)")
    att = [v for kk, v in prof.items() if kk.startswith("attend_") and kk.endswith("tc")][0]
    print(f"gathered+q/o bytes {byts / 1e6:.1f} MB -> {byts / (att[1] / att[0] * 1e-3) / 1e9:.0f} GB/s in the attention kernel")
    hb.trace_attend(1)
    run(False)
    tr = hb.trace_attend_read()
    hb.trace_attend(0)
    tot = tr["total"]
    tl = {kk for kk in tr if kk.startswith("t_")}
    print({kk: (round(3 * v / tot, 3) if kk not in ("rescales", "units", "tiles", "total") else v)
           for kk, v in tr.items() if kk not in tl})
    n = max(tr["t_ctas"], 1)
    span = (tr["t_exit_max"] - ((~tr["t_entry_inv"]) & (2 ** 64 - 1))) / 1e3
    print("per-CTA timeline (us):", {kk[2:]: round(tr[kk] / n / 1e3, 2)
                                      for kk in ("t_setup", "t_first_s", "t_tiles", "t_epilogue", "t_exit")},
          f"first entry -> last exit {span:.2f} us over {tr['t_ctas']} CTAs")
    print("device status", hb.device_status())


def main():
    if len(sys.argv) > 1 and sys.argv[1] == "decode":
        return decode_main()
    n_q = int(sys.argv[1]) if len(sys.argv) > 1 else 2048
    kind = sys.argv[2] if len(sys.argv) > 2 else "csa"
    c = int(sys.argv[3]) if len(sys.argv) > 3 else 512
    n_h = int(sys.argv[4]) if len(sys.argv) > 4 else 64
    B = int(sys.argv[5]) if len(sys.argv) > 5 else 1
    m = int(sys.argv[6]) if len(sys.argv) > 6 else 4
    rd, w, k = 64, 128, 512
    cap = n_q // m + 2
    dev = "cuda"
    q = synth.normal_on(dev, (B, n_q, n_h, c), 1, 1, dtype=torch.bfloat16)
    kv = synth.normal_on(dev, (B, cap, c), 1, 2, dtype=torch.bfloat16)
    win = synth.normal_on(dev, (B, n_q, c), 1, 3, dtype=torch.bfloat16)
    sink = synth.normal_on(dev, (n_h,), 1, 4)
    t = torch.arange(n_q, device=dev)
    V = (t + 1) // m
    nsel = torch.clamp(V, max=k)
    j = torch.arange(k, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    u = torch.rand(n_q, k, device=dev, generator=g)
    idx = torch.floor((j[None] + u) * V[:, None].double() / nsel.clamp(min=1)[:, None].double()).long()
    idx = torch.where(j[None] < nsel[:, None], idx, torch.full_like(idx, -1)).int()[None].expand(B, n_q, k).contiguous()
    o = torch.empty(B, n_q, n_h, c, dtype=torch.bfloat16, device=dev)
    d = hb.attn_desc(B, n_h, c, rd, w, m, k=k, dtype=hb.HCA_BF16)

    def run():
        if kind == "csa":
            hb.csa_attend(d, q, kv, cap, idx, win, 0, sink, n_q, 0, o)
        else:
            hb.hca_attend(d, q, kv, cap, win, 0, sink, n_q, 0, o)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(5):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / 5
    keys = 0
    for i in range(n_q):
        vv = (i + 1) // m
        keys += min(w, i + 1) + (min(k, vv) if kind == "csa" else vv)
    flops = B * keys * n_h * c * 4
    print(f"attend {kind} B={B} n_q={n_q} n_h={n_h} c={c} m={m}: {ms:.3f} ms, {flops / ms / 1e9:.1f} TFLOP/s")
    hb.trace_attend(1)
    run()
    tr = hb.trace_attend_read()
    hb.trace_attend(0)
    tot = tr["total"]   # summed over the three reporting roles
    print({kk: (round(3 * v / tot, 3) if kk not in ("rescales", "units", "tiles", "total") else v)
           for kk, v in tr.items()})
    print("device status", hb.device_status())


if __name__ == "__main__":
    main()
