"""GPU parity at the full sizes of the benchmark workloads, in the launch
configurations bench.py times, checked on sampled outputs the oracle computes
one by one (tolerances and the top-k gap rule as in the other parity tests)."""
import numpy as np
import pytest
import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth, workloads
from long_context_compressed_hca_b200.layer import LayerHandle
from oracle import hca_oracle as O
from tests.helpers import GAP, GAP_LAYER_BF16, TOL, assert_close, check_topk_row, to64
from tests.test_gpu_layer import PrefillIntermediates, check_prefill_tokens, run_decode_case

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16


@pytest.mark.parametrize("layer", [0, 1])
def test_decode_128k_batch32(cuda, layer):
    """Hybrid decode at 128K context, batch 32: every sequence checked (near-tie
    selections within the tie, and the output over the GPU's own selection)."""
    wl = workloads.HYBRID_DECODE_128K
    ties = run_decode_case(cuda, wl.layers[layer], wl.B, wl.pos, "bf16", seed=wl.seed)
    print(f"near-tie sequences (checked within the tie): {ties} of {wl.B}")


@pytest.mark.parametrize("layer", [0, 1])
def test_decode_1m_batch4_fp8_keys(cuda, layer):
    """1M-context decode, fp8-e4m3 indexer keys, top-k 1024: every sequence checked."""
    wl = workloads.HYBRID_DECODE_1M
    run_decode_case(cuda, wl.layers[layer], wl.B, wl.pos, wl.idx_key_dtype, seed=wl.seed)


def test_decode_128k_emitting_step(cuda):
    """A decode step that completes a block (entry emission) at 128K context."""
    wl = workloads.HYBRID_DECODE_128K
    run_decode_case(cuda, wl.layers[0], 8, wl.pos + 3, "bf16", seed=11)


def _layer_full(wl, cuda, toks_per_seq):
    L = wl.layers[0]
    W = synth.layer_weights_on(cuda, L, wl.d, wl.d_c, wl.seed, BF16)
    H = synth.normal_on(cuda, (wl.B, wl.n, wl.d), wl.seed, synth.STREAMS["H"], dtype=BF16)
    lh = LayerHandle(L, W, wl.d, wl.d_c, BF16, wl.B, device=cuda)
    ws = torch.empty(hb.layer_workspace_size(lh.struct, wl.n), dtype=torch.uint8, device=cuda)
    o = torch.empty(wl.B, wl.n, L.n_h, L.c, dtype=BF16, device=cuda)
    hb.hybrid_layer_forward(lh.struct, H, wl.n, None, o, ws)
    torch.cuda.synchronize()
    gi = PrefillIntermediates(lh, ws, L, wl.B, wl.n, BF16)
    W64 = {k: to64(v) for k, v in W.items()}
    rng = np.random.default_rng(wl.seed)
    ties = checked = 0
    for b in range(wl.B):
        toks = np.unique(np.concatenate([[0, 1, 2, 3, 127, 128, 511, 512, 2047, 2048, 2051, wl.n - 2, wl.n - 1],
                                         rng.integers(0, wl.n, toks_per_seq)]))
        c_, t_ = check_prefill_tokens(L, W64, to64(H[b]), gi, o, b, toks, wl.d_c, TOL[BF16])
        checked += c_
        ties += t_
    return ties, checked


def test_prefill_64k_csa_layer(cuda):
    """The 64K CSA prefill layer from hidden states (d_model 4096), sampled
    tokens, none skipped: stored intermediates, the GPU's selection against the
    oracle's (over the GPU's stored index operands, and bounded against the
    fp64 scores) and the output against the oracle's attention over that
    selection."""
    ties, checked = _layer_full(workloads.CSA_PREFILL, cuda, 60)
    print(f"64K layer: {checked} tokens checked, {ties} near ties (checked within the tie)")
    assert checked >= 60


def test_prefill_hca_8k_layer(cuda):
    """The 8K HCA prefill layer (batch 2, d_model 1024), sampled tokens."""
    ties, checked = _layer_full(workloads.HCA_PREFILL, cuda, 40)
    assert ties == 0 and checked >= 80


def test_index_topk_64k(cuda):
    """Indexer + top-k at the 64K prefill size (65536 queries x 16384 entries)."""
    n, m, k, nh, cI = 65536, 4, 512, 8, 64
    E = n // m
    qI = synth.normal_on(cuda, (1, n, nh, cI), 7, 1, dtype=BF16)
    wI = synth.normal_on(cuda, (1, n, nh), 7, 2, std=cI ** -0.5 * nh ** -0.5)
    KI = synth.normal_on(cuda, (1, E, cI), 7, 3, dtype=BF16)
    d = hb.attn_desc(1, 64, 512, 64, 128, m, k=k, n_hI=nh, c_I=cI, rd_I=64, dtype=hb.HCA_BF16)
    ws = torch.empty(hb.csa_index_topk_workspace_size(d, n, 0), dtype=torch.uint8, device=cuda)
    idx = torch.empty(1, n, k, dtype=torch.int32, device=cuda)
    hb.csa_index_topk(d, qI, wI, KI, None, E, n, 0, idx, ws=ws)
    torch.cuda.synchronize()
    K64 = to64(KI[0])
    rows = [0, 3, 4, 2047, 2048, 2051, 65535] + list(np.random.default_rng(1).integers(0, n, 40))
    ties = 0
    for t in rows:
        V = (t + 1) // m
        ref = O.index_scores(to64(qI[0, t]), to64(wI[0, t]), K64, V)
        ties += check_topk_row(idx[0, t].cpu().numpy(), ref, k, V)
    print(f"64K index/top-k: {ties} of {len(rows)} rows are near ties (checked within fp32 rounding)")


def test_csa_attend_64k(cuda):
    """Sparse attention at the 64K prefill size (64 heads x 512, window 128, top-512)."""
    n, m, k, nh, c, w = 65536, 4, 512, 64, 512, 128
    E = n // m
    q = synth.normal_on(cuda, (1, n, nh, c), 8, 1, dtype=BF16)
    kvc = synth.normal_on(cuda, (1, E, c), 8, 2, dtype=BF16)
    kvw = synth.normal_on(cuda, (1, n, c), 8, 3, dtype=BF16)
    sink = synth.normal_on(cuda, (nh,), 8, 4)
    # valid sorted index lists: one random entry per equal-width bucket of the visible range
    t = torch.arange(n, device=cuda)
    V = (t + 1) // m
    ns = torch.clamp(V, max=k)
    j = torch.arange(k, device=cuda)
    g = torch.Generator(device=cuda)
    g.manual_seed(5)
    u = torch.rand(n, k, device=cuda, generator=g)
    idx = torch.floor((j[None] + u) * V[:, None].double() / ns.clamp(min=1)[:, None].double()).long()
    idx = torch.where(j[None] < ns[:, None], idx, torch.full_like(idx, -1)).int()[None].contiguous()
    o = torch.empty(1, n, nh, c, dtype=BF16, device=cuda)
    d = hb.attn_desc(1, nh, c, 64, w, m, k=k, dtype=hb.HCA_BF16)
    hb.csa_attend(d, q, kvc, E, idx, kvw, 0, sink, n, 0, o)
    torch.cuda.synchronize()
    for tt in [0, 1, 127, 128, 4095, 65535] + list(np.random.default_rng(2).integers(0, n, 30)):
        tt = int(tt)
        sel = idx[0, tt].cpu().numpy()
        sel = sel[sel >= 0]
        rows = np.concatenate([to64(kvw[0, max(0, tt - w + 1):tt + 1]), to64(kvc[0][torch.from_numpy(sel).to(cuda).long()])])
        ref = O.attend_output(to64(q[0, tt]), rows, to64(sink), c ** -0.5, tt, 64)
        assert_close(to64(o[0, tt]), ref, TOL[BF16], f"o[{tt}]")
