"""FP4 indexer activations on the GPU against the oracle (juejin "DeepSeek-V4
技术报告简要解读" §4.4; 1zeryu "DeepSeek-V4：算法架构", Indexer): rows rotated
by the Hadamard butterflies in fp32 and FP4-quantised in blocks of 32, bit for
bit (both sides rotate in the same fp32 order, so the quantisation decisions
agree exactly)."""
import numpy as np
import pytest
import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth
from oracle import hca_oracle as O

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,dtype", [(1, torch.bfloat16), (1003, torch.bfloat16), (77, torch.float32), (0, torch.float32)])
def test_fp4_rotate_quant_matches_oracle(cuda, rows, dtype):
    x = synth.normal((max(rows, 1), 64), 61, 1) * torch.exp2(torch.randint(-20, 20, (max(rows, 1), 1)).float())
    if rows >= 4:
        x[1] = 0.0                               # an all-zero row
        x[2, :32] = 1e-30                        # a tiny block
        x[3] = torch.arange(64).float() - 31.5   # small integers: exact butterflies
    x = x[:rows].to(dtype)
    out = torch.full((max(rows, 1), 64), float("nan"), dtype=torch.bfloat16, device=cuda)
    hb.fp4_rotate_quant(x.to(cuda), hb.HCA_F32 if dtype == torch.float32 else hb.HCA_BF16, rows, 64, out)
    torch.cuda.synchronize()
    if rows == 0:
        assert torch.isnan(out.float()).all()
        return
    want = O.fp4_rotate_quant_gpu_order(x.double().numpy())
    got = out.double().cpu().numpy()
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(np.signbit(got), np.signbit(want))          # zero stored as +0


# ------------------------------------------------------------ the FP4 indexer path
def _bf16_ulp(x):
    """Spacing of bf16 values at |x| (the rounding step of the FP4 path's scores)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-38)))
    return np.exp2(e - 7)


def check_fp4_selection(gpu_idx, ref_scores, k, V):
    """The GPU keeps the oracle's bf16 top-k (ties to the lower index) up to
    entries whose oracle bf16 score lies within one bf16 step of the k-th
    score (the GPU rounds an fp32 accumulation to bf16, the oracle an exact
    sum: the two may sit one step apart at a rounding boundary)."""
    gi = np.asarray(gpu_idx)
    n = min(k, V)
    sel = gi[:n]
    assert (gi[n:] == -1).all() and ((sel >= 0) & (sel < V)).all()
    assert n <= 1 or (np.diff(sel) > 0).all()
    ref = O.topk_select(ref_scores, k)[:n]
    if n == V:
        np.testing.assert_array_equal(sel, ref)
        return 0
    kth = np.sort(ref_scores)[::-1][n - 1]
    diff = np.setxor1d(sel, ref)
    assert (np.abs(ref_scores[diff] - kth) <= _bf16_ulp(kth) * 1.0001).all(), "FP4 selection differs beyond a bf16 step"
    return len(diff)


@pytest.mark.parametrize("B,n_q,start_pos,k", [(2, 1, 8191, 512), (1, 64, 0, 16), (2, 1, 131071, 512)])
def test_fp4_index_topk_matches_oracle(cuda, B, n_q, start_pos, k):
    """csa_index_topk on the FP4 path: keys stored rotated and FP4-quantised
    (made by the oracle), q^I rotated and quantised by the library, scores
    rounded to bf16 before the selection (juejin §4.4)."""
    m, nh, cI = 4, 8, 64
    E = (start_pos + n_q) // m
    cap = E + 3
    Kraw = synth.normal((B, cap, cI), 63, 1)
    K4 = torch.from_numpy(O.fp4_rotate_quant_gpu_order(Kraw.double().numpy().reshape(-1, cI))).reshape(B, cap, cI)
    qI = synth.normal((B, n_q, nh, cI), 63, 2, dtype=torch.bfloat16)
    wI = synth.normal((B, n_q, nh), 63, 3, std=cI ** -0.5 * nh ** -0.5)
    d = hb.attn_desc(B, 4, 64, 16, 8, m, k=k, n_hI=nh, c_I=cI, rd_I=64, dtype=hb.HCA_BF16, idx_key_dtype=hb.HCA_FP4)
    ws = torch.empty(hb.csa_index_topk_workspace_size(d, n_q, start_pos), dtype=torch.uint8, device=cuda)
    idx = torch.full((B, n_q, k), -7, dtype=torch.int32, device=cuda)
    sc = torch.full((B, n_q, E), float("nan"), device=cuda)
    hb.csa_index_topk(d, qI.to(cuda), wI.to(cuda), K4.to(torch.bfloat16).to(cuda), None, cap, n_q, start_pos, idx,
                      sc, E, ws)
    torch.cuda.synchronize()
    gi, gs = idx.cpu().numpy(), sc.cpu().double().numpy()
    K64 = K4.double().numpy()
    moved = steps = 0
    for b in range(B):
        for i in range(n_q):
            V = (start_pos + i + 1) // m
            q4 = O.fp4_rotate_quant_gpu_order(qI[b, i].double().numpy())
            ref = O.bf16_bits_to_f64(O.bf16_encode(O.index_scores(q4, wI[b, i].double().numpy(), K64[b], V)))
            got = gs[b, i, :V]
            # scores: bf16 values, equal to the oracle's or one bf16 step away
            assert np.array_equal(O.bf16_bits_to_f64(O.bf16_encode(got)), got), "scores are not bf16 values"
            off = np.abs(got - ref) > 0
            assert (np.abs(got - ref)[off] <= _bf16_ulp(ref[off]) * 1.0001).all()
            steps += int(off.sum())
            moved += check_fp4_selection(gi[b, i], ref, k, V)
    total = sum((start_pos + i + 1) // m for i in range(n_q)) * B
    assert steps <= max(2, total // 200), (steps, total)
    print(f"FP4 path: {steps} of {total} scores one bf16 step from the oracle's; {moved} kept entries moved")


def test_fp4_compress_writes_rotated_fp4_entries(cuda):
    """Indexer keys written on the FP4 path (compressor out_dtype HCA_FP4):
    each entry is the oracle's entry (Eq.(11)-(12), norm, RoPE) in bf16,
    rotated and FP4-quantised -- exactly, except where the bf16 entry itself
    sits one rounding step from the oracle's (then within one FP4 step)."""
    B, n, width, m, rd = 2, 256, 64, 4, 64
    g = lambda s: synth.normal((B, n, width), 71, s)
    Ca, Cb, Za, Zb = g(1), g(2), g(3), g(4)
    Ba = synth.normal((m, width), 71, 5, std=0.5)
    Bb = synth.normal((m, width), 71, 6, std=0.5)
    E = n // m
    out = torch.full((B, E, width), float("nan"), dtype=torch.bfloat16, device=cuda)
    d = hb.compress_desc(B, width, m, 1, rd, hb.HCA_COMPRESS_NORM | hb.HCA_COMPRESS_ROPE, hb.HCA_F32, hb.HCA_FP4)
    c = lambda t: t.to(cuda).contiguous()
    hb.csa_compress(d, 0, n, c(Ca), c(Cb), c(Za), c(Zb), width, n * width, c(Ba), c(Bb), None, out, None, E,
                    None, None)
    torch.cuda.synchronize()
    exact = 0
    for b in range(B):
        ent = O.compress_prefill(Ca[b].double().numpy(), Za[b].double().numpy(), Ba.double().numpy(), m,
                                 Cb[b].double().numpy(), Zb[b].double().numpy(), Bb.double().numpy())
        ent = O.entry_epilogue(ent, m, rd=rd)
        ref = O.fp4_rotate_quant_gpu_order(O.bf16_bits_to_f64(O.bf16_encode(ent)))
        got = out[b].double().cpu().numpy()
        same = (got == ref).all(axis=1)
        exact += int(same.sum())
        # a differing row: within one FP4 grid step (2 x the block scale) per value
        for r in np.nonzero(~same)[0]:
            amax = np.abs(ref[r].reshape(2, 32)).max(axis=1)
            step = np.repeat(2.0 * np.exp2(np.floor(np.log2(np.maximum(amax, 1e-38))) - 2), 32)
            assert (np.abs(got[r] - ref[r]) <= step * 1.0001).all()
    assert exact >= 0.9 * B * E, (exact, B * E)
