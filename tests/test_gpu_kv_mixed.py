"""Mixed-precision KV rows on the GPU against the oracle (juejin "DeepSeek-V4
技术报告简要解读" §2.3.4; 1zeryu "DeepSeek-V4：算法架构", Q/K/V mapping and
Compressor): every code, scale and bf16 RoPE value of the records bit for bit
(both sides take the fp32 decisions the format defines), the padding zero, and
the dequantised rows equal to bf16(fp32(code * scale))."""
import numpy as np
import pytest
import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth
from oracle import hca_oracle as O

pytestmark = pytest.mark.gpu

CASES = [
    # rows, c, rd, dtype
    (1, 512, 64, torch.bfloat16),
    (1003, 512, 64, torch.bfloat16),      # ragged against the 8 rows of a block
    (37, 512, 64, torch.float32),
    (5, 128, 64, torch.bfloat16),          # one code block
    (9, 256, 64, torch.float32),
    (4, 64, 0, torch.bfloat16),            # no RoPE channels
    (0, 512, 64, torch.bfloat16),          # empty
]


def _rows(rows, c, dtype, seed):
    x = synth.normal((max(rows, 1), c), seed, 1)
    x = x * torch.exp2(torch.randint(-12, 12, (max(rows, 1), 1)).float())   # per-row magnitudes
    if rows >= 4:
        x[1, 64:128] = 0.0                    # an all-zero code block
        x[2, 5] = -0.0
        x[3] = 0.0                            # an all-zero row
        x[0, 7] = 1e-30                       # rounds to zero within its block
    return x[:rows].to(dtype)


@pytest.mark.parametrize("rows,c,rd,dtype", CASES)
def test_kv_quant_mixed_matches_oracle(cuda, rows, c, rd, dtype):
    rec = hb.kv_mixed_row_bytes(c, rd)
    nq = c - rd
    assert rec == ((nq + 2 * rd + nq // 16 + 15) // 16) * 16
    x = _rows(rows, c, dtype, 40 + c + rd)
    xd = x.to(cuda)
    out = torch.full((max(rows, 1), rec), 0xA5, dtype=torch.uint8, device=cuda)
    hb.kv_quant_mixed(xd, hb.HCA_F32 if dtype == torch.float32 else hb.HCA_BF16, rows, c, rd, out)
    back = torch.full((max(rows, 1), c), float("nan"), dtype=torch.bfloat16, device=cuda)
    hb.kv_dequant_mixed(out, rows, c, rd, back)
    torch.cuda.synchronize()
    if rows == 0:
        assert (out == 0xA5).all() and torch.isnan(back.float()).all()
        return
    got = out.cpu().numpy()
    codes, scales, rope = O.kv_row_quant(x.double().numpy(), rd)
    np.testing.assert_array_equal(got[:, :nq], codes)
    np.testing.assert_array_equal(got[:, nq:nq + 2 * rd].copy().view(np.uint16), rope)
    np.testing.assert_array_equal(got[:, nq + 2 * rd:nq + 2 * rd + nq // 16].copy().view(np.float32), scales)
    assert (got[:, nq + 2 * rd + nq // 16:] == 0).all()
    # the reader: bf16(fp32(code * scale)), the RoPE channels as stored
    prod = (O.e4m3_to_f64(codes).astype(np.float32) * np.repeat(scales, 64, axis=1)).astype(np.float32)
    want = np.concatenate([O.bf16_bits_to_f64(O.bf16_encode(prod)), O.bf16_bits_to_f64(rope)], axis=1)
    np.testing.assert_array_equal(back.double().cpu().numpy(), want)
    # and within the format's error of the exact rows
    exact = O.kv_row_dequant(codes, scales, rope)
    assert np.all(np.abs(back.double().cpu().numpy() - exact) <= np.abs(exact) * 2.0 ** -8)


# --------------------------------------------- attention over mixed-precision KV records
def _mixed_rows(x64, rd):
    """What a reader of the mixed format sees for bf16 rows x (the oracle's own
    quantisation of the same rows)."""
    return O.kv_row_dequant(*O.kv_row_quant(x64, rd))


@pytest.mark.parametrize("kind,ring,B,n_q,pos,c", [("csa", True, 3, 1, 4099, 512), ("hca", True, 2, 1, 5000, 512),
                                                   ("csa", False, 1, 150, 0, 512), ("hca", False, 2, 300, 0, 512),
                                                   ("hca", True, 2, 1, 1030, 128)])
def test_attend_reads_mixed_records(cuda, kind, ring, B, n_q, pos, c):
    """csa_attend / hca_attend with kv_mixed = 1 (juejin §2.3.4): the compressed
    rows and the window rows are 608-byte records (c = 512) that the attention
    dequantises on load; the output equals the oracle's attention over the
    dequantised rows (bf16 tolerance)."""
    n_h, rd, w = 64, 64, 128
    m, k = (4, 64) if kind == "csa" else (128, 0)
    cap = (pos + n_q) // m + 2
    rec = hb.kv_mixed_row_bytes(c, rd)
    bf = torch.bfloat16
    q = synth.normal((B, n_q, n_h, c), 41, 1, dtype=bf)
    kvc = synth.normal((B, cap, c), 41, 2, dtype=bf)
    win = synth.normal((B, w if ring else n_q, c), 41, 3, dtype=bf)
    sink = synth.normal((n_h,), 41, 4)
    rc = torch.zeros(B * cap * rec, dtype=torch.uint8, device=cuda)
    rw = torch.zeros(win.shape[0] * win.shape[1] * rec, dtype=torch.uint8, device=cuda)
    hb.kv_quant_mixed(kvc.to(cuda).contiguous(), hb.HCA_BF16, B * cap, c, rd, rc)
    hb.kv_quant_mixed(win.to(cuda).contiguous(), hb.HCA_BF16, win.shape[0] * win.shape[1], c, rd, rw)
    idx = None
    if kind == "csa":
        from tests.helpers import random_idx
        idx = random_idx(B, n_q, pos, m, k, seed=43, device=cuda)
    o = torch.full((B, n_q, n_h, c), float("nan"), dtype=bf, device=cuda)
    d = hb.attn_desc(B, n_h, c, rd, w, m, k=max(k, 1), dtype=hb.HCA_BF16, kv_mixed=1)
    if kind == "csa":
        hb.csa_attend(d, q.to(cuda), rc, cap, idx, rw, int(ring), sink.to(cuda), n_q, pos, o)
    else:
        hb.hca_attend(d, q.to(cuda), rc, cap, rw, int(ring), sink.to(cuda), n_q, pos, o)
    torch.cuda.synchronize()
    kvc64 = _mixed_rows(kvc.double().numpy(), rd)
    win64 = _mixed_rows(win.double().numpy(), rd)
    gi = idx.cpu().numpy() if idx is not None else None
    for b in range(B):
        for i in range(n_q):
            t = pos + i
            V = (t + 1) // m
            wpos = O.window_positions(t, w)
            wr = win64[b][[p % w for p in wpos]] if ring else win64[b][wpos]
            sel = gi[b, i][gi[b, i] >= 0] if kind == "csa" else np.arange(V)
            rows = np.concatenate([wr, kvc64[b][sel]])
            ref = O.attend_output(q[b, i].double().numpy(), rows, sink.double().numpy(), c ** -0.5, t, rd)
            got = o[b, i].double().cpu().numpy()
            err = np.abs(got - ref).max()
            assert err <= 2e-2, f"o[{b},{i}] max-abs {err}"
