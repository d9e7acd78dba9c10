"""GPU parity of each hot-path kernel against the oracle, through the C-ABI.

Small and ragged shapes that span several tiles and a ragged tail; the
full-size workloads are in test_gpu_workloads.py."""
import numpy as np
import pytest
import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth
from oracle import hca_oracle as O
from tests.helpers import TOL, assert_close, check_topk_row, random_idx, rnd, to64

pytestmark = pytest.mark.gpu

F32, BF16 = torch.float32, torch.bfloat16
CODE = {F32: hb.HCA_F32, BF16: hb.HCA_BF16}


# ----------------------------------------------------------------- compression
def _compress_inputs(B, n, width, m, in_dt, seed):
    Ca, Cb, Za, Zb = (rnd((B, n, width), seed, s, in_dt) for s in range(4))
    Ba = rnd((m, width), seed, 4, std=0.5)
    Bb = rnd((m, width), seed, 5, std=0.5)
    return Ca, Cb, Za, Zb, Ba, Bb


def _ref_entries(Ca, Cb, Za, Zb, Ba, Bb, m, overlap, flags, rd, b):
    if overlap:
        e = O.compress_prefill(to64(Ca[b]), to64(Za[b]), to64(Ba), m, to64(Cb[b]), to64(Zb[b]), to64(Bb))
    else:
        e = O.compress_prefill(to64(Ca[b]), to64(Za[b]), to64(Ba), m)
    return O.entry_epilogue(e, m, rd=rd if flags & hb.HCA_COMPRESS_ROPE else 0,
                            norm=bool(flags & hb.HCA_COMPRESS_NORM))


CASES = [
    # overlap, m, width, n, in, out, flags, rd
    (1, 4, 64, 103, F32, F32, 0, 0),
    (1, 4, 64, 103, F32, F32, 3, 16),
    (1, 4, 512, 256, BF16, BF16, 3, 64),
    (1, 4, 64, 201, BF16, BF16, 3, 64),
    (0, 128, 128, 1000, BF16, BF16, 3, 64),
    (0, 128, 512, 300, F32, F32, 1, 0),
    (1, 1, 32, 9, F32, F32, 0, 0),
    (1, 4, 64, 3, F32, F32, 3, 16),          # fewer tokens than one block
]


@pytest.mark.parametrize("overlap,m,width,n,in_dt,out_dt,flags,rd", CASES)
def test_compress_prefill(cuda, overlap, m, width, n, in_dt, out_dt, flags, rd):
    B = 2
    Ca, Cb, Za, Zb, Ba, Bb = _compress_inputs(B, n, width, m, in_dt, seed=m * 7 + width)
    E = n // m
    out = torch.full((B, max(E, 1), width), float("nan"), dtype=out_dt, device=cuda)
    R, Cw = (2 * m, 2 * width) if overlap else (m, width)
    skv = torch.empty(B, R, Cw, device=cuda)
    ssc = torch.empty(B, R, Cw, device=cuda)
    d = hb.compress_desc(B, width, m, overlap, rd, flags, CODE[in_dt], CODE[out_dt])
    # the non-overlapped (HCA) cases go through the hca_compress name of the same call
    hb.csa_compress(d, 0, n, Ca, Cb if overlap else None, Za, Zb if overlap else None, width, n * width,
                    Ba, Bb if overlap else None, None, out, None, max(E, 1), skv, ssc, hca_name=not overlap)
    torch.cuda.synchronize()
    for b in range(B):
        ref = _ref_entries(Ca, Cb, Za, Zb, Ba, Bb, m, overlap, flags, rd, b)
        assert_close(to64(out[b, :E]), ref, TOL[out_dt] if out_dt == F32 else 2e-2, f"entries b={b}")
    # state layout: previous block / tail rows with the bias folded into the logits
    cutoff = E * m
    rem = n - cutoff
    kv, sc = to64(skv), to64(ssc)
    for b in range(B):
        def rows(C, Z, Bias, tok, j):
            return to64(C[b, tok]), to64(Z[b, tok]) + to64(Bias[j])
        for r in range(R):
            if overlap:
                tok, j = ((cutoff - m + r, r) if r < m and cutoff >= m else
                          (cutoff + r - m, r - m) if r >= m and r - m < rem else (None, None))
            else:
                tok, j = (cutoff + r, r) if r < rem else (None, None)
            if tok is None:
                assert (kv[b, r] == 0).all() and np.isneginf(sc[b, r]).all()
                continue
            if overlap:
                cb, zb = rows(Cb, Zb, Bb, tok, j)
                ca, za = rows(Ca, Za, Ba, tok, j)
                np.testing.assert_allclose(kv[b, r], np.concatenate([cb, ca]), rtol=0, atol=0)
                np.testing.assert_allclose(sc[b, r], np.concatenate([zb, za]), rtol=1e-6, atol=1e-6)
            else:
                ca, za = rows(Ca, Za, Ba, tok, j)
                np.testing.assert_allclose(kv[b, r], ca, rtol=0, atol=0)
                np.testing.assert_allclose(sc[b, r], za, rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("overlap,m,width,n0,steps", [(1, 4, 64, 10, 23), (0, 8, 128, 5, 30), (1, 4, 512, 64, 9),
                                                      (0, 128, 128, 100, 160)])
def test_compress_decode_matches_prefill(cuda, overlap, m, width, n0, steps):
    """prefill(n0) then one decode step per token == prefill(n0 + steps)."""
    B = 2
    n = n0 + steps
    Ca, Cb, Za, Zb, Ba, Bb = _compress_inputs(B, n, width, m, F32, seed=31 + m)
    cap = n // m + 2
    out = torch.full((B, cap, width), float("nan"), device=cuda)
    R, Cw = (2 * m, 2 * width) if overlap else (m, width)
    skv = torch.empty(B, R, Cw, device=cuda)
    ssc = torch.empty(B, R, Cw, device=cuda)
    flags, rd = 3, 16
    d = hb.compress_desc(B, width, m, overlap, rd, flags, hb.HCA_F32, hb.HCA_F32)
    ov = lambda t: t if overlap else None
    hb.csa_compress(d, 0, n0, Ca[:, :n0].contiguous(), ov(Cb[:, :n0].contiguous()), Za[:, :n0].contiguous(),
                    ov(Zb[:, :n0].contiguous()), width, n0 * width, Ba, ov(Bb), None, out, None, cap, skv, ssc)
    for pos in range(n0, n):
        row = lambda t: t[:, pos].contiguous()
        hb.csa_compress(d, pos, 1, row(Ca), ov(row(Cb)), row(Za), ov(row(Zb)), width, width, Ba, ov(Bb), None,
                        out, None, cap, skv, ssc)
    torch.cuda.synchronize()
    E = n // m
    for b in range(B):
        ref = _ref_entries(Ca, Cb, Za, Zb, Ba, Bb, m, overlap, flags, rd, b)
        assert_close(to64(out[b, :E]), ref, 1e-4, f"entries b={b}")


def test_compress_fp8_output(cuda):
    B, n, width, m, rd = 2, 64, 64, 4, 64
    Ca, Cb, Za, Zb, Ba, Bb = _compress_inputs(B, n, width, m, F32, seed=77)
    E = n // m
    out = torch.zeros(B, E, width, dtype=torch.uint8, device=cuda)
    scale = torch.zeros(B, E, device=cuda)
    d = hb.compress_desc(B, width, m, 1, rd, 3, hb.HCA_F32, hb.HCA_FP8E4M3)
    hb.csa_compress(d, 0, n, Ca, Cb, Za, Zb, width, n * width, Ba, Bb, None, out, scale, E, None, None)
    torch.cuda.synchronize()
    mism = 0
    for b in range(B):
        ref = _ref_entries(Ca, Cb, Za, Zb, Ba, Bb, m, 1, 3, rd, b)
        ref_scale = np.abs(ref).max(1) / 448.0
        np.testing.assert_allclose(to64(scale[b]), ref_scale, rtol=1e-5)
        ref_codes = O.e4m3_encode(ref / to64(scale[b])[:, None])
        got = out[b].cpu().numpy()
        diff = got != ref_codes
        mism += diff.sum()
        # a mismatch may only be a rounding-boundary neighbour
        dec_g, dec_r = O.e4m3_to_f64(got), O.e4m3_to_f64(ref_codes)
        assert (np.abs(dec_g - dec_r)[diff] <= np.abs(dec_r[diff]) * 0.13 + 2 ** -9).all()
    assert mism <= 0.002 * out.numel()


# ----------------------------------------------------------------- index + top-k
IDX_CASES = [
    # B, n_q, start_pos, m, k, n_hI, c_I, q dtype, key dtype
    (1, 64, 0, 4, 16, 4, 32, F32, "f32"),
    (2, 37, 0, 4, 8, 8, 64, BF16, "bf16"),
    (1, 300, 0, 4, 64, 8, 64, BF16, "bf16"),
    (3, 1, 50000, 4, 512, 8, 64, BF16, "bf16"),      # decode-like: chunked two-pass select
    (2, 1, 70001, 4, 1024, 8, 64, BF16, "fp8"),
    (2, 5, 1000, 4, 40, 8, 64, BF16, "fp8"),
    (1, 40, 0, 4, 16, 8, 64, BF16, "fp8"),            # prefill-shaped blocks with fp8 keys
    (2, 530, 100, 4, 64, 8, 64, BF16, "bf16"),        # several 16-query blocks, ragged tail
]


@pytest.mark.parametrize("B,n_q,start_pos,m,k,n_hI,c_I,qdt,kdt", IDX_CASES)
def test_index_topk(cuda, B, n_q, start_pos, m, k, n_hI, c_I, qdt, kdt):
    seed = n_q + k
    E = (start_pos + n_q) // m
    cap = E + 3
    qI = rnd((B, n_q, n_hI, c_I), seed, 1, qdt)
    wI = rnd((B, n_q, n_hI), seed, 2, std=c_I ** -0.5 * n_hI ** -0.5)
    KIf = synth.normal((B, cap, c_I), seed, 3)
    KI_scale = None
    if kdt == "fp8":
        KI, KI_scale = synth.fp8_rows(KIf)
        KI, KI_scale = KI.to(cuda), KI_scale.to(cuda)
        KI64 = O.e4m3_to_f64(KI.cpu().numpy()) * to64(KI_scale)[..., None]
        kcode = hb.HCA_FP8E4M3
    else:
        kt = F32 if kdt == "f32" else BF16
        KI = KIf.to(kt).to(cuda)
        KI64 = to64(KI)
        kcode = CODE[kt]
    d = hb.attn_desc(B, 4, 64, 16, 8, m, k=k, n_hI=n_hI, c_I=c_I, rd_I=16, dtype=CODE[qdt], idx_key_dtype=kcode)
    ws = torch.empty(max(hb.csa_index_topk_workspace_size(d, n_q, start_pos), 16), dtype=torch.uint8, device=cuda)
    idx = torch.full((B, n_q, k), -7, dtype=torch.int32, device=cuda)
    scores = torch.full((B, n_q, max(E, 1)), float("nan"), device=cuda)
    hb.csa_index_topk(d, qI, wI, KI, KI_scale, cap, n_q, start_pos, idx, scores, max(E, 1), ws)
    torch.cuda.synchronize()
    q64, w64, gi, gs = to64(qI), to64(wI), idx.cpu().numpy(), to64(scores)
    ties = 0
    for b in range(B):
        for i in range(n_q):
            t = start_pos + i
            V = (t + 1) // m
            ref = O.index_scores(q64[b, i], w64[b, i], KI64[b], V)
            if V:
                np.testing.assert_allclose(gs[b, i, :V], ref, rtol=2e-5, atol=2e-5 * np.abs(ref).max())
            ties += check_topk_row(gi[b, i], ref, k, V)


TIE_CASES = [
    # B, n_q, start_pos, k, key dtype.  Many rows of up to 32768 keys: one CTA
    # per row (128..1024 threads); few rows all longer than k: a cluster of
    # CTAs per row (up to 262144 keys); many long rows: a cluster per row
    # segment (the 64 rows of 50000 keys)
    (2, 64, 0, 64, "bf16"),
    (2, 8, 16000, 64, "bf16"),
    (3, 1, 131071, 512, "bf16"),
    (2, 1, 163839, 512, "bf16"),
    (1, 2, 300000, 512, "bf16"),
    (1, 64, 200000, 512, "bf16"),
    (2, 1, 1048575, 1024, "fp8"),
]


@pytest.mark.parametrize("B,n_q,start_pos,k,kdt", TIE_CASES)
def test_index_topk_exact_ties(cuda, B, n_q, start_pos, k, kdt):
    """Entries share one of three index keys, so each row holds three score
    values repeated thousands of times: the selection must take the whole
    upper classes and then the lowest indices of the class that the k-th
    score falls in (Eq.(17), ties to the lower index), across every CTA of
    the cluster and every segment of the row."""
    m, n_hI, c_I = 4, 8, 64
    E = (start_pos + n_q) // m
    cap = E + 1
    base = synth.normal((B, 3, c_I), 77, 1)
    s_ids = np.arange(cap)
    cls = np.where(s_ids % 97 == 5, 0, 1 + (s_ids * 7 // 3) % 2)   # a rare class and two common ones
    KIf = base[:, torch.from_numpy(cls)]
    qI = rnd((B, n_q, n_hI, c_I), 78, 1, BF16)
    wI = rnd((B, n_q, n_hI), 78, 2, std=c_I ** -0.5 * n_hI ** -0.5)
    KI_scale = None
    if kdt == "fp8":
        KI, KI_scale = synth.fp8_rows(KIf)
        KI, KI_scale = KI.to(cuda), KI_scale.to(cuda)
        KI64 = O.e4m3_to_f64(KI.cpu().numpy()) * to64(KI_scale)[..., None]
        kcode = hb.HCA_FP8E4M3
    else:
        KI = KIf.to(BF16).to(cuda)
        KI64 = to64(KI)
        kcode = CODE[BF16]
    d = hb.attn_desc(B, 4, 64, 16, 8, m, k=k, n_hI=n_hI, c_I=c_I, rd_I=16, dtype=CODE[BF16], idx_key_dtype=kcode)
    ws = torch.empty(hb.csa_index_topk_workspace_size(d, n_q, start_pos), dtype=torch.uint8, device=cuda)
    idx = torch.full((B, n_q, k), -7, dtype=torch.int32, device=cuda)
    hb.csa_index_topk(d, qI, wI, KI, KI_scale, cap, n_q, start_pos, idx, None, 0, ws)
    torch.cuda.synchronize()
    q64, w64, gi = to64(qI), to64(wI), idx.cpu().numpy()
    for b in range(B):
        for i in range(n_q):
            V = (start_pos + i + 1) // m
            ref = O.index_scores(q64[b, i], w64[b, i], KI64[b], V)
            vals = np.unique(ref)
            if len(vals) > 1:   # the classes are far apart, so fp32 cannot reorder them
                assert np.diff(vals).min() > 1e-3 * np.abs(vals).max()
            np.testing.assert_array_equal(gi[b, i], O.topk_select(ref, k))


POW2_CASES = [
    # start_pos (one query, m = 4): a cluster of 8 CTAs (32768 entries) and of 4 (12500)
    131071,
    49999,
]


@pytest.mark.parametrize("start_pos", POW2_CASES)
def test_index_topk_pow2_classes(cuda, start_pos):
    """Every index key is one key scaled by a power of two, so with positive
    head weights each score is that key's score times the same power of two,
    exactly: the scores form classes of equal values one binade apart.  Row 0
    puts the k-th score inside a class of 1500 entries scattered over the
    row (ties across CTAs, resolved towards the lower index, Eq.(17)); row 1
    ends the top k exactly at a class boundary."""
    B, n_q, m, k, n_hI, c_I = 2, 1, 4, 512, 8, 64
    E = (start_pos + n_q) // m
    cap = E + 1
    rng = np.random.default_rng(start_pos)
    expo = np.zeros((B, cap), dtype=np.int64)
    for b, sizes in enumerate(((100, 300, 1500), (100, 412))):
        perm = rng.permutation(E)
        e = rng.integers(0, 9, size=cap)          # the bulk: exponents 0..8
        at = 0
        for j, n in enumerate(sizes):             # the top classes: exponents 11, 10, 9
            e[perm[at:at + n]] = 11 - j
            at += n
        expo[b] = e
    base = synth.normal((B, 1, c_I), 91, 1).to(BF16).float()
    KI = (base * torch.from_numpy(np.exp2(expo)).float()[..., None]).to(BF16).to(cuda)
    qI = rnd((B, n_q, n_hI, c_I), 91, 2, BF16)
    wI = rnd((B, n_q, n_hI), 91, 3, std=c_I ** -0.5).abs().to(cuda)
    d = hb.attn_desc(B, 4, 64, 16, 8, m, k=k, n_hI=n_hI, c_I=c_I, rd_I=16, dtype=CODE[BF16],
                     idx_key_dtype=CODE[BF16])
    ws = torch.empty(hb.csa_index_topk_workspace_size(d, n_q, start_pos), dtype=torch.uint8, device=cuda)
    idx = torch.full((B, n_q, k), -7, dtype=torch.int32, device=cuda)
    hb.csa_index_topk(d, qI, wI, KI, None, cap, n_q, start_pos, idx, None, 0, ws)
    torch.cuda.synchronize()
    q64, w64, K64, gi = to64(qI), to64(wI), to64(KI), idx.cpu().numpy()
    for b in range(B):
        ref = O.index_scores(q64[b, 0], w64[b, 0], K64[b], E)
        assert ref.max() > 0 and len(np.unique(ref)) <= 12
        np.testing.assert_array_equal(gi[b, 0], O.topk_select(ref, k))


# ----------------------------------------------------------------- attention
ATT_CASES = [
    # kind, dtype, B, n_q, n_h, c, rd, w, m, k
    ("csa", F32, 1, 70, 4, 64, 16, 32, 4, 16),
    ("hca", F32, 2, 300, 4, 64, 16, 32, 128, 0),
    ("csa", BF16, 1, 150, 64, 512, 64, 37, 4, 100),
    ("hca", BF16, 2, 700, 16, 128, 64, 128, 128, 0),
    ("csa", BF16, 2, 90, 64, 512, 64, 128, 4, 512),
    ("hca", BF16, 1, 260, 64, 512, 64, 128, 4, 0),
    ("csa", BF16, 1, 40, 16, 256, 32, 0, 1, 64),      # no window, ratio 1
]


def _run_attend(kind, dt, B, n_q, n_h, c, rd, w, m, k, cuda, start_pos=0, ring=False, seed=5, max_ctas=0):
    cap = (start_pos + n_q) // m + 2
    q = rnd((B, n_q, n_h, c), seed, 1, dt)
    kv_comp = rnd((B, cap, c), seed, 2, dt)
    kv_win = rnd((B, w if ring else n_q, c), seed, 3, dt)
    sink = rnd((n_h,), seed, 4)
    idx = random_idx(B, n_q, start_pos, m, k, seed) if kind == "csa" else None
    o = torch.full((B, n_q, n_h, c), float("nan"), dtype=dt, device=cuda)
    d = hb.attn_desc(B, n_h, c, rd, w, m, k=k, dtype=CODE[dt], max_ctas=max_ctas)
    if kind == "csa":
        hb.csa_attend(d, q, kv_comp, cap, idx, kv_win, ring, sink, n_q, start_pos, o)
    else:
        hb.hca_attend(d, q, kv_comp, cap, kv_win, ring, sink, n_q, start_pos, o)
    torch.cuda.synchronize()
    return q, kv_comp, kv_win, sink, idx, o


def _ref_attend(kind, q, kv_comp, kv_win, sink, idx, b, i, start_pos, w, m, k, rd, ring):
    t = start_pos + i
    V = (t + 1) // m
    c = q.shape[-1]
    wpos = O.window_positions(t, w) if w else np.zeros(0, int)
    win = to64(kv_win[b])
    wrows = win[[p % w for p in wpos]] if ring else win[wpos]
    comp = to64(kv_comp[b])
    if kind == "csa":
        sel = idx[b, i].cpu().numpy()
        sel = sel[:min(k, V)]
        crows = comp[sel[sel >= 0]]
    else:
        crows = comp[:V]
    rows = np.concatenate([wrows.reshape(-1, c), crows], 0)
    return O.attend_output(to64(q[b, i]), rows, to64(sink), c ** -0.5, t, rd)


@pytest.mark.parametrize("kind,dt,B,n_q,n_h,c,rd,w,m,k", ATT_CASES)
def test_attend_prefill(cuda, kind, dt, B, n_q, n_h, c, rd, w, m, k):
    q, kv_comp, kv_win, sink, idx, o = _run_attend(kind, dt, B, n_q, n_h, c, rd, w, m, k, cuda)
    tol = TOL[dt]
    rng = np.random.default_rng(0)
    toks = sorted(set([0, 1, n_q - 1] + list(rng.integers(0, n_q, size=min(n_q, 40)))))
    for b in range(B):
        for i in toks:
            ref = _ref_attend(kind, q, kv_comp, kv_win, sink, idx, b, i, 0, w, m, k, rd, False)
            assert_close(to64(o[b, i]), ref, tol, f"o[{b},{i}]")


@pytest.mark.parametrize("kind,pos", [("csa", 1001), ("csa", 1003), ("hca", 5000), ("csa", 60)])
def test_attend_decode_ring(cuda, kind, pos):
    B, n_h, c, rd, w = 3, 64, 512, 64, 128
    m, k = (4, 512) if kind == "csa" else (128, 0)
    q, kv_comp, kv_win, sink, idx, o = _run_attend(kind, BF16, B, 1, n_h, c, rd, w, m, k, cuda,
                                                   start_pos=pos, ring=True)
    for b in range(B):
        ref = _ref_attend(kind, q, kv_comp, kv_win, sink, idx, b, 0, pos, w, m, k, rd, True)
        assert_close(to64(o[b, 0]), ref, 2e-2, f"o[{b}]")


@pytest.mark.parametrize("kind,B,pos", [("csa", 5, 1700), ("hca", 2, 100000), ("csa", 32, 131071)])
def test_attend_decode_cluster_merge(cuda, kind, B, pos):
    """Decode with few sequences: each query's key tiles are split over the
    CTAs of one cluster (here 4 splits of 9 tiles, the last one empty; 7
    splits; the 128K batch) and merged through distributed shared memory."""
    n_h, c, rd, w = 64, 512, 64, 128
    m, k = (4, 512) if kind == "csa" else (128, 0)
    q, kv_comp, kv_win, sink, idx, o = _run_attend(kind, BF16, B, 1, n_h, c, rd, w, m, k, cuda,
                                                   start_pos=pos, ring=True)
    for b in range(0, B, max(1, B // 4)):
        ref = _ref_attend(kind, q, kv_comp, kv_win, sink, idx, b, 0, pos, w, m, k, rd, True)
        assert_close(to64(o[b, 0]), ref, 2e-2, f"o[{b}]")


@pytest.mark.parametrize("kind,B,pos,max_ctas", [("hca", 32, 131071, 64), ("hca", 32, 131071, 32),
                                                 ("hca", 2, 100000, 6), ("csa", 5, 1700, 12)])
def test_attend_decode_cta_budget(cuda, kind, B, pos, max_ctas):
    """A CTA budget (max_ctas) bounds the splits per query -- 2, 1, 3 and 2
    here instead of 4, 4, 7 and 4 -- without changing what is computed."""
    n_h, c, rd, w = 64, 512, 64, 128
    m, k = (4, 512) if kind == "csa" else (128, 0)
    q, kv_comp, kv_win, sink, idx, o = _run_attend(kind, BF16, B, 1, n_h, c, rd, w, m, k, cuda,
                                                   start_pos=pos, ring=True, max_ctas=max_ctas)
    for b in range(0, B, max(1, B // 4)):
        ref = _ref_attend(kind, q, kv_comp, kv_win, sink, idx, b, 0, pos, w, m, k, rd, True)
        assert_close(to64(o[b, 0]), ref, 2e-2, f"o[{b}]")


def test_attend_prefill_cta_budget(cuda):
    """Prefill under a budget of 5 CTAs: the persistent grid shrinks to 5 and
    each CTA works through 30 of the 150 query units."""
    kind, dt, B, n_q, n_h, c, rd, w, m, k = "csa", BF16, 1, 150, 64, 512, 64, 37, 4, 100
    q, kv_comp, kv_win, sink, idx, o = _run_attend(kind, dt, B, n_q, n_h, c, rd, w, m, k, cuda, max_ctas=5)
    for i in (0, 1, 77, n_q - 1):
        ref = _ref_attend(kind, q, kv_comp, kv_win, sink, idx, 0, i, 0, w, m, k, rd, False)
        assert_close(to64(o[0, i]), ref, TOL[dt], f"o[0,{i}]")


def test_attend_is_deterministic(cuda):
    runs = [_run_attend("csa", BF16, 1, 64, 64, 512, 64, 128, 4, 128, cuda)[-1] for _ in range(2)]
    assert torch.equal(runs[0], runs[1])


GROUP_CASES = [
    # B, n_q, n_h, c, rd, w, m, start_pos, max_ctas
    (2, 701, 16, 128, 64, 128, 128, 0, 0),       # 8 queries on 128 rows, the last group of 5
    (1, 603, 32, 256, 64, 100, 16, 0, 0),        # 4 on 128 rows; the visible entries change every 16 tokens
    (1, 400, 64, 128, 64, 128, 16, 0, 0),        # 2 on 128 rows
    (2, 1205, 16, 128, 64, 128, 128, 3000, 0),   # a chunk after 3000 tokens: the window's halo rows
    (2, 600, 16, 128, 64, 5, 128, 0, 0),         # 12-key windows: the tile's upper 32 keys are all masked
    (2, 600, 16, 128, 64, 0, 128, 0, 0),         # no window: queries before the first entry see no key
    (2, 450, 16, 128, 64, 128, 128, 1000, 0),    # 57 groups of 8 per sequence are too few: 4 on 64 rows
    (1, 599, 16, 512, 64, 37, 4, 77, 0),         # c = 512: 4 on 64 rows; short window, m = 4
    (1, 399, 16, 512, 64, 37, 4, 77, 0),         # 100 groups leave SMs idle: one query per unit
]


@pytest.mark.parametrize("B,n_q,n_h,c,rd,w,m,start_pos,max_ctas", GROUP_CASES)
def test_attend_query_groups(cuda, B, n_q, n_h, c, rd, w, m, start_pos, max_ctas):
    """All-entries (HCA) attention over many queries runs 128 / n_h (c <= 256)
    or 64 / n_h consecutive queries per unit: the union of their key sets is
    gathered once and each query masks the keys outside its own window and
    visible entries (juejin "DeepSeek-V4 技术报告简要解读" §2.3.2 Eq.(20)-(23)).
    Every query is compared with the oracle over its own rows."""
    seed = 8
    halo = min(w - 1, start_pos)
    win_tok0 = start_pos - halo
    cap = (start_pos + n_q) // m + 1
    q = rnd((B, n_q, n_h, c), seed, 1, BF16)
    kv_comp = rnd((B, cap, c), seed, 2, BF16)
    kv_win = rnd((B, n_q + halo, c), seed, 3, BF16)
    sink = rnd((n_h,), seed, 4)
    o = torch.full((B, n_q, n_h, c), float("nan"), dtype=BF16, device=cuda)
    d = hb.attn_desc(B, n_h, c, rd, w, m, dtype=hb.HCA_BF16, max_ctas=max_ctas)
    hb.hca_attend(d, q, kv_comp, cap, kv_win, False, sink, n_q, start_pos, o)
    torch.cuda.synchronize()
    s64, go = to64(sink), to64(o)
    for b in range(B):
        q64, comp, win = to64(q[b]), to64(kv_comp[b]), to64(kv_win[b])
        for i in range(n_q):
            t = start_pos + i
            wpos = O.window_positions(t, w)
            rows = np.concatenate([win[wpos - win_tok0], comp[:(t + 1) // m]], 0)
            ref = O.attend_output(q64[i], rows, s64, c ** -0.5, t, rd)
            assert_close(go[b, i], ref, 2e-2, f"o[{b},{i}]")
