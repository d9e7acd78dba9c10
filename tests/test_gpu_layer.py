"""GPU parity of whole layers: prefill from hidden states (hybrid_layer_forward)
and single-token decode over a cache (hybrid_decode_step), against the oracle."""
import numpy as np
import pytest
import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth, workloads
from long_context_compressed_hca_b200.layer import CacheHandle, LayerHandle, TokenInputs
from oracle import hca_oracle as O
from tests.helpers import (GAP, GAP_LAYER_BF16, TOL, assert_close, check_selection_bound, check_topk_row,
                           oracle_attend_over, to64)

pytestmark = pytest.mark.gpu
F32, BF16 = torch.float32, torch.bfloat16


def _w64(W):
    return {k: to64(v) for k, v in W.items()}


def _run_layer(wl, L, dt, cuda, n=None, cache=None, keep_ws=False):
    n = n or wl.n
    W = synth.layer_weights(L, wl.d, wl.d_c, wl.seed, dt)
    H = synth.hidden_states(wl.B, n, wl.d, wl.seed, dt)
    lh = LayerHandle(L, W, wl.d, wl.d_c, dt, wl.B, device=cuda)
    ws = torch.empty(hb.layer_workspace_size(lh.struct, n), dtype=torch.uint8, device=cuda)
    o = torch.full((wl.B, n, L.n_h, L.c), float("nan"), dtype=dt, device=cuda)
    hb.hybrid_layer_forward(lh.struct, H.to(cuda), n, cache.struct if cache else None, o, ws)
    torch.cuda.synchronize()
    if keep_ws:
        return W, H, o, lh, ws
    return W, H, o


class PrefillIntermediates:
    """The GPU's stored intermediates of one hybrid_layer_forward call (no
    cache), read through hybrid_workspace_map."""

    def __init__(self, lh, ws, L, B, n, dt):
        mp = hb.workspace_map(lh.struct, n)
        E = max(n // L.m, 1)
        v = lambda key, shape, d: hb.ws_view(ws, mp[key], shape, d) if mp[key] is not None else None
        self.q = v("q", (B, n, L.n_h, L.c), dt)
        self.kv_win = v("kv_win", (B, n, L.c), dt)
        self.kv_comp = v("kv_comp", (B, E, L.c), dt)
        self.idx = v("idx", (B, n, L.k), torch.int32) if L.kind == "csa" else None
        if L.kind == "csa":
            self.qI = v("qI", (B, n, L.n_hI, L.c_I), dt)
            self.wI = v("wI", (B, n, L.n_hI), torch.float32)
            self.KI = v("key_I", (B, E, L.c_I), dt)


def check_prefill_tokens(L, W64, H64, gi: PrefillIntermediates, o, b, toks, d_c, tol):
    """Every sampled token of sequence b, with nothing skipped:
      - the stored intermediates (queries, window rows, compressed entries,
        indexer queries / keys) against the oracle's;
      - CSA: the GPU's top-k against the oracle's selection over the GPU's
        stored index operands (bit-exact where the k-th/(k+1)-th gap exceeds
        1e-3, else within the tie), and bounded against the fp64 scores;
      - the output against the oracle's attention over the GPU's selection.
    Returns (tokens checked, near ties among them)."""
    ref = O.layer_prefill(H64, W64, L, d_c, tokens=toks, return_intermediates=True)
    E = (int(toks.max()) + 1) // L.m
    assert_close(to64(gi.q[b, toks]), ref["q"], tol, "q")
    need = sorted(ref["kv_win"])
    assert_close(to64(gi.kv_win[b, need]), np.stack([ref["kv_win"][p] for p in need]), tol, "window rows")
    if E:
        assert_close(to64(gi.kv_comp[b, :E]), ref["kv_comp"][:E], tol, "kv_comp")
    sink = W64["sink"]
    ties = 0
    if L.kind == "csa":
        if E:
            assert_close(to64(gi.KI[b, :E]), ref["KI"][:E], tol, "key_I")
        assert_close(to64(gi.qI[b, toks]), ref["qI"], tol, "qI")
        wref = ref["wI"]
        assert_close(to64(gi.wI[b, toks]), wref, 1e-2 * np.abs(wref).max(), "wI")
        KIg = to64(gi.KI[b])
        idx = gi.idx[b, toks].cpu().numpy()
        qIg, wIg = to64(gi.qI[b, toks]), to64(gi.wI[b, toks])
    for j, t in enumerate(toks):
        t = int(t)
        V = (t + 1) // L.m
        sel = None
        same_sel = True
        if L.kind == "csa":
            s_shared = O.index_scores(qIg[j], wIg[j], KIg, V)
            ties += check_topk_row(idx[j], s_shared, L.k, V)
            delta = check_selection_bound(idx[j], ref["scores"][j], s_shared, L.k, V)
            sel = idx[j]
            if V > L.k:
                srt = np.sort(ref["scores"][j])[::-1]
                # the fp64 selection is provably the GPU's only where the k-th /
                # (k+1)-th gap exceeds what the stored operands' rounding can move
                same_sel = srt[L.k - 1] - srt[L.k] > 2 * delta
        else:
            sel = np.arange(V)
        wrows = [ref["kv_win"][p] for p in O.window_positions(t, L.w)]
        o_ref = oracle_attend_over(ref["q"][j], wrows, ref["kv_comp"], sel, sink, L.c, t, L.rd)
        assert_close(to64(o[b, t]), o_ref, tol, f"o[{b},{t}]")
        if same_sel:
            assert_close(to64(o[b, t]), ref["o"][j], tol, f"o[{b},{t}] (oracle selection)")
    return len(toks), ties


def test_layer_tiny_csa_fp32(cuda):
    wl = workloads.TINY_CSA
    L = wl.layers[0]
    W, H, o, lh, ws = _run_layer(wl, L, F32, cuda, keep_ws=True)
    gi = PrefillIntermediates(lh, ws, L, wl.B, wl.n, F32)
    checked, ties = check_prefill_tokens(L, _w64(W), to64(H[0]), gi, o, 0, np.arange(wl.n), wl.d_c, TOL[F32])
    print(f"tiny CSA fp32: {checked} tokens checked, {ties} near ties (checked within the tie)")


def test_layer_hca_bf16(cuda):
    wl = workloads.HCA_PREFILL
    L = wl.layers[0]
    n = 2048   # the oracle over all 8192 tokens is covered by the full-size test
    W, H, o, lh, ws = _run_layer(wl, L, BF16, cuda, n=n, keep_ws=True)
    gi = PrefillIntermediates(lh, ws, L, wl.B, n, BF16)
    W64 = _w64(W)
    for b in range(wl.B):
        toks = np.unique(np.concatenate([np.arange(0, 300), np.arange(n - 300, n),
                                         np.random.default_rng(b).integers(0, n, 200)]))
        check_prefill_tokens(L, W64, to64(H[b]), gi, o, b, toks, wl.d_c, TOL[BF16])


def test_layer_csa_bf16_small(cuda):
    """CSA layer with the 64K workload's attention shapes at 4096 tokens, where
    queries past token 2047 see more than k = 512 entries, so the selection
    drops entries on every such token."""
    wl = workloads.CSA_PREFILL.with_(n=4096, d=512, d_c=256)
    L = wl.layers[0]
    W, H, o, lh, ws = _run_layer(wl, L, BF16, cuda, keep_ws=True)
    gi = PrefillIntermediates(lh, ws, L, wl.B, wl.n, BF16)
    toks = np.unique(np.concatenate([np.arange(0, 40), np.arange(2040, 2060), np.arange(wl.n - 40, wl.n),
                                     np.random.default_rng(3).integers(0, wl.n, 80)]))
    checked, ties = check_prefill_tokens(L, _w64(W), to64(H[0]), gi, o, 0, toks, wl.d_c, TOL[BF16])
    assert sum((int(t) + 1) // L.m > L.k for t in toks) >= 60
    print(f"CSA bf16 4096 tokens: {checked} tokens checked, {ties} near ties (checked within the tie)")


def test_prefill_then_decode_matches_longer_prefill(cuda):
    """prefill(n) + decode steps n..n+r-1 reproduces prefill(n+r) at those tokens
    (the cache and compressor states carry everything decode needs)."""
    wl = workloads.TINY_CSA
    L = wl.layers[0]
    n, r = 200, 13
    W = synth.layer_weights(L, wl.d, wl.d_c, wl.seed, F32, bias_std=0.3)
    H = synth.hidden_states(wl.B, n + r, wl.d, wl.seed, F32)
    lh = LayerHandle(L, W, wl.d, wl.d_c, F32, wl.B, device=cuda)
    cache = CacheHandle(L, wl.B, cap=64, dtype=F32, device=cuda)
    ws = torch.empty(hb.layer_workspace_size(lh.struct, n), dtype=torch.uint8, device=cuda)
    o = torch.empty(wl.B, n, L.n_h, L.c, device=cuda)
    hb.hybrid_layer_forward(lh.struct, H[:, :n].contiguous().to(cuda), n, cache.struct, o, ws)
    # the decode inputs are the oracle-independent projections of the new tokens,
    # computed here with torch in fp64 from the same weights (input preparation)
    W64 = {k: v.double() for k, v in W.items()}
    Hd = H.double()
    ref = O.layer_prefill(to64(H[0]), _w64(W), L, wl.d_c, return_intermediates=True)
    dws = torch.empty(max(hb.decode_workspace_size(lh.struct, n + r), 16), dtype=torch.uint8, device=cuda)
    for pos in range(n, n + r):
        h = Hd[:, pos]
        comp = torch.cat([h @ W64[k].T for k in ("W_aKV", "W_bKV", "W_aZ", "W_bZ")], -1)
        compI = torch.cat([h @ W64[k].T for k in ("W_IaKV", "W_IbKV", "W_IaZ", "W_IbZ")], -1)
        x = TokenInputs(q=torch.from_numpy(ref["q"][pos]).float()[None].to(cuda).contiguous(),
                        kv=torch.from_numpy(ref["kv_win"][pos]).float()[None].to(cuda).contiguous(),
                        comp=comp.float().to(cuda).contiguous(), compI=compI.float().to(cuda).contiguous(),
                        qI=torch.from_numpy(ref["qI"][pos]).float()[None].to(cuda).contiguous(),
                        wI=torch.from_numpy(ref["wI"][pos]).float()[None].to(cuda).contiguous())
        od = torch.empty(wl.B, L.n_h, L.c, device=cuda)
        hb.hybrid_decode_step(lh.struct, x.struct, cache.struct, pos, od, dws)
        torch.cuda.synchronize()
        if O.topk_gap(ref["scores"][pos], L.k) > GAP:
            assert_close(to64(od[0]), ref["o"][pos], 1e-4, f"decode o[{pos}]")
    # emitted entries equal the prefill's entries
    E = (n + r) // L.m
    assert_close(to64(cache.kv_comp[0, :E]), ref["kv_comp"][:E], 1e-4, "kv_comp")
    assert_close(to64(cache.key_I[0, :E]), ref["KI"][:E], 1e-4, "key_I")


# ----------------------------------------------------------------- decode step over a synthetic cache
def _fill_state(state_kv, state_score, overlap, m, width, prev, cur, Ba, Bb):
    """Write the ABI's compressor-state layout from raw rows (test-side input
    preparation): prev = (Cb, Zb) of the previous block, cur = (Ca, Cb, Za, Zb)
    of the current block's earlier tokens."""
    kv = torch.zeros_like(state_kv)
    sc = torch.full_like(state_score, float("-inf"))
    if overlap:
        if prev is not None:
            Cb, Zb = prev
            kv[:, :m, :width] = Cb
            sc[:, :m, :width] = Zb + Bb[None]
            kv[:, :m, width:] = 7.0          # unused half of the previous block
            sc[:, :m, width:] = 3.0
        Ca, Cb, Za, Zb = cur
        j = Ca.shape[1]
        kv[:, m:m + j, :width] = Cb
        sc[:, m:m + j, :width] = Zb + Bb[None, :j]
        kv[:, m:m + j, width:] = Ca
        sc[:, m:m + j, width:] = Za + Ba[None, :j]
    else:
        Ca, _, Za, _ = cur
        j = Ca.shape[1]
        kv[:, :j] = Ca
        sc[:, :j] = Za + Ba[None, :j]
    state_kv.copy_(kv)
    state_score.copy_(sc)


def _bf16_round(x):
    return torch.from_numpy(np.asarray(x)).to(BF16).double().numpy()


def _mixed(x64, rd):
    """Rows as a reader of the mixed-precision KV format sees them (the oracle's
    own quantisation of the same bf16 rows)."""
    return O.kv_row_dequant(*O.kv_row_quant(np.asarray(x64, np.float64), rd))


def run_decode_case(cuda, L, B, pos, idx_key_dtype, seed, kv_mixed=False):
    c, m, w = L.c, L.m, L.w
    csa = L.kind == "csa"
    dt = BF16
    cap = pos // m + 4
    Ecur = pos // m                          # complete entries before this token
    W = synth.layer_weights(L, 256, 64, seed, dt, bias_std=0.5)
    lh = LayerHandle(L, W, 256, 64, dt, B, idx_key_dtype=idx_key_dtype, device=cuda, kv_mixed=kv_mixed)
    cache = CacheHandle(L, B, cap, dt, idx_key_dtype=idx_key_dtype, device=cuda, kv_mixed=kv_mixed)
    g = lambda shape, s, std=1.0, d=torch.float32: synth.normal(shape, seed, s, std=std, dtype=d)
    gd = lambda shape, s, d=torch.float32: synth.normal_on(cuda, shape, seed, s, dtype=d)
    kvc_rows = gd((B, cap, c), 100, d=dt)
    win_rows = g((B, w, c), 101, d=dt).to(cuda)
    if kv_mixed:
        hb.kv_quant_mixed(kvc_rows, hb.HCA_BF16, B * cap, c, L.rd, cache.kv_comp)
        hb.kv_quant_mixed(win_rows, hb.HCA_BF16, B * w, c, L.rd, cache.win)
    else:
        cache.kv_comp.copy_(kvc_rows)
        cache.win.copy_(win_rows)
    j = pos % m
    raw = {nm: g((B, m, c), 102 + i) for i, nm in enumerate(("pCb", "pZb", "Ca", "Cb", "Za", "Zb"))}
    Ba, Bb = (W["B_a"], W["B_b"]) if csa else (W["B"], None)
    _fill_state(cache.state_kv, cache.state_score, L.overlap, m, c,
                (raw["pCb"], raw["pZb"]) if (L.overlap and Ecur > 0) else None,
                tuple(raw[k][:, :j] for k in ("Ca", "Cb", "Za", "Zb")), Ba.float(),
                Bb.float() if Bb is not None else None)
    x = dict(q=g((B, L.n_h, c), 110, d=dt), kv=g((B, c), 111, d=dt), comp=g((B, (4 if csa else 2) * c), 112))
    if csa:
        cI = L.c_I
        KIf = gd((B, cap, cI), 120)
        if idx_key_dtype == "fp8":
            kb, ks = synth.fp8_rows(KIf)
            cache.key_I.copy_(kb)
            cache.key_I_scale.copy_(ks)
        else:
            cache.key_I.copy_(KIf.to(dt))
        rawI = {nm: g((B, m, cI), 130 + i) for i, nm in enumerate(("pCb", "pZb", "Ca", "Cb", "Za", "Zb"))}
        _fill_state(cache.stateI_kv, cache.stateI_score, L.overlap, m, cI,
                    (rawI["pCb"], rawI["pZb"]) if Ecur > 0 else None,
                    tuple(rawI[k][:, :j] for k in ("Ca", "Cb", "Za", "Zb")), W["B_Ia"].float(), W["B_Ib"].float())
        x.update(qI=g((B, L.n_hI, cI), 113, d=dt), wI=g((B, L.n_hI), 114, std=cI ** -0.5 * L.n_hI ** -0.5),
                 compI=g((B, 4 * cI), 115))
    # the bf16 rows behind the cache (the step mutates the cache; host copies are made per sequence)
    kvc0, win0 = kvc_rows, win_rows
    if csa:
        KI0 = cache.key_I.clone()
        KI0s = cache.key_I_scale.clone() if idx_key_dtype == "fp8" else None
    xt = TokenInputs(**{k: v.to(cuda).contiguous() for k, v in x.items()})
    o = torch.full((B, L.n_h, c), float("nan"), dtype=dt, device=cuda)
    ws = torch.empty(max(hb.decode_workspace_size(lh.struct, pos), 16), dtype=torch.uint8, device=cuda)
    hb.hybrid_decode_step(lh.struct, xt.struct, cache.struct, pos, o, ws)
    torch.cuda.synchronize()
    emit = (pos + 1) % m == 0
    ties = 0
    if csa:
        mp = hb.workspace_map(lh.struct, pos, decode=True)
        gidx = hb.ws_view(ws, mp["idx"], (B, 1, L.k), torch.int32).cpu().numpy()
    rec = hb.kv_mixed_row_bytes(c, L.rd) if kv_mixed else 0
    for b in range(B):
        comp = to64(x["comp"][b])
        kvc = to64(kvc0[b][:(pos + 1) // m + 1])
        if kv_mixed:
            kvc = _mixed(kvc, L.rd)
        if emit:
            if csa:
                Ca = np.concatenate([to64(raw["Ca"][b, :j]), comp[None, 0:c]])
                Za = np.concatenate([to64(raw["Za"][b, :j]), comp[None, 2 * c:3 * c]])
                prev = (to64(raw["pCb"][b]), to64(raw["pZb"][b])) if Ecur > 0 else (None, None)
                e = O.decode_new_entry(pos, m, Ca, Za, to64(W["B_a"]), prev[0], prev[1], to64(W["B_b"]))
            else:
                Ca = np.concatenate([to64(raw["Ca"][b, :j]), comp[None, 0:c]])
                Za = np.concatenate([to64(raw["Za"][b, :j]), comp[None, c:2 * c]])
                e = O.decode_new_entry(pos, m, Ca, Za, to64(W["B"]))
            e = O.entry_epilogue(e[None], m, first_entry=Ecur, rd=L.rd)[0]
            if kv_mixed:
                # the emitted record, read back: the oracle's quantisation of the
                # bf16 entry (a value may sit one e4m3 step away where the two
                # bf16 entries differ in their last bit)
                got = torch.empty(1, c, dtype=BF16, device=cuda)
                hb.kv_dequant_mixed(cache.kv_comp[b, Ecur].contiguous(), 1, c, L.rd, got)
                ref = _mixed(_bf16_round(e)[None], L.rd)[0]
                d = np.abs(to64(got[0]) - _bf16_round(ref))      # the reader rounds code x scale to bf16
                assert (d <= 0.126 * np.abs(ref) + 1e-6).all() and (d == 0).mean() >= 0.95, "emitted record"
                kvc[Ecur] = ref
            else:
                assert_close(to64(cache.kv_comp[b, Ecur]), e, 2e-2, "emitted entry")
                kvc[Ecur] = _bf16_round(e)
        wpos = O.window_positions(pos, w)
        win = to64(win0[b])
        win[pos % w] = to64(x["kv"][b])
        if kv_mixed:
            win = _mixed(win, L.rd)
        wrows = win[[p % w for p in wpos]]
        kw = {}
        if csa:
            Vb = (pos + 1) // m + 1
            if idx_key_dtype == "fp8":
                KI = O.e4m3_to_f64(KI0[b][:Vb].cpu().numpy()) * to64(KI0s[b][:Vb])[..., None]
            else:
                KI = to64(KI0[b][:Vb])
            if emit:
                cI = L.c_I
                cI64 = to64(x["compI"][b])
                Ca = np.concatenate([to64(rawI["Ca"][b, :j]), cI64[None, 0:cI]])
                Za = np.concatenate([to64(rawI["Za"][b, :j]), cI64[None, 2 * cI:3 * cI]])
                prev = (to64(rawI["pCb"][b]), to64(rawI["pZb"][b])) if Ecur > 0 else (None, None)
                e = O.decode_new_entry(pos, m, Ca, Za, to64(W["B_Ia"]), prev[0], prev[1], to64(W["B_Ib"]))
                e = O.entry_epilogue(e[None], m, first_entry=Ecur, rd=L.rd_I)[0]
                if idx_key_dtype == "fp8":
                    sc = np.abs(e).max() / 448.0
                    KI[Ecur] = O.e4m3_to_f64(O.e4m3_encode(e / sc)) * sc
                else:
                    KI[Ecur] = _bf16_round(e)
            kw = dict(qI_t=to64(x["qI"][b]), w_t=to64(x["wI"][b]), KI=KI)
            V = (pos + 1) // m
            scores = O.index_scores(kw["qI_t"], kw["w_t"], KI, V)
            # the step's own selection (it keeps the index lists at the start of
            # its workspace): exact where the gap rule applies, else within the tie
            gsel = gidx[b, 0]
            ties += check_topk_row(gsel, scores, L.k, V)
            o_sel = oracle_attend_over(to64(x["q"][b]), wrows, kvc, gsel, to64(W["sink"]), c, pos, L.rd)
            assert_close(to64(o[b]), o_sel, 2e-2, f"decode o[b={b}] (over the GPU's selection)")
            if V > L.k and O.topk_gap(scores, L.k) <= GAP:
                continue
        ref, _ = O.layer_decode(L, pos, to64(x["q"][b]), kvc, wrows, to64(W["sink"]), **kw)
        assert_close(to64(o[b]), ref, 2e-2, f"decode o[b={b}]")
    return ties


@pytest.mark.parametrize("kind,pos,kdt", [("csa", 2047, "bf16"), ("csa", 2050, "bf16"), ("csa", 3, "bf16"),
                                           ("csa", 4099, "fp8"), ("csa", 4098, "fp8"),
                                           ("hca", 4095, "bf16"), ("hca", 5000, "bf16"), ("hca", 130, "bf16")])
def test_decode_step(cuda, kind, pos, kdt):
    L = workloads.HYBRID_DECODE_128K.layers[0 if kind == "csa" else 1]
    run_decode_case(cuda, L, 3, pos, kdt, seed=pos)


@pytest.mark.parametrize("kind,pos", [("csa", 2047), ("csa", 2050), ("hca", 4095), ("hca", 5000)])
def test_decode_step_mixed_kv(cuda, kind, pos):
    """A decode step over a mixed-precision KV cache ([J] §2.3.4): the step
    stores its window row and (on a block's last token) its new entry as
    records, and the attention reads records; checked against the oracle over
    the oracle's own quantisation of the same rows."""
    L = workloads.HYBRID_DECODE_128K.layers[0 if kind == "csa" else 1]
    run_decode_case(cuda, L, 3, pos, "bf16", seed=pos + 7, kv_mixed=True)
