"""Decode from hidden states and layer chaining (the CSA layer's output feeds
the HCA layer), on the GPU against the oracle.

hybrid_decode_inputs projects one token per sequence from hidden states
(juejin "DeepSeek-V4 技术报告简要解读" Eq.(9)-(10), (13)-(15), (18), (20)-(21));
the chain is: CSA decode inputs from h0 -> CSA decode step -> grouped output
projection (§2.3.1(d)) -> HCA decode inputs -> HCA decode step.  Every stage's
GPU result is compared with the oracle applied to the GPU's inputs of that
stage (so a stage's bf16 rounding does not compound into the next check)."""
import numpy as np
import pytest
import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth, workloads
from long_context_compressed_hca_b200.layer import CacheHandle, LayerHandle, TokenInputs
from oracle import hca_oracle as O
from tests.helpers import assert_close, to64

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16
D, DC = 512, 256              # d_model and the query compression width of this test


def _oracle_inputs(L, W, h, pos):
    """The oracle's projections of one token per sequence at position pos."""
    W = {k: to64(v) for k, v in W.items()}
    out = {}
    if L.kind == "csa":
        out["comp"] = np.concatenate([O.project(h, W[n]) for n in ("W_aKV", "W_bKV", "W_aZ", "W_bZ")], axis=1)
        out["compI"] = np.concatenate([O.project(h, W[n]) for n in ("W_IaKV", "W_IbKV", "W_IaZ", "W_IbZ")], axis=1)
    else:
        out["comp"] = np.concatenate([O.project(h, W["W_KVc"]), O.project(h, W["W_Zc"])], axis=1)
    cQ = O.rmsnorm(O.project(h, W["W_DQ"]))
    q = O.rmsnorm(O.project(cQ, W["W_UQ"]).reshape(h.shape[0], L.n_h, L.c))
    out["q"] = O.rope(q, np.full((h.shape[0], 1), pos), L.rd)
    out["kv"] = O.rope(O.rmsnorm(O.project(h, W["W_KV"])), np.full(h.shape[0], pos), L.rd)
    if L.kind == "csa":
        qI = O.project(cQ, W["W_IUQ"]).reshape(h.shape[0], L.n_hI, L.c_I)
        out["qI"] = O.rope(qI, np.full((h.shape[0], 1), pos), L.rd_I)
        out["wI"] = O.project(h, W["W_w"]) * (L.c_I ** -0.5 * L.n_hI ** -0.5)
    return out


def _check_inputs(L, x, ref):
    # fp32 outputs of bf16 operands: fp32 accumulation over d = 512
    for k in ("comp", "compI", "wI"):
        if k in ref:
            assert_close(to64(x.t[k]), ref[k], 1e-4 * max(1.0, np.abs(ref[k]).max()), k)
    # bf16 outputs (c^Q is rounded to bf16 between the two query GEMMs)
    for k in ("q", "kv", "qI"):
        if k in ref:
            assert_close(to64(x.t[k]), ref[k], 2e-2, k)


def _layer(L, li, B, cuda, seed):
    W = synth.layer_weights(L, D, DC, seed, BF16, layer_id=li, bias_std=0.5)
    lh = LayerHandle(L, W, D, DC, BF16, B, device=cuda)
    return W, lh


def _cache(L, B, pos, cuda, seed):
    cap = pos // L.m + 4
    ch = CacheHandle(L, B, cap, BF16, device=cuda)
    ch.kv_comp.copy_(synth.normal_on(cuda, ch.kv_comp.shape, seed, 1, dtype=BF16))
    ch.win.copy_(synth.normal_on(cuda, ch.win.shape, seed, 2, dtype=BF16))
    ch.state_kv.copy_(synth.normal_on(cuda, ch.state_kv.shape, seed, 3))
    ch.state_score.copy_(synth.normal_on(cuda, ch.state_score.shape, seed, 4))
    if L.kind == "csa":
        ch.key_I.copy_(synth.normal_on(cuda, ch.key_I.shape, seed, 5, dtype=BF16))
        ch.stateI_kv.copy_(synth.normal_on(cuda, ch.stateI_kv.shape, seed, 6))
        ch.stateI_score.copy_(synth.normal_on(cuda, ch.stateI_score.shape, seed, 7))
    return ch


def _oracle_step(L, ch, x, lh, pos, B):
    """The oracle's decode output per sequence over the GPU's caches (the step
    wrote the token's window row; no entry is emitted at this position)."""
    V = (pos + 1) // L.m
    sink = to64(lh.t["sink"])
    outs = []
    for b in range(B):
        win = to64(ch.win[b])
        rows = win[[p % L.w for p in O.window_positions(pos, L.w)]]
        kw = {}
        if L.kind == "csa":
            kw = dict(qI_t=to64(x.t["qI"][b]), w_t=to64(x.t["wI"][b]), KI=to64(ch.key_I[b, :V]))
        o, _ = O.layer_decode(L, pos, to64(x.t["q"][b]), to64(ch.kv_comp[b, :V]), rows, sink, **kw)
        outs.append(o)
    return np.stack(outs)


def test_decode_inputs_and_chained_csa_hca_step(cuda):
    wl = workloads.HYBRID_DECODE_128K
    Lc, Lh = wl.layers
    B, pos = 4, 2000                      # no entry emission at this position for m = 4 or 128
    assert (pos + 1) % Lc.m and (pos + 1) % Lh.m
    Wc, lc = _layer(Lc, 0, B, cuda, 31)
    Wh, lh = _layer(Lh, 1, B, cuda, 31)
    cc, chh = _cache(Lc, B, pos, cuda, 32), _cache(Lh, B, pos, cuda, 33)

    # 1. CSA decode inputs from hidden states h0
    h0 = synth.normal_on(cuda, (B, D), 34, 1, dtype=BF16)
    xc = TokenInputs.empty(Lc, B, BF16, cuda)
    wsi = torch.empty(max(hb.decode_inputs_workspace_size(lc.struct), 16), dtype=torch.uint8, device=cuda)
    hb.hybrid_decode_inputs(lc.struct, h0, pos, xc.struct, wsi)
    torch.cuda.synchronize()
    _check_inputs(Lc, xc, _oracle_inputs(Lc, Wc, to64(h0), pos))

    # 2. the CSA decode step
    oc = torch.empty(B, Lc.n_h, Lc.c, dtype=BF16, device=cuda)
    ws = torch.empty(max(hb.decode_workspace_size(lc.struct, pos), 16), dtype=torch.uint8, device=cuda)
    hb.hybrid_decode_step(lc.struct, xc.struct, cc.struct, pos, oc, ws)
    torch.cuda.synchronize()
    assert_close(to64(oc), _oracle_step(Lc, cc, xc, lc, pos, B), 2e-2, "o (CSA)")

    # 3. grouped output projection of the CSA output to the next layer's hidden states
    g, d_g = 8, 256
    gw = Lc.n_h * Lc.c // g
    wo_a = synth.normal_on(cuda, (g, d_g, gw), 35, 1, std=gw ** -0.5, dtype=BF16)
    wo_b = synth.normal_on(cuda, (D, g * d_g), 35, 2, std=(g * d_g) ** -0.5, dtype=BF16)
    od = hb.oproj_desc(B, Lc.n_h, Lc.c, g, d_g, D, hb.HCA_BF16, hb.HCA_BF16)
    wso = torch.empty(max(hb.output_projection_workspace_size(od), 16), dtype=torch.uint8, device=cuda)
    h1 = torch.empty(B, D, dtype=BF16, device=cuda)
    hb.output_projection(od, oc, wo_a, wo_b, h1, wso)
    torch.cuda.synchronize()
    assert_close(to64(h1), O.output_projection(to64(oc), to64(wo_a), to64(wo_b), g), 2e-2, "h1")

    # 4. HCA decode inputs from h1, then the HCA decode step
    xh = TokenInputs.empty(Lh, B, BF16, cuda)
    wsh = torch.empty(max(hb.decode_inputs_workspace_size(lh.struct), 16), dtype=torch.uint8, device=cuda)
    hb.hybrid_decode_inputs(lh.struct, h1, pos, xh.struct, wsh)
    torch.cuda.synchronize()
    _check_inputs(Lh, xh, _oracle_inputs(Lh, Wh, to64(h1), pos))
    oh = torch.empty(B, Lh.n_h, Lh.c, dtype=BF16, device=cuda)
    ws2 = torch.empty(max(hb.decode_workspace_size(lh.struct, pos), 16), dtype=torch.uint8, device=cuda)
    hb.hybrid_decode_step(lh.struct, xh.struct, chh.struct, pos, oh, ws2)
    torch.cuda.synchronize()
    assert_close(to64(oh), _oracle_step(Lh, chh, xh, lh, pos, B), 2e-2, "o (HCA)")


def test_decode_inputs_rejects_missing_buffers():
    import ctypes
    wl = workloads.HYBRID_DECODE_128K
    Lc = wl.layers[0]
    W = synth.layer_weights(Lc, D, DC, 1, BF16)
    lc = LayerHandle(Lc, W, D, DC, BF16, 2, device="cuda")
    x = hb.TokenIn()
    rc = hb.lib().hybrid_decode_inputs(ctypes.byref(lc.struct), 16, 5, ctypes.byref(x), 16, 1 << 20, None)
    assert rc == hb.HCA_ERR_INVALID and "missing output buffer" in hb.last_error()
