"""Oracle for DeepSeek-V4 hybrid compressed attention (CSA + HCA): plain, slow, fp64.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module; only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
reference arm may use it.  It shares no code with the CUDA path.

Every function restates one step of the method in float64 with numpy, in the
order and notation of the pages:

  [J]  juejin.cn "DeepSeek-V4 技术报告简要解读" — §2.3.1 (CSA) Eq.(9)-(19),
       §2.3.2 (HCA) Eq.(20)-(23), §2.3.3 (QK norm, partial RoPE, sliding window,
       attention sink Eq.(27)), Appendix A.
  [Z]  1zeryu.github.io "DeepSeek-V4：算法架构" — "Q, K, V 映射与位置编码注入"
       (query/window-KV path), "Sparse Attention" (window + compressed index
       sets), "CSA 选择器层代码实现" (Compressor, Indexer), "HCA 选择函数代码实现"
       (visible-entry rule), "输出投影" (inverse RoPE on the output).

Readings taken where the pages are silent or disagree:
  * visibility: entry s is visible to query t iff (s+1)*m <= t+1 ([Z] Indexer
    mask and get_compress_topk_idxs; [J] Eq.(16)'s s < floor(t/m) with 1-based t);
  * RoPE: theta = 10000, interleaved pairs (2i, 2i+1) of the last rd dims,
    frequency theta^(-2i/rd); entry i sits at position i*m, tokens at t;
  * attention scale c^-1/2; the sink logit is unscaled and only in the
    denominator ([J] Eq.(27));
  * window = tokens max(0, t-w+1) .. t, concatenated with the compressed set
    without de-duplication ([Z] Sparse Attention);
  * top-k keeps min(k, V_t) entries, ties to the lower index, output in
    ascending index order, -1 padding ([J] Eq.(17), [Z] Indexer);
  * the Hadamard rotation of indexer q/k is orthonormal and omitted; no FP4
    simulation; no intermediate rounding (exact arithmetic);
  * mixed-precision KV rows: e4m3 codes with one fp32 scale (block amax / 448)
    per 64 non-RoPE channels, decided in fp32, all-zero blocks with scale 0;
    the RoPE channels in bf16 (nearest, ties to even);
  * FP4 indexer path: orthonormal Sylvester-Hadamard rotation, E2M1 (ties to
    even, saturating at 6) with one power-of-two scale 2^(floor(log2 amax)-2)
    per 32 values, scores rounded to bf16 before the selection.

Parity pins: every function here is pinned by tests/test_oracle_pins.py against
closed forms, brute force and invariants (no page prints a worked example).
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# exact decoding of the stored number formats
# ---------------------------------------------------------------------------


def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16 as any int array) -> exact float64 values."""
    b = np.asarray(bits).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_to_f64(bits) -> np.ndarray:
    """fp8 e4m3 (OCP 'fn' variant: bias 7, no inf, S.1111.111 = NaN) -> float64.

    Written from the format definition: value = (-1)^s * 2^(e-7) * (1 + f/8)
    for e > 0, and (-1)^s * 2^-6 * (f/8) for e = 0.
    """
    b = np.asarray(bits).astype(np.int64) & 0xFF
    s = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    f = (b & 7).astype(np.float64)
    normal = np.ldexp(1.0 + f / 8.0, (e - 7).astype(np.int64))
    sub = np.ldexp(f / 8.0, -6)
    v = s * np.where(e == 0, sub, normal)
    return np.where((e == 15) & ((b & 7) == 7), np.nan, v)


# ---------------------------------------------------------------------------
# normalisation and partial RoPE  ([J] §2.3.3; [Z] 位置编码注入)
# ---------------------------------------------------------------------------


def rmsnorm(x: np.ndarray, gamma=None, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gamma."""
    x = np.asarray(x, dtype=np.float64)
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, dtype=np.float64)
    return y


def rope(x: np.ndarray, pos, rd: int, theta: float = 10000.0, inverse: bool = False) -> np.ndarray:
    """Rotate the last rd dims of x in interleaved pairs (2i, 2i+1).

    Pair i turns by angle pos * theta^(-2i/rd) (by -angle when inverse).  pos
    broadcasts against x's leading axes.  Other dims pass through unchanged.
    """
    x = np.asarray(x, dtype=np.float64)
    if rd == 0:
        return x.copy()
    c = x.shape[-1]
    assert rd % 2 == 0 and rd <= c
    i = np.arange(rd // 2, dtype=np.float64)
    freq = theta ** (-2.0 * i / rd)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq
    if inverse:
        ang = -ang
    cos, sin = np.cos(ang), np.sin(ang)
    y = x.copy()
    a = x[..., c - rd::2]
    b = x[..., c - rd + 1::2]
    y[..., c - rd::2] = a * cos - b * sin
    y[..., c - rd + 1::2] = a * sin + b * cos
    return y


# ---------------------------------------------------------------------------
# block compression  ([J] Eq.(11)-(12) CSA, Eq.(22)-(23) HCA; [Z] Compressor)
# ---------------------------------------------------------------------------


def compress_entry(Ca_blk, Za_blk, Ba, Cb_prev=None, Zb_prev=None, Bb=None) -> np.ndarray:
    """One compressed entry.

    CSA (Eq.(11)-(12)): per channel, softmax over the 2m logits
    {Z_a[mi..m(i+1)-1] + B_a} U {Z_b[m(i-1)..mi-1] + B_b}, then
    C_i = sum S_a * C_a + sum S_b * C_b.  Pass Cb_prev=None for entry 0 (the
    b-half is -inf / 0 there) and for HCA (Eq.(22)-(23): softmax over the m'
    rows of the block with bias B, no overlap).
    Inputs are [rows, c]; returns [c].
    """
    logits = [np.asarray(Za_blk, np.float64) + np.asarray(Ba, np.float64)]
    values = [np.asarray(Ca_blk, np.float64)]
    if Cb_prev is not None:
        logits.append(np.asarray(Zb_prev, np.float64) + np.asarray(Bb, np.float64))
        values.append(np.asarray(Cb_prev, np.float64))
    L = np.concatenate(logits, axis=0)
    V = np.concatenate(values, axis=0)
    L = L - L.max(axis=0, keepdims=True)
    S = np.exp(L)
    S = S / S.sum(axis=0, keepdims=True)           # Softmax_row over the rows, per channel
    return (S * V).sum(axis=0)


def compress_prefill(Ca, Za, Ba, m: int, Cb=None, Zb=None, Bb=None) -> np.ndarray:
    """All floor(n/m) entries of a sequence of n tokens ([n, c] inputs).

    Overlapped (CSA) when Cb is given, plain (HCA) otherwise.
    """
    n = Ca.shape[0]
    E = n // m
    out = np.zeros((E, Ca.shape[1]), dtype=np.float64)
    for i in range(E):
        blk = slice(m * i, m * (i + 1))
        if Cb is not None and i > 0:
            prev = slice(m * (i - 1), m * i)
            out[i] = compress_entry(Ca[blk], Za[blk], Ba, Cb[prev], Zb[prev], Bb)
        else:
            out[i] = compress_entry(Ca[blk], Za[blk], Ba)
    return out


def entry_epilogue(entries, m: int, first_entry: int = 0, gamma=None, eps: float = 1e-6,
                   rd: int = 0, theta: float = 10000.0, norm: bool = True) -> np.ndarray:
    """RMSNorm of each compressed entry, then RoPE of its last rd dims at the
    entry's block start i*m ([J] §2.3.3 QK normalisation / partial RoPE; [Z]
    Compressor: norm, then rotary at positions 0, m, 2m, ...)."""
    x = np.asarray(entries, np.float64)
    if norm:
        x = rmsnorm(x, gamma, eps)
    pos = (first_entry + np.arange(x.shape[0])) * m
    return rope(x, pos, rd, theta)


# ---------------------------------------------------------------------------
# visibility, index score, top-k  ([J] Eq.(16)-(17); [Z] Indexer)
# ---------------------------------------------------------------------------


def visible_entries(t: int, m: int) -> int:
    """Number of compressed entries query t may see: entry s is visible iff its
    block is complete including token t, i.e. (s+1)*m <= t+1."""
    return (t + 1) // m


def index_scores(qI_t, w_t, KI, V: int) -> np.ndarray:
    """Eq.(16): I[t,s] = sum_h w[t,h] * ReLU(q^I[t,h] . K^I[s]) for s < V.

    qI_t [n_hI, c_I], w_t [n_hI], KI [>=V, c_I] (dequantised).  Returns [V].
    """
    dots = np.asarray(KI, np.float64)[:V] @ np.asarray(qI_t, np.float64).T   # [V, n_hI]
    return (np.maximum(dots, 0.0) * np.asarray(w_t, np.float64)[None, :]).sum(axis=1)


def topk_select(scores, k: int) -> np.ndarray:
    """Eq.(17): keep the min(k, V) highest scores; ties go to the lower index.

    Returns int32 [k]: the kept entry indices in ascending order, then -1s.
    """
    s = np.asarray(scores, np.float64)
    V = s.shape[0]
    order = np.lexsort((np.arange(V), -s))          # score desc, index asc
    kept = np.sort(order[:min(k, V)])
    out = np.full(k, -1, dtype=np.int32)
    out[:kept.shape[0]] = kept
    return out


def topk_gap(scores, k: int) -> float:
    """Relative gap between the k-th and (k+1)-th highest score (inf if V <= k)."""
    s = np.sort(np.asarray(scores, np.float64))[::-1]
    if s.shape[0] <= k:
        return np.inf
    a, b = s[k - 1], s[k]
    return abs(a - b) / max(abs(a), abs(b), 1e-30)


# ---------------------------------------------------------------------------
# candidate sets and the shared-KV MQA core with sink
# ([J] Eq.(18)-(19), (27), §2.3.3; [Z] Sparse Attention, HCA selection)
# ---------------------------------------------------------------------------


def window_positions(t: int, w: int) -> np.ndarray:
    """Tokens of the sliding-window branch for query t: max(0, t-w+1) .. t."""
    return np.arange(max(0, t - w + 1), t + 1)


def attend_token(q_t, rows, sink, scale: float) -> np.ndarray:
    """Shared-KV MQA for one query token with a per-head sink (Eq.(19), (27)).

    q_t [n_h, c]; rows [R, c] serve as keys and values; sink [n_h] logits.
    o_h = sum_j exp(z_hj) v_j / (sum_j exp(z_hj) + exp(z'_h)), z = scale q.k.
    """
    q = np.asarray(q_t, np.float64)
    kv = np.asarray(rows, np.float64)
    sink = np.asarray(sink, np.float64)
    z = (q @ kv.T) * scale                                  # [n_h, R]
    M = np.maximum(z.max(axis=1) if kv.shape[0] else -np.inf, sink)
    e = np.exp(z - M[:, None])
    denom = e.sum(axis=1) + np.exp(sink - M)
    return (e @ kv) / denom[:, None]


def attend_output(q_t, rows, sink, scale: float, t: int, rd: int, theta: float = 10000.0):
    """attend_token followed by the inverse RoPE of the output's last rd dims at
    the query position t ([J] §2.3.3 partial RoPE; [Z] 输出投影)."""
    return rope(attend_token(q_t, rows, sink, scale), t, rd, theta, inverse=True)


# ---------------------------------------------------------------------------
# the layer from hidden states (prefill)  ([J] Eq.(9)-(19), (20)-(23); [Z])
# ---------------------------------------------------------------------------


def project(H, W) -> np.ndarray:
    """H [n, d_in] times a weight stored [d_out, d_in] (Linear convention)."""
    return np.asarray(H, np.float64) @ np.asarray(W, np.float64).T


def layer_prefill(H, W: dict, L, d_c: int, eps: float = 1e-6, theta: float = 10000.0,
                  tokens=None, return_intermediates: bool = False):
    """One attention layer over a whole sequence from position 0.

    H [n, d].  W holds fp64 arrays (stored [d_out, d_in]):
      CSA: W_aKV, W_bKV, W_aZ, W_bZ [c, d]; B_a, B_b [m, c];
           indexer W_IaKV, W_IbKV, W_IaZ, W_IbZ [c_I, d]; B_Ia, B_Ib [m, c_I];
           W_IUQ [n_hI*c_I, d_c]; W_w [n_hI, d]
      HCA: W_KVc, W_Zc [c, d]; B [m, c]
      both: W_DQ [d_c, d]; W_UQ [n_h*c, d_c]; W_KV [c, d] (window branch); sink [n_h]
    L is a LayerShape.  Returns o [len(tokens), n_h, c] (inverse-RoPE'd).
    RMSNorm weights are 1 (a reading: the workloads list none).
    """
    H = np.asarray(H, np.float64)
    n = H.shape[0]
    tokens = np.arange(n) if tokens is None else np.asarray(tokens)
    m, c, rd = L.m, L.c, L.rd
    scale = c ** -0.5

    # compressed main KV entries (Eq.(9)-(12) or (20)-(23)), normed and RoPE'd
    if L.kind == "csa" and L.overlap:
        ent = compress_prefill(project(H, W["W_aKV"]), project(H, W["W_aZ"]), W["B_a"], m,
                               project(H, W["W_bKV"]), project(H, W["W_bZ"]), W["B_b"])
    elif L.kind == "csa":
        ent = compress_prefill(project(H, W["W_aKV"]), project(H, W["W_aZ"]), W["B_a"], m)
    else:
        ent = compress_prefill(project(H, W["W_KVc"]), project(H, W["W_Zc"]), W["B"], m)
    kv_comp = entry_epilogue(ent, m, eps=eps, rd=rd, theta=theta)

    # window branch: kv = RMSNorm(h W_KV), RoPE at the token's own position
    need = sorted({p for t in tokens for p in window_positions(int(t), L.w)})
    kv_win = {}
    if need:
        rows = rope(rmsnorm(project(H[need], W["W_KV"]), eps=eps), np.asarray(need), rd, theta)
        kv_win = {p: rows[i] for i, p in enumerate(need)}

    # queries (Eq.(13), (18)): c^Q = RMSNorm(h W_DQ); q = c^Q W_UQ; per-head
    # unweighted RMS normalisation; RoPE at t
    cQ = rmsnorm(project(H[tokens], W["W_DQ"]), eps=eps)
    q = project(cQ, W["W_UQ"]).reshape(len(tokens), L.n_h, c)
    q = rmsnorm(q, eps=eps)
    q = rope(q, tokens[:, None], rd, theta)

    if L.kind == "csa":
        if L.overlap:
            KIraw = compress_prefill(project(H, W["W_IaKV"]), project(H, W["W_IaZ"]), W["B_Ia"],
                                     m, project(H, W["W_IbKV"]), project(H, W["W_IbZ"]),
                                     W["B_Ib"])
        else:
            KIraw = compress_prefill(project(H, W["W_IaKV"]), project(H, W["W_IaZ"]), W["B_Ia"], m)
        KI = entry_epilogue(KIraw, m, eps=eps, rd=L.rd_I, theta=theta)
        qI = project(cQ, W["W_IUQ"]).reshape(len(tokens), L.n_hI, L.c_I)   # Eq.(14)
        qI = rope(qI, tokens[:, None], L.rd_I, theta)
        wI = project(H[tokens], W["W_w"]) * (L.c_I ** -0.5 * L.n_hI ** -0.5)   # Eq.(15)

    o = np.zeros((len(tokens), L.n_h, c))
    idx_all, scores_all = [], []
    for j, t in enumerate(tokens):
        t = int(t)
        V = visible_entries(t, m)
        if L.kind == "csa":
            sc = index_scores(qI[j], wI[j], KI, V)
            idx = topk_select(sc, L.k)
            idx_all.append(idx)
            scores_all.append(sc)
            comp_rows = kv_comp[idx[idx >= 0]]
        else:
            comp_rows = kv_comp[:V]
        win_rows = np.stack([kv_win[p] for p in window_positions(t, L.w)]) if L.w else \
            np.zeros((0, c))
        rows = np.concatenate([win_rows, comp_rows], axis=0)
        o[j] = attend_output(q[j], rows, W["sink"], scale, t, rd, theta)
    if not return_intermediates:
        return o
    out = dict(o=o, kv_comp=kv_comp, q=q, kv_win=kv_win)
    if L.kind == "csa":
        out.update(KI=KI, qI=qI, wI=wI, idx=np.stack(idx_all) if idx_all else None,
                   scores=scores_all)
    return out


# ---------------------------------------------------------------------------
# single-token decode over a compressed cache  ([Z] Compressor decode branch,
# Indexer / get_compress_topk_idxs with start_pos > 0)
# ---------------------------------------------------------------------------


# ---------------------------------------------------------------------------
# grouped output projection  ([J] §2.3.1(d); [Z] 输出投影)
# ---------------------------------------------------------------------------


def output_projection(o, wo_a, wo_b, g: int) -> np.ndarray:
    """The attention output of one token, o [n_h, c] (inverse RoPE already
    applied), split into g groups of n_h/g heads; group i's flattened
    n_h*c/g values go through wo_a[i] ([d_g, n_h*c/g]) to d_g values, the g
    results are concatenated (group order) and wo_b ([d, g*d_g]) maps them
    to the layer output [d].  o may carry leading token dims."""
    o = np.asarray(o, np.float64)
    lead = o.shape[:-2]
    n_h, c = o.shape[-2:]
    wo_a = np.asarray(wo_a, np.float64)
    wo_b = np.asarray(wo_b, np.float64)
    d_g = wo_a.shape[1]
    grp = o.reshape(lead + (g, n_h * c // g))
    mid = np.empty(lead + (g, d_g))
    for i in range(g):
        mid[..., i, :] = grp[..., i, :] @ wo_a[i].T
    return mid.reshape(lead + (g * d_g,)) @ wo_b.T


def decode_new_entry(pos: int, m: int, cur_Ca, cur_Za, Ba, prev_Cb=None, prev_Zb=None, Bb=None):
    """The entry a decode step emits, or None.

    Token pos completes block pos//m when (pos+1) % m == 0.  cur_Ca/cur_Za
    hold the block's m projected rows (the new token's row last); prev_Cb /
    prev_Zb the previous block's b-series rows (CSA, block index > 0), else None.
    The entry is the same Eq.(12)/(23) reduction as in prefill.
    """
    if (pos + 1) % m != 0:
        return None
    return compress_entry(cur_Ca, cur_Za, Ba, prev_Cb, prev_Zb, Bb)


def layer_decode(L, pos: int, q_t, kv_comp, win_rows, sink, qI_t=None, w_t=None, KI=None,
                 theta: float = 10000.0):
    """Attention output of one decode step for one sequence.

    q_t [n_h, c] (normed, RoPE'd at pos); kv_comp: the compressed entries
    visible after this step (at least (pos+1)//m rows, the emitted one
    included); win_rows [R, c]: the window rows of tokens
    max(0, pos-w+1) .. pos in position order (the new token's row last).
    CSA also takes qI_t [n_hI, c_I], w_t [n_hI] and KI (dequantised indexer
    keys, at least (pos+1)//m rows).  Returns (o [n_h, c], idx or None).
    """
    V = visible_entries(pos, L.m)
    if L.kind == "csa":
        idx = topk_select(index_scores(qI_t, w_t, KI, V), L.k)
        comp_rows = np.asarray(kv_comp, np.float64)[idx[idx >= 0]]
    else:
        idx = None
        comp_rows = np.asarray(kv_comp, np.float64)[:V]
    rows = np.concatenate([np.asarray(win_rows, np.float64).reshape(-1, L.c), comp_rows], axis=0)
    o = attend_output(q_t, rows, sink, L.c ** -0.5, pos, L.rd, theta)
    return o, idx


def e4m3_encode(x) -> np.ndarray:
    """Round float64 values to the nearest fp8 e4m3 value (ties to even
    mantissa), saturating at +-448; returns the bit patterns (uint8).

    Brute force over the 254 finite codes, from the format definition."""
    codes = np.arange(256, dtype=np.int64)
    vals = e4m3_to_f64(codes)
    finite = ~np.isnan(vals)
    codes, vals = codes[finite], vals[finite]
    order = np.argsort(vals, kind="stable")
    codes, vals = codes[order], vals[order]
    # drop -0 (keep +0 for zero)
    keep = ~((vals == 0) & (codes == 0x80))
    codes, vals = codes[keep], vals[keep]
    x = np.clip(np.asarray(x, np.float64), -448.0, 448.0)
    hi = np.clip(np.searchsorted(vals, x, side="left"), 0, len(vals) - 1)
    lo = np.clip(hi - 1, 0, len(vals) - 1)
    dlo, dhi = np.abs(x - vals[lo]), np.abs(vals[hi] - x)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((codes[hi] & 1) == 0))
    out = np.where(pick_hi, codes[hi], codes[lo])
    return out.astype(np.uint8)


# ---------------------------------------------------------------------------
# mixed-precision KV rows ([J] §2.3.4 效率对比: RoPE dims kept in BF16, the
# other dims in FP8, which nearly halves the KV cache; [Z] "Q, K, V 映射与位置
# 编码注入" and the Compressor: after RoPE, the non-RoPE dims of every KV row
# are quantised to FP8 in blocks of 64 channels)
# ---------------------------------------------------------------------------
KV_FP8_BLOCK = 64


def bf16_encode(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even); returns
    the bit patterns (uint16).  From the format: 8 significant bits, exponent
    range of fp32 (subnormal spacing 2^-133), overflow to infinity."""
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)                                    # x = m * 2^e, 0.5 <= |m| < 1
    q = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)         # 8 significant bits, ties to even
    sub = np.ldexp(np.rint(np.ldexp(x, 133)), -133)      # below 2^-126: fixed spacing 2^-133
    q = np.where(np.abs(x) < 2.0 ** -126, sub, q)
    q = np.where(np.abs(q) >= 2.0 ** 128, np.copysign(np.inf, x), q)
    with np.errstate(over="ignore"):
        f = q.astype(np.float32)                         # exact: q has at most 8 significant bits
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def kv_row_quant(row, rd: int, block: int = KV_FP8_BLOCK):
    """Store KV rows (last axis = c channels) in the mixed format.

    The first c - rd channels, in blocks of `block`: scale = block amax / 448
    and code = e4m3(x / scale), so the block's largest magnitude maps to 448;
    these decisions are taken in fp32 (the row rounded to fp32, the scale and
    the quotient each rounded to fp32, then nearest e4m3 with ties to even);
    an all-zero block gets scale 0 and codes 0.  The last rd (RoPE) channels:
    bf16, nearest with ties to even.  Returns (codes uint8 [..., c-rd],
    scales float32 [..., (c-rd)/block], rope bf16 bits uint16 [..., rd])."""
    x = np.asarray(row, np.float64)
    c = x.shape[-1]
    nq = c - rd
    assert nq >= 0 and nq % block == 0, "c - rd must be a multiple of the block"
    xb = x[..., :nq].astype(np.float32).reshape(*x.shape[:-1], nq // block, block)
    amax = np.abs(xb).max(axis=-1, keepdims=True)
    scale = (amax / np.float32(448.0)).astype(np.float32)
    quot = (xb / np.where(scale > 0, scale, np.float32(1.0))).astype(np.float32)
    codes = e4m3_encode(quot.astype(np.float64)).reshape(*x.shape[:-1], nq)
    return codes, scale[..., 0], bf16_encode(x[..., nq:])


def kv_row_dequant(codes, scales, rope_bits, block: int = KV_FP8_BLOCK) -> np.ndarray:
    """The float64 KV rows a reader of the mixed format sees: each fp8 code
    times its block's scale, then the bf16 RoPE channels."""
    v = e4m3_to_f64(codes)
    sc = np.repeat(np.asarray(scales, np.float64), block, axis=-1)
    return np.concatenate([v * sc, bf16_bits_to_f64(rope_bits)], axis=-1)


def mixed_kv_row_bytes(c: int, rd: int, block: int = KV_FP8_BLOCK) -> int:
    """Bytes one row occupies in the mixed format: fp8 codes, fp32 block
    scales and bf16 RoPE channels."""
    return (c - rd) + 4 * ((c - rd) // block) + 2 * rd


# ---------------------------------------------------------------------------
# FP4 indexer path ([J] §4.4 FP4 量化感知训练: the CSA indexer's QK activations
# are cached, loaded and multiplied in FP4, FP4 (E2M1) sub-blocks of 1 x 32
# carry fine-grained scales that FP8's two extra exponent bits absorb, so FP4
# -> FP8 dequantisation is lossless; the index scores go from FP32 to BF16.
# [Z] Indexer and its Compressor: q and the compressed keys are rotated by a
# Hadamard transform (rotate_activation) before the FP4 simulation)
# ---------------------------------------------------------------------------
FP4_BLOCK = 32
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def hadamard(n: int) -> np.ndarray:
    """The n x n Sylvester-Hadamard matrix scaled by n^-1/2 (orthonormal and
    symmetric); n a power of two."""
    assert n >= 1 and n & (n - 1) == 0
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h / np.sqrt(n)


def hadamard_rotate(x) -> np.ndarray:
    """Rotate the last axis by the orthonormal Hadamard matrix."""
    x = np.asarray(x, np.float64)
    return x @ hadamard(x.shape[-1])


def e2m1_encode(x) -> np.ndarray:
    """Nearest FP4 E2M1 value (sign, 2 exponent bits with bias 1, 1 mantissa
    bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), ties to the even mantissa,
    saturating at +-6; returns the 4-bit codes (sign in bit 3)."""
    x = np.asarray(x, np.float64)
    a = np.minimum(np.abs(x), 6.0)
    hi = np.clip(np.searchsorted(E2M1_MAGNITUDES, a, side="left"), 0, 7)
    lo = np.clip(hi - 1, 0, 7)
    dlo, dhi = a - E2M1_MAGNITUDES[lo], E2M1_MAGNITUDES[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((hi & 1) == 0))   # code parity = mantissa bit
    mag = np.where(pick_hi, hi, lo)
    return (np.where((x < 0) & (mag > 0), 8, 0) + mag).astype(np.uint8)


def e2m1_to_f64(codes) -> np.ndarray:
    c = np.asarray(codes).astype(np.int64) & 0xF
    return np.where(c & 8, -1.0, 1.0) * E2M1_MAGNITUDES[c & 7]


def fp4_block_quant(x, block: int = FP4_BLOCK):
    """FP4 with one power-of-two scale per `block` consecutive values of the
    last axis (the OCP MX layout, reading of "1 x 32 sub-blocks whose scales
    FP8 absorbs losslessly"): scale = 2^(floor(log2 amax) - 2), so the block's
    largest magnitude lands in [4, 8) before rounding, codes = E2M1 of
    x / scale; an all-zero block gets scale 1.  Returns (codes [...], scale
    exponents int [..., n/block])."""
    x = np.asarray(x, np.float64)
    n = x.shape[-1]
    assert n % block == 0
    xb = x.reshape(*x.shape[:-1], n // block, block)
    amax = np.abs(xb).max(axis=-1)
    e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2, 0).astype(np.int64)
    codes = e2m1_encode(xb / np.ldexp(1.0, e)[..., None])
    return codes.reshape(x.shape), e


def fp4_block_dequant(codes, exps, block: int = FP4_BLOCK) -> np.ndarray:
    v = e2m1_to_f64(codes)
    return v * np.repeat(np.ldexp(1.0, np.asarray(exps)), block, axis=-1)


def fp4_simulate(x, block: int = FP4_BLOCK) -> np.ndarray:
    """Quantise to FP4 blocks and back (the indexer's FP4 simulation)."""
    c, e = fp4_block_quant(x, block)
    return fp4_block_dequant(c, e, block)


def index_scores_fp4(qI_t, w_t, KI, V: int) -> np.ndarray:
    """Index scores on the FP4 path: q^I and K^I rotated by the Hadamard
    transform and FP4-simulated, Eq.(16) over them, the result rounded to
    BF16 (the top-k then runs on the BF16 scores, ties to the lower index)."""
    qr = fp4_simulate(hadamard_rotate(qI_t))
    kr = fp4_simulate(hadamard_rotate(np.asarray(KI, np.float64)[:V]))
    return bf16_bits_to_f64(bf16_encode(index_scores(qr, w_t, kr, V)))



def hadamard_rotate_fwht32(x) -> np.ndarray:
    """The Hadamard rotation of the last axis (a power of two) as the GPU takes
    it, for decisions made on its result: fast Walsh-Hadamard butterflies in
    fp32, strides 1, 2, 4, ... (lower element a, upper b: a + b, a - b, each
    rounded to fp32), then the exact scale n^-1/2 for n = 4^j.  Equal to
    hadamard_rotate up to fp32 rounding."""
    y = np.array(np.asarray(x, np.float64).astype(np.float32), copy=True)
    n = y.shape[-1]
    assert n & (n - 1) == 0 and (n.bit_length() - 1) % 2 == 0, "n must be a power of 4"
    s = 1
    while s < n:
        v = y.reshape(*y.shape[:-1], n // (2 * s), 2, s)
        a, b = v[..., 0, :].copy(), v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        y = v.reshape(*y.shape[:-1], n)
        s *= 2
    return (y * np.float32(2.0 ** (-(n.bit_length() - 1) // 2))).astype(np.float64)


def fp4_rotate_quant_gpu_order(x, block: int = FP4_BLOCK) -> np.ndarray:
    """The FP4 values (as float64) of rows rotated in the GPU's fp32 order and
    block-quantised: what an indexer stores for q^I / K^I on the FP4 path."""
    return fp4_simulate(hadamard_rotate_fwht32(x), block)
