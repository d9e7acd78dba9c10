"""Pins of the CPU oracle against what the pages and the mathematics fix.

No page prints a worked numeric example, so the oracle is pinned by closed forms
derived by hand from the equations, brute force on tiny inputs, library
routines for the number formats, and the invariants the method must satisfy
(juejin "DeepSeek-V4 技术报告简要解读" §2.3.1-§2.3.3; 1zeryu "DeepSeek-V4：算法架构").
These run on the CPU (not marked gpu).
"""
import json
import math
import os
from types import SimpleNamespace

import numpy as np
import pytest
import torch

from oracle import hca_oracle as O
from long_context_compressed_hca_b200 import synth
from long_context_compressed_hca_b200.workloads import LayerShape

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def f64(t):
    return t.double().numpy() if isinstance(t, torch.Tensor) else np.asarray(t, np.float64)


# ----------------------------------------------------------------- formats

def test_bf16_decode_matches_torch():
    x = torch.randn(4096) * 100
    b = x.to(torch.bfloat16)
    bits = synth.bf16_bits(b).numpy()
    np.testing.assert_array_equal(O.bf16_bits_to_f64(bits), b.double().numpy())


def test_e4m3_decode_known_values_and_torch():
    known = {0x00: 0.0, 0x38: 1.0, 0x40: 2.0, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x08: 2.0 ** -6,
             0xB8: -1.0, 0x3C: 1.5, 0x07: 7 * 2.0 ** -9}
    for code, val in known.items():
        assert O.e4m3_to_f64(code) == val, hex(code)
    assert np.isnan(O.e4m3_to_f64(0x7F)) and np.isnan(O.e4m3_to_f64(0xFF))
    codes = torch.arange(256, dtype=torch.int64).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    got = O.e4m3_to_f64(np.arange(256))
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def test_e4m3_encode_round_trip_and_torch():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF, 0x80)])
    np.testing.assert_array_equal(O.e4m3_encode(O.e4m3_to_f64(codes)), codes.astype(np.uint8))
    x = rng.standard_normal(20000) * 60
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode(x)
    # compare decoded values (a -0 / +0 pair would compare equal)
    np.testing.assert_array_equal(O.e4m3_to_f64(got), O.e4m3_to_f64(ref))


# ----------------------------------------------------------------- norm / rope

def test_rmsnorm_closed_form():
    y = O.rmsnorm(np.array([3.0, 4.0]), eps=0.0)
    np.testing.assert_allclose(y, np.array([3.0, 4.0]) / math.sqrt(12.5), rtol=0, atol=1e-15)
    y = O.rmsnorm(np.array([3.0, 4.0]), gamma=np.array([2.0, -1.0]), eps=1.0)
    np.testing.assert_allclose(y, np.array([6.0, -4.0]) / math.sqrt(13.5), atol=1e-15)


@pytest.mark.parametrize("pair", [0, 1, 7])
def test_rope_unit_vector_closed_form(pair):
    c, rd, pos, theta = 32, 16, 37, 10000.0
    x = np.zeros(c)
    x[c - rd + 2 * pair] = 1.0
    y = O.rope(x, pos, rd, theta)
    ang = pos * theta ** (-2.0 * pair / rd)
    exp = np.zeros(c)
    exp[c - rd + 2 * pair] = math.cos(ang)
    exp[c - rd + 2 * pair + 1] = math.sin(ang)
    np.testing.assert_allclose(y, exp, atol=1e-14)


def test_rope_norm_inverse_and_passthrough():
    x = rng.standard_normal((5, 64))
    pos = np.arange(5) * 1000 + 3
    y = O.rope(x, pos, 16)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_array_equal(y[:, :48], x[:, :48])
    np.testing.assert_allclose(O.rope(y, pos, 16, inverse=True), x, atol=1e-12)
    # rotations compose: R(a) R(b) = R(a+b)
    np.testing.assert_allclose(O.rope(O.rope(x, 5, 16), 7, 16), O.rope(x, 12, 16), atol=1e-12)


# ----------------------------------------------------------------- compression

def test_compress_golden_closed_form():
    g = json.load(open(os.path.join(GOLDEN, "compress_m2_closed_form.json")))
    col = lambda k: np.asarray(g[k], np.float64)[:, None]
    ent = O.compress_prefill(col("C_a"), col("Z_a"), col("B_a"), g["m"],
                             col("C_b"), col("Z_b"), col("B_b"))
    np.testing.assert_allclose(ent[:, 0], g["entries"], rtol=0, atol=1e-14)


@pytest.mark.parametrize("overlap", [True, False])
def test_compress_identical_rows_give_that_row(overlap):
    m, c, n = 4, 8, 32
    v = rng.standard_normal(c)
    C = np.tile(v, (n, 1))
    Za, Zb = rng.standard_normal((n, c)) * 3, rng.standard_normal((n, c)) * 3
    Ba, Bb = rng.standard_normal((m, c)), rng.standard_normal((m, c))
    ent = O.compress_prefill(C, Za, Ba, m, C if overlap else None, Zb if overlap else None,
                             Bb if overlap else None)
    np.testing.assert_allclose(ent, np.tile(v, (n // m, 1)), rtol=1e-14, atol=1e-14)


def test_compress_weights_sum_to_one():
    m, c, n = 4, 6, 40
    ones = np.ones((n, c))
    Za, Zb = rng.standard_normal((n, c)) * 5, rng.standard_normal((n, c)) * 5
    Ba, Bb = rng.standard_normal((m, c)), rng.standard_normal((m, c))
    np.testing.assert_allclose(O.compress_prefill(ones, Za, Ba, m, ones, Zb, Bb), 1.0,
                               atol=1e-14)
    np.testing.assert_allclose(O.compress_prefill(ones, Za, Ba, m), 1.0, atol=1e-14)


def test_compress_ratio_one_is_identity():
    C = rng.standard_normal((9, 5))
    Z = rng.standard_normal((9, 5))
    np.testing.assert_allclose(O.compress_prefill(C, Z, np.zeros((1, 5)), 1), C, atol=1e-15)


def test_compress_brute_force_with_biases():
    """Eq.(11)-(12) written with explicit loops, independently of the oracle."""
    m, c, n = 3, 4, 13
    Ca, Cb, Za, Zb = (rng.standard_normal((n, c)) for _ in range(4))
    Ba, Bb = rng.standard_normal((m, c)), rng.standard_normal((m, c))
    ent = O.compress_prefill(Ca, Za, Ba, m, Cb, Zb, Bb)
    assert ent.shape == (n // m, c)
    for i in range(n // m):
        for ch in range(c):
            terms = []   # (logit, value); entry 0's b-half is -inf / 0 (drops out)
            for j in range(m):
                terms.append((Za[m * i + j, ch] + Ba[j, ch], Ca[m * i + j, ch]))
                if i > 0:
                    terms.append((Zb[m * (i - 1) + j, ch] + Bb[j, ch], Cb[m * (i - 1) + j, ch]))
            den = sum(math.exp(l) for l, _ in terms)
            val = sum(math.exp(l) * v for l, v in terms) / den
            assert abs(ent[i, ch] - val) < 1e-12


def test_entry_epilogue_positions():
    e = rng.standard_normal((6, 32))
    out = O.entry_epilogue(e, m=4, first_entry=2, rd=8)
    for i in range(6):
        np.testing.assert_allclose(out[i], O.rope(O.rmsnorm(e[i]), (2 + i) * 4, 8), atol=1e-14)


# ----------------------------------------------------------------- visibility / index / top-k

def test_visible_entries_brute_force():
    for m in (1, 2, 4, 128):
        for t in range(0, 600, 7):
            assert O.visible_entries(t, m) == sum(1 for s in range(1000) if (s + 1) * m <= t + 1)


def test_index_scores_brute_force():
    nh, cI, E = 3, 5, 9
    q, K = rng.standard_normal((nh, cI)), rng.standard_normal((E, cI))
    w = rng.standard_normal(nh)
    got = O.index_scores(q, w, K, 7)
    assert got.shape == (7,)
    for s in range(7):
        val = 0.0
        for h in range(nh):
            dot = sum(q[h, j] * K[s, j] for j in range(cI))
            val += w[h] * (dot if dot > 0 else 0.0)
        assert abs(got[s] - val) < 1e-12


def test_index_scores_relu_hand_example():
    q = np.array([[1.0, 0.0], [0.0, 1.0]])
    w = np.array([2.0, 3.0])
    K = np.array([[1.0, -1.0], [-2.0, 5.0]])
    # s=0: 2*relu(1) + 3*relu(-1) = 2 ; s=1: 2*relu(-2) + 3*relu(5) = 15
    np.testing.assert_allclose(O.index_scores(q, w, K, 2), [2.0, 15.0])


def test_topk_brute_force_with_ties():
    for trial in range(200):
        V = int(rng.integers(0, 40))
        k = int(rng.integers(1, 20))
        s = rng.integers(-3, 4, size=V).astype(np.float64)   # many ties
        got = O.topk_select(s, k)
        ranked = sorted(range(V), key=lambda j: (-s[j], j))
        exp = sorted(ranked[:min(k, V)]) + [-1] * (k - min(k, V))
        assert list(got) == exp


def test_topk_k_at_least_visible_selects_all():
    s = rng.standard_normal(11)
    np.testing.assert_array_equal(O.topk_select(s, 16), list(range(11)) + [-1] * 5)


# ----------------------------------------------------------------- attention core

def _textbook_attention(q, K, sink, scale):
    out = np.zeros((q.shape[0], K.shape[1]))
    for h in range(q.shape[0]):
        z = [scale * float(np.dot(q[h], K[j])) for j in range(K.shape[0])]
        den = sum(math.exp(v) for v in z) + math.exp(sink[h])
        for j in range(K.shape[0]):
            out[h] += math.exp(z[j]) / den * K[j]
    return out


def test_attend_token_brute_force():
    q, K = rng.standard_normal((3, 8)), rng.standard_normal((6, 8))
    sink = rng.standard_normal(3)
    np.testing.assert_allclose(O.attend_token(q, K, sink, 0.3), _textbook_attention(q, K, sink, 0.3),
                               atol=1e-13)


def test_sink_scales_mass_exactly():
    q, K = rng.standard_normal((4, 16)), rng.standard_normal((9, 16))
    sink = np.array([-1.0, 0.0, 2.0, 5.0])
    scale = 0.25
    o_sink = O.attend_token(q, K, sink, scale)
    o_plain = O.attend_token(q, K, np.full(4, -np.inf), scale)
    z = (q @ K.T) * scale
    se = np.exp(z).sum(1)
    np.testing.assert_allclose(o_sink, o_plain * (se / (se + np.exp(sink)))[:, None], rtol=1e-12)
    # sink -> -inf recovers the plain softmax
    p = np.exp(z - z.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(o_plain, p @ K, atol=1e-13)


def test_empty_candidate_set_gives_zero():
    q = rng.standard_normal((2, 4))
    np.testing.assert_array_equal(O.attend_token(q, np.zeros((0, 4)), np.zeros(2), 1.0), 0.0)


def test_rope_relative_position_invariance_of_output():
    """Logits depend on s - t only, and the inverse rotation at t removes the
    absolute part of the output ([J] §2.3.3 partial RoPE)."""
    c, rd, nh = 32, 16, 2
    q0, K0 = rng.standard_normal((nh, c)), rng.standard_normal((7, c))
    sink = rng.standard_normal(nh)
    t, spos = 20, np.array([0, 4, 8, 12, 17, 19, 20])
    outs = []
    for delta in (0, 1000, 65537):
        q = O.rope(q0, t + delta, rd)
        K = O.rope(K0, spos + delta, rd)
        outs.append(O.attend_output(q, K, sink, c ** -0.5, t + delta, rd))
    np.testing.assert_allclose(outs[1], outs[0], atol=1e-10)
    np.testing.assert_allclose(outs[2], outs[0], atol=1e-10)


# ----------------------------------------------------------------- layer-level pins

def _layer(kind, m, overlap=None, w=8, k=64, n_h=2, c=16, rd=8, n_hI=2, c_I=8, sink_std=1.0):
    L = LayerShape(kind, m=m, n_h=n_h, c=c, rd=rd, w=w, k=k, n_hI=n_hI, c_I=c_I,
                   sink_std=sink_std)
    if overlap is None:
        return L
    return SimpleNamespace(**{f: getattr(L, f) for f in L.__dataclass_fields__},
                           overlap=overlap, rd_I=L.rd_I)


def _weights(L, d, d_c, seed=7, bias_std=0.0):
    W = synth.layer_weights(L, d, d_c, seed, torch.float32, bias_std=bias_std)
    return {k: f64(v) for k, v in W.items()}


def _brute_causal_mqa(H, W, L, keys, key_pos, d_c, eps=1e-6):
    """Causal MQA written independently: q from the low-rank path, each token t
    attends to the keys at positions <= t, sink in the denominator, output
    rotated back by -t."""
    n = H.shape[0]
    out = np.zeros((n, L.n_h, L.c))
    cQ = H @ W["W_DQ"].T
    cQ = cQ / np.sqrt((cQ ** 2).mean(-1, keepdims=True) + eps)
    for t in range(n):
        q = (cQ[t] @ W["W_UQ"].T).reshape(L.n_h, L.c)
        q = q / np.sqrt((q ** 2).mean(-1, keepdims=True) + eps)
        q = O.rope(q, t, L.rd)
        vis = [j for j in range(len(key_pos)) if key_pos[j] <= t]
        o = _textbook_attention(q, keys[vis], W["sink"], L.c ** -0.5)
        out[t] = O.rope(o, t, L.rd, inverse=True)
    return out


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_ratio_one_no_window_is_causal_mqa(kind):
    """m = 1, no overlap, k >= entries, w = 0: compressed attention is causal MQA
    over RMSNorm(h W)·RoPE keys (spec pin)."""
    n, d, d_c = 24, 16, 8
    L = _layer(kind, 1, overlap=False, w=0, k=64)
    W = _weights(L, d, d_c)
    H = f64(synth.normal((n, d), 3, 0))
    got = O.layer_prefill(H, W, L, d_c)
    Wkv = W["W_aKV"] if kind == "csa" else W["W_KVc"]
    x = H @ Wkv.T
    keys = O.rope(x / np.sqrt((x ** 2).mean(-1, keepdims=True) + 1e-6), np.arange(n), L.rd)
    exp = _brute_causal_mqa(H, W, L, keys, np.arange(n), d_c)
    np.testing.assert_allclose(got, exp, atol=1e-11)


def test_ratio_one_with_overlap_is_mqa_over_two_row_entries():
    """m = 1 with overlap: entry i is the 2-row softmax of (C_a[i], C_b[i-1])."""
    n, d, d_c = 20, 16, 8
    L = _layer("csa", 1, overlap=True, w=0, k=64)
    W = _weights(L, d, d_c, bias_std=0.5)
    H = f64(synth.normal((n, d), 5, 0))
    got = O.layer_prefill(H, W, L, d_c)
    Ca, Cb, Za, Zb = (H @ W[k].T for k in ("W_aKV", "W_bKV", "W_aZ", "W_bZ"))
    ent = np.zeros_like(Ca)
    for i in range(n):
        ea = np.exp(Za[i] + W["B_a"][0])
        if i == 0:
            ent[i] = Ca[i]
        else:
            eb = np.exp(Zb[i - 1] + W["B_b"][0])
            ent[i] = (ea * Ca[i] + eb * Cb[i - 1]) / (ea + eb)
    keys = O.rope(ent / np.sqrt((ent ** 2).mean(-1, keepdims=True) + 1e-6), np.arange(n), L.rd)
    exp = _brute_causal_mqa(H, W, L, keys, np.arange(n), d_c)
    np.testing.assert_allclose(got, exp, atol=1e-11)


def test_causality_perturbing_future_token():
    n, d, d_c = 40, 16, 8
    L = _layer("csa", 4, w=6, k=3)
    W = _weights(L, d, d_c)
    H = f64(synth.normal((n, d), 9, 0))
    base = O.layer_prefill(H, W, L, d_c)
    for j in (5, 17, 31):
        H2 = H.copy()
        H2[j] += 3.0
        o2 = O.layer_prefill(H2, W, L, d_c)
        np.testing.assert_array_equal(o2[:j], base[:j])
        assert np.abs(o2[j:] - base[j:]).max() > 0


def test_entry_invisible_until_block_completes():
    """An entry of block s reaches no query before token (s+1)m-1; from that
    token on, the indexer can see it."""
    n, d, d_c, m = 48, 16, 8, 4
    L = _layer("csa", m, w=1, k=64)      # k >= entries: all visible entries are kept
    W = _weights(L, d, d_c)
    H = f64(synth.normal((n, d), 11, 0))
    r = O.layer_prefill(H, W, L, d_c, return_intermediates=True)
    for t in range(n):
        sel = r["idx"][t]
        sel = set(sel[sel >= 0].tolist())
        assert sel == set(range((t + 1) // m))


def test_decode_matches_prefill():
    """A decode step at position p over the cache a prefill built gives the
    prefill's output at token p (the decode branch of the Compressor/Indexer
    reproduces the prefill definition)."""
    n, d, d_c, m = 37, 16, 8, 4
    for kind in ("csa", "hca"):
        L = _layer(kind, m if kind == "csa" else 8, w=5, k=3)
        W = _weights(L, d, d_c, bias_std=0.3)
        H = f64(synth.normal((n, d), 13, 0))
        r = O.layer_prefill(H, W, L, d_c, return_intermediates=True)
        for p in (0, 3, 7, 8, 20, 36):
            win = np.stack([r["kv_win"][j] for j in O.window_positions(p, L.w)])
            kw = dict(qI_t=r["qI"][p], w_t=r["wI"][p], KI=r["KI"]) if kind == "csa" else {}
            o, idx = O.layer_decode(L, p, r["q"][p], r["kv_comp"], win, W["sink"], **kw)
            np.testing.assert_allclose(o, r["o"][p], atol=1e-12)
            if kind == "csa":
                np.testing.assert_array_equal(idx, r["idx"][p])


def test_decode_emission_equals_prefill_entries():
    """Entries emitted one token at a time equal the prefill entries."""
    m, c, n = 4, 6, 30
    Ca, Cb, Za, Zb = (rng.standard_normal((n, c)) for _ in range(4))
    Ba, Bb = rng.standard_normal((m, c)), rng.standard_normal((m, c))
    ref = O.compress_prefill(Ca, Za, Ba, m, Cb, Zb, Bb)
    got, at = [], []
    for pos in range(n):
        b = pos // m
        blk = slice(b * m, pos + 1)
        prev = slice((b - 1) * m, b * m) if b > 0 else None
        e = O.decode_new_entry(pos, m, Ca[blk], Za[blk], Ba,
                               Cb[prev] if prev else None, Zb[prev] if prev else None, Bb)
        if e is not None:
            got.append(e)
            at.append(pos)
    assert at == list(range(m - 1, n, m))          # a block's entry appears with its last token
    np.testing.assert_allclose(np.stack(got), ref, atol=1e-14)


# ----------------------------------------------------------- grouped output projection
def test_output_projection_equals_block_diagonal_projection():
    """Grouping = one projection whose first matrix is block diagonal over the
    groups (assembled here element by element, not by the grouping code)."""
    rng = np.random.default_rng(7)
    n_h, c, g, d_g, d = 8, 6, 4, 5, 9
    o = rng.normal(size=(3, n_h, c))
    wo_a = rng.normal(size=(g, d_g, n_h * c // g))
    wo_b = rng.normal(size=(d, g * d_g))
    big = np.zeros((g * d_g, n_h * c))
    w = n_h * c // g
    for i in range(g):
        for r in range(d_g):
            for j in range(w):
                big[i * d_g + r, i * w + j] = wo_a[i, r, j]
    ref = np.stack([wo_b @ (big @ o[t].reshape(-1)) for t in range(3)])
    np.testing.assert_allclose(O.output_projection(o, wo_a, wo_b, g), ref, rtol=1e-12, atol=1e-12)


def test_output_projection_group_permutation_invariance():
    """Relabelling the groups (heads, wo_a blocks and wo_b column blocks
    together) leaves the output unchanged; swapping only the heads does not."""
    rng = np.random.default_rng(8)
    n_h, c, g, d_g, d = 8, 4, 4, 3, 5
    o = rng.normal(size=(n_h, c))
    wo_a = rng.normal(size=(g, d_g, n_h * c // g))
    wo_b = rng.normal(size=(d, g * d_g))
    perm = np.array([2, 0, 3, 1])
    hpg = n_h // g
    o_p = o.reshape(g, hpg, c)[perm].reshape(n_h, c)
    wb_p = wo_b.reshape(d, g, d_g)[:, perm].reshape(d, g * d_g)
    base = O.output_projection(o, wo_a, wo_b, g)
    np.testing.assert_allclose(O.output_projection(o_p, wo_a[perm], wb_p, g), base, rtol=1e-12, atol=1e-12)
    assert not np.allclose(O.output_projection(o_p, wo_a, wo_b, g), base)


def test_output_projection_hand_example():
    """Two heads of one channel, two groups of one output each, a square wo_b
    (so a transposed operand would still fit): mid = (a p, b q), out = wo_b mid."""
    a, b, p, q = 2.0, -3.0, 5.0, 7.0
    o = np.array([[a], [b]])
    wo_a = np.array([[[p]], [[q]]])
    wo_b = np.array([[1.0, 2.0], [3.0, 4.0]])
    np.testing.assert_array_equal(O.output_projection(o, wo_a, wo_b, 2),
                                  [a * p + 2 * b * q, 3 * a * p + 4 * b * q])


def test_window_positions_hand_table():
    """Reading 10: the window of query t is tokens max(0, t-w+1) .. t, its own
    token included (w rows once t >= w-1)."""
    table = {(5, 3): [3, 4, 5], (1, 3): [0, 1], (0, 1): [0], (7, 1): [7], (4, 0): []}
    for (t, w), want in table.items():
        np.testing.assert_array_equal(O.window_positions(t, w), want)


def test_output_projection_identity_weights_flatten():
    """d_g = n_h*c/g with identity blocks and wo_b = I returns o flattened."""
    rng = np.random.default_rng(9)
    n_h, c, g = 4, 3, 2
    w = n_h * c // g
    o = rng.normal(size=(n_h, c))
    wo_a = np.stack([np.eye(w)] * g)
    wo_b = np.eye(g * w)
    np.testing.assert_allclose(O.output_projection(o, wo_a, wo_b, g), o.reshape(-1), rtol=0, atol=0)


# ----------------------------------------------------------------- mixed-precision KV rows

def test_bf16_encode_matches_torch_and_hand_ties():
    # float32 inputs: torch's float32 -> bf16 conversion is nearest, ties to even
    x = (torch.randn(20000) * torch.exp2(torch.randint(-30, 30, (20000,)).float())).float()
    ref = synth.bf16_bits(x.to(torch.bfloat16)).numpy()
    np.testing.assert_array_equal(O.bf16_encode(x.double().numpy()).astype(np.int64), ref)
    # ties by hand: 1 + 2^-8 lies halfway between 1 (even) and 1 + 2^-7 (odd);
    # 1 + 3*2^-8 halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
    assert O.bf16_encode(1 + 2 ** -8) == 0x3F80
    assert O.bf16_encode(1 + 3 * 2 ** -8) == 0x3F82
    assert O.bf16_encode(-(1 + 2 ** -8 + 2 ** -40)) == 0xBF81        # just above the tie
    assert O.bf16_encode(2.0 ** -133) == 0x0001 and O.bf16_encode(3.5e38) == 0x7F80


def test_kv_quant_exact_on_the_grid():
    """Rows built from e4m3 values times a power-of-two scale, each block
    holding +-448, with bf16-exact RoPE channels, come back bit for bit."""
    c, rd = 512, 64
    codes = rng.integers(0, 0x7E, size=(5, c - rd))
    codes[:, ::64] = 0x7E                                   # every block's amax is 448
    sign = np.where(rng.random((5, c - rd)) < 0.5, -1.0, 1.0)
    scale = 2.0 ** rng.integers(-8, 4, size=(5, (c - rd) // 64))
    x = sign * O.e4m3_to_f64(codes) * np.repeat(scale, 64, axis=1)
    rope = O.bf16_bits_to_f64(O.bf16_encode(rng.standard_normal((5, rd))))
    row = np.concatenate([x, rope], axis=1)
    q, s, r = O.kv_row_quant(row, rd)
    np.testing.assert_array_equal(s, scale)
    np.testing.assert_array_equal(O.kv_row_dequant(q, s, r), row)


def test_kv_quant_error_bound_and_block_amax():
    """e4m3 keeps 3 mantissa bits: a normal value is within 2^-4 of itself
    relative, a subnormal one within half the spacing 2^-9 (times the scale);
    the block's largest magnitude maps to 448 exactly."""
    c, rd = 512, 64
    row = rng.standard_normal((64, c)) * np.exp(rng.uniform(-6, 6, size=(64, 1)))
    q, s, r = O.kv_row_quant(row, rd)
    d = O.kv_row_dequant(q, s, r)
    x32 = row[:, :c - rd].astype(np.float32).astype(np.float64)
    sc = np.repeat(s.astype(np.float64), 64, axis=1)
    err = np.abs(d[:, :c - rd] - x32)
    assert (err <= 2.0 ** -4 * np.abs(x32) * (1 + 2 ** -20) + sc * 2.0 ** -10).all()
    blocks = np.abs(x32).reshape(64, -1, 64)
    at = blocks.argmax(axis=2)
    top = np.take_along_axis(q.reshape(64, -1, 64), at[..., None], axis=2)[..., 0]
    assert ((top & 0x7F) == 0x7E).all()
    # RoPE channels: exactly the bf16 rounding
    np.testing.assert_array_equal(r, O.bf16_encode(row[:, c - rd:]))


def test_kv_quant_blocks_are_independent_and_zero_blocks():
    c, rd = 256, 64
    row = rng.standard_normal(c)
    row[64:128] = 0.0                                       # an all-zero block
    q, s, r = O.kv_row_quant(row, rd)
    assert s[1] == 0 and (q[64:128] == 0).all()
    np.testing.assert_array_equal(O.kv_row_dequant(q, s, r)[64:128], 0.0)
    row2 = row.copy()
    row2[130] = 10.0 * np.abs(row[128:192]).max()           # block 2's new amax, no other block
    q2, s2, r2 = O.kv_row_quant(row2, rd)
    np.testing.assert_array_equal(np.delete(q2, np.s_[128:192]), np.delete(q, np.s_[128:192]))
    np.testing.assert_array_equal(np.delete(s2, 2), np.delete(s, 2))
    assert s2[2] != s[2]
    np.testing.assert_array_equal(r2, r)


def test_mixed_kv_row_bytes_nearly_halve_the_cache():
    """[J] §2.3.4: BF16 RoPE dims + FP8 for the rest nearly halves the KV
    cache: 448 fp8 bytes + 7 fp32 scales + 64 bf16 values = 604 of 1024."""
    assert O.mixed_kv_row_bytes(512, 64) == 448 + 28 + 128 == 604
    assert 0.5 < O.mixed_kv_row_bytes(512, 64) / (512 * 2) < 0.6


# ----------------------------------------------------------------- FP4 indexer path

@pytest.mark.parametrize("n", [1, 2, 4, 8, 64, 128])
def test_hadamard_orthonormal_symmetric(n):
    h = O.hadamard(n)
    np.testing.assert_allclose(h @ h.T, np.eye(n), atol=1e-12)
    np.testing.assert_array_equal(h, h.T)
    assert np.all(np.abs(np.abs(h) - n ** -0.5) < 1e-15)


def test_hadamard_rotation_closed_form_and_dot_products():
    a, b = 3.0, -1.25
    np.testing.assert_allclose(O.hadamard_rotate([a, b]), [(a + b) / 2 ** 0.5, (a - b) / 2 ** 0.5])
    q, k = rng.standard_normal((5, 64)), rng.standard_normal((7, 64))
    np.testing.assert_allclose(O.hadamard_rotate(q) @ O.hadamard_rotate(k).T, q @ k.T, atol=1e-11)
    # the exact index scores do not see the rotation
    w = rng.standard_normal(5)
    np.testing.assert_allclose(O.index_scores(O.hadamard_rotate(q), w, O.hadamard_rotate(k), 7),
                               O.index_scores(q, w, k, 7), atol=1e-11)


def test_e2m1_table_ties_and_saturation():
    np.testing.assert_array_equal(O.e2m1_to_f64(np.arange(16)),
                                  [0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6])
    # halfway cases go to the even mantissa (code bit 0 clear)
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for x, want in ties.items():
        assert O.e2m1_to_f64(O.e2m1_encode(x)) == want, x
        assert O.e2m1_to_f64(O.e2m1_encode(-x)) == -want, -x
    assert O.e2m1_to_f64(O.e2m1_encode(7.9)) == 6.0 and O.e2m1_to_f64(O.e2m1_encode(-1e9)) == -6.0
    # round trip of every non-negative-zero code, and nearest by brute force
    codes = np.array([c for c in range(16) if c != 8])
    np.testing.assert_array_equal(O.e2m1_encode(O.e2m1_to_f64(codes)), codes)
    x = rng.uniform(-6, 6, 5000)
    got = O.e2m1_to_f64(O.e2m1_encode(x))
    vals = np.unique(O.e2m1_to_f64(np.arange(16)))
    best = np.abs(x[:, None] - vals[None]).min(axis=1)
    np.testing.assert_allclose(np.abs(got - x), best, atol=0)


def test_fp4_into_e4m3_is_lossless():
    """[J] §4.4: FP8 (E4M3) has two more exponent bits, so FP4 values times
    their power-of-two block scales are E4M3 values (within E4M3's range)."""
    for k in range(-7, 7):
        v = O.e2m1_to_f64(np.arange(16)) * 2.0 ** k
        v = v[np.abs(v) <= 448]
        np.testing.assert_array_equal(O.e4m3_to_f64(O.e4m3_encode(v)), v)


def test_fp4_block_quant_scale_grid_and_error():
    x = rng.standard_normal((16, 128)) * np.exp(rng.uniform(-5, 5, (16, 1)))
    codes, e = O.fp4_block_quant(x)
    assert codes.shape == x.shape and e.shape == (16, 4)            # one scale per 32 values
    amax = np.abs(x.reshape(16, 4, 32)).max(axis=-1)
    r = amax / np.ldexp(1.0, e)
    assert np.all((r >= 4) & (r < 8))
    xh = O.fp4_block_dequant(codes, e)
    s = np.repeat(np.ldexp(1.0, e), 32, axis=1)
    assert np.all(np.abs(xh - x) <= 2 * s)                           # saturation region (6, 8)
    inside = np.abs(x) <= 6 * s
    assert np.all(np.abs(xh - x)[inside] <= s[inside])              # half the widest spacing (2)
    # values on the grid come back exactly; an all-zero block stays zero
    g = O.e2m1_to_f64(rng.integers(0, 16, (3, 64))) * 2.0 ** 3
    g[:, ::32] = 6 * 2.0 ** 3
    np.testing.assert_array_equal(O.fp4_simulate(g), g)
    z = np.zeros((1, 32))
    np.testing.assert_array_equal(O.fp4_simulate(z), z)


def test_index_scores_fp4_bf16_and_power_of_two_scaling():
    q, k = rng.standard_normal((8, 64)), rng.standard_normal((40, 64))
    w = np.abs(rng.standard_normal(8)) * 0.05
    sc = O.index_scores_fp4(q, w, k, 40)
    np.testing.assert_array_equal(O.bf16_bits_to_f64(O.bf16_encode(sc)), sc)   # BF16 values
    # FP4 block scales are powers of two and BF16 rounding is scale-free: scaling
    # q by 2^j scales every score by 2^j exactly
    np.testing.assert_array_equal(O.index_scores_fp4(4 * q, w, k, 40), 4 * sc)
    # the FP4 path stays close to the exact scores on this data
    ex = O.index_scores(q, w, k, 40)
    assert np.abs(sc - ex).max() <= 0.25 * np.abs(ex).max()


def test_fwht32_matches_the_hadamard_matrix():
    x = rng.standard_normal((50, 64)) * 10
    np.testing.assert_allclose(O.hadamard_rotate_fwht32(x), O.hadamard_rotate(x.astype(np.float32)),
                               rtol=0, atol=1e-5 * np.abs(x).max())
    # small integers: every butterfly sum is exact in fp32, so the two agree exactly
    xi = rng.integers(-50, 50, (20, 64)).astype(np.float64)
    np.testing.assert_array_equal(O.hadamard_rotate_fwht32(xi), O.hadamard_rotate(xi))
    # the butterfly order of the 4-point case by hand: [a+b+c+d, a-b+c-d, a+b-c-d, a-b-c+d] / 2
    a, b, c, d = 1.0, 2.0, 4.0, 8.0
    np.testing.assert_array_equal(O.hadamard_rotate_fwht32([a, b, c, d]),
                                  np.array([a + b + c + d, a - b + c - d, a + b - c - d, a - b - c + d]) / 2)


def test_fp4_rotate_quant_values_are_bf16_and_fp4():
    x = rng.standard_normal((30, 64))
    y = O.fp4_rotate_quant_gpu_order(x)
    np.testing.assert_array_equal(O.bf16_bits_to_f64(O.bf16_encode(y)), y)      # exact in bf16
    codes, e = O.fp4_block_quant(y)
    np.testing.assert_array_equal(O.fp4_block_dequant(codes, e), y)             # already on the grid
