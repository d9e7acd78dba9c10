"""Pins of the C++ oracle (oracle/hca_oracle_c.cpp), on the CPU.

The C++ oracle is a second, independent restatement of the method's steps
(juejin "DeepSeek-V4 技术报告简要解读" §2.3.1-§2.3.3; 1zeryu "DeepSeek-V4：算法架构").
It is pinned by the same kinds of facts as the numpy oracle -- closed forms,
brute force on tiny inputs, invariants -- and by agreement with the numpy
oracle (itself pinned in test_oracle_pins.py) on random inputs, function by
function and through the decode / prefill composites.
"""
import numpy as np
import pytest

from oracle import hca_oracle as O
from oracle import hca_oracle_c as OC

rng = np.random.default_rng(77)


@pytest.fixture(scope="module", autouse=True)
def built():
    OC.build()
    yield
    OC.num_threads(0)


def close(a, b, rtol=1e-12, atol=1e-12):
    np.testing.assert_allclose(a, b, rtol=rtol, atol=atol)


# ------------------------------------------------------------ closed forms

@pytest.mark.parametrize("overlap", [False, True])
def test_identical_rows_compress_to_that_row(overlap):
    n, c, m = 12, 6, 4
    row = rng.standard_normal(c)
    C = np.tile(row, (n, 1))
    Z = rng.standard_normal((n, c)) * 3
    B = rng.standard_normal((m, c))
    out = OC.compress(C, Z, B, m, C if overlap else None, Z if overlap else None, B if overlap else None)
    close(out, np.tile(row, (n // m, 1)))


def test_weights_sum_to_one_and_ratio_one_is_identity():
    n, c, m = 8, 5, 1
    C = rng.standard_normal((n, c))
    Z = rng.standard_normal((n, c)) * 10
    close(OC.compress(C, Z, np.zeros((m, c)), m), C)


def test_compress_two_row_hand_example():
    # one entry over two rows: softmax of logits (0, ln 3) weights the values (1, 5): (1 + 3*5) / 4 = 4
    C = np.array([[1.0], [5.0]])
    Z = np.array([[0.0], [np.log(3.0)]])
    close(OC.compress(C, Z, np.zeros((2, 1)), 2), [[4.0]])


def test_index_scores_relu_hand_example():
    qI = np.array([[1.0, 0.0], [0.0, 1.0]])
    w = np.array([2.0, -1.0])
    KI = np.array([[3.0, 4.0], [-1.0, 2.0], [1.0, -5.0]])
    # entry 0: 2*3 - 1*4 = 2; entry 1: 2*0 - 1*2 = -2; entry 2: 2*1 - 0 = 2
    close(OC.index_scores(qI, w, KI, 3), [2.0, -2.0, 2.0])


def test_topk_brute_force_with_ties():
    for _ in range(50):
        V = int(rng.integers(1, 40))
        k = int(rng.integers(1, 20))
        s = rng.integers(0, 5, V).astype(np.float64)
        order = sorted(range(V), key=lambda i: (-s[i], i))[:min(k, V)]
        want = sorted(order) + [-1] * (k - min(k, V))
        np.testing.assert_array_equal(OC.topk_select(s, k), want)


def test_sink_scales_mass_exactly():
    n_h, c, R = 3, 8, 5
    q = rng.standard_normal((n_h, c))
    rows = np.tile(rng.standard_normal(c), (R, 1))     # identical rows: o = row * sum / (sum + e^s)
    sink = rng.standard_normal(n_h)
    out = OC.attend_output(q, rows, sink, c ** -0.5, 0, 0)
    z = (q @ rows[0]) * c ** -0.5
    mass = R * np.exp(z) / (R * np.exp(z) + np.exp(sink))
    close(out, mass[:, None] * rows[0][None, :])


def test_ratio_one_no_window_is_causal_mqa():
    """m = 1, k >= V, no window: the CSA token t attends the entries 0..t, i.e.
    (with ratio 1 and no overlap every entry is its token's row) causal MQA."""
    n, n_h, c, rd = 9, 2, 8, 4
    rows = rng.standard_normal((n, c))
    q = rng.standard_normal((n, n_h, c))
    qI = rng.standard_normal((n, 2, 4))
    w = rng.standard_normal((n, 2))
    KI = rng.standard_normal((n, 4))
    sink = rng.standard_normal(n_h)
    ts = np.arange(n)
    out = OC.prefill_tokens("csa", ts, q, rows, 0, rows, 1, sink, rd, k=n, qI=qI, w=w, KI=KI)
    for t in range(n):
        z = q[t] @ rows[:t + 1].T * c ** -0.5
        M = np.maximum(z.max(axis=1), sink)
        e = np.exp(z - M[:, None])
        o = (e @ rows[:t + 1]) / (e.sum(axis=1) + np.exp(sink - M))[:, None]
        close(out[t], O.rope(o, t, rd, inverse=True))


# ------------------------------------------------- agreement with the numpy oracle

@pytest.mark.parametrize("overlap,m", [(True, 4), (False, 16)])
def test_compress_and_epilogue_match_numpy_oracle(overlap, m):
    n, c = 64, 32
    Ca, Za, Cb, Zb = (rng.standard_normal((n, c)) for _ in range(4))
    Ba, Bb = rng.standard_normal((m, c)), rng.standard_normal((m, c))
    a = OC.compress(Ca, Za, Ba, m, Cb if overlap else None, Zb if overlap else None, Bb if overlap else None)
    b = O.compress_prefill(Ca, Za, Ba, m, Cb if overlap else None, Zb if overlap else None, Bb if overlap else None)
    close(a, b)
    g = rng.standard_normal(c)
    close(OC.entry_epilogue(a, m, 3, g, 1e-6, 8), O.entry_epilogue(b, m, 3, g, 1e-6, 8))


def test_index_scores_topk_and_attend_match_numpy_oracle():
    for _ in range(5):
        V, n_hI, c_I, k = 300, 4, 16, 37
        qI, w, KI = rng.standard_normal((n_hI, c_I)), rng.standard_normal(n_hI), rng.standard_normal((V, c_I))
        s = OC.index_scores(qI, w, KI, V)
        close(s, O.index_scores(qI, w, KI, V))
        np.testing.assert_array_equal(OC.topk_select(s, k), O.topk_select(s, k))
        q, rows, sink = rng.standard_normal((8, 64)), rng.standard_normal((50, 64)), rng.standard_normal(8)
        close(OC.attend_output(q, rows, sink, 64 ** -0.5, 1234, 16), O.attend_output(q, rows, sink, 64 ** -0.5, 1234, 16))


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_decode_batch_matches_numpy_layer_decode(kind):
    B, n_h, c, rd, w, m, k, n_hI, c_I = 3, 4, 32, 8, 5, 4 if kind == "csa" else 16, 7, 2, 8
    pos = 203
    V = (pos + 1) // m
    from types import SimpleNamespace
    L = SimpleNamespace(kind=kind, m=m, k=k, c=c, rd=rd)
    q = rng.standard_normal((B, n_h, c))
    win = rng.standard_normal((B, w, c))
    kvc = rng.standard_normal((B, V + 2, c))
    qI, wI, KI = rng.standard_normal((B, n_hI, c_I)), rng.standard_normal((B, n_hI)), rng.standard_normal((B, V + 2, c_I))
    sink = rng.standard_normal(n_h)
    out = OC.decode_batch(kind, q, win, np.arange(w), kvc, m, sink, rd, pos, k=k, qI=qI if kind == "csa" else None,
                          w=wI if kind == "csa" else None, KI=KI if kind == "csa" else None)
    for b in range(B):
        ref, _ = O.layer_decode(L, pos, q[b], kvc[b], win[b], sink, qI[b], wI[b], KI[b])
        close(out[b], ref)


def test_thread_count_does_not_change_results():
    B, n_h, c, rd, w, m, k = 6, 4, 32, 8, 5, 4, 9
    pos = 99
    q = rng.standard_normal((B, n_h, c))
    win, kvc = rng.standard_normal((B, w, c)), rng.standard_normal((B, 40, c))
    qI, wI, KI = rng.standard_normal((B, 2, 8)), rng.standard_normal((B, 2)), rng.standard_normal((B, 40, 8))
    sink = rng.standard_normal(n_h)
    outs = []
    for nt in (1, 4):
        OC.num_threads(nt)
        outs.append(OC.decode_batch("csa", q, win, np.arange(w), kvc, m, sink, rd, pos, k=k, qI=qI, w=wI, KI=KI))
    np.testing.assert_array_equal(outs[0], outs[1])


def test_bad_arguments_are_rejected():
    with pytest.raises(ValueError):
        OC.topk_select(np.zeros(3), 0)


def test_stored_formats_decode_exactly():
    """bf16 bits and e4m3 codes x scale read by the composites equal the
    numpy oracle's exact decodings of the same bytes."""
    import torch
    from long_context_compressed_hca_b200 import synth
    B, n_h, c, rd, w, m, k, n_hI, c_I = 2, 4, 32, 8, 6, 4, 5, 2, 16
    pos = 61
    V = (pos + 1) // m
    kvc = torch.randn(B, V + 1, c).to(torch.bfloat16)
    win = torch.randn(B, w, c).to(torch.bfloat16)
    KIf = torch.randn(B, V + 1, c_I)
    codes, scale = synth.fp8_rows(KIf)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    q = rng.standard_normal((B, n_h, c))
    qI, wI = rng.standard_normal((B, n_hI, c_I)), rng.standard_normal((B, n_hI))
    sink = rng.standard_normal(n_h)
    order = np.array([p % w for p in O.window_positions(pos, w)])
    out = OC.decode_batch("csa", q, bits(win), order, bits(kvc), m, sink, rd, pos, k=k, qI=qI, w=wI,
                          KI=codes.numpy(), KI_scale=scale.numpy())
    from types import SimpleNamespace
    L = SimpleNamespace(kind="csa", m=m, k=k, c=c, rd=rd)
    for b in range(B):
        KI64 = O.e4m3_to_f64(codes[b].numpy()) * scale[b].double().numpy()[:, None]
        ref, _ = O.layer_decode(L, pos, q[b], kvc[b].double().numpy(), win[b].double().numpy()[order], sink,
                                qI[b], wI[b], KI64)
        close(out[b], ref)
