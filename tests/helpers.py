"""Shared helpers for the parity tests: exact host copies, seeded inputs,
and comparisons with the tolerances the workloads state (max-abs 1e-4 for
fp32 paths, 2e-2 for bf16 paths; top-k sets exact where the oracle's k-th /
(k+1)-th score gap exceeds 1e-3 relative)."""
import numpy as np
import torch

from long_context_compressed_hca_b200 import synth
from oracle import hca_oracle as O

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
GAP = 1e-3          # top-k must match exactly where the k-th/(k+1)-th gap exceeds this
# Where the GPU and the oracle score identical stored inputs (decode over a
# given cache), their scores agree to ~1e-6 relative, so outputs are compared
# wherever the gap exceeds this much smaller threshold (stricter than GAP).
GAP_STRICT = 2e-5
# From hidden states the bf16 path stores q^I and K^I in bf16, which moves an
# index score by up to ~1-2% relative (64-term dot products of rounded
# operands), so end-to-end bf16 layer outputs are compared where the gap
# exceeds this; the exact rule is applied where the stored inputs are shared.
GAP_LAYER_BF16 = 2e-2


def to64(t):
    """Exact float64 copy of a device/host tensor (bf16 and fp32 widen exactly)."""
    return t.detach().to("cpu").double().numpy()


def rnd(shape, seed, stream, dtype=torch.float32, std=1.0, device="cuda"):
    return synth.normal(shape, seed, stream, std=std, dtype=dtype).to(device)


def random_idx(B, n_q, start_pos, m, k, seed, device="cuda"):
    """Random valid top-k lists: for each query a sorted random subset of its
    visible entries of size min(k, V), then -1 padding."""
    g = synth.generator(seed, 999)
    out = torch.full((B, n_q, k), -1, dtype=torch.int32)
    for b in range(B):
        for i in range(n_q):
            V = (start_pos + i + 1) // m
            n = min(k, V)
            if n:
                sel = torch.randperm(V, generator=g)[:n].sort().values
                out[b, i, :n] = sel.to(torch.int32)
    return out.to(device)


def assert_close(got, ref, tol, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    err = np.abs(got - ref)
    bad = ~(err <= tol)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(np.isnan(err), np.inf, err)), err.shape)
        raise AssertionError(f"{what}: max-abs {np.nanmax(err):.3e} > {tol} at {i}: got {got[i]} ref {ref[i]}"
                             f" ({bad.sum()} of {bad.size} elements out of tolerance)")
    return float(err.max()) if err.size else 0.0


def check_topk_row(gpu_idx, ref_scores, k, V):
    """Top-k parity of one query: exact set where the gap rule applies, else a
    valid selection.  Returns True when the row was a near tie."""
    gi = np.asarray(gpu_idx)
    n = min(k, V)
    sel = gi[:n]
    assert (gi[n:] == -1).all(), "padding must be -1"
    assert (np.diff(sel) > 0).all() if n > 1 else True, "indices must be ascending and unique"
    assert ((sel >= 0) & (sel < V)).all(), "indices must be visible entries"
    ref = O.topk_select(ref_scores, k)
    if O.topk_gap(ref_scores, k) > GAP:
        np.testing.assert_array_equal(gi, ref)
        return False
    # near tie: the sets may differ only in entries whose oracle score is
    # within fp32 rounding of the k-th score
    kth = np.sort(ref_scores)[::-1][n - 1]
    diff = np.setxor1d(sel, ref[:n])
    tol = 1e-5 * max(abs(kth), 1e-30) + 1e-7 * np.abs(ref_scores).max()
    assert (np.abs(ref_scores[diff] - kth) <= tol).all(), "selection differs beyond the tie"
    return True


def check_selection_bound(gpu_idx, s_exact, s_shared, k, V):
    """The GPU's selection against the oracle's fp64 scores s_exact when the
    GPU stored its index operands in a narrower type: s_shared are the oracle's
    scores over the GPU's stored (rounded) operands, delta the largest change
    that rounding made to any score of the row.  A selection exact for
    s_shared keeps only entries whose s_exact is >= the fp64 k-th score minus
    2*delta (each side moves by at most delta), which is asserted."""
    n = min(k, V)
    if n >= V or n == 0:
        return 0.0
    sel = np.asarray(gpu_idx)[:n]
    s_exact = np.asarray(s_exact, np.float64)
    delta = float(np.abs(s_exact - np.asarray(s_shared, np.float64)).max())
    kth = np.sort(s_exact)[::-1][n - 1]
    slack = 2 * delta + 1e-6 * float(np.abs(s_exact).max())
    worst = float(kth - s_exact[sel].min())
    assert worst <= slack, f"a kept entry lies {worst:.3e} below the fp64 k-th score (allowed {slack:.3e})"
    return delta


def oracle_attend_over(q_t, win_rows, kv_comp, sel, sink, c, t, rd):
    """The oracle's attention output of query t over its window rows and the
    compressed rows `sel` (the GPU's own selection, already validated against
    the oracle's), so that near-tie selections leave no output unchecked."""
    sel = np.asarray(sel)
    sel = sel[sel >= 0]
    rows = np.concatenate([np.asarray(win_rows, np.float64).reshape(-1, c),
                           np.asarray(kv_comp, np.float64)[sel]], axis=0)
    return O.attend_output(q_t, rows, sink, c ** -0.5, t, rd)
