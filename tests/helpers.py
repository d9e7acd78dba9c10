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
