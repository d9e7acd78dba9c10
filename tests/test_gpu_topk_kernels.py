"""Every top-k selection kernel against the oracle's exact selection of the
same fp32 scores (the scores the GPU scorer wrote, read back), row by row and
bit for bit: the min(k, V) highest, ties to the lower index, ascending, padded
with -1 (juejin "DeepSeek-V4 技术报告简要解读" §2.3.1(b), Eq.(17)).  The kernels:
a CTA per row, a warp per row, the segmented cluster select, a cluster per
row, and the choice by shape."""
import numpy as np
import pytest
import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth
from oracle import hca_oracle as O
from tests.helpers import rnd

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16

MODES = [hb.TOPK_AUTO, hb.TOPK_ROW, hb.TOPK_WARP, hb.TOPK_CLUSTER, hb.TOPK_ROW_CLUSTER]
CASES = [
    # B, n_q, start_pos, k
    (1, 16, 0, 8),          # short rows: V <= k for most
    (2, 64, 2000, 64),      # V ~ 500: the whole row is the warp kernel's sample
    (2, 40, 16000, 64),     # V ~ 4000
    (1, 300, 30000, 512),   # 300 rows of ~7500 keys (by shape: a warp per row)
    (3, 1, 131071, 512),    # the longest rows the row and warp kernels take (32768)
]


def _select(cuda, mode, B, n_q, start_pos, k, ties):
    m, n_hI, c_I = 4, 8, 64
    E = (start_pos + n_q) // m
    cap = E + 1
    if ties:
        # three index keys: every row holds three score values, repeated
        base = synth.normal((B, 3, c_I), 77, 1)
        s_ids = np.arange(cap)
        cls = np.where(s_ids % 97 == 5, 0, 1 + (s_ids * 7 // 3) % 2)
        KI = base[:, torch.from_numpy(cls)].to(BF16).to(cuda)
    else:
        KI = synth.normal((B, cap, c_I), 5, 3).to(BF16).to(cuda)
    qI = rnd((B, n_q, n_hI, c_I), 78, 1, BF16)
    wI = rnd((B, n_q, n_hI), 78, 2, std=c_I ** -0.5 * n_hI ** -0.5)
    d = hb.attn_desc(B, 4, 64, 16, 8, m, k=k, n_hI=n_hI, c_I=c_I, rd_I=16, dtype=hb.HCA_BF16,
                     idx_key_dtype=hb.HCA_BF16)
    prev = hb.topk_kernel(mode)
    try:
        ws = torch.empty(max(hb.csa_index_topk_workspace_size(d, n_q, start_pos), 16), dtype=torch.uint8,
                         device=cuda)
        idx = torch.full((B, n_q, k), -7, dtype=torch.int32, device=cuda)
        scores = torch.full((B, n_q, max(E, 1)), float("nan"), device=cuda)
        hb.csa_index_topk(d, qI, wI, KI, None, cap, n_q, start_pos, idx, scores, max(E, 1), ws)
        torch.cuda.synchronize()
    finally:
        hb.topk_kernel(prev)
    gi, gs = idx.cpu().numpy(), scores.cpu().numpy().astype(np.float64)
    for b in range(B):
        for i in range(n_q):
            V = (start_pos + i + 1) // m
            np.testing.assert_array_equal(gi[b, i], O.topk_select(gs[b, i, :V], k), err_msg=f"row ({b}, {i}), V {V}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("B,n_q,start_pos,k", CASES)
def test_selection_kernel_exact(cuda, mode, B, n_q, start_pos, k):
    _select(cuda, mode, B, n_q, start_pos, k, ties=False)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("B,n_q,start_pos,k", CASES[1:])
def test_selection_kernel_exact_ties(cuda, mode, B, n_q, start_pos, k):
    """Three score values per row, thousands of each: the k-th score falls in
    a class of equal scores, kept from the lowest index up."""
    _select(cuda, mode, B, n_q, start_pos, k, ties=True)

