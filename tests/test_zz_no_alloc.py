"""csa_index_topk_static_scratch: the index score + top-k call whose scratch is
a fixed device array inside the library instead of a caller workspace.  It
must give exactly what csa_index_topk gives on the same inputs, call after
call (the array is reused and never cleared), and refuse calls that need more
than the array holds.  Collected last so that it also runs after every other
test has used the device."""
import pytest
import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth
from tests.helpers import rnd

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16

CASES = [
    # B, n_q, start_pos, k, key dtype
    (32, 1, 131071, 512, "bf16"),      # decode step of 32 sequences at 128K tokens (4 MiB of scores)
    (1, 300, 0, 64, "bf16"),           # prefill-shaped rows of every length up to 75
    (4, 1, 1048575, 1024, "fp8"),      # 1M-token decode: segmented selection plus merge
]


def _desc(B, k, kdt):
    return hb.attn_desc(B, 4, 64, 16, 8, 4, k=k, n_hI=8, c_I=64, rd_I=16, dtype=hb.HCA_BF16,
                        idx_key_dtype=hb.HCA_FP8E4M3 if kdt == "fp8" else hb.HCA_BF16)


def _inputs(B, n_q, start_pos, k, kdt, seed, cuda):
    m, n_hI, c_I = 4, 8, 64
    cap = (start_pos + n_q) // m + 1
    qI = rnd((B, n_q, n_hI, c_I), seed, 1, BF16)
    wI = rnd((B, n_q, n_hI), seed, 2, std=c_I ** -0.5 * n_hI ** -0.5)
    KIf = synth.normal((B, cap, c_I), seed, 3)
    if kdt == "fp8":
        KI, KI_scale = synth.fp8_rows(KIf)
        KI, KI_scale = KI.to(cuda), KI_scale.to(cuda)
    else:
        KI, KI_scale = KIf.to(BF16).to(cuda), None
    return _desc(B, k, kdt), qI, wI, KI, KI_scale, cap


def _with_workspace(d, qI, wI, KI, KI_scale, cap, B, n_q, start_pos, k, cuda):
    E = max((start_pos + n_q) // 4, 1)
    ws = torch.empty(hb.csa_index_topk_workspace_size(d, n_q, start_pos), dtype=torch.uint8, device=cuda)
    idx = torch.full((B, n_q, k), -7, dtype=torch.int32, device=cuda)
    sc = torch.zeros((B, n_q, E), device=cuda)
    hb.csa_index_topk(d, qI, wI, KI, KI_scale, cap, n_q, start_pos, idx, sc, E, ws)
    return idx, sc


@pytest.mark.parametrize("B,n_q,start_pos,k,kdt", CASES)
def test_static_scratch_matches_workspace_call(cuda, B, n_q, start_pos, k, kdt):
    assert hb.csa_index_topk_workspace_size(_desc(B, k, kdt), n_q, start_pos) <= hb.static_scratch_bytes()
    E = max((start_pos + n_q) // 4, 1)
    runs = []
    # two calls in a row on different inputs, each into its own outputs
    for seed in (11, 12):
        args = _inputs(B, n_q, start_pos, k, kdt, seed, cuda)
        idx = torch.full((B, n_q, k), -7, dtype=torch.int32, device=cuda)
        sc = torch.zeros((B, n_q, E), device=cuda)
        hb.csa_index_topk_static_scratch(*args, n_q, start_pos, idx, sc, E)
        runs.append((args, idx, sc))
    # and once more without the score output, as a decode step calls it
    idx_only = torch.full((B, n_q, k), -7, dtype=torch.int32, device=cuda)
    hb.csa_index_topk_static_scratch(*runs[0][0], n_q, start_pos, idx_only)
    torch.cuda.synchronize()
    for args, idx, sc in runs:
        ref_idx, ref_sc = _with_workspace(*args, B, n_q, start_pos, k, cuda)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        for i in range(n_q):
            V = (start_pos + i + 1) // 4
            assert torch.equal(sc[:, i, :V], ref_sc[:, i, :V])
    assert torch.equal(idx_only, runs[0][1])
    assert not torch.equal(runs[0][1], runs[1][1])   # the two inputs really differ


def test_static_scratch_refuses_calls_beyond_its_size(cuda):
    # 65 sequences at 128K tokens need 65 * 32768 * 4 bytes of scores > 8 MiB
    B, n_q, start_pos, k = 65, 1, 131071, 512
    args = _inputs(B, n_q, start_pos, k, "bf16", 13, cuda)
    assert hb.csa_index_topk_workspace_size(args[0], n_q, start_pos) > hb.static_scratch_bytes()
    idx = torch.full((B, n_q, k), -7, dtype=torch.int32, device=cuda)
    with pytest.raises(hb.HcaError) as e:
        hb.csa_index_topk_static_scratch(*args, n_q, start_pos, idx)
    assert "static scratch holds 8388608" in str(e.value)
    torch.cuda.synchronize()
    assert (idx == -7).all()   # nothing was launched
