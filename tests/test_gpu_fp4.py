"""FP4 indexer activations on the GPU against the oracle (juejin "DeepSeek-V4
技术报告简要解读" §4.4; 1zeryu "DeepSeek-V4：算法架构", Indexer): rows rotated
by the Hadamard butterflies in fp32 and FP4-quantised in blocks of 32, bit for
bit (both sides rotate in the same fp32 order, so the quantisation decisions
agree exactly)."""
import numpy as np
import pytest
import torch

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import synth
from oracle import hca_oracle as O

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,dtype", [(1, torch.bfloat16), (1003, torch.bfloat16), (77, torch.float32), (0, torch.float32)])
def test_fp4_rotate_quant_matches_oracle(cuda, rows, dtype):
    x = synth.normal((max(rows, 1), 64), 61, 1) * torch.exp2(torch.randint(-20, 20, (max(rows, 1), 1)).float())
    if rows >= 4:
        x[1] = 0.0                               # an all-zero row
        x[2, :32] = 1e-30                        # a tiny block
        x[3] = torch.arange(64).float() - 31.5   # small integers: exact butterflies
    x = x[:rows].to(dtype)
    out = torch.full((max(rows, 1), 64), float("nan"), dtype=torch.bfloat16, device=cuda)
    hb.fp4_rotate_quant(x.to(cuda), hb.HCA_F32 if dtype == torch.float32 else hb.HCA_BF16, rows, 64, out)
    torch.cuda.synchronize()
    if rows == 0:
        assert torch.isnan(out.float()).all()
        return
    want = O.fp4_rotate_quant_gpu_order(x.double().numpy())
    got = out.double().cpu().numpy()
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(np.signbit(got), np.signbit(want))          # zero stored as +0
