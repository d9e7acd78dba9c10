"""Grouped output projection ([J] §2.3.1(d)) on the GPU against the oracle."""
import numpy as np
import pytest
import torch

from long_context_compressed_hca_b200 import binding as hb
from oracle import hca_oracle as O
from tests.helpers import assert_close, rnd, to64

BF16, F32 = torch.bfloat16, torch.float32
CODE = {BF16: hb.HCA_BF16, F32: hb.HCA_F32}

CASES = [
    # T, n_h, c, g, d_g, d, dtype
    (160, 64, 512, 8, 1024, 4096, BF16),   # V4-Flash widths; a ragged 128-row tile (tensor-core GEMMs)
    (300, 16, 128, 4, 256, 512, BF16),
    (50, 16, 128, 4, 256, 512, BF16),      # few rows: the swapped skinny tensor-core tile (64 tokens)
    (32, 64, 512, 8, 1024, 4096, BF16),    # a decode batch of 32 tokens (skinny tile of 32)
    (5, 16, 128, 4, 256, 512, BF16),       # a ragged skinny tile
    (37, 8, 64, 2, 32, 48, F32),
]


@pytest.mark.gpu
@pytest.mark.parametrize("T,n_h,c,g,d_g,d,dt", CASES)
def test_output_projection(cuda, T, n_h, c, g, d_g, d, dt):
    gw = n_h * c // g
    o = rnd((T, n_h, c), 41, 1, dt)
    wo_a = rnd((g, d_g, gw), 41, 2, dt, std=gw ** -0.5)
    wo_b = rnd((d, g * d_g), 41, 3, dt, std=(g * d_g) ** -0.5)
    desc = hb.oproj_desc(T, n_h, c, g, d_g, d, CODE[dt], hb.HCA_F32)
    ws = torch.empty(max(hb.output_projection_workspace_size(desc), 16), dtype=torch.uint8, device=cuda)
    out = torch.full((T, d), float("nan"), device=cuda)
    hb.output_projection(desc, o, wo_a, wo_b, out, ws)
    torch.cuda.synchronize()
    ref = O.output_projection(to64(o), to64(wo_a), to64(wo_b), g)
    # bf16: the intermediate [T, g*d_g] is rounded to bf16 (outputs are O(1))
    assert_close(to64(out), ref, 2e-2 if dt == BF16 else 1e-4, "out")


def test_output_projection_rejects_bad_groups():
    import ctypes
    d = hb.oproj_desc(4, 6, 8, 4, 8, 8)
    rc = hb.lib().hca_output_projection(ctypes.byref(d), 16, 16, 16, 16, 16, 1 << 20, None)
    assert rc == hb.HCA_ERR_INVALID and "multiple of g" in hb.last_error()
