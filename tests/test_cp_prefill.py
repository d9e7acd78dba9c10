"""Context-parallel prefill (juejin "DeepSeek-V4 技术报告简要解读" §4.5, the
two-stage communication of compressed attention): a sequence's tokens are cut
into ranges, one per rank; each rank compresses its range, one all-gather
collects every range's entries and indexer keys, and each rank attends its
queries against the gathered caches.

CPU (gloo, 2 and 3 ranks): the driver's partitioning, halo exchange and
entry all-gather, with the rank stages written from the oracle, reproduce
the oracle's whole-sequence layer.  GPU (one device): libhca's two stages,
run for every range in turn with the all-gathers done by concatenation,
reproduce hybrid_layer_forward on the whole sequence (no kernel of one range
waits on another's)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from long_context_compressed_hca_b200 import cp_prefill as CP
from long_context_compressed_hca_b200 import synth, workloads
from oracle import hca_oracle as O


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_cp_ranges_cover_the_sequence_on_block_starts():
    for n, world, align in ((512, 2, 4), (512, 3, 4), (8192, 8, 128), (1000, 4, 128), (7, 4, 1)):
        rs = CP.cp_ranges(n, world, align)
        assert len(rs) == world
        assert sum(r[1] for r in rs) == n
        t = 0
        for t0, n_loc in rs:
            assert t0 == t and t0 % align == 0 or n_loc == 0
            t += n_loc
        assert all(r[1] % align == 0 for r in rs[:-1] if rs[rs.index(r) + 1][1] > 0)
    assert CP.lcm_align(4, 128) == 128 and CP.lcm_align(4, 6) == 12


def _case(name):
    if name == "csa":
        wl = workloads.TINY_CSA
        return wl, wl.layers[0], wl.n, torch.float32
    wl = workloads.HCA_PREFILL.with_(B=1, n=1024, d=256, d_c=64)
    return wl, wl.layers[0], wl.n, torch.float32


def _worker(rank, world, port, name, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from tests.cp_oracle_stages import OracleCPStages
        wl, L, n, dt = _case(name)
        W = synth.layer_weights(L, wl.d, wl.d_c, wl.seed, dt, bias_std=0.3)
        W64 = {k: v.double().numpy() for k, v in W.items()}
        H = synth.hidden_states(1, n, wl.d, wl.seed, dt).double()
        st = OracleCPStages(L, W64, wl.d_c)
        t0, n_loc = CP.cp_ranges(n, world, L.m)[rank]
        o = CP.cp_prefill(st, H[:, t0:t0 + n_loc].contiguous(), n, L.m)
        out[rank] = (t0, n_loc, o.numpy())
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("name,world", [("csa", 2), ("csa", 3), ("hca", 2)])
def test_cp_prefill_gloo_ranks_match_the_oracle(name, world):
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, _free_port(), name, out), nprocs=world, join=True)
        res = dict(out)
    wl, L, n, dt = _case(name)
    W = synth.layer_weights(L, wl.d, wl.d_c, wl.seed, dt, bias_std=0.3)
    W64 = {k: v.double().numpy() for k, v in W.items()}
    H = synth.hidden_states(1, n, wl.d, wl.seed, dt).double()
    ref = O.layer_prefill(H[0].numpy(), W64, L, wl.d_c)
    got = np.concatenate([res[r][2][0] for r in range(world)], axis=0)
    assert got.shape == ref.shape
    assert sum(res[r][1] for r in range(world)) == n
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-9)


# ----------------------------------------------------------------- GPU: libhca's stages
@pytest.mark.gpu
@pytest.mark.parametrize("name,world,dt", [("csa", 2, "f32"), ("csa", 3, "f32"), ("csa4k", 4, "bf16"),
                                           ("hca", 2, "bf16")])
def test_cp_stages_on_gpu_match_the_whole_sequence(cuda, name, world, dt):
    from long_context_compressed_hca_b200 import binding as hb
    from long_context_compressed_hca_b200.layer import LayerHandle
    from tests.helpers import TOL, assert_close, check_topk_row, to64
    dtype = torch.float32 if dt == "f32" else torch.bfloat16
    if name == "csa":
        wl = workloads.TINY_CSA.with_(B=2)
    elif name == "csa4k":
        wl = workloads.CSA_PREFILL.with_(n=4096, d=512, d_c=256, B=2)
    else:
        wl = workloads.HCA_PREFILL.with_(n=2048)
    L = wl.layers[0]
    n = wl.n
    W = synth.layer_weights(L, wl.d, wl.d_c, wl.seed, dtype, bias_std=0.3)
    H = synth.hidden_states(wl.B, n, wl.d, wl.seed, dtype).to(cuda)
    lh = LayerHandle(L, W, wl.d, wl.d_c, dtype, wl.B, device=cuda)
    # the whole sequence in one call
    ws = torch.empty(hb.layer_workspace_size(lh.struct, n), dtype=torch.uint8, device=cuda)
    o_ref = torch.empty(wl.B, n, L.n_h, L.c, dtype=dtype, device=cuda)
    hb.hybrid_layer_forward(lh.struct, H, n, None, o_ref, ws)
    mp_ = hb.workspace_map(lh.struct, n)
    idx_ref = hb.ws_view(ws, mp_["idx"], (wl.B, n, L.k), torch.int32).clone() if L.kind == "csa" else None
    # the same sequence cut into ranges: stage 1 for every range, the gathers, stage 2
    st = CP.CPLayer(lh)
    ranges = CP.cp_ranges(n, world, L.m)
    Hs, parts = [], []
    for t0, n_loc in ranges:
        h = st.halo(t0)
        Hr = H[:, t0 - h:t0 + n_loc].contiguous()
        Hs.append(Hr)
        parts.append(st.compress(Hr, t0, n_loc))
    kv = torch.cat([p[0] for p in parts], 1).contiguous()
    kI = torch.cat([p[1] for p in parts], 1).contiguous() if L.kind == "csa" else None
    outs = [st.attend(Hs[i], t0, n_loc, kv, kI, None) for i, (t0, n_loc) in enumerate(ranges)]
    o = torch.cat(outs, 1)
    torch.cuda.synchronize()
    # the caches equal the whole-sequence prefill's
    E = n // L.m
    kv_ref = hb.ws_view(ws, mp_["kv_comp"], (wl.B, E, L.c), dtype)
    tol = TOL[dtype]
    assert_close(to64(kv), to64(kv_ref), tol, "gathered entries")
    if L.kind == "csa":
        kI_ref = hb.ws_view(ws, mp_["key_I"], (wl.B, E, L.c_I), dtype)
        assert_close(to64(kI), to64(kI_ref), tol, "gathered indexer keys")
    # the outputs: equal where the selections agree (the ranges compute the same
    # rounded operands, so they do unless a score tie is split differently)
    assert_close(to64(o), to64(o_ref), tol, "o")
