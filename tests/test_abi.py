"""The C-ABI library loads and exports every symbol include/hca.h declares, and
host-side validation rejects bad calls before anything is launched (no GPU
needed: invalid calls return before touching the device)."""
import ctypes

import pytest

from long_context_compressed_hca_b200 import binding as hb
from long_context_compressed_hca_b200 import build as hbuild


@pytest.fixture(scope="module")
def L():
    hbuild.build()
    return hb.lib()


def test_header_declares_the_hot_path():
    names = set(hb.header_functions())
    for f in ("csa_compress", "csa_index_topk", "csa_attend", "hca_attend", "hybrid_layer_forward",
              "hybrid_decode_step", "hca_last_error", "hca_check_status"):
        assert f in names, f


def test_every_declared_symbol_is_exported(L):
    for name in hb.header_functions():
        assert hasattr(L, name), name
    out = __import__("subprocess").run(["nm", "-D", "--defined-only", hb.LIB_PATH],
                                       capture_output=True, text=True).stdout
    for name in hb.header_functions():
        assert f" T {name}" in out, name


def test_version(L):
    assert L.hca_version() >= 1


def _bad(rc, text):
    assert rc == hb.HCA_ERR_INVALID
    assert text in hb.last_error()


def test_compress_rejects_bad_arguments(L):
    d = hb.compress_desc(1, 12, 4, 1, 0, 0, hb.HCA_F32, hb.HCA_F32)   # width not a multiple of 8
    _bad(L.csa_compress(ctypes.byref(d), 0, 8, 16, 16, 16, 16, 12, 96, 16, 16, None, 16, None, 2,
                        None, None, None), "width")
    d = hb.compress_desc(1, 16, 4, 1, 0, 0, hb.HCA_F32, hb.HCA_F32)
    _bad(L.csa_compress(ctypes.byref(d), 0, 8, 16, None, 16, 16, 16, 128, 16, 16, None, 16, None, 2,
                        None, None, None), "overlap needs")
    _bad(L.csa_compress(ctypes.byref(d), 0, 8, 24, 16, 16, 16, 16, 128, 16, 16, None, 16, None, 2,
                        None, None, None), "aligned")
    _bad(L.csa_compress(ctypes.byref(d), 5, 2, 16, 16, 16, 16, 16, 128, 16, 16, None, 16, None, 2,
                        16, 16, None), "exactly one token")
    _bad(L.csa_compress(ctypes.byref(d), 5, 1, 16, 16, 16, 16, 16, 128, 16, 16, None, 16, None, 2,
                        None, None, None), "state")
    d8 = hb.compress_desc(1, 16, 4, 0, 0, 0, hb.HCA_F32, hb.HCA_FP8E4M3)
    _bad(L.csa_compress(ctypes.byref(d8), 0, 8, 16, None, 16, None, 16, 128, 16, None, None, 16,
                        None, 2, None, None, None), "out_scale")


def test_attend_rejects_bad_arguments(L):
    d = hb.attn_desc(1, 4, 64, 16, 8, 4, k=4)
    # cap smaller than the visible entries
    _bad(L.hca_attend(ctypes.byref(d), 16, 16, 1, 16, 0, 16, 64, 0, 16, None, 0, None), "cap")
    # ring window with several queries
    _bad(L.hca_attend(ctypes.byref(d), 16, 16, 100, 16, 1, 16, 4, 0, 16, None, 0, None), "ring")
    dbad = hb.attn_desc(1, 4, 48, 16, 8, 4, k=4)
    _bad(L.hca_attend(ctypes.byref(dbad), 16, 16, 100, 16, 0, 16, 4, 0, 16, None, 0, None), "multiple of 32")
    _bad(L.csa_attend(ctypes.byref(d), 16, 16, 100, None, 16, 0, 16, 4, 0, 16, None, 0, None), "idx")
    dneg = hb.attn_desc(1, 4, 64, 16, 8, 4, k=4, max_ctas=-1)
    _bad(L.hca_attend(ctypes.byref(dneg), 16, 16, 100, 16, 0, 16, 4, 0, 16, None, 0, None), "max_ctas")


def test_index_rejects_bad_arguments(L):
    d = hb.attn_desc(1, 4, 64, 16, 8, 4, k=0, n_hI=4, c_I=32, rd_I=16)
    _bad(L.csa_index_topk(ctypes.byref(d), 16, 16, 16, None, 100, 4, 0, 16, None, 0, None, 0, None), "k must")
    d = hb.attn_desc(1, 4, 64, 16, 8, 4, k=4, n_hI=4, c_I=32, rd_I=16, idx_key_dtype=hb.HCA_FP8E4M3)
    _bad(L.csa_index_topk(ctypes.byref(d), 16, 16, 16, None, 100, 4, 0, 16, None, 0, None, 0, None), "KI_scale")
    d = hb.attn_desc(1, 4, 64, 16, 8, 4, k=4, n_hI=4, c_I=32, rd_I=16)
    _bad(L.csa_index_topk(ctypes.byref(d), 16, 16, 16, None, 1, 64, 0, 16, None, 0, None, 0, None), "cap")


def test_layer_rejects_bad_arguments(L):
    lay = hb.Layer()
    lay.kind = hb.HCA_LAYER_CSA
    lay.a = hb.attn_desc(1, 4, 64, 16, 8, 4, overlap=1, k=4, n_hI=4, c_I=32, rd_I=16)
    lay.d, lay.d_c = 64, 16
    lay.sink = 16
    _bad(L.hybrid_layer_forward(ctypes.byref(lay), 16, 8, None, 16, 16, 1 << 20, None), "missing layer weight")
    assert L.hybrid_layer_forward_workspace_size(ctypes.byref(lay), 64) > 0


def test_kv_mixed_sizes_and_rejections(L):
    assert L.hca_kv_mixed_row_bytes(512, 64) == 608          # 448 + 128 + 28 = 604, padded to 16
    assert L.hca_kv_mixed_row_bytes(128, 64) == 208          # 64 + 128 + 4 = 196 -> 208
    for c, rd in ((512, 60), (640, 64), (512, 32), (64, 80)):
        assert L.hca_kv_mixed_row_bytes(c, rd) == 0, (c, rd)
    _bad(L.hca_kv_quant_mixed(16, hb.HCA_BF16, 4, 512, 32, 16, None), "unsupported")
    _bad(L.hca_kv_quant_mixed(16, hb.HCA_FP8E4M3, 4, 512, 64, 16, None), "x_dtype")
    _bad(L.hca_kv_quant_mixed(16, hb.HCA_BF16, -1, 512, 64, 16, None), "rows")
    _bad(L.hca_kv_quant_mixed(24, hb.HCA_BF16, 4, 512, 64, 16, None), "aligned")
    _bad(L.hca_kv_quant_mixed(None, hb.HCA_BF16, 4, 512, 64, 16, None), "non-null")
    _bad(L.hca_kv_dequant_mixed(16, 4, 512, 64, 40, None), "aligned")
    assert L.hca_kv_dequant_mixed(None, 0, 512, 64, None, None) == hb.HCA_OK   # empty call


def test_attention_cta_budget_sets_the_split_plan(L):
    """The CTA budget bounds the split-KV count per query, visible here through
    the workspace a call needs: splits beyond 8 go through an fp32 workspace
    of q * splits * 64 rows of c floats (+ 64 (max, sum) pairs each); up to 8
    merge inside a thread-block cluster and need none.  4 sequences at the 1M
    position: HCA has 130 key tiles per query, CSA (k = 1024) 18."""
    def ws(kind, max_ctas):
        k = 1024 if kind == "csa" else 0
        m = 4 if kind == "csa" else 128
        d = hb.attn_desc(4, 64, 512, 64, 128, m, k=k, dtype=hb.HCA_BF16, max_ctas=max_ctas)
        f = L.csa_attend_workspace_size if kind == "csa" else L.hca_attend_workspace_size
        return f(ctypes.byref(d), 1, 1048576)

    def split_ws(ns, q=4, c=512):
        return q * ns * 64 * c * 4 + q * ns * 64 * 8
    sms = 148
    assert ws("hca", 0) == split_ws(min(sms // 4, 65, 32))       # 32 splits
    assert ws("hca", 64) == split_ws(16)
    assert ws("hca", 32) == 0                                    # 8 splits: cluster merge
    assert ws("hca", 4) == 0                                     # 1 split
    assert ws("csa", 0) == split_ws(9)                           # 18 tiles -> 9 splits
    assert ws("csa", 32) == 0


def test_fp4_rotate_quant_rejects_bad_arguments(L):
    _bad(L.hca_fp4_rotate_quant(16, hb.HCA_BF16, 4, 32, 16, None), "n must be 64")
    _bad(L.hca_fp4_rotate_quant(16, hb.HCA_FP8E4M3, 4, 64, 16, None), "x_dtype")
    _bad(L.hca_fp4_rotate_quant(24, hb.HCA_BF16, 4, 64, 16, None), "aligned")
    assert L.hca_fp4_rotate_quant(None, hb.HCA_BF16, 0, 64, None, None) == hb.HCA_OK


def test_static_scratch_size_matches_header(L):
    assert L.hca_static_scratch_bytes() == hb.STATIC_SCRATCH_BYTES == hb.static_scratch_bytes()


def test_hca_compress_alias_validates_like_csa_compress(L):
    d = hb.compress_desc(1, 12, 4, 0, 0, 0, hb.HCA_F32, hb.HCA_F32)   # width not a multiple of 8
    _bad(L.hca_compress(ctypes.byref(d), 0, 8, 16, None, 16, None, 12, 96, 16, None, None, 16, None, 2,
                        None, None, None), "width")


def test_workspace_map_places_intermediates_inside_the_workspace(L):
    """hybrid_workspace_map: every prefill intermediate lies inside the
    workspace hybrid_layer_forward_workspace_size asks for, 256-byte aligned,
    without overlaps; decode keeps its index lists at offset 0."""
    from long_context_compressed_hca_b200 import workloads
    for wl in (workloads.TINY_CSA, workloads.CSA_PREFILL.with_(n=4096, d=512, d_c=256), workloads.HCA_PREFILL):
        Ls = wl.layers[0]
        csa = Ls.kind == "csa"
        lay = hb.Layer()
        lay.kind = hb.HCA_LAYER_CSA if csa else hb.HCA_LAYER_HCA
        lay.a = hb.attn_desc(wl.B, Ls.n_h, Ls.c, Ls.rd, Ls.w, Ls.m, overlap=Ls.overlap, k=Ls.k,
                             n_hI=Ls.n_hI, c_I=Ls.c_I, rd_I=Ls.rd_I if csa else 0, dtype=hb.HCA_BF16)
        lay.d, lay.d_c = wl.d, wl.d_c
        lay.sink = 16
        n = wl.n
        total = L.hybrid_layer_forward_workspace_size(ctypes.byref(lay), n)
        mp = hb.workspace_map(lay, n)
        B, E = wl.B, max(n // Ls.m, 1)
        sizes = dict(q=B * n * Ls.n_h * Ls.c * 2, kv_win=B * n * Ls.c * 2, kv_comp=B * E * Ls.c * 2)
        if csa:
            sizes.update(idx=B * n * Ls.k * 4, qI=B * n * Ls.n_hI * Ls.c_I * 2, wI=B * n * Ls.n_hI * 4,
                         key_I=B * E * Ls.c_I * 2)
        else:
            assert mp["idx"] is None and mp["qI"] is None and mp["key_I"] is None
        spans = []
        for key, size in sizes.items():
            off = mp[key]
            assert off is not None and off % 256 == 0 and off + size <= total, (wl.name, key, off, size, total)
            spans.append((off, off + size))
        spans.sort()
        assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:])), spans
        dm = hb.workspace_map(lay, 131072, decode=True)
        assert (dm["idx"] == 0) if csa else (dm["idx"] is None)
        assert L.hybrid_workspace_map(ctypes.byref(lay), 0, 1, ctypes.byref(hb.WsMap())) == hb.HCA_ERR_INVALID


def test_step_trace_rejects_bad_buffers(L):
    _bad(L.hca_step_trace(12, 1024), "8-byte aligned")
    _bad(L.hca_step_trace(16, 32), "8-byte aligned")


def test_topk_kernel_knob_round_trip(L):
    prev = hb.topk_kernel(hb.TOPK_WARP)
    try:
        assert hb.topk_kernel(-1) == hb.TOPK_WARP
    finally:
        hb.topk_kernel(prev)
    assert hb.topk_kernel(-1) == prev
    _bad(L.hca_topk_kernel(5), "top-k kernel mode")
