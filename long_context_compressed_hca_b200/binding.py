"""Thin ctypes binding of libhca (include/hca.h): argument marshalling only.

Every step of the path runs in the library's CUDA kernels; PyTorch supplies
device memory and streams.  Loading fails loudly if libhca.so is missing.
"""
from __future__ import annotations

import ctypes as C
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhca.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "hca.h")

HCA_OK, HCA_ERR_INVALID, HCA_ERR_UNSUPPORTED, HCA_ERR_CUDA, HCA_ERR_TIMEOUT = 0, -1, -2, -3, -4
HCA_F32, HCA_BF16, HCA_FP8E4M3, HCA_FP4 = 0, 1, 2, 3
HCA_COMPRESS_NORM, HCA_COMPRESS_ROPE = 1, 2
HCA_LAYER_CSA, HCA_LAYER_HCA, HCA_LAYER_SWA = 0, 1, 2
# HCA_STATIC_SCRATCH_BYTES of include/hca.h; lib() checks that the loaded library agrees.
STATIC_SCRATCH_BYTES = 8 << 20

DTYPE_CODE = {torch.float32: HCA_F32, torch.bfloat16: HCA_BF16, torch.uint8: HCA_FP8E4M3,
              torch.float8_e4m3fn: HCA_FP8E4M3}


class HcaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libhca error {code}: {msg}")
        self.code = code


class AttnDesc(C.Structure):
    _fields_ = [("B", C.c_int), ("n_h", C.c_int), ("c", C.c_int), ("rd", C.c_int), ("w", C.c_int),
                ("m", C.c_int), ("overlap", C.c_int), ("k", C.c_int), ("n_hI", C.c_int),
                ("c_I", C.c_int), ("rd_I", C.c_int), ("dtype", C.c_int), ("idx_key_dtype", C.c_int),
                ("scale", C.c_float), ("eps", C.c_float), ("rope_theta", C.c_float), ("max_ctas", C.c_int),
                ("kv_mixed", C.c_int)]


class CompressDesc(C.Structure):
    _fields_ = [("B", C.c_int), ("width", C.c_int), ("m", C.c_int), ("overlap", C.c_int),
                ("rd", C.c_int), ("flags", C.c_int), ("eps", C.c_float), ("rope_theta", C.c_float),
                ("in_dtype", C.c_int), ("out_dtype", C.c_int)]


class Layer(C.Structure):
    _fields_ = [("kind", C.c_int), ("a", AttnDesc), ("d", C.c_int), ("d_c", C.c_int),
                ("W_comp", C.c_void_p), ("B_comp", C.c_void_p), ("W_compI", C.c_void_p),
                ("B_compI", C.c_void_p), ("W_DQ", C.c_void_p), ("W_UQ", C.c_void_p),
                ("W_IUQ", C.c_void_p), ("W_w", C.c_void_p), ("W_KV", C.c_void_p),
                ("sink", C.c_void_p)]


class Cache(C.Structure):
    _fields_ = [("cap", C.c_int), ("kv_comp", C.c_void_p), ("key_I", C.c_void_p),
                ("key_I_scale", C.c_void_p), ("win", C.c_void_p), ("state_kv", C.c_void_p),
                ("state_score", C.c_void_p), ("stateI_kv", C.c_void_p), ("stateI_score", C.c_void_p)]


class OprojDesc(C.Structure):
    _fields_ = [("T", C.c_int), ("n_h", C.c_int), ("c", C.c_int), ("g", C.c_int), ("d_g", C.c_int),
                ("d", C.c_int), ("dtype", C.c_int), ("out_dtype", C.c_int)]


class WsMap(C.Structure):
    _fields_ = [(f, C.c_longlong) for f in ("idx", "q", "qI", "wI", "key_I", "kv_comp", "kv_win")]


class TokenIn(C.Structure):
    _fields_ = [("q", C.c_void_p), ("qI", C.c_void_p), ("wI", C.c_void_p), ("kv", C.c_void_p),
                ("comp", C.c_void_p), ("compI", C.c_void_p)]


_lib = None
VP, I, LL, SZ = C.c_void_p, C.c_int, C.c_longlong, C.c_size_t


def _declare(L):
    sig = {
        "hca_last_error": (C.c_char_p, []),
        "hca_version": (I, []),
        "hca_launch_count": (LL, []),
        "hca_check_status": (I, [VP, C.POINTER(C.c_int)]),
        "hca_selftest_wait": (I, [C.c_ulonglong, VP]),
        "hca_profile_enable": (I, [I]),
        "hca_profile_sample": (I, []),
        "hca_profile_collect": (I, [C.c_char_p, SZ]),
        "hca_trace_attend": (I, [I, C.POINTER(C.c_ulonglong), I]),
        "hca_topk_kernel": (I, [I]),
        "csa_compress": (I, [C.POINTER(CompressDesc), I, I, VP, VP, VP, VP, LL, LL, VP, VP, VP, VP,
                             VP, LL, VP, VP, VP]),
        "csa_index_topk_workspace_size": (SZ, [C.POINTER(AttnDesc), I, I]),
        "csa_index_topk": (I, [C.POINTER(AttnDesc), VP, VP, VP, VP, I, I, I, VP, VP, LL, VP, SZ, VP]),
        "csa_index_topk_static_scratch": (I, [C.POINTER(AttnDesc), VP, VP, VP, VP, I, I, I, VP, VP, LL, VP]),
        "csa_attend_workspace_size": (SZ, [C.POINTER(AttnDesc), I, I]),
        "csa_attend": (I, [C.POINTER(AttnDesc), VP, VP, I, VP, VP, I, VP, I, I, VP, VP, SZ, VP]),
        "hca_attend_workspace_size": (SZ, [C.POINTER(AttnDesc), I, I]),
        "hca_attend": (I, [C.POINTER(AttnDesc), VP, VP, I, VP, I, VP, I, I, VP, VP, SZ, VP]),
        "hybrid_layer_forward_workspace_size": (SZ, [C.POINTER(Layer), I]),
        "hybrid_layer_forward": (I, [C.POINTER(Layer), VP, I, C.POINTER(Cache), VP, VP, SZ, VP]),
        "hybrid_decode_step_workspace_size": (SZ, [C.POINTER(Layer), I]),
        "hca_output_projection_workspace_size": (SZ, [C.POINTER(OprojDesc)]),
        "hca_output_projection": (I, [C.POINTER(OprojDesc), VP, VP, VP, VP, VP, SZ, VP]),
        "hybrid_decode_step": (I, [C.POINTER(Layer), C.POINTER(TokenIn), C.POINTER(Cache), I, VP, VP,
                                   SZ, VP]),
        "hca_kv_mixed_row_bytes": (SZ, [I, I]),
        "hybrid_decode_inputs_workspace_size": (SZ, [C.POINTER(Layer)]),
        "hybrid_decode_inputs": (I, [C.POINTER(Layer), VP, I, C.POINTER(TokenIn), VP, SZ, VP]),
        "hca_static_scratch_bytes": (SZ, []),
        "hca_compress": (I, [C.POINTER(CompressDesc), I, I, VP, VP, VP, VP, LL, LL, VP, VP, VP, VP,
                             VP, LL, VP, VP, VP]),
        "hybrid_workspace_map": (I, [C.POINTER(Layer), I, I, C.POINTER(WsMap)]),
        "hca_fp4_rotate_quant": (I, [VP, I, LL, I, VP, VP]),

        "hca_step_trace": (I, [VP, SZ]),
        "hybrid_cp_halo": (I, [C.POINTER(Layer), I]),
        "hybrid_cp_workspace_size": (SZ, [C.POINTER(Layer), I, I]),
        "hybrid_cp_compress": (I, [C.POINTER(Layer), VP, I, I, VP, VP, VP, I, VP, SZ, VP]),
        "hybrid_cp_attend": (I, [C.POINTER(Layer), VP, I, I, VP, VP, VP, I, VP, VP, SZ, VP]),
        "hca_kv_quant_mixed": (I, [VP, I, LL, I, I, VP, VP]),
        "hca_kv_dequant_mixed": (I, [VP, LL, I, I, VP, VP]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args


def lib():
    """Load libhca.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise HcaError(HCA_ERR_UNSUPPORTED,
                           f"{LIB_PATH} is missing: build it with "
                           "`python -m long_context_compressed_hca_b200.build`")
        L = C.CDLL(LIB_PATH)
        _declare(L)
        if L.hca_static_scratch_bytes() != STATIC_SCRATCH_BYTES:
            raise HcaError(HCA_ERR_UNSUPPORTED, "libhca.so was built with a different static scratch size "
                           f"({L.hca_static_scratch_bytes()} != {STATIC_SCRATCH_BYTES}): rebuild it")
        _lib = L
    return _lib


def header_functions() -> list:
    """Names of the functions include/hca.h declares."""
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?(?:int|size_t|long long|char\s*\*|const char\s*\*)\s*\**\s*"
                                 r"([a-z_][a-z0-9_]*)\s*\(", txt, flags=re.M)))


def ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def stream_handle(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def check(rc: int):
    if rc != HCA_OK:
        raise HcaError(rc, lib().hca_last_error().decode(errors="replace"))
    return rc


def last_error() -> str:
    return lib().hca_last_error().decode(errors="replace")


def device_status(stream=None) -> int:
    v = C.c_int(0)
    check(lib().hca_check_status(stream_handle(stream), C.byref(v)))
    return v.value


def selftest_wait(limit_ns: int, stream=None):
    """Launch the bounded-wait self-test kernel (its wait always expires)."""
    return check(lib().hca_selftest_wait(limit_ns, stream_handle(stream)))


def launch_count() -> int:
    return lib().hca_launch_count()


def profile_enable(on: bool = True):
    check(lib().hca_profile_enable(int(on)))


def profile_sample():
    check(lib().hca_profile_sample())


def profile_collect() -> dict:
    """{kernel name: (launches, total ms)} since the last collect."""
    buf = C.create_string_buffer(1 << 16)
    check(lib().hca_profile_collect(buf, len(buf)))
    out = {}
    for line in buf.value.decode().splitlines():
        name, n, ms = line.split("\t")
        out[name] = (int(n), float(ms))
    return out


TRACE_SLOTS = ("prod_q_free", "prod_stage_free", "mma_q_ready", "mma_tile_ready", "mma_s_free",
               "mma_p_ready", "mma_o_free", "smax_s_ready", "smax_pbuf_free", "smax_rescale_wait",
               "smax_epi_wait", "smax_unit_setup", "epilogue", "total", "rescales", "units", "tiles", "smax_pair_xchg",
               "merge_wait_ready", "merge_wait_full", "merge_push", "merge_weights", "merge_loop",
               "t_setup", "t_first_s", "t_tiles", "t_epilogue", "t_exit", "t_entry_inv", "t_exit_max", "t_ctas")


TOPK_AUTO, TOPK_ROW, TOPK_WARP, TOPK_CLUSTER, TOPK_ROW_CLUSTER = 0, 1, 2, 3, 4


def topk_kernel(mode: int = -1) -> int:
    """Select the top-k kernel (TOPK_*; -1 only reads); returns the previous mode."""
    r = lib().hca_topk_kernel(mode)
    if r < 0:
        check(r)
    return r


def trace_attend(enable: int):
    """Switch the attention wait-cycle trace on (1) / off (0) and reset it."""
    check(lib().hca_trace_attend(enable, None, 0))


def trace_attend_read() -> dict:
    buf = (C.c_ulonglong * 32)()
    check(lib().hca_trace_attend(-1, buf, 32))
    return {k: int(buf[i]) for i, k in enumerate(TRACE_SLOTS) if k != "-"}


def attn_desc(B, n_h, c, rd, w, m, overlap=0, k=0, n_hI=0, c_I=0, rd_I=0, dtype=HCA_BF16,
              idx_key_dtype=None, scale=0.0, eps=1e-6, rope_theta=10000.0, max_ctas=0, kv_mixed=0) -> AttnDesc:
    return AttnDesc(B, n_h, c, rd, w, m, int(overlap), k, n_hI, c_I, rd_I, dtype,
                    dtype if idx_key_dtype is None else idx_key_dtype, scale, eps, rope_theta, max_ctas,
                    int(kv_mixed))


def compress_desc(B, width, m, overlap, rd, flags, in_dtype, out_dtype, eps=1e-6,
                  rope_theta=10000.0) -> CompressDesc:
    return CompressDesc(B, width, m, int(overlap), rd, flags, eps, rope_theta, in_dtype, out_dtype)


# --------------------------------------------------------------------- calls
def csa_compress(d: CompressDesc, start_pos, n, Ca, Cb, Za, Zb, row_stride, seq_stride, Ba, Bb,
                 gamma, out, out_scale, out_seq_stride, state_kv, state_score, stream=None, hca_name=False):
    fn = lib().hca_compress if hca_name else lib().csa_compress
    return check(fn(C.byref(d), start_pos, n, ptr(Ca), ptr(Cb), ptr(Za), ptr(Zb),
                                    row_stride, seq_stride, ptr(Ba), ptr(Bb), ptr(gamma), ptr(out),
                                    ptr(out_scale), out_seq_stride, ptr(state_kv), ptr(state_score),
                                    stream_handle(stream)))


def csa_index_topk_workspace_size(d: AttnDesc, n_q, start_pos) -> int:
    return lib().csa_index_topk_workspace_size(C.byref(d), n_q, start_pos)


def csa_index_topk(d: AttnDesc, qI, wI, KI, KI_scale, cap, n_q, start_pos, idx, scores=None,
                   score_stride=0, ws=None, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    return check(lib().csa_index_topk(C.byref(d), ptr(qI), ptr(wI), ptr(KI), ptr(KI_scale), cap, n_q,
                                      start_pos, ptr(idx), ptr(scores), score_stride, ptr(ws), nbytes,
                                      stream_handle(stream)))


def static_scratch_bytes() -> int:
    """Size of the library's fixed scratch array (csa_index_topk_static_scratch)."""
    return lib().hca_static_scratch_bytes()


def csa_index_topk_static_scratch(d: AttnDesc, qI, wI, KI, KI_scale, cap, n_q, start_pos, idx, scores=None,
                                  score_stride=0, stream=None):
    return check(lib().csa_index_topk_static_scratch(C.byref(d), ptr(qI), ptr(wI), ptr(KI), ptr(KI_scale), cap,
                                                     n_q, start_pos, ptr(idx), ptr(scores), score_stride,
                                                     stream_handle(stream)))


def csa_attend_workspace_size(d: AttnDesc, n_q, start_pos) -> int:
    return lib().csa_attend_workspace_size(C.byref(d), n_q, start_pos)


def hca_attend_workspace_size(d: AttnDesc, n_q, start_pos) -> int:
    return lib().hca_attend_workspace_size(C.byref(d), n_q, start_pos)


def csa_attend(d: AttnDesc, q, kv_comp, cap, idx, kv_win, win_is_ring, sink, n_q, start_pos, o,
               ws=None, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    return check(lib().csa_attend(C.byref(d), ptr(q), ptr(kv_comp), cap, ptr(idx), ptr(kv_win),
                                  int(win_is_ring), ptr(sink), n_q, start_pos, ptr(o), ptr(ws), nbytes,
                                  stream_handle(stream)))


def hca_attend(d: AttnDesc, q, kv_comp, cap, kv_win, win_is_ring, sink, n_q, start_pos, o, ws=None,
               stream=None):
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    return check(lib().hca_attend(C.byref(d), ptr(q), ptr(kv_comp), cap, ptr(kv_win), int(win_is_ring),
                                  ptr(sink), n_q, start_pos, ptr(o), ptr(ws), nbytes,
                                  stream_handle(stream)))


def layer_workspace_size(L: Layer, n: int) -> int:
    return lib().hybrid_layer_forward_workspace_size(C.byref(L), n)


def ctypes_byref(x):
    return C.byref(x)


def hybrid_cp_compress(L: Layer, H, t0, n_loc, kv_comp, key_I, key_I_scale, out_cap, ws, stream=None):
    nbytes = ws.numel() * ws.element_size()
    return check(lib().hybrid_cp_compress(C.byref(L), ptr(H), t0, n_loc, ptr(kv_comp), ptr(key_I), ptr(key_I_scale),
                                          out_cap, ptr(ws), nbytes, stream_handle(stream)))


def hybrid_cp_attend(L: Layer, H, t0, n_loc, kv_comp, key_I, key_I_scale, cap, o, ws, stream=None):
    nbytes = ws.numel() * ws.element_size()
    return check(lib().hybrid_cp_attend(C.byref(L), ptr(H), t0, n_loc, ptr(kv_comp), ptr(key_I), ptr(key_I_scale),
                                        cap, ptr(o), ptr(ws), nbytes, stream_handle(stream)))


def workspace_map(L: Layer, n: int, decode: bool = False) -> dict:
    """Byte offsets of the intermediates hybrid_layer_forward (decode=False,
    n tokens) or hybrid_decode_step (decode=True, pos n) leaves in its
    workspace; None where the call has no such buffer."""
    m = WsMap()
    check(lib().hybrid_workspace_map(C.byref(L), n, int(decode), C.byref(m)))
    return {f: (getattr(m, f) if getattr(m, f) >= 0 else None) for f, _ in WsMap._fields_}


def ws_view(ws, offset: int, shape, dtype):
    """A tensor view of `shape` / `dtype` at byte `offset` of a uint8 workspace."""
    n = 1
    for x in shape:
        n *= x
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    return ws[offset:offset + nbytes].view(dtype).view(*shape)


def hybrid_layer_forward(L: Layer, H, n, cache: Cache | None, o, ws, stream=None):
    nbytes = ws.numel() * ws.element_size()
    return check(lib().hybrid_layer_forward(C.byref(L), ptr(H), n, C.byref(cache) if cache else None,
                                            ptr(o), ptr(ws), nbytes, stream_handle(stream)))


def decode_inputs_workspace_size(L: Layer) -> int:
    return lib().hybrid_decode_inputs_workspace_size(C.byref(L))


def hybrid_decode_inputs(L: Layer, h, pos, x: TokenIn, ws, stream=None):
    """Write the decode token inputs x (buffers the caller allocated) from hidden states h [B, d]."""
    nbytes = ws.numel() * ws.element_size()
    return check(lib().hybrid_decode_inputs(C.byref(L), ptr(h), pos, C.byref(x), ptr(ws), nbytes,
                                            stream_handle(stream)))


def decode_workspace_size(L: Layer, pos: int) -> int:
    return lib().hybrid_decode_step_workspace_size(C.byref(L), pos)


def hybrid_decode_step(L: Layer, x: TokenIn, cache: Cache, pos, o, ws, stream=None):
    nbytes = ws.numel() * ws.element_size()
    return check(lib().hybrid_decode_step(C.byref(L), C.byref(x), C.byref(cache), pos, ptr(o), ptr(ws),
                                          nbytes, stream_handle(stream)))


def oproj_desc(T, n_h, c, g, d_g, d, dtype=HCA_BF16, out_dtype=HCA_F32) -> OprojDesc:
    return OprojDesc(T, n_h, c, g, d_g, d, dtype, out_dtype)


def output_projection_workspace_size(d: OprojDesc) -> int:
    return lib().hca_output_projection_workspace_size(C.byref(d))


def fp4_rotate_quant(x, x_dtype, rows, n, out, stream=None):
    return check(lib().hca_fp4_rotate_quant(ptr(x), x_dtype, rows, n, ptr(out), stream_handle(stream)))


STEP_TRACE_KERNELS = {1: "ingest", 2: "indexer", 3: "top-k", 4: "attend CSA", 5: "attend HCA"}


def step_trace(buf):
    """Point the decode-step kernels at `buf` (a zeroed uint64 device tensor:
    counter, then 4 words per CTA record), or switch the trace off (None)."""
    nbytes = buf.numel() * buf.element_size() if buf is not None else 0
    return check(lib().hca_step_trace(ptr(buf), nbytes))


def step_trace_records(buf):
    """The records of a trace buffer as a list of dicts (host copy)."""
    h = buf.cpu().numpy().view("uint64")
    n = min(int(h[0]), (h.shape[0] - 1) // 4)
    recs = h[1:1 + 4 * n].reshape(n, 4)
    return [{"kernel": STEP_TRACE_KERNELS.get(int(r[3] >> 48), str(int(r[3] >> 48))),
             "sm": int((r[3] >> 32) & 0xFFFF), "cta": int(r[3] & 0xFFFFFFFF),
             "entry": int(r[0]), "ready": int(r[1]), "exit": int(r[2])} for r in recs]


def kv_mixed_row_bytes(c, rd) -> int:
    """Bytes of one row record in the mixed-precision KV format (0 = unsupported)."""
    return lib().hca_kv_mixed_row_bytes(c, rd)


def kv_quant_mixed(x, x_dtype, rows, c, rd, out, stream=None):
    return check(lib().hca_kv_quant_mixed(ptr(x), x_dtype, rows, c, rd, ptr(out), stream_handle(stream)))


def kv_dequant_mixed(inp, rows, c, rd, out, stream=None):
    return check(lib().hca_kv_dequant_mixed(ptr(inp), rows, c, rd, ptr(out), stream_handle(stream)))


def output_projection(d: OprojDesc, o, wo_a, wo_b, out, ws, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    return check(lib().hca_output_projection(C.byref(d), ptr(o), ptr(wo_a), ptr(wo_b), ptr(out), ptr(ws), nbytes,
                                             stream_handle(stream)))
