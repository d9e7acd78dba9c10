"""ctypes wrapper of the C++ oracle (oracle/hca_oracle_c.cpp).

TEST INFRASTRUCTURE ONLY: used by tests/, __graft_entry__.smoke() and bench.py's
CPU baseline and reference arm, never by the product path.  It builds
oracle/libhca_oracle_c.so with g++ (-O3, OpenMP) when the library is missing or
older than its source.  Arguments are converted to contiguous float64 / int32
numpy arrays; every function restates one step of the method (see the source).
"""
import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hca_oracle_c.cpp")
LIB = os.path.join(HERE, "libhca_oracle_c.so")
_lib = None

class Rows(C.Structure):
    """Cache rows as stored (hco_rows): dtype 0 float64, 1 bf16 bits, 2 e4m3 codes x scale."""
    _fields_ = [("p", C.c_void_p), ("dtype", C.c_int), ("scale", C.POINTER(C.c_float)), ("n_rows", C.c_longlong)]


D = C.POINTER(C.c_double)
I32 = C.POINTER(C.c_int32)
I64 = C.POINTER(C.c_longlong)
i, ll, dbl = C.c_int, C.c_longlong, C.c_double


def build(force: bool = False) -> str:
    """Compile the C++ oracle into oracle/libhca_oracle_c.so (g++ -O3 -fopenmp)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp"
        subprocess.run(["g++", "-O3", "-std=c++17", "-fopenmp", "-shared", "-fPIC", SRC, "-o", tmp], check=True)
        os.replace(tmp, LIB)
    return LIB


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(build())
        sig = {
            "hco_num_threads": [i],
            "hco_compress": [D, D, D, D, D, D, i, i, i, D],
            "hco_entry_epilogue": [D, i, i, i, i, D, dbl, i, dbl, i],
            "hco_index_scores": [D, D, D, i, i, i, D],
            "hco_topk_select": [D, i, i, I32],
            "hco_attend": [D, D, i, D, i, i, dbl, ll, i, dbl, D],
            "hco_token": [i, ll, D, Rows, I32, i, Rows, i, i, D, D, Rows, i, i, D, i, i, i, dbl, ll, D, I32],
            "hco_decode_batch": [i, i, D, Rows, I32, i, Rows, i, i, D, D, Rows, i, i, D, i, i, i, dbl, ll, D],
            "hco_prefill_tokens": [i, ll, i, I64, D, Rows, i, Rows, i, i, D, D, Rows, i, i, D, i, i, i, dbl, D],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = i
        _lib = L
    return _lib


def _d(x):
    if x is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    return a, a.ctypes.data_as(D)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"C++ oracle: {what} rejected its arguments")


def num_threads(n: int = 0) -> int:
    """Set the OpenMP thread count (n > 0) and return it."""
    return lib().hco_num_threads(n)


def compress(Ca, Za, Ba, m, Cb=None, Zb=None, Bb=None):
    """[n, c] inputs -> the n/m entries [n/m, c] (overlapped when Cb is given)."""
    Ca, pCa = _d(Ca); Za, pZa = _d(Za); Ba, pBa = _d(Ba)
    Cb, pCb = _d(Cb); Zb, pZb = _d(Zb); Bb, pBb = _d(Bb)
    n, c = Ca.shape
    out = np.zeros((n // m, c))
    _check(lib().hco_compress(pCa, pZa, pBa, pCb, pZb, pBb, n, c, m, out.ctypes.data_as(D)), "compress")
    return out


def entry_epilogue(entries, m, first_entry=0, gamma=None, eps=1e-6, rd=0, theta=10000.0, norm=True):
    x = np.array(entries, dtype=np.float64, copy=True, order="C")
    g, pg = _d(gamma)
    _check(lib().hco_entry_epilogue(x.ctypes.data_as(D), x.shape[0], x.shape[1], m, first_entry, pg, eps, rd, theta,
                                    1 if norm else 0), "entry_epilogue")
    return x


def index_scores(qI_t, w_t, KI, V):
    q, pq = _d(qI_t); w, pw = _d(w_t); K, pK = _d(np.asarray(KI)[:V])
    out = np.zeros(max(V, 1))
    _check(lib().hco_index_scores(pq, pw, pK, q.shape[0], q.shape[1], V, out.ctypes.data_as(D)), "index_scores")
    return out[:V]


def topk_select(scores, k):
    s, ps = _d(scores)
    out = np.zeros(k, dtype=np.int32)
    _check(lib().hco_topk_select(ps, s.shape[0], k, out.ctypes.data_as(I32)), "topk_select")
    return out


def attend_output(q_t, rows, sink, scale, t, rd, theta=10000.0):
    q, pq = _d(q_t); r, pr = _d(np.asarray(rows).reshape(-1, np.asarray(q_t).shape[-1])); s, psk = _d(sink)
    out = np.zeros_like(q)
    _check(lib().hco_attend(pq, pr, r.shape[0], psk, q.shape[0], q.shape[1], scale, t, rd, theta,
                            out.ctypes.data_as(D)), "attend")
    return out


def rows(x, scale=None):
    """A cache [seqs, rows, c] (or [rows, c]) as hco_rows: float arrays as
    float64, uint16 as bf16 bits, uint8 as e4m3 codes with `scale` [seqs, rows]
    fp32.  Returns (Rows, keep-alive list)."""
    a = np.asarray(x)
    if a.dtype == np.uint16:
        dt = 1
    elif a.dtype == np.uint8:
        dt = 2
    else:
        a, dt = a.astype(np.float64), 0
    a = np.ascontiguousarray(a)
    keep = [a]
    sp = None
    if dt == 2:
        sc = np.ascontiguousarray(np.asarray(scale, dtype=np.float32))
        keep.append(sc)
        sp = sc.ctypes.data_as(C.POINTER(C.c_float))
    n_rows = a.shape[-2] if a.ndim >= 2 else 0
    return Rows(a.ctypes.data, dt, sp, n_rows), keep


def decode_batch(kind, q, win, win_idx, comp, m, sink, rd, t, k=0, qI=None, w=None, KI=None, KI_scale=None,
                 theta=10000.0):
    """One decode token per sequence: q [B, n_h, c]; win [B, w, c] ring rows
    with win_idx the slots of tokens max(0, t-w+1)..t in position order;
    comp [B, cap, c]; CSA also qI [B, n_hI, c_I], w [B, n_hI], KI [B, cap, c_I]
    (+ KI_scale for e4m3 codes).  Caches may be float, bf16 bits (uint16) or
    e4m3 codes (uint8).  Returns o [B, n_h, c] (float64)."""
    q, pq = _d(q); sk, psk = _d(sink)
    B, n_h, c = q.shape
    csa = kind == "csa"
    rw, k1 = rows(win); rc_, k2 = rows(comp)
    rk, k3 = rows(KI, KI_scale) if csa else (Rows(None, 0, None, 0), [])
    wi = np.ascontiguousarray(np.asarray(win_idx, dtype=np.int32))
    qI_, pqI = _d(qI); w_, pw = _d(w)
    out = np.zeros_like(q)
    _check(lib().hco_decode_batch(1 if csa else 0, B, pq, rw, wi.ctypes.data_as(I32), wi.shape[0], rc_, m, k, pqI, pw,
                                  rk, qI_.shape[1] if csa else 1, qI_.shape[2] if csa else 1, psk, n_h, c, rd, theta,
                                  t, out.ctypes.data_as(D)), "decode_batch")
    return out


def prefill_tokens(kind, ts, q, kv_win, w_len, kv_comp, m, sink, rd, k=0, qI=None, w=None, KI=None, KI_scale=None,
                   theta=10000.0, seq=0):
    """Prefill attention of the listed tokens ts of sequence `seq`: q
    [len(ts), n_h, c] (those tokens' queries), kv_win [n, c] (or [B, n, c])
    token rows, kv_comp [E, c] (or [B, E, c]); CSA also qI [len(ts), n_hI,
    c_I], w [len(ts), n_hI], KI [E, c_I] (or [B, E, c_I])."""
    tsa = np.ascontiguousarray(np.asarray(ts, dtype=np.int64))
    q, pq = _d(q); sk, psk = _d(sink)
    n_tok, n_h, c = q.shape
    csa = kind == "csa"
    rw, k1 = rows(kv_win); rc_, k2 = rows(kv_comp)
    rk, k3 = rows(KI, KI_scale) if csa else (Rows(None, 0, None, 0), [])
    qI_, pqI = _d(qI); w_, pw = _d(w)
    out = np.zeros_like(q)
    _check(lib().hco_prefill_tokens(1 if csa else 0, seq, n_tok, tsa.ctypes.data_as(I64), pq, rw, w_len, rc_, m, k,
                                    pqI, pw, rk, qI_.shape[1] if csa else 1, qI_.shape[2] if csa else 1, psk, n_h, c,
                                    rd, theta, out.ctypes.data_as(D)), "prefill_tokens")
    return out
