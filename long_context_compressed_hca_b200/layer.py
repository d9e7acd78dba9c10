"""Python-side construction of the C-ABI layer / cache / token structs.

Argument marshalling only: weights are laid out as the ABI wants them
(concatenated compressor projections, stacked position biases) and kept
alive with the struct; all arithmetic runs in libhca.
"""
from __future__ import annotations

import torch

from . import binding as hb


def _code(dtype: torch.dtype) -> int:
    return hb.DTYPE_CODE[dtype]


class LayerHandle:
    """One attention layer: weights on `device` plus the hca_layer struct."""

    def __init__(self, L, W: dict, d: int, d_c: int, dtype: torch.dtype, B: int,
                 idx_key_dtype: str = "bf16", device="cuda", max_ctas: int = 0, kv_mixed: bool = False):
        self.shape, self.d, self.d_c, self.dtype, self.B = L, d, d_c, dtype, B
        dev = lambda t, dt=None: t.to(device=device, dtype=dt or t.dtype).contiguous()
        csa = L.kind == "csa"
        self.t = {}
        if csa:
            self.t["W_comp"] = dev(torch.cat([W["W_aKV"], W["W_bKV"], W["W_aZ"], W["W_bZ"]], 0), dtype)
            self.t["B_comp"] = dev(torch.stack([W["B_a"], W["B_b"]], 0), torch.float32)
            self.t["W_compI"] = dev(torch.cat([W["W_IaKV"], W["W_IbKV"], W["W_IaZ"], W["W_IbZ"]], 0), dtype)
            self.t["B_compI"] = dev(torch.stack([W["B_Ia"], W["B_Ib"]], 0), torch.float32)
            self.t["W_IUQ"] = dev(W["W_IUQ"], dtype)
            self.t["W_w"] = dev(W["W_w"], dtype)
        else:
            self.t["W_comp"] = dev(torch.cat([W["W_KVc"], W["W_Zc"]], 0), dtype)
            self.t["B_comp"] = dev(W["B"], torch.float32)
        for nm in ("W_DQ", "W_UQ", "W_KV"):
            self.t[nm] = dev(W[nm], dtype)
        self.t["sink"] = dev(W["sink"], torch.float32)
        kdt = {"bf16": _code(dtype), "fp8": hb.HCA_FP8E4M3, "fp4": hb.HCA_FP4}[idx_key_dtype] if csa else _code(dtype)
        self.idx_key_dtype = idx_key_dtype
        self.desc = hb.attn_desc(B, L.n_h, L.c, L.rd, L.w, L.m, overlap=L.overlap, k=L.k,
                                 n_hI=L.n_hI, c_I=L.c_I, rd_I=L.rd_I if csa else 0,
                                 dtype=_code(dtype), idx_key_dtype=kdt, max_ctas=max_ctas, kv_mixed=int(kv_mixed))
        g = lambda nm: hb.ptr(self.t.get(nm))
        self.struct = hb.Layer(hb.HCA_LAYER_CSA if csa else hb.HCA_LAYER_HCA, self.desc, d, d_c,
                               g("W_comp"), g("B_comp"), g("W_compI"), g("B_compI"), g("W_DQ"),
                               g("W_UQ"), g("W_IUQ"), g("W_w"), g("W_KV"), g("sink"))


class CacheHandle:
    """Decode cache of one layer (caller-owned device buffers)."""

    def __init__(self, L, B: int, cap: int, dtype: torch.dtype, idx_key_dtype: str = "bf16",
                 device="cuda", kv_mixed: bool = False):
        self.shape, self.B, self.cap = L, B, cap
        z = lambda *s, dt=torch.float32: torch.zeros(*s, dtype=dt, device=device)
        if kv_mixed:
            # mixed-precision records (hca_kv_mixed_row_bytes per row)
            rec = hb.kv_mixed_row_bytes(L.c, L.rd)
            self.kv_comp = z(B, cap, rec, dt=torch.uint8)
            self.win = z(B, max(L.w, 1), rec, dt=torch.uint8)
        else:
            self.kv_comp = z(B, cap, L.c, dt=dtype)
            self.win = z(B, max(L.w, 1), L.c, dt=dtype)
        R = 2 * L.m if L.overlap else L.m
        Cw = 2 * L.c if L.overlap else L.c
        self.state_kv = z(B, R, Cw)
        self.state_score = torch.full((B, R, Cw), float("-inf"), device=device)
        self.key_I = self.key_I_scale = self.stateI_kv = self.stateI_score = None
        if L.kind == "csa":
            # fp8: e4m3 bytes + row scales; fp4: rotated FP4 values carried in bf16
            kdt = torch.uint8 if idx_key_dtype == "fp8" else (torch.bfloat16 if idx_key_dtype == "fp4" else dtype)
            self.key_I = z(B, cap, L.c_I, dt=kdt)
            if idx_key_dtype == "fp8":
                self.key_I_scale = z(B, cap)
            RI, CI = (2 * L.m, 2 * L.c_I) if L.overlap else (L.m, L.c_I)
            self.stateI_kv = z(B, RI, CI)
            self.stateI_score = torch.full((B, RI, CI), float("-inf"), device=device)
        p = hb.ptr
        self.struct = hb.Cache(cap, p(self.kv_comp), p(self.key_I), p(self.key_I_scale), p(self.win),
                               p(self.state_kv), p(self.state_score), p(self.stateI_kv),
                               p(self.stateI_score))


class TokenInputs:
    """Projected inputs of one decode token per sequence."""

    def __init__(self, q, kv, comp, qI=None, wI=None, compI=None):
        self.t = dict(q=q, kv=kv, comp=comp, qI=qI, wI=wI, compI=compI)
        p = hb.ptr
        self.struct = hb.TokenIn(p(q), p(qI), p(wI), p(kv), p(comp), p(compI))

    @classmethod
    def empty(cls, L, B: int, dtype: torch.dtype, device="cuda"):
        """Buffers for one decode token per sequence of layer shape L (for
        hybrid_decode_inputs to fill)."""
        csa = L.kind == "csa"
        e = lambda *s, dt=dtype: torch.empty(*s, dtype=dt, device=device)
        return cls(q=e(B, L.n_h, L.c), kv=e(B, L.c), comp=e(B, (4 if csa else 2) * L.c, dt=torch.float32),
                   qI=e(B, L.n_hI, L.c_I) if csa else None, wI=e(B, L.n_hI, dt=torch.float32) if csa else None,
                   compI=e(B, 4 * L.c_I, dt=torch.float32) if csa else None)
