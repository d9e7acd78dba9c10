"""Context-parallel prefill of one compressed attention layer.

juejin "DeepSeek-V4 技术报告简要解读" §4.5 (two-stage communication for the
compressed attention under context parallelism); ranhao "DeepSeek-V4 技术报告"
(context parallelism of the prefill).  The tokens of every sequence are cut
into contiguous ranges, one per rank, each starting on a compression block:

  0. halo   every rank needs the hidden states of the h tokens before its
            range (window rows of its first queries; for CSA the previous
            block, whose b series its first entry needs): one all-gather of
            the ranges' last rows;
  1. stage 1 (libhca hybrid_cp_compress): the range's compressed entries and
            indexer keys, computed locally;
  2. one all-gather of every rank's entries and keys, concatenated in rank
            order = the whole sequence's caches;
  3. stage 2 (libhca hybrid_cp_attend): the range's queries are scored,
            selected and attended against the gathered caches, locally.

The two collectives go through torch.distributed (NCCL between GPUs); no
kernel waits on another rank.  `CPLayer` runs the stages in libhca; the
driver `cp_prefill` is written against the small stage interface it
implements, so that the partitioning and exchange logic can be exercised with
other stage implementations too.
"""
from __future__ import annotations

import math

import torch

from . import binding as hb


def cp_ranges(n: int, world: int, align: int):
    """[(t0, n_loc)] of each rank: contiguous ranges covering n tokens, every
    start a multiple of `align` (the compression ratio, or the lcm of the
    ratios of the layers that share the split), as equal as that allows."""
    if n < 1 or world < 1 or align < 1:
        raise ValueError("n, world and align must be >= 1")
    per = -(-n // world)
    per = -(-per // align) * align
    out, t0 = [], 0
    for _ in range(world):
        n_loc = max(0, min(per, n - t0))
        out.append((t0, n_loc))
        t0 += n_loc
    return out


class CPLayer:
    """The two stages of one rank in libhca (hybrid_cp_compress /
    hybrid_cp_attend) for a LayerHandle."""

    def __init__(self, lh):
        self.lh = lh
        L = lh.shape
        self.csa = L.kind == "csa"
        self.m = L.m
        self.B = lh.B
        self.dtype = lh.dtype
        self.fp8 = self.csa and lh.idx_key_dtype == "fp8"

    def halo(self, t0: int) -> int:
        return hb.lib().hybrid_cp_halo(hb.ctypes_byref(self.lh.struct), t0)

    def _ws(self, t0, n_loc, device):
        size = hb.lib().hybrid_cp_workspace_size(hb.ctypes_byref(self.lh.struct), t0, n_loc)
        return torch.empty(max(size, 16), dtype=torch.uint8, device=device)

    def compress(self, H, t0: int, n_loc: int):
        """H [B, h + n_loc, d] -> (entries [B, E_loc, c], indexer keys or None,
        their fp32 scales or None), E_loc = n_loc // m."""
        L = self.lh.shape
        E = n_loc // self.m
        dev = H.device
        kv = torch.empty(self.B, max(E, 1), L.c, dtype=self.dtype, device=dev)
        kI = kIs = None
        if self.csa:
            kI = torch.empty(self.B, max(E, 1), L.c_I, dtype=torch.uint8 if self.fp8 else self.dtype, device=dev)
            kIs = torch.empty(self.B, max(E, 1), device=dev) if self.fp8 else None
        ws = self._ws(t0, n_loc, dev)
        hb.hybrid_cp_compress(self.lh.struct, H, t0, n_loc, kv, kI, kIs, max(E, 1), ws)
        return kv[:, :E], (kI[:, :E] if kI is not None else None), (kIs[:, :E] if kIs is not None else None)

    def attend(self, H, t0: int, n_loc: int, kv, kI, kIs):
        """o [B, n_loc, n_h, c] of the range against the gathered caches."""
        L = self.lh.shape
        o = torch.empty(self.B, n_loc, L.n_h, L.c, dtype=self.dtype, device=H.device)
        ws = self._ws(t0, n_loc, H.device)
        hb.hybrid_cp_attend(self.lh.struct, H, t0, n_loc, kv.contiguous(),
                            kI.contiguous() if kI is not None else None,
                            kIs.contiguous() if kIs is not None else None, kv.shape[1], o, ws)
        return o


def _all_gather(t, group):
    world = torch.distributed.get_world_size(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    torch.distributed.all_gather(parts, t.contiguous(), group=group)
    return parts


def gather_entries(parts, n_entries):
    """Concatenate the ranks' entries (each [B, E_pad, ...]) in rank order,
    each trimmed to its own count, along the entry dimension."""
    return torch.cat([p[:, :e] for p, e in zip(parts, n_entries)], dim=1).contiguous()


def cp_prefill(stages, H_local, n: int, align: int, group=None):
    """One rank of a context-parallel prefill.  H_local [B, n_loc, d] holds
    this rank's range of the hidden states (cp_ranges(n, world, align));
    returns o [B, n_loc, n_h, c].  Every rank calls it with its own range."""
    rank = torch.distributed.get_rank(group)
    world = torch.distributed.get_world_size(group)
    ranges = cp_ranges(n, world, align)
    t0, n_loc = ranges[rank]
    if H_local.shape[1] != n_loc:
        raise ValueError(f"rank {rank} holds {H_local.shape[1]} tokens, its range has {n_loc}")
    # 0. halo: the last h_max rows of every range (zero-padded where a range is shorter)
    h_max = max(stages.halo(r0) for r0, _ in ranges)
    B, _, d = H_local.shape
    tail = torch.zeros(B, h_max, d, dtype=H_local.dtype, device=H_local.device)
    if h_max:
        k = min(h_max, n_loc)
        if k:
            tail[:, h_max - k:] = H_local[:, n_loc - k:]
    tails = _all_gather(tail, group) if h_max else None
    h = stages.halo(t0)
    if h:
        prev = tails[rank - 1]
        if ranges[rank - 1][1] < h:
            raise ValueError("each range must be at least as long as the halo")
        H = torch.cat([prev[:, h_max - h:], H_local], dim=1).contiguous()
    else:
        H = H_local.contiguous()
    # 1. local compression
    kv, kI, kIs = stages.compress(H, t0, n_loc)
    # 2. one all-gather of entries and indexer keys (padded to the longest range)
    counts = [r[1] // stages.m for r in ranges]
    e_pad = max(max(counts), 1)

    def padded(t):
        if t is None:
            return None
        out = torch.zeros((t.shape[0], e_pad) + tuple(t.shape[2:]), dtype=t.dtype, device=t.device)
        out[:, :t.shape[1]] = t
        return out
    kv_all = gather_entries(_all_gather(padded(kv), group), counts)
    kI_all = gather_entries(_all_gather(padded(kI), group), counts) if kI is not None else None
    kIs_all = gather_entries(_all_gather(padded(kIs), group), counts) if kIs is not None else None
    if n_loc == 0:
        return torch.empty(B, 0, *kv.shape[2:], dtype=kv.dtype, device=kv.device)
    # 3. local scoring, selection and attention
    return stages.attend(H, t0, n_loc, kv_all, kI_all, kIs_all)


def lcm_align(*ratios: int) -> int:
    """The alignment of ranges shared by layers with these compression ratios."""
    a = 1
    for r in ratios:
        a = a * r // math.gcd(a, r)
    return a
