"""Seeded synthetic inputs for the hybrid compressed attention workloads.

This module is shared by the CUDA path's tests/benchmark and by the oracle's
tests.  It holds none of the attention method's arithmetic: it only draws
random tensors with the distributions the workloads state (N(0,1) activations,
N(0, 1/d_in) weights, N(0,1) caches and sinks) and converts them to the
storage types the kernels read (bf16 round-to-nearest-even, fp8-e4m3 with a
per-row fp32 scale).

Every tensor has its own counter-derived generator (seed, stream id), so the
values of one tensor do not depend on which other tensors were drawn before it.
"""
from __future__ import annotations

import torch

_MIX = 0x9E3779B97F4A7C15
_MASK63 = (1 << 63) - 1


def _sub_seed(seed: int, stream: int) -> int:
    # splitmix64 finaliser over (seed, stream) -> a 63-bit torch seed
    z = (seed * 0x100000001B3 + (stream + 1) * _MIX) & ((1 << 64) - 1)
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & ((1 << 64) - 1)
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & ((1 << 64) - 1)
    z ^= z >> 31
    return z & _MASK63


def generator(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(_sub_seed(seed, stream))
    return g


def normal(shape, seed: int, stream: int, std: float = 1.0,
           dtype: torch.dtype = torch.float32) -> torch.Tensor:
    """N(0, std^2) samples drawn in fp32 on the CPU, then cast (RNE) to dtype."""
    x = torch.randn(tuple(shape), generator=generator(seed, stream), dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x if dtype == torch.float32 else x.to(dtype)


def uniform_int(shape, low: int, high: int, seed: int, stream: int) -> torch.Tensor:
    return torch.randint(low, high, tuple(shape), generator=generator(seed, stream),
                         dtype=torch.int64)


def fp8_rows(x: torch.Tensor):
    """Store fp32 rows as fp8-e4m3 bytes plus one fp32 scale per row (amax/448).

    Returns (uint8 tensor of the e4m3 bit patterns, fp32 scale per row).  This
    is how the synthetic fp8 indexer-key cache is made; readers decode the
    bytes and multiply by the row scale.
    """
    amax = x.abs().amax(dim=-1, keepdim=True).clamp_min(1e-12)
    scale = (amax / 448.0).to(torch.float32)
    q = (x / scale).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    return q.view(torch.uint8), scale.squeeze(-1).contiguous()


def bf16_bits(x: torch.Tensor) -> torch.Tensor:
    """Raw uint16 bit patterns of a bf16 tensor (for readers that decode bytes)."""
    assert x.dtype == torch.bfloat16
    return x.contiguous().view(torch.int16).to(torch.int32).bitwise_and(0xFFFF)


# Stream ids of the per-layer tensors (fixed so that each tensor's values do
# not depend on which others are drawn).
STREAMS = {
    "H": 1, "W_aKV": 2, "W_bKV": 3, "W_aZ": 4, "W_bZ": 5, "W_KVc": 6, "W_Zc": 7,
    "W_IaKV": 8, "W_IbKV": 9, "W_IaZ": 10, "W_IbZ": 11, "W_DQ": 12, "W_UQ": 13,
    "W_IUQ": 14, "W_w": 15, "W_KV": 16, "sink": 17, "B_a": 18, "B_b": 19, "B": 20,
    "B_Ia": 21, "B_Ib": 22,
}


def layer_weights(L, d: int, d_c: int, seed: int, dtype: torch.dtype,
                  layer_id: int = 0, bias_std: float = 0.0) -> dict:
    """Random weights of one attention layer, stored [d_out, d_in] ~ N(0, 1/d_in).

    Position biases B_a/B_b/B (and the indexer's) are N(0, bias_std^2), zero by
    default; sinks are N(0, L.sink_std^2) in fp32.
    """
    s = seed * 131 + layer_id

    def w(name, d_out, d_in):
        return normal((d_out, d_in), s, STREAMS[name], std=d_in ** -0.5, dtype=dtype)

    def bias(name, rows, cols):
        if bias_std == 0.0:
            return torch.zeros(rows, cols, dtype=torch.float32)
        return normal((rows, cols), s, STREAMS[name], std=bias_std)

    W = {}
    if L.kind == "csa":
        for nm in ("W_aKV", "W_bKV", "W_aZ", "W_bZ"):
            W[nm] = w(nm, L.c, d)
        W["B_a"], W["B_b"] = bias("B_a", L.m, L.c), bias("B_b", L.m, L.c)
        for nm in ("W_IaKV", "W_IbKV", "W_IaZ", "W_IbZ"):
            W[nm] = w(nm, L.c_I, d)
        W["B_Ia"], W["B_Ib"] = bias("B_Ia", L.m, L.c_I), bias("B_Ib", L.m, L.c_I)
        W["W_IUQ"] = w("W_IUQ", L.n_hI * L.c_I, d_c)
        W["W_w"] = w("W_w", L.n_hI, d)
    else:
        W["W_KVc"], W["W_Zc"] = w("W_KVc", L.c, d), w("W_Zc", L.c, d)
        W["B"] = bias("B", L.m, L.c)
    W["W_DQ"] = w("W_DQ", d_c, d)
    W["W_UQ"] = w("W_UQ", L.n_h * L.c, d_c)
    W["W_KV"] = w("W_KV", L.c, d)
    if L.sink_std == 0.0:
        W["sink"] = torch.zeros(L.n_h, dtype=torch.float32)
    else:
        W["sink"] = normal((L.n_h,), s, STREAMS["sink"], std=L.sink_std)
    return W


def hidden_states(B: int, n: int, d: int, seed: int, dtype: torch.dtype) -> torch.Tensor:
    return normal((B, n, d), seed, STREAMS["H"], dtype=dtype)


def normal_on(device, shape, seed: int, stream: int, std: float = 1.0,
              dtype: torch.dtype = torch.float32) -> torch.Tensor:
    """N(0, std^2) drawn directly on `device` (for large benchmark inputs)."""
    g = torch.Generator(device=device)
    g.manual_seed(_sub_seed(seed, stream))
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x if dtype == torch.float32 else x.to(dtype)


def layer_weights_on(device, L, d: int, d_c: int, seed: int, dtype: torch.dtype,
                     layer_id: int = 0) -> dict:
    """layer_weights() drawn directly on `device` (large benchmark layers);
    position biases zero, sinks N(0, L.sink_std^2)."""
    s = seed * 131 + layer_id

    def w(name, d_out, d_in):
        return normal_on(device, (d_out, d_in), s, STREAMS[name], std=d_in ** -0.5, dtype=dtype)

    W = {}
    if L.kind == "csa":
        for nm in ("W_aKV", "W_bKV", "W_aZ", "W_bZ"):
            W[nm] = w(nm, L.c, d)
        W["B_a"] = torch.zeros(L.m, L.c, device=device)
        W["B_b"] = torch.zeros(L.m, L.c, device=device)
        for nm in ("W_IaKV", "W_IbKV", "W_IaZ", "W_IbZ"):
            W[nm] = w(nm, L.c_I, d)
        W["B_Ia"] = torch.zeros(L.m, L.c_I, device=device)
        W["B_Ib"] = torch.zeros(L.m, L.c_I, device=device)
        W["W_IUQ"] = w("W_IUQ", L.n_hI * L.c_I, d_c)
        W["W_w"] = w("W_w", L.n_hI, d)
    else:
        W["W_KVc"], W["W_Zc"] = w("W_KVc", L.c, d), w("W_Zc", L.c, d)
        W["B"] = torch.zeros(L.m, L.c, device=device)
    W["W_DQ"] = w("W_DQ", d_c, d)
    W["W_UQ"] = w("W_UQ", L.n_h * L.c, d_c)
    W["W_KV"] = w("W_KV", L.c, d)
    W["sink"] = (normal_on(device, (L.n_h,), s, STREAMS["sink"], std=L.sink_std)
                 if L.sink_std else torch.zeros(L.n_h, device=device))
    return W
