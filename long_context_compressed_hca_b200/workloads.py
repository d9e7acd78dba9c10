"""The five synthetic workloads of the hybrid compressed attention path, as plain data.

Sizes follow the DeepSeek-V4 digests' hyper-parameter tables (juejin
"DeepSeek-V4 技术报告简要解读" §2.3.1 CSA table and Appendix A) at the scales
named for each workload; values the pages leave open carry the reading used
for them (see the field comments).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace


@dataclass(frozen=True)
class LayerShape:
    kind: str            # "csa" (overlapped, indexer + top-k) or "hca" (dense over entries)
    m: int               # compression ratio (m for CSA, m' for HCA)
    n_h: int             # query heads
    c: int               # shared KV / head dim
    rd: int              # RoPE dims (last rd of c)
    w: int               # sliding window
    k: int = 0           # top-k (CSA only)
    n_hI: int = 0        # indexer heads (CSA only)
    c_I: int = 0         # indexer head dim (CSA only)
    sink_std: float = 1.0  # per-head sink logits ~ N(0, sink_std^2); 0 = all zero

    @property
    def overlap(self) -> bool:
        return self.kind == "csa"

    @property
    def rd_I(self) -> int:
        return min(self.rd, self.c_I)


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    dtype: str           # "f32" or "bf16": q / kv / o storage type
    B: int
    layers: tuple        # LayerShape per layer in one step
    mode: str            # "prefill" (from hidden states) or "decode" (one token over a cache)
    n: int = 0           # prefill tokens per sequence
    d: int = 0           # d_model (prefill)
    d_c: int = 0         # query compression rank (prefill)
    pos: int = 0         # decode: position of the new token (= cached context length)
    idx_key_dtype: str = "bf16"   # indexer key cache type ("bf16" or "fp8")
    notes: str = ""

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# Tiny CSA layer, fp32.  n_hI = 4 and c_I = 32 are a reading (the workload does
# not state the indexer size); d_c = 32 follows its W^DQ of 256 x 32.
TINY_CSA = Workload(
    name="tiny_csa_fp32_b1_s512", seed=0, dtype="f32", B=1, mode="prefill",
    n=512, d=256, d_c=32,
    layers=(LayerShape("csa", m=4, n_h=4, c=64, rd=16, w=32, k=16, n_hI=4, c_I=32,
                       sink_std=0.0),),
)

# HCA layer, bf16.  d_c = 256 (= d/4, V4-Flash's ratio) is a reading.
HCA_PREFILL = Workload(
    name="hca_prefill_bf16_b2_s8192", seed=1, dtype="bf16", B=2, mode="prefill",
    n=8192, d=1024, d_c=256,
    layers=(LayerShape("hca", m=128, n_h=16, c=128, rd=64, w=128),),
)

# CSA prefill at 64K, bf16 (V4-Flash attention sizes, d_c = 1024).
CSA_PREFILL = Workload(
    name="csa_prefill_bf16_b1_s65536", seed=2, dtype="bf16", B=1, mode="prefill",
    n=65536, d=4096, d_c=1024,
    layers=(LayerShape("csa", m=4, n_h=64, c=512, rd=64, w=128, k=512, n_hI=8, c_I=64),),
)

# The same CSA layer prefilled over 128K tokens.
CSA_PREFILL_128K = Workload(
    name="csa_prefill_bf16_b1_s131072", seed=2, dtype="bf16", B=1, mode="prefill",
    n=131072, d=4096, d_c=1024,
    layers=(LayerShape("csa", m=4, n_h=64, c=512, rd=64, w=128, k=512, n_hI=8, c_I=64),),
)

# Hybrid decode at 128K: one CSA layer then one HCA layer per step.
HYBRID_DECODE_128K = Workload(
    name="hybrid_decode_bf16_b32_ctx131072", seed=3, dtype="bf16", B=32, mode="decode",
    pos=131072,
    layers=(LayerShape("csa", m=4, n_h=64, c=512, rd=64, w=128, k=512, n_hI=8, c_I=64),
            LayerShape("hca", m=128, n_h=64, c=512, rd=64, w=128)),
)

# 1M-context decode with fp8-e4m3 indexer keys; indexer 8 x 64 is a reading.
HYBRID_DECODE_1M = Workload(
    name="hybrid_decode_bf16_fp8idx_b4_ctx1048576", seed=4, dtype="bf16", B=4,
    mode="decode", pos=1048576, idx_key_dtype="fp8",
    layers=(LayerShape("csa", m=4, n_h=64, c=512, rd=64, w=128, k=1024, n_hI=8, c_I=64),
            LayerShape("hca", m=128, n_h=64, c=512, rd=64, w=128)),
)

ALL = (TINY_CSA, HCA_PREFILL, CSA_PREFILL, HYBRID_DECODE_128K, HYBRID_DECODE_1M)
BY_NAME = {w.name: w for w in ALL}
