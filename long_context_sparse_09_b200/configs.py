"""The five synthetic workloads of the CSA / HCA forward pass.

Dimensions follow the DeepSeek-V4 pages: V4-Flash (d=4096, 64 query heads,
entry dim c=512 with RoPE on the last 64 dims, m=4, a 64-head x 128-dim
indexer, top-k 512, window 128) and V4-Pro (d=7168, 128 heads, top-k 1024,
448 FP8 dims + 64 BF16 RoPE dims per entry); HCA groups m'=128 tokens
("02 · DeepSeek-V4: 压缩注意力撑起 1M 上下文", sections 2.1-2.5; "DeepSeekV4
技术报告阅读笔记", section 2.3-2.5); the grouped output projection has g = 8
(Flash) or 16 (Pro) groups of width d_g = 1024 (PaperTrace 2.2).  This module holds sizes only, no arithmetic
of the method.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str          # "prefill" (all queries of a sequence) or "decode"
    variant: str       # "csa" (compress + index + top-k + attend) or "hca"
    B: int             # sequences
    T: int             # prefill: tokens per sequence; decode: context length L
    d: int             # hidden size
    n_h: int           # query heads
    c: int             # shared-KV entry width
    rope_dims: int     # RoPE on the last rope_dims of c
    m: int             # tokens per compressed entry (m for CSA, m' for HCA)
    n_hI: int          # indexer heads (0 for HCA)
    c_I: int           # indexer key width (0 for HCA)
    d_c: int           # query low-rank width (documents the query path only)
    topk: int          # selected entries per query (0 for HCA)
    n_win: int         # sliding-window tokens
    act: str           # "f32" or "bf16": activations, weights, queries
    kv: str            # "f32", "bf16" or "fp8mix": KV-cache format
    seed: int
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    g_out: int = 8     # output-projection groups (V4-Flash 8, V4-Pro 16)
    d_g: int = 1024    # width of each group's projection

    @property
    def overlap(self) -> int:
        return 1 if self.variant == "csa" else 0

    @property
    def softmax_scale(self) -> float:
        return 1.0 / (self.c ** 0.5)

    @property
    def n_entries(self) -> int:
        """Compressed entries per sequence: complete groups of m tokens."""
        return self.T // self.m

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_csa_prefill_f32": Workload(
        "tiny_csa_prefill_f32", "prefill", "csa", B=1, T=256, d=512, n_h=8,
        c=128, rope_dims=32, m=4, n_hI=4, c_I=32, d_c=128, topk=16, n_win=16,
        act="f32", kv="f32", seed=0),
    "flash_csa_decode_64k": Workload(
        "flash_csa_decode_64k", "decode", "csa", B=32, T=65536, d=4096,
        n_h=64, c=512, rope_dims=64, m=4, n_hI=64, c_I=128, d_c=1024,
        topk=512, n_win=128, act="bf16", kv="bf16", seed=1),
    "flash_csa_prefill_32k": Workload(
        "flash_csa_prefill_32k", "prefill", "csa", B=1, T=32768, d=4096,
        n_h=64, c=512, rope_dims=64, m=4, n_hI=64, c_I=128, d_c=1024,
        topk=512, n_win=128, act="bf16", kv="bf16", seed=2),
    "pro_csa_decode_1m": Workload(
        "pro_csa_decode_1m", "decode", "csa", B=4, T=1048576, d=7168,
        n_h=128, c=512, rope_dims=64, m=4, n_hI=64, c_I=128, d_c=1536,
        topk=1024, n_win=128, act="bf16", kv="fp8mix", seed=3, g_out=16),
    "hca_decode_1m": Workload(
        "hca_decode_1m", "decode", "hca", B=16, T=1048576, d=4096, n_h=64,
        c=512, rope_dims=64, m=128, n_hI=0, c_I=0, d_c=1024, topk=0,
        n_win=128, act="bf16", kv="bf16", seed=4),
}

# the workload a benchmark step runs by default: 1M-context CSA decode
DEFAULT_BENCH = "pro_csa_decode_1m"
