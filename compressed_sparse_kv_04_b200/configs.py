"""The five workloads of the CSA/HCA hot path, named by what they are.

Shapes follow the V4-Pro attention block of "DeepSeek V4-Pro" (llm-arch-kb),
section "Hybrid attention: CSA + HCA replace MLA": 128 query heads of head dim
512 over one shared KV head, RoPE on the last 64 dims, a 128-token window,
64 indexer heads of dim 128, top-k 1024, m = 4 (CSA) and m' = 128 (HCA).
The 1M-token CSA case (262,144 compressed entries narrowed to 1,024) is the
one "DeepSeek V4-Pro Architecture: KV Cache Compression ..." describes under
"Key points".  The tiny case exists for parity at oracle speed.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "csa_decode" | "hca_decode" | "csa_prefill" | "hca_prefill"
    B: int               # sequences
    L: int               # context tokens per sequence (decode: the query is token L-1)
    d: int               # KV entry dim == head dim D
    m: int               # compression ratio
    H: int               # query heads
    rope_dim: int
    W: int               # sliding window
    H_I: int = 0         # indexer heads (CSA)
    D_I: int = 0         # indexer dim (CSA)
    k: int = 0           # top-k (CSA)
    P: int = 0           # prefill: prior tokens
    T: int = 0           # prefill: new tokens
    seed: int = 0
    yarn: tuple | None = None  # (factor, beta_fast, beta_slow, original_len) or plain RoPE
    overlap: int = 0     # compression: tokens of block i-1 that entry i also pools

    @property
    def D(self) -> int:
        return self.d

    @property
    def N_c(self) -> int:
        """Compressed entries of the full context, ceil(L/m)."""
        return -(-self.L // self.m)

    @property
    def csa(self) -> bool:
        return self.kind in ("csa_decode", "csa_prefill")


TINY_CSA = Workload("csa_decode_tiny_4k", "csa_decode", B=1, L=4096, d=128, m=4, H=16,
                    rope_dim=32, W=128, H_I=4, D_I=64, k=128, seed=20260001)
CSA_128K = Workload("csa_decode_128k_b8", "csa_decode", B=8, L=131072, d=512, m=4, H=128,
                    rope_dim=64, W=128, H_I=64, D_I=128, k=1024, seed=20260002)
HCA_1M = Workload("hca_decode_1m_b8", "hca_decode", B=8, L=1048576, d=512, m=128, H=128,
                  rope_dim=64, W=128, seed=20260003)
CSA_1M = Workload("csa_decode_1m_b4", "csa_decode", B=4, L=1048576, d=512, m=4, H=128,
                  rope_dim=64, W=128, H_I=64, D_I=128, k=1024, seed=20260004)
CSA_PREFILL = Workload("csa_prefill_4096_after_65536", "csa_prefill", B=1, L=65536 + 4096,
                       d=512, m=4, H=128, rope_dim=64, W=128, H_I=64, D_I=128, k=1024,
                       P=65536, T=4096, seed=20260005)

# V4-Flash attention ("DeepSeek V4-Pro" (llm-arch-kb), "Family"): 64 query
# heads and top-k 512, the rest as V4-Pro; RoPE with the YaRN frequencies of
# "5. 1M context, gradually" (factor 16, beta_fast 32, beta_slow 1) over an
# original context of 1,048,576 / 16 tokens.
YARN_V4 = (16.0, 32.0, 1.0, 1048576 / 16)
CSA_FLASH_128K = Workload("csa_flash_decode_128k_b8", "csa_decode", B=8, L=131072, d=512, m=4,
                          H=64, rope_dim=64, W=128, H_I=64, D_I=128, k=512, seed=20260006,
                          yarn=YARN_V4)

# HCA prefill: the same 4096-token chunk after 65,536 cached tokens as the CSA
# prefill, through the HCA layer (m' = 128: 512 cached + 32 new entries).
HCA_PREFILL = Workload("hca_prefill_4096_after_65536", "hca_prefill", B=1, L=65536 + 4096,
                       d=512, m=128, H=128, rope_dim=64, W=128, P=65536, T=4096,
                       seed=20260007)

# Reduced cases for profiler captures (a few GB on the device): the 128K CSA
# decode with a 32K context (the same per-row attention work: 1024 selected
# entries + the window), the HCA decode at 256K (2048 entries per row), and
# the 1M CSA decode's batch of 4 at 32K.
CSA_32K_PROFILE = Workload("csa_decode_32k_b8", "csa_decode", B=8, L=32768, d=512, m=4, H=128,
                           rope_dim=64, W=128, H_I=64, D_I=128, k=1024, seed=20260009)
HCA_256K_PROFILE = Workload("hca_decode_256k_b8", "hca_decode", B=8, L=262144, d=512, m=128,
                            H=128, rope_dim=64, W=128, seed=20260010)
# The 1M CSA decode's attention work (4 sequences x (1024 selected entries +
# the window)) with a 32K context.
CSA_32K_B4_PROFILE = Workload("csa_decode_32k_b4", "csa_decode", B=4, L=32768, d=512, m=4, H=128,
                              rope_dim=64, W=128, H_I=64, D_I=128, k=1024, seed=20260011)

ALL = [TINY_CSA, CSA_128K, HCA_1M, CSA_1M, CSA_PREFILL, CSA_FLASH_128K, HCA_PREFILL,
       CSA_32K_PROFILE, HCA_256K_PROFILE, CSA_32K_B4_PROFILE]
BY_NAME = {w.name: w for w in ALL}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some sizes changed (parity tests at reduced size)."""
    return replace(w, **kw)
