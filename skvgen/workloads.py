"""Workload recipes: shapes, seeds and structure of the synthetic inputs.

The five named workloads follow the decode settings the pages measure on
(Llama-3.1-8B-like shapes: 32 query heads, 8 KV heads, head dim 128, contexts of
4K to 128K tokens), with seeded synthetic tensors standing in for the
LongBench / RULER style inputs the pages evaluate on.
"""
from dataclasses import dataclass, field, replace
from typing import List, Optional

import numpy as np


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int                      # context length (uniform unless `lens` is given)
    d: int = 128
    bs: int = 64                # tokens per KV block / page
    Tq: int = 1                 # query tokens per sequence
    seed: int = 0x5EED0000
    lens: Optional[List[int]] = None
    structured: bool = False    # token-0 sink (+6 qhat) and 1% heavy tokens (+4 qhat)
    paging: str = "identity"    # "identity" | "perm" | "window"
    mixture: bool = False       # Gaussian-mixture keys, cluster-contiguous
    shared_context: bool = False  # every request reads one context (that of request 0)
    c_log2: int = 10            # 1024 clusters
    topk: int = 102
    # ART (recency-first traversal)
    tau: float = 1e-3
    phi: float = 1e-4
    patience: int = 4
    # sink + recent window of sparse (routed) layers
    sink: int = 64
    recent: int = 4096
    # sharded exact merge with a causal query chunk
    shards: int = 1
    chunk: int = 0              # number of chunk tokens appended after the context
    n_layers: int = 1
    softmax_scale: Optional[float] = None  # default 1/sqrt(d)
    extra: dict = field(default_factory=dict)

    @property
    def G(self):
        return self.Hq // self.Hkv

    @property
    def scale(self):
        if self.softmax_scale is not None:
            return float(self.softmax_scale)
        return 1.0 / float(np.sqrt(self.d))

    def seq_len(self, b):
        return int(self.lens[b]) if self.lens is not None else int(self.L)

    @property
    def Lmax(self):
        return max(self.seq_len(b) for b in range(self.B))

    @property
    def max_blocks(self):
        return (self.Lmax + self.bs - 1) // self.bs

    def nb(self, b):
        return (self.seq_len(b) + self.bs - 1) // self.bs

    def kv_bytes(self):
        """Algorithmic K+V bytes of a full traversal."""
        return sum(self.seq_len(b) for b in range(self.B)) * self.Hkv * self.d * 2 * 2

    def with_(self, **kw):
        return replace(self, **kw)


def window_blocks(L, bs, sink, recent):
    """Logical blocks holding tokens [0, sink) U [L - recent, L)."""
    nb = (L + bs - 1) // bs
    if sink <= 0 and recent <= 0:
        return list(range(nb))
    blocks = set(range((min(sink, L) + bs - 1) // bs))
    lo = max(0, L - recent)
    blocks.update(range(lo // bs, nb))
    return sorted(blocks)


def block_table_host(wl: Workload, layer=0):
    """block_table int32 [B][max_blocks] and the pool size.

    identity: sequence b's blocks occupy pages b*max_blocks + j.
    perm:     pages are a seeded Fisher-Yates permutation of the whole pool.
    window:   only the blocks of the sink + recent window are mapped (the
              minimal KV a sparse layer keeps); the rest are -1.
    Unmapped entries (j >= nb) are -1.
    """
    from . import host_perm, S_PERM
    mb = wl.max_blocks
    bt = np.full((wl.B, mb), -1, dtype=np.int32)
    if wl.paging == "window":
        nxt = 0
        for b in range(wl.B):
            for j in window_blocks(wl.seq_len(b), wl.bs, wl.sink, wl.recent):
                bt[b, j] = nxt
                nxt += 1
        return bt, nxt
    total = sum(wl.nb(b) for b in range(wl.B))
    if wl.paging == "perm":
        perm = host_perm(wl.seed, total, S_PERM, layer)
    else:
        perm = np.arange(total, dtype=np.int32)
    o = 0
    for b in range(wl.B):
        n = wl.nb(b)
        bt[b, :n] = perm[o:o + n]
        o += n
    return bt, total


WORKLOADS = {
    # single decode step, full traversal, no termination
    "cfg1_b1_h8_l4k": Workload("cfg1_b1_h8_l4k", B=1, Hq=8, Hkv=2, L=4096, seed=0x5EED0001),
    # Llama-3.1-8B-shaped decode with ART; also run full
    "cfg2_b16_h32_l32k": Workload("cfg2_b16_h32_l32k", B=16, Hq=32, Hkv=8, L=32768, seed=0x5EED0002,
                                  structured=True, paging="perm"),
    # centroid-selected decode over a 1024-component Gaussian mixture per KV head
    "cfg3_b8_h32_l64k_c1024_k102": Workload("cfg3_b8_h32_l64k_c1024_k102", B=8, Hq=32, Hkv=8, L=65536,
                                            seed=0x5EED0003, mixture=True, c_log2=10, topk=102),
    # centroid-selected decode of 8 requests over ONE shared fixed context
    # (clustered once, per KV head, reused by every request)
    "cfg3s_b8_h32_l64k_shared": Workload("cfg3s_b8_h32_l64k_shared", B=8, Hq=32, Hkv=8, L=65536,
                                         seed=0x5EED0006, mixture=True, c_log2=10, topk=102,
                                         shared_context=True),
    # 8 shards of 16384 context keys + a causal 128-token query chunk
    "cfg4_b4_h32_l128k_chunk128": Workload("cfg4_b4_h32_l128k_chunk128", B=4, Hq=32, Hkv=8,
                                           L=131072 + 128, Tq=128, seed=0x5EED0004, shards=8, chunk=128),
    # lookahead prefetch on cfg5's layers: a full layer on the GPU, the next layer's KV in
    # host memory, its top-16 blocks (of 2048) chosen by the Forecast and fetched meanwhile
    "cfg5p_b8_h32_l128k_lookahead16": Workload("cfg5p_b8_h32_l128k_lookahead16", B=8, Hq=32, Hkv=8,
                                               L=131072, seed=0x5EED0005, structured=True, n_layers=32,
                                               extra={"lookahead_blocks": 16}),
    # 32-layer routed attention-only decode stack
    "cfg5_b8_h32_l128k_32layers": Workload("cfg5_b8_h32_l128k_32layers", B=8, Hq=32, Hkv=8, L=131072,
                                           seed=0x5EED0005, structured=True, n_layers=32),
}
