"""Seeded synthetic decode workloads shared by the tests, the bench and the oracle.

This module only describes shapes and draws random numbers. It holds none of
the paged-attention arithmetic: no block tables, no slots, no softmax. Both the
CUDA path (through the C ABI) and the float64 oracle consume what it returns.

Every draw comes from its own ``torch.Generator('cpu')`` whose seed is derived
from the workload seed and a tag, so any piece (one sequence's keys, say) can be
regenerated on its own without replaying the others. Values are float32
N(0, 1) rounded to nearest-even into the workload's source dtype.

The five named workloads follow the decode batches the vLLM pages talk about
(7B / 8B / 70B-style heads, 2K to 128K contexts, 16-token blocks); the ``*_small``
variants keep each one's structure (GQA group, dtype, prefix sharing, split
partitions, ragged tails) at sizes a CPU oracle finishes in seconds.
"""
from __future__ import annotations

import dataclasses
import functools
import zlib
from typing import Dict, List, Optional, Tuple

import torch

BLOCK_SIZE = 16

_TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and seed of one synthetic decode batch.

    ``ctx`` is either ``("fixed", (c0, c1, ...))`` (one length per sequence, or a
    single length for all), or ``("uniform", lo, hi)`` (inclusive bounds, one
    draw per sequence). With ``shared_prefix_tokens`` > 0 every sequence starts
    with the same prefix and ``ctx`` describes the unique suffix length only.
    """

    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    kv_dtype: str  # "f16" | "bf16" | "e4m3"
    q_dtype: str  # "f16" | "bf16"
    num_blocks: int  # physical pool size, in blocks
    ctx: Tuple
    seed: int
    shared_prefix_tokens: int = 0
    partition_tokens: int = 0  # 0: let the library choose
    block_size: int = BLOCK_SIZE

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def source_dtype(self) -> torch.dtype:
        """dtype the K/V source values are drawn in (bf16 for an e4m3 cache)."""
        return torch.bfloat16 if self.kv_dtype == "e4m3" else _TORCH_DTYPES[self.kv_dtype]

    @property
    def q_torch_dtype(self) -> torch.dtype:
        return _TORCH_DTYPES[self.q_dtype]

    @property
    def kv_elem_bytes(self) -> int:
        return 1 if self.kv_dtype == "e4m3" else 2

    @property
    def scale(self) -> float:
        return 1.0 / float(self.head_dim) ** 0.5


def _gen(seed: int, tag: str) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((zlib.crc32(f"{seed}/{tag}".encode()) << 8) ^ seed)
    return g


def context_lens(w: Workload) -> torch.Tensor:
    """Per-sequence context length (int32), including the token written this step."""
    kind = w.ctx[0]
    if kind == "fixed":
        vals = list(w.ctx[1])
        if len(vals) == 1:
            vals = vals * w.num_seqs
        assert len(vals) == w.num_seqs
        lens = torch.tensor(vals, dtype=torch.int64)
    elif kind == "uniform":
        lo, hi = w.ctx[1], w.ctx[2]
        lens = torch.randint(lo, hi + 1, (w.num_seqs,), generator=_gen(w.seed, "ctx"))
    else:
        raise ValueError(kind)
    lens = lens + w.shared_prefix_tokens
    return lens.to(torch.int32)


def block_order(w: Workload) -> torch.Tensor:
    """A seeded permutation of the pool's block ids: the order the free list hands them out."""
    return torch.randperm(w.num_blocks, generator=_gen(w.seed, "perm")).to(torch.int32)


def query(w: Workload) -> torch.Tensor:
    """q [num_seqs, num_q_heads, head_dim] in the workload's q dtype."""
    x = torch.randn(w.num_seqs, w.num_q_heads, w.head_dim, generator=_gen(w.seed, "q"))
    return x.to(w.q_torch_dtype)


def _normal(w: Workload, n: int, tag: str) -> torch.Tensor:
    x = torch.randn(n, w.num_kv_heads, w.head_dim, generator=_gen(w.seed, tag))
    return x.to(w.source_dtype)


def kv_source(w: Workload, seq: int, which: str, lens: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Logical K or V rows of one sequence, [ctx, num_kv_heads, head_dim], source dtype.

    Row t is the key (value) of position t. With a shared prefix the first
    ``shared_prefix_tokens`` rows are the same tensor for every sequence.
    """
    assert which in ("k", "v")
    if lens is None:
        lens = context_lens(w)
    n = int(lens[seq])
    p = w.shared_prefix_tokens
    if p == 0:
        return _normal(w, n, f"{which}/{seq}")
    prefix = _normal(w, p, f"{which}/prefix")
    return torch.cat([prefix, _normal(w, n - p, f"{which}/{seq}")], dim=0)


def kv_prefix(w: Workload, which: str) -> torch.Tensor:
    """The shared prefix rows alone (empty when the workload has none)."""
    if w.shared_prefix_tokens == 0:
        return torch.empty(0, w.num_kv_heads, w.head_dim, dtype=w.source_dtype)
    return _normal(w, w.shared_prefix_tokens, f"{which}/prefix")


def sentinel_pool(w: Workload, seed_tag: str = "sentinel") -> torch.Tensor:
    """Seeded random bytes the pool is pre-filled with, [num_blocks, Hkv, 16, D * elem] uint8.

    Untouched slots must keep exactly these bytes after any write.
    """
    g = _gen(w.seed, seed_tag)
    nbytes = w.num_blocks * w.num_kv_heads * w.block_size * w.head_dim * w.kv_elem_bytes
    b = torch.randint(0, 256, (nbytes,), generator=g, dtype=torch.uint8)
    return b.view(w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim * w.kv_elem_bytes)


@functools.lru_cache(maxsize=None)
def fp8_scales(w: Workload) -> Tuple[float, float]:
    """Per-tensor (k_scale, v_scale) of an e4m3 cache: float32(amax |source|) / 448 in float32.

    The amax runs over every K (V) source row of the workload, shared prefix
    included, so the whole source range maps onto e4m3's finite range.
    """
    if w.kv_dtype != "e4m3":
        return 1.0, 1.0
    lens = context_lens(w)
    amax = {"k": 0.0, "v": 0.0}
    for which in ("k", "v"):
        for s in range(w.num_seqs):
            amax[which] = max(amax[which], float(kv_source(w, s, which, lens).float().abs().max()))
    c448 = torch.tensor(448.0, dtype=torch.float32)
    return (float(torch.tensor(amax["k"], dtype=torch.float32) / c448),
            float(torch.tensor(amax["v"], dtype=torch.float32) / c448))


def max_blocks_per_seq(w: Workload, lens: Optional[torch.Tensor] = None) -> int:
    if lens is None:
        lens = context_lens(w)
    m = int(lens.max())
    return max(1, -(-m // w.block_size))


# --- the five workloads -----------------------------------------------------

TINY = Workload("tiny", 4, 4, 4, 64, "f16", "f16", 64, ("fixed", (1, 17, 33, 100)), seed=1001)
LLAMA7B_MHA = Workload("llama7b_mha", 32, 32, 32, 128, "f16", "f16", 5120, ("fixed", (2048,)), seed=1002)
LLAMA3_8B_GQA = Workload("llama3_8b_gqa", 64, 32, 8, 128, "bf16", "bf16", 36864, ("uniform", 128, 8192), seed=1003)
PREFIX_GQA = Workload("prefix_gqa", 128, 32, 8, 128, "bf16", "bf16", 8192, ("uniform", 1, 512), seed=1004,
                      shared_prefix_tokens=1024)
LONG70B_FP8 = Workload("long70b_fp8", 8, 64, 8, 128, "e4m3", "bf16", 73728, ("uniform", 32768, 131072), seed=1005,
                       partition_tokens=512)

# Same structure at sizes the float64 oracle finishes in seconds: several
# pages and partitions per sequence, ragged last blocks and partitions.
LLAMA7B_MHA_SMALL = Workload("llama7b_mha_small", 3, 4, 4, 128, "f16", "f16", 256, ("fixed", (2048, 777, 1)),
                             seed=2002)
LLAMA3_8B_GQA_SMALL = Workload("llama3_8b_gqa_small", 5, 8, 2, 128, "bf16", "bf16", 512, ("uniform", 128, 1300),
                               seed=2003)
PREFIX_GQA_SMALL = Workload("prefix_gqa_small", 6, 8, 2, 128, "bf16", "bf16", 256, ("uniform", 1, 90), seed=2004,
                            shared_prefix_tokens=64)
LONG70B_FP8_SMALL = Workload("long70b_fp8_small", 2, 16, 2, 128, "e4m3", "bf16", 512, ("uniform", 1500, 3100),
                             seed=2005, partition_tokens=512)
MQA_SMALL = Workload("mqa_small", 3, 16, 1, 128, "f16", "f16", 128, ("fixed", (300, 45, 513)), seed=2006)
D64_GQA_SMALL = Workload("d64_gqa_small", 4, 8, 4, 64, "bf16", "bf16", 128, ("fixed", (16, 32, 250, 2)), seed=2007)

FULL: Dict[str, Workload] = {w.name: w for w in (TINY, LLAMA7B_MHA, LLAMA3_8B_GQA, PREFIX_GQA, LONG70B_FP8)}
SMALL: Dict[str, Workload] = {w.name: w for w in (TINY, LLAMA7B_MHA_SMALL, LLAMA3_8B_GQA_SMALL, PREFIX_GQA_SMALL,
                                                  LONG70B_FP8_SMALL, MQA_SMALL, D64_GQA_SMALL)}
ALL: Dict[str, Workload] = {**FULL, **SMALL}


def request_stream(seed: int, num_requests: int, max_tokens: int = 2048):
    """Synthetic request mix for the KV-memory utilisation measurement: (prompt, output) lengths.

    Prompts uniform in [16, 1024]; outputs exponential with mean 256, at least 1; prompt + output
    capped at max_tokens (the length a contiguous allocator would have to reserve).
    """
    g = _gen(seed, "requests")
    prompt = torch.randint(16, 1025, (num_requests,), generator=g)
    out = (torch.empty(num_requests).exponential_(1.0 / 256.0, generator=g).ceil().clamp(min=1)).to(torch.int64)
    out = torch.minimum(out, max_tokens - prompt)
    return prompt.tolist(), out.tolist()


def kv_bytes_read(w: Workload, lens: Optional[torch.Tensor] = None) -> int:
    """Algorithmic K+V bytes one decode step reads: sum_s ctx_s * Hkv * D * elem * 2."""
    if lens is None:
        lens = context_lens(w)
    return int(lens.to(torch.int64).sum()) * w.num_kv_heads * w.head_dim * w.kv_elem_bytes * 2


__all__: List[str] = [
    "Workload", "BLOCK_SIZE", "context_lens", "block_order", "query", "kv_source", "kv_prefix", "sentinel_pool",
    "max_blocks_per_seq", "kv_bytes_read", "fp8_scales", "FULL", "SMALL", "ALL", "TINY", "LLAMA7B_MHA", "LLAMA3_8B_GQA",
    "PREFIX_GQA", "LONG70B_FP8",
]
