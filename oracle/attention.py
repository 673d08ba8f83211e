"""Decode attention of the oracle, as its plain definition in float64 (test infrastructure).

For sequence s with context length n, query head h and its KV head
hk = h // G (G = num_q_heads / num_kv_heads):

    K~[t] = Kpool[bt[s][t // 16], hk, t % 16, :],  V~ likewise,  t in [0, n)
    out[s, h, :] = sum_t softmax_t(scale * q[s, h] . K~[t]) * V~[t]

Sources: vLLM pages, "PagedAttention" (dingiv.github.io/ai/compute/engine/vllm)
and "vLLM 前世今生" section 3.2 (pages of 16 tokens reached through a block
table, page of a position = position // block_size); the kernels section of
the first page names GQA (LLaMA) and MQA (ChatGLM) kernels, where several query
heads share one KV head.

Readings taken where the pages are silent:
* query heads are grouped contiguously: query head h reads KV head h // G
  (the LLaMA ``repeat_kv`` convention);
* ``context_lens`` already counts the token written this step;
* a sequence with context length 0 has output 0;
* ``scale`` multiplies q.k before the softmax.

Paged decode reaches exactly this result up to rounding, so the oracle is the
definition: one max-subtracted softmax over the whole context, float64, no
online rescaling, no partitions.
"""
from __future__ import annotations

from typing import Sequence

import numpy as np

from . import cache


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * K q) V for one query vector; float64; zeros for an empty context."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    s = float(scale) * (K @ q)
    s = s - s.max()
    w = np.exp(s)
    return (w @ V) / w.sum()


def gather_context(pool_bytes: np.ndarray, block_table_row: np.ndarray, n: int, kv_head: int, kv_dtype: str,
                   scale: float = 1.0, block_size: int = 16) -> np.ndarray:
    """Logical rows [n, D] (float64) of one (sequence, KV head), read through the block table.

    ``pool_bytes`` is a byte pool [NB, Hkv, BS, D * elem]; only the gathered
    rows are converted to values.
    """
    t = np.arange(n)
    blocks = block_table_row[t // block_size].astype(np.int64)
    rows = pool_bytes[blocks, kv_head, t % block_size, :]
    return cache.pool_values(rows, kv_dtype, scale)


def decode_paged(q: np.ndarray, k_pool: np.ndarray, v_pool: np.ndarray, block_tables: np.ndarray,
                 context_lens: Sequence[int], scale: float, num_kv_heads: int, kv_dtype: str,
                 k_scale: float = 1.0, v_scale: float = 1.0, block_size: int = 16) -> np.ndarray:
    """Decode through the byte pools (path B): float64 [B, Hq, D]."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    G = Hq // num_kv_heads
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for s in range(B):
        n = int(context_lens[s])
        for hk in range(num_kv_heads):
            K = gather_context(k_pool, block_tables[s], n, hk, kv_dtype, k_scale, block_size)
            V = gather_context(v_pool, block_tables[s], n, hk, kv_dtype, v_scale, block_size)
            for h in range(hk * G, (hk + 1) * G):
                out[s, h] = attend(q[s, h], K, V, scale)
    return out


def decode_logical(q: np.ndarray, k_seqs: Sequence[np.ndarray], v_seqs: Sequence[np.ndarray], scale: float,
                   num_kv_heads: int) -> np.ndarray:
    """Decode from each sequence's logical float64 rows [n, Hkv, D] (path A): no pool, no block table."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for s in range(B):
        for h in range(Hq):
            out[s, h] = decode_logical_one(q[s, h], k_seqs[s], v_seqs[s], h, Hq, num_kv_heads, scale)
    return out


def decode_logical_one(q_vec: np.ndarray, k_seq: np.ndarray, v_seq: np.ndarray, q_head: int, num_q_heads: int,
                       num_kv_heads: int, scale: float) -> np.ndarray:
    """One (sequence, query head) output from the logical rows: what sampled full-size checks call."""
    hk = q_head // (num_q_heads // num_kv_heads)
    return attend(q_vec, k_seq[:, hk, :], v_seq[:, hk, :], scale)


def prefill_paged(q: np.ndarray, k_pool: np.ndarray, v_pool: np.ndarray, block_tables: np.ndarray,
                  query_start: Sequence[int], context_lens: Sequence[int], scale: float, num_kv_heads: int,
                  kv_dtype: str, block_size: int = 16) -> np.ndarray:
    """Causal attention of a chunk of new tokens per sequence over its paged context (float64).

    Sequence s owns query rows query_start[s] .. query_start[s + 1] - 1, the last
    n_s = query_start[s + 1] - query_start[s] tokens of its context_lens[s] tokens (all already
    written to the pool). Row i of the chunk is position p = context_lens[s] - n_s + i and attends
    over positions 0 .. p (itself included): out = softmax(scale * q K[0..p]^T) V[0..p].
    Source: the notes page's kernels section (attention over paged KV, FlashAttention adapted to
    paging) and "vLLM 前世今生" §5.4 (chunked prefill: a long prompt's prefill split into chunks).
    """
    q = np.asarray(q, dtype=np.float64)
    T, Hq, D = q.shape
    G = Hq // num_kv_heads
    out = np.zeros((T, Hq, D), dtype=np.float64)
    for s in range(len(context_lens)):
        r0, r1 = int(query_start[s]), int(query_start[s + 1])
        n = int(context_lens[s])
        start = n - (r1 - r0)
        for hk in range(num_kv_heads):
            K = gather_context(k_pool, block_tables[s], n, hk, kv_dtype, 1.0, block_size)
            V = gather_context(v_pool, block_tables[s], n, hk, kv_dtype, 1.0, block_size)
            for i in range(r1 - r0):
                p = start + i
                for h in range(hk * G, (hk + 1) * G):
                    out[r0 + i, h] = attend(q[r0 + i, h], K[:p + 1], V[:p + 1], scale)
    return out
